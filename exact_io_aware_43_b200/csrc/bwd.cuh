// bwd.cuh -- attention backward for sm_100a, by recomputation (robocikowo.com "Flash Attention":
// the backward recomputes the attention matrix from the saved O and L instead of storing it).
//
// Three kernels on the caller's stream.  The main kernel is fa_bwd_kernel_q128 (bwd_q128.cuh,
// 128-query steps) for d = 64 and 128, and fa_bwd_kernel_pair (bwd_pair.cuh, CTA pairs) for
// d = 256; this file's fa_bwd_kernel is the alternative the build selects with FA_BWD_Q128=0 or
// FA_BWD_PAIR=0:
//   fa_bwd_pre_kernel   D_i = sum_c dO_ic O_ic, L2_i = L_i log2(e) (padded rows: +inf, 0),
//                       and zeroes the fp32 dQ accumulator (and the dK, dV accumulators when
//                       a group's query heads are split over CTAs).                  (HBM bound)
//   fa_bwd_kernel       one CTA per (block of 128 keys, key/value head [, 128-wide slice of d]
//                       [, share of the group's query heads]): K_j, V_j stay in shared memory
//                       while the CTA loops over 64-query blocks i of each of its query heads:
//                         S^T  = K_j Q_i^T               tcgen05.mma -> TMEM (keys on lanes)
//                         P^T  = exp2(S^T s log2e - L2_i)   recomputed from L
//                         dV  += P^T dO_i                A = P^T (bf16, TMEM)
//                         dP^T = V_j dO_i^T
//                         dS^T = P^T * (dP^T - D_i)
//                         dK  += dS^T Q_i                A = dS^T (bf16, TMEM)
//                         dQ_i^T += K_j^T dS^T           -> fp32 reduction into the accumulator
//                       dK is scaled by s in the epilogue, dQ when it is reduced.
//   fa_bwd_post_kernel  dq = bf16(dQ accumulator) (and dk, dv from their accumulators).
// No N x N buffer exists: the score and probability tiles live in tensor memory.
//
// Warp roles of fa_bwd_kernel (FA_BWD_SPLIT, the default): warps 0-7 compute P and dS, two
// warpgroups of 32 query columns each (thread = key row = TMEM lane); warps 8-11 drain dQ^T from
// tensor memory into the accumulator; warp 12 issues TMA loads; warp 13 allocates tensor memory
// and issues the MMAs.  With FA_BWD_SPLIT=0: one P/dS warpgroup, drain warps 4-7, warps 8, 9.
#pragma once

#include "sm100.cuh"

// Tuning knobs (compile time).  FA_BWD_STAGES128: depth of the Q_i/dO_i ring for d=128.
#ifndef FA_BWD_STAGES128
#define FA_BWD_STAGES128 3
#endif
// FA_BWD_MASKFAST: query blocks entirely below the diagonal (and without padded keys) skip the
// per-element mask test.
#ifndef FA_BWD_MASKFAST
#define FA_BWD_MASKFAST 1
#endif
// FA_BWD_SPLIT: two P/dS warpgroups, each owning 32 of the 64 query columns of S^T / dP^T (the
// arithmetic is elementwise, so the halves are independent); 0: one warpgroup, all 64 columns.
#ifndef FA_BWD_SPLIT
#define FA_BWD_SPLIT 1
#endif
// FA_BWD_ORDER: 1 issues dP^T(i+1) as soon as the dS warps have read dP^T(i), ahead of dK(i) and
// dQ^T(i) (which wait for dS(i)); 0 issues it after them.
#ifndef FA_BWD_ORDER
#define FA_BWD_ORDER 0
#endif

namespace fattn {

struct BwdParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  const float* lse;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dq_acc;   // [BH, N, D] fp32
  float* L2;       // [BH, Npad] fp32: lse * log2(e), +inf on padded rows
  float* Drow;     // [BH, Npad] fp32: rowsum(dO * O), 0 on padded rows
  uint8_t* aug;    // d = 128 only: per 128-query block, 4 KB of MMA operand holding -L/s and -D
                   // as three bf16 terms each (see fa_bwd_pre_kernel); nullptr otherwise
  int BH;          // batch * query heads (rows of dq_acc, L2, Drow)
  int N;
  int Npad;        // N rounded up to 128
  int nkb;         // key blocks of 128 per head
  int H;           // query heads per batch
  int Hkv;         // key/value heads per batch (H is a multiple of Hkv)
  int G;           // query heads per key/value head, H / Hkv
  int BHkv;        // batch * key/value heads (CTAs of the main kernels: BHkv x key blocks)
  int head_band;   // K/V heads per band of the CTA order (0: kBwdHeadBand)
  int gsplit;      // CTAs that share one (key block, key/value head), each taking gq query heads
  int gq;          //   of the group; with gsplit > 1 they add their dK, dV into dk_acc, dv_acc
  float* dk_acc;   // [BHkv, N, D] fp32 (scaled dK), used when gsplit > 1
  float* dv_acc;   // [BHkv, N, D] fp32
  float scale;
  float scale_log2;
  uint64_t limit_ns;
};

// Grouped heads in the main backward kernels.  A CTA owns key block j of key/value head kvh
// (= b * Hkv + hk) and runs nit_h query-block steps for each of its query heads b * H + hk * G +
// g, one head after the other; dK_j and dV_j accumulate over them in tensor memory (the gradient
// of a shared K/V row is the sum over the heads that read it).  When (key blocks x K/V heads)
// alone would leave SMs idle, the G heads are dealt out gq at a time to gsplit CTAs, which add
// their sums into fp32 accumulators at the end.
struct BwdGroup {
  int qh0;      // first query head of this CTA
  int nheads;   // query heads of this CTA
  int nit_h;    // query-block steps per query head
  int i_start;  // first query block
  __device__ __forceinline__ BwdGroup(const BwdParams& p, int kvh, int gs, int i0, int nqblk)
      : qh0((kvh / p.Hkv) * p.H + (kvh % p.Hkv) * p.G + gs * p.gq),
        nheads(min(p.gq, p.G - gs * p.gq)), nit_h(nqblk - i0), i_start(i0) {}
};

// One 32-column chunk of a dK or dV row leaving tensor memory: bf16 straight to the output, or,
// when the group's query heads are split over CTAs, an fp32 reduce-add into the accumulator.
__device__ __forceinline__ void bwd_store_chunk(const uint32_t (&v)[32], float mul, bool row_ok,
                                                __nv_bfloat16* dst, float* acc) {
  if (!row_ok) return;
  if (acc != nullptr) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      red_add_v4_f32(acc + 4 * e, __uint_as_float(v[4 * e]) * mul,
                     __uint_as_float(v[4 * e + 1]) * mul, __uint_as_float(v[4 * e + 2]) * mul,
                     __uint_as_float(v[4 * e + 3]) * mul);
    return;
  }
  uint4 pkd[4];
  uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
  for (int e = 0; e < 16; ++e)
    pw[e] = pack_bf16(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int e = 0; e < 4; ++e) d4[e] = pkd[e];
}
// CTA -> (key block j, key/value head, d slice).  Heads are taken in bands of kBwdHeadBand; within
// a band the key block is outermost, so the key blocks with the most query steps (causal: the
// first ones) of the band's heads start first, while the query tiles in flight stay those of a
// few heads (their reads are served from L2).
#ifndef FA_BWD_HEAD_BAND
#define FA_BWD_HEAD_BAND 4
#endif
constexpr int kBwdHeadBand = FA_BWD_HEAD_BAND;
struct BwdUnit {
  int j, kvh, gs, slice;
  __device__ __forceinline__ BwdUnit(int x, const BwdParams& p, int nsl) {
    const int per_head = nsl * p.gsplit;  // CTAs per (key block, K/V head)
    const int hb = p.head_band > 0 ? p.head_band : kBwdHeadBand;
    const int band_ctas = hb * p.nkb * per_head;
    const int band = x / band_ctas;
    const int h0 = band * hb;
    const int nh = min(hb, p.BHkv - h0);
    const int r = x - band * band_ctas;
    j = r / (nh * per_head);
    const int rem = r - j * (nh * per_head);
    kvh = h0 + rem / per_head;
    const int rem2 = rem - (rem / per_head) * per_head;
    gs = rem2 / nsl;
    slice = rem2 - gs * nsl;
  }
};

// Walks the steps of a BwdGroup in order (no division per step): `i` and `head` describe the
// current step; next() moves to the following one.
struct BwdCursor {
  int i, head, i_start, i_end;
  __device__ __forceinline__ explicit BwdCursor(const BwdGroup& g)
      : i(g.i_start), head(g.qh0), i_start(g.i_start), i_end(g.i_start + g.nit_h) {}
  __device__ __forceinline__ void next() {
    if (++i == i_end) {
      i = i_start;
      ++head;
    }
  }
};

// ------------------------------------------------------------------------------------------
// preprocess: D, L2, zero dQ accumulator
// ------------------------------------------------------------------------------------------
// x as three bf16 terms hi + mid + lo (each the rounding of what the previous ones left; about
// 24 significant bits together) in the first three of eight bf16 slots, the rest zero.
__device__ __forceinline__ uint4 split3_bf16(float x) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
  return make_uint4(uint32_t(__bfloat16_as_ushort(hi)) | (uint32_t(__bfloat16_as_ushort(mid)) << 16),
                    uint32_t(__bfloat16_as_ushort(lo)), 0u, 0u);
}

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p) {
  constexpr int G = D / 8;  // lanes per row, 8 bf16 (16 bytes) each
  const long long total_rows = (long long)p.BH * p.Npad;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  const int sub = lane % G;
  constexpr int ROWS_PER_WARP = 32 / G;
  // rows: D and L2.  The loop bound is warp-uniform so the shuffles see the whole warp.
  const long long warp_id = tid >> 5;
  const long long nwarps = nthreads >> 5;
  for (long long rb = warp_id * ROWS_PER_WARP; rb < total_rows; rb += nwarps * ROWS_PER_WARP) {
    const long long r = rb + lane / G;
    const bool in = r < total_rows;
    const int head = in ? int(r / p.Npad) : 0;
    const int q = in ? int(r % p.Npad) : p.N;
    float acc = 0.f;
    if (q < p.N) {
      const size_t off = (size_t(head) * p.N + q) * D + sub * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(p.o + off);
      const uint4 b = *reinterpret_cast<const uint4*>(p.dO + off);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(a2[e]);
        const float2 y = __bfloat1622float2(b2[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
#pragma unroll
    for (int w = G / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (in && sub == 0) {
      p.Drow[r] = acc;
      p.L2[r] = (q < p.N) ? p.lse[size_t(head) * p.N + q] * 1.4426950408889634f : INFINITY;
      if (p.aug != nullptr) {
        // the 128-query kernel's B operand for its ninth K step: row q of the block gets
        // [-L/s as hi, mid, lo, 0 x 5] in the first 8-element K half and [-D likewise] in the
        // second, each half a run of 8-row x 16-byte core matrices (rows 16 B apart, 8-row
        // groups 128 B apart, the two halves 2 KB apart).  A padded row gets a huge finite
        // -L/s (never inf: the other step multiplies it by zero), so its P is 0.
        const float xl = (q < p.N) ? -p.lse[size_t(head) * p.N + q] / p.scale : -0x1p100f;
        const int blk = q >> 7, rr = q & 127;
        uint8_t* tile = p.aug + (size_t(head) * (p.Npad >> 7) + blk) * 4096 +
                        (rr >> 3) * 128 + (rr & 7) * 16;
        *reinterpret_cast<uint4*>(tile) = split3_bf16(xl);
        *reinterpret_cast<uint4*>(tile + 2048) = split3_bf16(-acc);
      }
    }
  }
  // zero the dQ accumulator (its size is a multiple of 4 floats: D >= 64), and the dK, dV
  // accumulators when a group's query heads are split over CTAs
  const long long n4 = (long long)p.BH * p.N * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long i = tid; i < n4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p.gsplit > 1) {
    const long long m4 = (long long)p.BHkv * p.N * D / 4;
    float4* k4 = reinterpret_cast<float4*>(p.dk_acc);
    float4* v4 = reinterpret_cast<float4*>(p.dv_acc);
    for (long long i = tid; i < m4; i += nthreads) {
      k4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      v4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// ------------------------------------------------------------------------------------------
// postprocess: dq = bf16(accumulator)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float* __restrict__ acc,
                                                          __nv_bfloat16* __restrict__ dq,
                                                          long long n8) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long i = tid; i < n8; i += nthreads) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16(a.x, a.y);
    o.y = pack_bf16(a.z, a.w);
    o.z = pack_bf16(b.x, b.y);
    o.w = pack_bf16(b.z, b.w);
    reinterpret_cast<uint4*>(dq)[i] = o;
  }
}

// ------------------------------------------------------------------------------------------
// main backward kernel
// ------------------------------------------------------------------------------------------
template <int D>
struct BwdCfg {
  static constexpr int BC = 128;                  // keys per CTA (MMA M for S^T, dV, dK)
  static constexpr int BR = 64;                   // queries per inner step
  static constexpr int DO = D > 128 ? 128 : D;    // width of the dK/dV/dQ slice of this CTA
  static constexpr int NSL = D / DO;              // slices of d (CTAs per key block)
  static constexpr int KB = D / 64;               // 128-byte swizzle blocks across d
  static constexpr int KV_BLK = BC * 128;         // bytes of one 64-column block of K_j / V_j
  static constexpr int Q_BLK = BR * 128;          // bytes of one 64-column block of Q_i / dO_i
  static constexpr int KV_BYTES = KB * KV_BLK;
  static constexpr int Q_BYTES = KB * Q_BLK;
  static constexpr int STAGES = D == 64 ? 3 : (D == 128 ? FA_BWD_STAGES128 : 1);
  static constexpr bool SPLIT = FA_BWD_SPLIT != 0;
  static constexpr int CMP_WARPS = SPLIT ? 8 : 4;        // P/dS warps (one or two warpgroups)
  static constexpr int NCOL = SPLIT ? 32 : 64;           // query columns per P/dS thread
  static constexpr int THREADS = SPLIT ? 512 : 320;
  static constexpr int DQ_WARP0 = CMP_WARPS;
  static constexpr int PRODUCER_WARP = CMP_WARPS + 4;
  static constexpr int MMA_WARP = CMP_WARPS + 5;
  // tensor memory columns
  static constexpr int T_S = 0, T_DP = 64, T_P = 128, T_DS = 160, T_DQ = 192, T_DV = 256,
                       T_DK = 256 + DO;
  static constexpr int TMEM_COLS = (T_DK + DO) <= 256 ? 256 : 512;
  // shared memory map
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;                 // STAGES x Q_i
  static constexpr int OFF_DO = OFF_Q + STAGES * Q_BYTES;        // STAGES x dO_i
  static constexpr int OFF_DS = OFF_DO + STAGES * Q_BYTES;       // dS^T [128 keys][64 q] bf16
  static constexpr int OFF_ROWS = OFF_DS + BC * BR * 2;          // STAGES x (L2[64], D[64])
  // dQ staging: slots of [64 queries][64 d] fp32 reduced into the accumulator by TMA
  static constexpr int DQ_CH = DO / 64;                          // 64-wide chunks per tile
  static constexpr int DQ_SLOT = BR * 64 * 4;
  static constexpr int DQ_SLOTS = D == 64 ? 2 : (D == 128 ? (FA_BWD_STAGES128 > 2 ? 2 : 4) : 1);
  static constexpr int OFF_DQS = OFF_ROWS + STAGES * 2 * BR * 4;
  static constexpr int OFF_BAR = OFF_DQS + DQ_SLOTS * DQ_SLOT;
  // barriers: kv_full, q_full[S], q_empty[S], s_full, s_free, dp_full, dp_free, p_full,
  //           ds_full, dv_done, dq_full, dq_empty, drain
  static constexpr int NBAR = 1 + 2 * STAGES + 11;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t IDESC_ST = idesc_bf16_f32(BC, BR, 0, 0);  // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(BC, DO, 0, 1);  // dV, dK (A in TMEM)
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(DO, BR, 1, 1);  // dQ^T = K^T dS^T
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FA_TRACE_DECL;

  // ---- work unit: (key block j, key/value head, d slice) in the order of BwdUnit.  Steps run
  // over the group's query heads, each over its query blocks (see BwdGroup).
  const BwdUnit unit(blockIdx.x, p, C::NSL);
  const int j = unit.j, kvh = unit.kvh, slice = unit.slice;
  const int k0 = j * C::BC;
  const int nqblk = (p.N + C::BR - 1) / C::BR;
  const BwdGroup grp(p, kvh, unit.gs, CAUSAL ? (k0 / C::BR) : 0, nqblk);
  const int nit = grp.nheads * grp.nit_h;  // >= 1

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  const uint32_t BAR_KV = bar(0);
  auto BAR_QF = [&](int s) { return bar(1 + s); };
  auto BAR_QE = [&](int s) { return bar(1 + C::STAGES + s); };
  const int b0 = 1 + 2 * C::STAGES;
  const uint32_t BAR_SF = bar(b0 + 0), BAR_SFREE = bar(b0 + 1), BAR_DPF = bar(b0 + 2),
                 BAR_DPFREE = bar(b0 + 3), BAR_PF = bar(b0 + 4), BAR_DSF = bar(b0 + 5),
                 BAR_DVD = bar(b0 + 6), BAR_DQF = bar(b0 + 7), BAR_DQE = bar(b0 + 8),
                 BAR_DRAIN = bar(b0 + 9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const Waiter W{abort_flag, p.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(BAR_KV, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR_QF(s), 1);
      mbar_init(BAR_QE(s), 1);
    }
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_SFREE, C::CMP_WARPS);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_DPFREE, C::CMP_WARPS);
    mbar_init(BAR_PF, C::CMP_WARPS);
    mbar_init(BAR_DSF, C::CMP_WARPS);
    mbar_init(BAR_DVD, 1);
    mbar_init(BAR_DQF, 1);
    mbar_init(BAR_DQE, 4);
    mbar_init(BAR_DRAIN, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float* rows_smem = reinterpret_cast<const float*>(smem + C::OFF_ROWS);

  if (warp == C::PRODUCER_WARP) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(BAR_KV, 2 * C::KV_BYTES);
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_3d(sbase + C::OFF_K + kb * C::KV_BLK, &tmK, BAR_KV, kb * 64, k0, kvh);
        tma_load_3d(sbase + C::OFF_V + kb * C::KV_BLK, &tmV, BAR_KV, kb * 64, k0, kvh);
      }
      int it = 0;
      BwdCursor cur(grp);
      for (; it < nit; ++it) {
        const int i = cur.i, head = cur.head;
        cur.next();
        const int s = it % C::STAGES;
        if (!W.wait(BAR_QE(s), ((it / C::STAGES) & 1) ^ 1, 31)) break;
        FA_TRACE_EV(20, it);
        mbar_arrive_expect_tx(BAR_QF(s), 2 * C::Q_BYTES + 2 * C::BR * 4);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_3d(sbase + C::OFF_Q + s * C::Q_BYTES + kb * C::Q_BLK, &tmQ, BAR_QF(s), kb * 64,
                      i * C::BR, head);
          tma_load_3d(sbase + C::OFF_DO + s * C::Q_BYTES + kb * C::Q_BLK, &tmdO, BAR_QF(s),
                      kb * 64, i * C::BR, head);
        }
        const size_t roff = size_t(head) * p.Npad + size_t(i) * C::BR;
        bulk_load(sbase + C::OFF_ROWS + s * 2 * C::BR * 4, p.L2 + roff, C::BR * 4, BAR_QF(s));
        bulk_load(sbase + C::OFF_ROWS + s * 2 * C::BR * 4 + C::BR * 4, p.Drow + roff, C::BR * 4,
                  BAR_QF(s));
      }
      if (W.aborted()) {
        W.drain(BAR_KV, 0);
        for (int jj = max(0, it - C::STAGES); jj < it; ++jj)
          W.drain(BAR_QF(jj % C::STAGES), (jj / C::STAGES) & 1);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t k_addr = sbase + C::OFF_K, v_addr = sbase + C::OFF_V;
      const uint32_t ds_addr = sbase + C::OFF_DS;
      auto issue_st = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
        // [S^T | dP^T] (128 x 64) = A (128 keys x D) * B (64 queries x D)^T, both K-major
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * C::KV_BLK + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * C::Q_BLK + (kk & 3) * 32;
          mma_ss(tmem + d_col, sdesc_sw128(a_base + ka, 16, 1024),
                 sdesc_sw128(b_base + kb, 16, 1024), C::IDESC_ST, kk > 0);
        }
      };
      auto issue_kv = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool acc) {
        // [dV | dK] (128 x DO) += A (tmem, 128 keys x 64 queries) * B (DO x 64 queries, MN-major)
#pragma unroll
        for (int kk = 0; kk < C::BR / 16; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + kk * 8,
                 sdesc_sw128(b_base + slice * 2 * C::Q_BLK + kk * 2048, C::Q_BLK, 1024),
                 C::IDESC_KV, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = W.wait(BAR_KV, 0, 40);
      if (ok) ok = W.wait(BAR_QF(0), 0, 41);
      if (ok) {
        tc_fence_after();
        issue_st(C::T_S, k_addr, sbase + C::OFF_Q);
        tc_commit(BAR_SF);
        issue_st(C::T_DP, v_addr, sbase + C::OFF_DO);
        tc_commit(BAR_DPF);
      }
      for (int it = 0; ok && it < nit; ++it) {
        const int s = it % C::STAGES;
        const int sn = (it + 1) % C::STAGES;
        const uint32_t q_addr = sbase + C::OFF_Q + s * C::Q_BYTES;
        const uint32_t do_addr = sbase + C::OFF_DO + s * C::Q_BYTES;
        // dV += P^T dO_i
        FA_TRACE_EV(1, it);
        if (!(ok = W.wait(BAR_PF, it & 1, 42))) break;
        FA_TRACE_EV(2, it);
        tc_fence_after();
        issue_kv(C::T_DV, C::T_P, do_addr, it > 0);
        tc_commit(BAR_DVD);
        // S^T for the next query block as soon as its tile and the S^T columns are free.  With a
        // single stage the next tile can only arrive after this one is released, further down.
        const bool more = it + 1 < nit;
        auto issue_next_st = [&]() -> bool {
          if (!W.wait(BAR_QF(sn), ((it + 1) / C::STAGES) & 1, 43)) return false;
          if (!W.wait(BAR_SFREE, it & 1, 44)) return false;
          FA_TRACE_EV(3, it);
          tc_fence_after();
          issue_st(C::T_S, k_addr, sbase + C::OFF_Q + sn * C::Q_BYTES);
          tc_commit(BAR_SF);
          return true;
        };
        if (more && C::STAGES > 1 && !(ok = issue_next_st())) break;
        const bool early_dp = FA_BWD_ORDER && C::STAGES > 1 && more;
        if (early_dp) {
          if (!(ok = W.wait(BAR_DPFREE, it & 1, 47))) break;
          FA_TRACE_EV(7, it);
          tc_fence_after();
          issue_st(C::T_DP, v_addr, sbase + C::OFF_DO + sn * C::Q_BYTES);
          tc_commit(BAR_DPF);
        }
        // dK += dS^T Q_i ; dQ_i^T = K_j^T dS^T
        FA_TRACE_EV(4, it);
        if (!(ok = W.wait(BAR_DSF, it & 1, 45))) break;
        FA_TRACE_EV(5, it);
        if (it > 0 && !(ok = W.wait(BAR_DQE, (it - 1) & 1, 46))) break;
        FA_TRACE_EV(6, it);
        tc_fence_after();
        issue_kv(C::T_DK, C::T_DS, q_addr, it > 0);
#pragma unroll
        for (int kk = 0; kk < C::BC / 16; ++kk)
          mma_ss(tmem + C::T_DQ,
                 sdesc_sw128(k_addr + slice * 2 * C::KV_BLK + kk * 2048, C::KV_BLK, 1024),
                 sdesc_sw128(ds_addr + kk * 2048, C::Q_BLK, 1024), C::IDESC_DQ, kk > 0);
        tc_commit(BAR_DQF);
        tc_commit(BAR_QE(s));
        if (more && !early_dp) {
          if (C::STAGES == 1 && !(ok = issue_next_st())) break;
          if (!(ok = W.wait(BAR_DPFREE, it & 1, 47))) break;
          FA_TRACE_EV(7, it);
          tc_fence_after();
          issue_st(C::T_DP, v_addr, sbase + C::OFF_DO + sn * C::Q_BYTES);
          tc_commit(BAR_DPF);
        }
      }
      tc_commit(BAR_DRAIN);
      W.drain(BAR_DRAIN, 0);
    }
  } else if (warp < C::CMP_WARPS) {
    // ---------------------------------------------------------------- P / dS warpgroup(s)
    // Thread = key row (TMEM lane).  With two warpgroups, warpgroup h owns query columns
    // [32h, 32h+32) of every tile; the arithmetic is elementwise, so the halves never meet.
    constexpr int NC = C::NCOL;
    const int h = warp >> 2;                 // column half (0 when not split)
    const int c0 = h * NC;                   // first query column of this thread
    const int r = (warp & 3) * 32 + lane;    // key row within the block == TMEM lane
    const int key = k0 + r;
    const bool key_ok = key < p.N;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    uint8_t* ds_row = smem + C::OFF_DS + r * 128;
    bool ok = true;
    BwdCursor cur(grp);
    for (int it = 0; it < nit; ++it) {
      const int i = cur.i;
      cur.next();
      const int s = it % C::STAGES;
      const float* L2s = rows_smem + s * 2 * C::BR + c0;
      const float* Ds = rows_smem + s * 2 * C::BR + C::BR + c0;
      FA_TRACE_EV(10, it);
      if (!(ok = W.wait_warp(BAR_SF, it & 1, 50))) break;
      if (!(ok = W.wait_warp(BAR_QF(s), (it / C::STAGES) & 1, 51))) break;
      FA_TRACE_EV(11, it);
      tc_fence_after();
      uint32_t st[NC / 32][32];
#pragma unroll
      for (int q = 0; q < NC / 32; ++q) tmem_ld32(tmem + lane_base + C::T_S + c0 + 32 * q, st[q]);
#pragma unroll
      for (int q = 0; q < NC / 32; ++q) tmem_wait_ld(st[q]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_SFREE);
      // P^T = exp2(S^T s log2e - L2); zero for masked (causal key > query) and padded keys
      float pr[NC];
      const int qbase = i * C::BR + c0;
      const bool need_mask = !FA_BWD_MASKFAST || !key_ok || (CAUSAL && qbase < k0 + C::BC);
      if (need_mask) {
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float4 l4 = reinterpret_cast<const float4*>(L2s)[c4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e;
            const float x = fmaf(__uint_as_float(st[c >> 5][c & 31]), p.scale_log2, -lv[e]);
            bool valid = key_ok;
            if (CAUSAL) valid = valid && (key <= qbase + c);
            pr[c] = valid ? ex2(x) : 0.f;
          }
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float4 l4 = reinterpret_cast<const float4*>(L2s)[c4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e;
            pr[c] = ex2(fmaf(__uint_as_float(st[c >> 5][c & 31]), p.scale_log2, -lv[e]));
          }
        }
      }
      uint32_t pk[NC / 2];
#pragma unroll
      for (int c = 0; c < NC / 2; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
      // P^T columns are free once dV(it-1) has read them
      if (it > 0 && !(ok = W.wait_warp(BAR_DVD, (it - 1) & 1, 52))) break;
      tc_fence_after();
      if (NC == 64)
        tmem_st32(tmem + lane_base + C::T_P, *reinterpret_cast<uint32_t(*)[32]>(pk));
      else
        tmem_st16(tmem + lane_base + C::T_P + c0 / 2, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_PF);
      FA_TRACE_EV(12, it);
      // dS^T = P^T * (dP^T - D)
      if (!(ok = W.wait_warp(BAR_DPF, it & 1, 53))) break;
      FA_TRACE_EV(13, it);
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < NC / 32; ++q) tmem_ld32(tmem + lane_base + C::T_DP + c0 + 32 * q, st[q]);
#pragma unroll
      for (int q = 0; q < NC / 32; ++q) tmem_wait_ld(st[q]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DPFREE);
#pragma unroll
      for (int c4 = 0; c4 < NC / 4; ++c4) {
        const float4 d4 = reinterpret_cast<const float4*>(Ds)[c4];
        const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 4 * c4 + 2 * e;
          const float d0 = pr[c] * (__uint_as_float(st[c >> 5][c & 31]) - dv4[2 * e]);
          const float d1 = pr[c + 1] * (__uint_as_float(st[(c + 1) >> 5][(c + 1) & 31]) - dv4[2 * e + 1]);
          pk[c >> 1] = pack_bf16(d0, d1);
        }
      }
      // dS^T columns and the dS smem tile are free once dK(it-1) and dQ(it-1) have read them
      if (it > 0 && !(ok = W.wait_warp(BAR_DQF, (it - 1) & 1, 54))) break;
      tc_fence_after();
      if (NC == 64)
        tmem_st32(tmem + lane_base + C::T_DS, *reinterpret_cast<uint32_t(*)[32]>(pk));
      else
        tmem_st16(tmem + lane_base + C::T_DS + c0 / 2, pk);
#pragma unroll
      for (int c = 0; c < NC / 8; ++c) {
        const int chunk = c0 / 8 + c;  // 16-byte chunk = 8 queries of this key's row
        const uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) = v;
      }
      fence_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DSF);
      FA_TRACE_EV(14, it);
    }
    if (ok) {
      // ---- epilogue: dV, dK (x scale) -> bf16 -> global (split: warpgroup 0 dV, 1 dK)
      ok = W.wait_warp(BAR_DQF, (nit - 1) & 1, 55);
      if (ok) {
        tc_fence_after();
        const size_t base = (size_t(kvh) * p.N + key) * D + slice * C::DO;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          if (C::SPLIT && which != h) continue;
          const uint32_t col = which == 0 ? C::T_DV : C::T_DK;
          const float mul = which == 0 ? 1.f : p.scale;
          __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + base;
          float* acc = p.gsplit > 1 ? (which == 0 ? p.dv_acc : p.dk_acc) + base : nullptr;
#pragma unroll
          for (int c = 0; c < C::DO / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + col + 32 * c, v);
            tmem_wait_ld(v);
            bwd_store_chunk(v, mul, key_ok, dst + 32 * c, acc ? acc + 32 * c : nullptr);
          }
        }
      }
    }
    tc_fence_before();
  } else if (warp < C::DQ_WARP0 + 4) {
    // ---------------------------------------------------------------- dQ drain warpgroup
    // dQ^T (d on TMEM lanes, 64 queries on columns) -> x scale -> shared staging slots laid out
    // [64 queries][64 d] fp32 -> TMA bulk reduce-add into the fp32 accumulator (rows past N are
    // clipped by the tensor map).
    const int wq = warp - C::DQ_WARP0;
    const int tq = threadIdx.x - C::DQ_WARP0 * 32;  // 0..127
    const bool issuer = tq == 0;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    // dQ^T rows are d indices.  M = 128: lane i of warp w holds row 32w+i.  M = 64: rows
    // 16w..16w+15 sit in lanes 0..15 of warp w's lane quarter; lanes 16..31 hold nothing.
    const int drow = (C::DO == 128) ? (wq * 32 + lane) : (wq * 16 + lane);
    const bool row_ok = (C::DO == 128) || (lane < 16);
    const int my_chunk = drow >> 6;
    float* slots = reinterpret_cast<float*>(smem + C::OFF_DQS);
    if (issuer) tma_prefetch_desc(&tmdQ);
    int group = 0;
    BwdCursor cur(grp);
    for (int it = 0; it < nit; ++it) {
      const int i = cur.i, head = cur.head;
      cur.next();
      // the four drain warps leave the loop together (they share named barriers below)
      if (!named_bar_and(1, 128, W.wait_warp(BAR_DQF, it & 1, 60))) break;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(tmem + lane_base + C::T_DQ, v[0]);
      tmem_ld32(tmem + lane_base + C::T_DQ + 32, v[1]);
      tmem_wait_ld(v[0]);
      tmem_wait_ld(v[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DQE);
#pragma unroll
      for (int ch = 0; ch < C::DQ_CH; ++ch, ++group) {
        const int slot = group % C::DQ_SLOTS;
        if (issuer) bulk_wait_group_read<C::DQ_SLOTS - 1>();  // slot's previous reduce has read it
        named_bar_sync(1, 128);
        if (row_ok && my_chunk == ch) {
          float* dst = slots + slot * (C::BR * 64) + (drow & 63);
#pragma unroll
          for (int c = 0; c < C::BR; ++c) dst[c * 64] = __uint_as_float(v[c >> 5][c & 31]) * p.scale;
        }
        fence_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
          tma_reduce_add_3d(&tmdQ, smem_u32(slots + slot * (C::BR * 64)), slice * C::DO + ch * 64,
                            i * C::BR, head);
          bulk_commit_group();
        }
      }
    }
    if (issuer) bulk_wait_group_all();
    tc_fence_before();
  }

  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
