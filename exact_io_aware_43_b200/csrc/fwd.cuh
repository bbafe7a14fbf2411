// fwd.cuh -- fused attention forward for sm_100a.
//
// A work unit is NQT query tiles of 128 rows of one (batch, head) -- or, in the general variant,
// a range of the keys for them, or the packed query heads of one key/value head (see FwdUnit).
// For each unit the CTA streams its K_j, V_j tiles of 128 keys through a shared-memory ring (chipfoundryservices.com glossary
// "Flash Attention", "Tiling Algorithm" steps 1-2; robocikowo.com "Flash Attention": a Q block
// is loaded once, then the loop runs over the K, V blocks).  Per KV tile and query tile:
//   S   = Q_t K_j^T                  tcgen05.mma, bf16 x bf16 -> fp32 in tensor memory (step 3)
//   m   = max(m, rowmax(S*s))        one softmax thread owns one row (one TMEM lane)   (step 4)
//   P~  = exp2(S*s*log2e - m)        rounded to bf16 and written back into tensor memory
//   O  *= exp2(m_old - m_new)        rescale of the running output (robocikowo.com update rule)
//   O  += P~ V_j                     tcgen05.mma with A = P~ from tensor memory         (step 5)
// and after the last tile O /= l, L = (m + log2 l) ln 2 (step 6; L is kept for the backward).
// The score tile lives only in tensor memory: the N x N matrix never reaches HBM
// (systems-analysis.info "FlashAttention (PL)", "Scalanie operacji w jedno jadro CUDA").
//
// The kernel is persistent: CTA c takes units c, 2G-1-c, 2G+c, ... (a zig-zag over rounds of G =
// gridDim.x units, with the units ordered heaviest first when causal), keeping its tensor memory
// and barriers across units.  Q of the next unit is loaded as soon as the current unit's last S
// MMA has been issued, so its latency hides behind the last PV and the epilogue.  With a grid of
// one CTA per unit the same code runs one unit per CTA.
//
// Warp roles: warps [0, 4*NQT) are the softmax warpgroups (warpgroup t owns query tile t); the
// next warpgroup holds the TMA producer warp and the MMA-issuing warp (which also allocates
// tensor memory).  With NQT = 2 the two query tiles ping-pong: the tensor core works on one tile
// while the softmax warpgroup of the other computes its exponentials.
#pragma once

#include "sm100.cuh"

// Tuning knobs (compile time), each chosen by measurement on the long-context workload.
// FA_FWD_RSUM: how O's normaliser is formed -- 0: the fp32 sum (also used for
// L); 1: sum of the bf16-rounded weights via integer unpack; 2: the same sum with mixed
// bf16 + fp32 adds.  FA_FWD_RESCALE: the reference max moves (and O is rescaled) only when a row's
// max grows by more than this many log2 units (0: on every increase).  FA_FWD_MAX3: three-input
// max for the row maximum.
#ifndef FA_FWD_RSUM
#define FA_FWD_RSUM 2
#endif
// FA_FWD_POLY_MASK: bit g set computes the exponentials of scores [4g, 4g+4) of every 32 on the
// FMA pipe (exp2_fma2) instead of the MUFU unit; -1: a quarter (groups 0 and 4) at d = 64, where
// an exponential comes with half the MMA work of d = 128 and MUFU binds, none otherwise.
#ifndef FA_FWD_POLY_MASK
#define FA_FWD_POLY_MASK -1
#endif
#ifndef FA_FWD_RESCALE
#define FA_FWD_RESCALE 8.0f
#endif
#ifndef FA_FWD_MAX3
#define FA_FWD_MAX3 0
#endif
// FA_FWD_ONES_SUM: at d = 64 (where tensor memory has room) the PV MMA also multiplies P~ by a
// block of ones appended to V, so 16 extra O columns carry the sum of the bf16-rounded weights --
// rescaled with O, and no longer summed by the softmax threads.
#ifndef FA_FWD_ONES_SUM
#define FA_FWD_ONES_SUM 1
#endif
// FA_FWD_VST: V ring depth at d = 128 with two query tiles (the K ring keeps 2 stages).
#ifndef FA_FWD_VST
#define FA_FWD_VST 2
#endif
// FA_FWD_MMA_POLL: the two-tile MMA warp waits on its barriers with plain try_wait polling
// instead of try_wait with a suspend hint (-1: at d = 128 only).
#ifndef FA_FWD_MMA_POLL
#define FA_FWD_MMA_POLL -1
#endif
// FA_FWD_INORDER: 1 issues S_t(j+1) right behind PV_t(j) without waiting for PV_t(j) to
// complete.  S_t(j+1) overwrites the tensor memory that PV_t(j) reads P_t(j) from; the MMAs of
// one issuing thread run through the tensor core in issue order, so PV_t(j) has read its
// operands before S_t(j+1) writes (the same reliance as the sm100 attention collectives of
// CUTLASS, which issue Q K^T of the next tile straight after P V of the previous one).
#ifndef FA_FWD_INORDER
#define FA_FWD_INORDER 1
#endif

namespace fattn {

struct FwdParams {
  __nv_bfloat16* o;  // [BH, Nq, D] bf16 (one split) ...
  float* lse;        // [BH, Nq]
  float* o_part;     // ... or, with several splits, [splits, BH, Nq, D] fp32 partial outputs
  float* lse_part;   //     and [splits, BH, Nq] their logsumexps (natural log, -inf if empty)
  int Nq;            // queries per head
  int Nk;            // keys per head
  int off;           // causal alignment: query i sees keys j <= i + off (off = Nk - Nq)
  int BH;            // batch * query heads
  int H;             // query heads per batch
  int G;             // query heads per key/value head (grouped-query attention; 1 = one each)
  int nqb;           // query blocks (of NQT*128 rows) per head
  int splits;        // key ranges per (head, query block); 1 = the whole key sequence
  int pack;          // > 1: the pack = G query heads of a key/value head share one query tile
                     // (rows g * Nq + i; needs G * Nq <= 128), one unit per (K/V head, range)
  int Hkv;           // key/value heads per batch
  int kv_chunk;      // KV tiles of 128 keys per split
  int units;         // BH * nqb * splits, or more with a split tail (below)
  int tail_base;     // work items from here on are single query tiles: the units of the last
                     // (partial) round, each cut in two so that the round is shorter (plain
                     // non-causal forward with two query tiles); = units when not used
  float scale_log2;  // scale * log2(e)
  uint64_t limit_ns;
};

template <int D, int NQT>
struct FwdCfg {
  static constexpr int BM = 128;                 // query rows per tile (MMA M)
  static constexpr int BN = 128;                 // keys per KV tile
  static constexpr int KB = D / 64;              // 128-byte swizzle blocks across d
  static constexpr int QTILE_BYTES = BM * D * 2;
  static constexpr int KVTILE_BYTES = BN * D * 2;
  // K/V ring depth.  With one query tile (d = 256, and packed decoding at d = 64 / 128, where
  // a second tile would stay empty) the freed query buffer holds more stages.
  static constexpr int STAGES = NQT == 1 ? (D == 64 ? 6 : (D == 128 ? 3 : 1))
                                         : (D == 64 ? 4 : (D == 128 ? 2 : 1));
  static constexpr int KST = STAGES;                                        // K ring
  static constexpr int VST = (NQT == 2 && D == 128) ? FA_FWD_VST : STAGES;  // V ring
  static constexpr int SOFTMAX_WARPS = 4 * NQT;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;  // control warpgroup: producer, MMA, 2 idle
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int THREADS = (SOFTMAX_WARPS + 4) * 32;
  // Register split with two softmax warpgroups (384 threads launched at 168 registers each):
  // control warpgroup / softmax warpgroups 112 / 192 at d = 128 (with 104 for the control
  // warpgroup its MMA-issue path spilled; 112 / 192 compiles spill-free and measured 3% faster on
  // the long-context forward) and 104 / 200 at d = 64 (whose softmax path, with the ones-column
  // row sums, needs the larger share).  CTRL*128 + SOFTMAX*256 <= 384*168 in both.
  static constexpr bool REALLOC = NQT == 2;
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int CTRL_REGS = D == 64 ? 104 : 112;
  static constexpr int SOFTMAX_REGS = D == 64 ? 200 : 192;
  static_assert(!REALLOC || CTRL_REGS * 128 + SOFTMAX_REGS * 256 <= LAUNCH_REGS * THREADS,
                "register split exceeds the launch allocation");
  // ones-column row sums (FA_FWD_ONES_SUM): O_t gets EXTRA more columns, V a ones block
  static constexpr int EXTRA = (D == 64 && FA_FWD_ONES_SUM) ? 16 : 0;
  static constexpr int OCOLS = D + EXTRA;
  static constexpr int TMEM_S = 0;               // S_t at column t*BN (P_t aliases its first BN/2)
  static constexpr int TMEM_O = NQT * BN;        // O_t at TMEM_O + t*OCOLS
  static constexpr int TMEM_COLS = 512;
  static_assert(NQT * (BN + OCOLS) <= TMEM_COLS, "tensor memory budget");
  // One query tile: tensor memory has room for a second score buffer, so consecutive key tiles
  // alternate between S buffers (column 0 and TMEM_S1) and S(j+1) need not wait for PV(j).
  static constexpr bool DBUF = NQT == 1;
  static constexpr int TMEM_S1 = TMEM_O + OCOLS <= 256 ? 256 : 384;
  static_assert(!DBUF || TMEM_S1 + BN <= TMEM_COLS, "tensor memory budget (second S buffer)");
  static constexpr int NB = DBUF ? 2 : NQT;      // score / P / PV-done barrier slots
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQT * QTILE_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KVTILE_BYTES;
  static constexpr int OFF_ONES = OFF_V + VST * KVTILE_BYTES;  // [BN keys][64] bf16 ones
  // O written by TMA tensor stores from swizzled shared blocks of [128 rows][64 columns] (16 KB):
  // one per query tile at d = 64 (two tiles), two alternating at d = 256.  d = 128 stores its
  // rows directly: there the staging's warpgroup barriers cost more than the stores save (long
  // causal forward 1023 vs 1044 TFLOP/s), and the one-tile configurations of d = 64 / 128 have no
  // room for it.
  static constexpr bool TMA_EPI = (NQT == 2 && D == 64) || D == 256;
  static constexpr int STG_BLK = BM * 128;
  static constexpr int OFF_STG = OFF_ONES + (EXTRA ? BN * 128 : 0);
  static constexpr int OFF_BAR = OFF_STG + (TMA_EPI ? 2 * STG_BLK : 0);
  // barriers: q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST],
  //           s_full[NB], p_full[NB], o_done[NB], o_free[NQT], drain (slot = query tile, or
  //           with one query tile the S buffer)
  static constexpr int NBAR = 2 + 2 * KST + 2 * VST + 3 * NB + NQT + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem address + abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);   // Q, K both K-major
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, OCOLS, 0, 1);  // P (tmem), V MN-major
};

// The k-th unit of CTA c among G CTAs (zig-zag over rounds of G units), or -1 when none is left.
__device__ __forceinline__ int fwd_unit_of(int k, int c, int G, int units) {
  const int u = k * G + ((k & 1) ? (G - 1 - c) : c);
  return u < units ? u : -1;
}

// Unit u -> (head, its key/value head, split, first query row, first KV tile, KV tiles per
// query tile).  Units are numbered query block major (heaviest, i.e. latest, query blocks first
// when causal), then split, heads inner, so the query heads that share a key/value head run side
// by side and share its tiles in L2.  A split covers KV tiles [kt0, kt0 + kv_chunk); a query
// tile takes those of them that hold at least one key it may see.
template <int NQT, bool CAUSAL, bool GENERAL>
struct FwdUnit {
  int head, kv_head, split, q0, kt0, J;
  int nkv[NQT];
  __device__ __forceinline__ FwdUnit(int u, const FwdParams& p) {
    const int n_kv_total = (p.Nk + 127) / 128;
    if (GENERAL && p.pack > 1) {
      // packed query heads: unit = (range, K/V head); `head` is the group's first query head
      const int bhkv = p.BH / p.G;
      split = u / bhkv;
      kv_head = u - split * bhkv;
      head = (kv_head / p.Hkv) * p.H + (kv_head % p.Hkv) * p.G;
      q0 = 0;
      kt0 = split * p.kv_chunk;
      const int kt1 = min(n_kv_total, kt0 + p.kv_chunk);
      const int last = CAUSAL ? min(p.Nk - 1, p.Nq - 1 + p.off) : p.Nk - 1;
      nkv[0] = max(0, min(kt1, last / 128 + 1) - kt0);
#pragma unroll
      for (int t = 1; t < NQT; ++t) nkv[t] = 0;
      J = nkv[0];
      return;
    }
    // a split tail: work item u >= tail_base is query tile (u - tail_base) & 1 of unit
    // tail_base + (u - tail_base) / 2, run as a one-tile unit
    int half = -1;
    if (!CAUSAL && !GENERAL && NQT == 2 && u >= p.tail_base) {
      half = (u - p.tail_base) & 1;
      u = p.tail_base + ((u - p.tail_base) >> 1);
    }
    const int per_qb = p.BH * p.splits;
    const int qi = u / per_qb;
    const int rem = u - qi * per_qb;
    split = rem / p.BH;
    head = rem - split * p.BH;
    kv_head = (head / p.H) * (p.H / p.G) + (head % p.H) / p.G;
    const int qb = CAUSAL ? (p.nqb - 1 - qi) : qi;
    q0 = qb * NQT * 128;
    kt0 = split * p.kv_chunk;
    const int kt1 = min(n_kv_total, kt0 + p.kv_chunk);
    J = 0;
#pragma unroll
    for (int t = 0; t < NQT; ++t) {
      const int r0 = q0 + t * 128;
      int n = 0;
      if (r0 < p.Nq) {
        // last key any row of the tile may see, and the KV tile holding it
        const int last = CAUSAL ? min(p.Nk - 1, min(r0 + 127, p.Nq - 1) + p.off) : p.Nk - 1;
        n = max(0, min(kt1, last / 128 + 1) - kt0);
      }
      nkv[t] = n;
      J = max(J, n);
    }
    if (half >= 0) {
      // tile `half` of the unit, moved into tile slot 0; slot 1 stays empty
      q0 += half * 128;
      nkv[0] = nkv[half];
#pragma unroll
      for (int t = 1; t < NQT; ++t) nkv[t] = 0;
      J = nkv[0];
    }
  }
};

// SPLIT: the general variant -- partial outputs per key range and packed query heads (see
// FwdParams).  Only with ranges can a row meet one that holds no key it may see, so only this
// variant carries the empty-row guards; plain calls use the lean one.
template <int D, bool CAUSAL, int NQT, bool SPLIT>
__global__ void __launch_bounds__(FwdCfg<D, NQT>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D, NQT>;
  using Unit = FwdUnit<NQT, CAUSAL, SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  FA_TRACE_DECL;

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  const uint32_t BAR_Q = bar(0);
  const uint32_t BAR_QE = bar(1);
  auto BAR_KF = [&](int s) { return bar(2 + s); };
  constexpr int KV_BARS = 2 * C::KST + 2 * C::VST;
  auto BAR_KE = [&](int s) { return bar(2 + C::KST + s); };
  auto BAR_VF = [&](int s) { return bar(2 + 2 * C::KST + s); };
  auto BAR_VE = [&](int s) { return bar(2 + 2 * C::KST + C::VST + s); };
  auto BAR_SF = [&](int b) { return bar(2 + KV_BARS + b); };
  auto BAR_PF = [&](int b) { return bar(2 + KV_BARS + C::NB + b); };
  auto BAR_OD = [&](int b) { return bar(2 + KV_BARS + 2 * C::NB + b); };
  auto BAR_OF = [&](int t) { return bar(2 + KV_BARS + 3 * C::NB + t); };
  // With the double score buffer (one query tile), key tile g (counted over the CTA's whole run)
  // uses S buffer / barrier slot g & 1, and is the (g >> 1)-th use of that slot.
  auto sbuf_col = [&](int g) -> uint32_t { return (g & 1) ? C::TMEM_S1 : C::TMEM_S; };
  const uint32_t BAR_DRAIN = bar(C::NBAR - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  Waiter W{abort_flag, p.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    mbar_init(BAR_QE, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(BAR_KF(s), 1);
      mbar_init(BAR_KE(s), 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(BAR_VF(s), 1);
      mbar_init(BAR_VE(s), 1);
    }
    for (int b = 0; b < C::NB; ++b) {
      mbar_init(BAR_SF(b), 1);
      mbar_init(BAR_PF(b), 4);
      mbar_init(BAR_OD(b), 1);
    }
    for (int t = 0; t < NQT; ++t) mbar_init(BAR_OF(t), 4);
    mbar_init(BAR_DRAIN, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  if constexpr (C::EXTRA > 0) {
    // the ones block V is extended with (every bf16 of it 1.0, so its swizzle does not matter)
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    for (int i = threadIdx.x; i < C::BN * 128 / 4; i += C::THREADS) ones[i] = 0x3F803F80u;
    fence_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  FA_TRACE_EV(30, 0);

  if (warp >= C::SOFTMAX_WARPS) {
    // ================================================================ control warpgroup
    if constexpr (C::REALLOC) regs_dec<C::CTRL_REGS>();
    if (warp == C::PRODUCER_WARP) {
      // -------------------------------------------------------------- TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int kv_it = 0;   // KV tiles loaded so far (ring position)
        int kq = 0;      // units with work so far (the Q barriers' phase)
        int q_n = 0;     // Q loads issued, and K / V loads issued per ring stage: each issued load
        int k_n[C::KST], v_n[C::VST];  // is one phase of its full barrier (drain below)
#pragma unroll
        for (int s = 0; s < C::KST; ++s) k_n[s] = 0;
#pragma unroll
        for (int s = 0; s < C::VST; ++s) v_n[s] = 0;
        bool ok = true;
        for (int k = 0;; ++k) {
          const int u = fwd_unit_of(k, cta, G, p.units);
          if (u < 0) break;
          const Unit un(u, p);
          if (un.J == 0) continue;  // a key range none of its queries may see (split mode)
          // Q of this unit replaces the previous unit's once its last S MMA has completed
          if (kq > 0 && !(ok = W.wait(BAR_QE, (kq - 1) & 1, 3))) break;
          if (SPLIT && p.pack > 1) {
            // the group's G query heads as rows g * Nq + i of tile 0: one box of Nq x G rows
            mbar_arrive_expect_tx(BAR_Q, C::KB * p.pack * p.Nq * 128);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_Q + kb * (C::BM * 128), &tmQ, BAR_Q, kb * 64, 0, un.head);
            ++q_n;
          } else {
            int q_tiles = 0;
            for (int t = 0; t < NQT; ++t) q_tiles += (un.nkv[t] > 0);
            mbar_arrive_expect_tx(BAR_Q, q_tiles * C::QTILE_BYTES);
            for (int t = 0; t < NQT; ++t) {
              if (un.nkv[t] == 0) continue;
              for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(sbase + C::OFF_Q + t * C::QTILE_BYTES + kb * (C::BM * 128), &tmQ, BAR_Q,
                            kb * 64, un.q0 + t * C::BM, un.head);
            }
            ++q_n;
          }
          for (int j = 0; j < un.J; ++j) {
            const int g = kv_it + j;
            const int s = g % C::KST;
            const uint32_t ph = (g / C::KST) & 1;
            const int sv = g % C::VST;
            const uint32_t phv = (g / C::VST) & 1;
#ifdef FA_TEST_STARVE
            // Test build only (libfattn_starve.so): CTA 0 never issues the second K/V tile of its
            // first unit, so the MMA warp's bounded wait for it runs out and the kernel must
            // report FA_ERR_TIMEOUT and tear down cleanly.  Nothing is left in flight: the loads
            // issued so far are drained below like after any other abort.
            if (cta == 0 && k == 0 && j == 1) {
              ok = false;
              break;
            }
#endif
            if (!(ok = W.wait(BAR_KE(s), ph ^ 1, 1))) break;
            FA_TRACE_EV(20, j);
            mbar_arrive_expect_tx(BAR_KF(s), C::KVTILE_BYTES);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_K + s * C::KVTILE_BYTES + kb * (C::BN * 128), &tmK,
                          BAR_KF(s), kb * 64, (un.kt0 + j) * C::BN, un.kv_head);
            ++k_n[s];
            if (!(ok = W.wait(BAR_VE(sv), phv ^ 1, 2))) break;
            FA_TRACE_EV(21, j);
            mbar_arrive_expect_tx(BAR_VF(sv), C::KVTILE_BYTES);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_V + sv * C::KVTILE_BYTES + kb * (C::BN * 128), &tmV,
                          BAR_VF(sv), kb * 64, (un.kt0 + j) * C::BN, un.kv_head);
            ++v_n[sv];
          }
          if (!ok) break;
          kv_it += un.J;
          ++kq;
        }
        if (!ok) {
          // drain (bounded): every load issued so far lands before the CTA exits.  A barrier has
          // at most its last phase outstanding (a load is issued only after the previous one on
          // the same buffer was consumed), so waiting for the phase of its last issued load is
          // enough; a barrier with no load issued is skipped.
          if (q_n > 0) W.drain(BAR_Q, (q_n - 1) & 1);
#pragma unroll
          for (int s = 0; s < C::KST; ++s)
            if (k_n[s] > 0) W.drain(BAR_KF(s), (k_n[s] - 1) & 1);
#pragma unroll
          for (int s = 0; s < C::VST; ++s)
            if (v_n[s] > 0) W.drain(BAR_VF(s), (v_n[s] - 1) & 1);
        }
      }
    } else if (warp == C::MMA_WARP && C::DBUF) {
      // -------------------------------------------------------------- MMA issuer, one query tile
      // Key tile g's scores go to S buffer g & 1, so S(g+1) only has to wait for PV(g-1), which
      // read the P that buffer held.  S(g+1) is issued ahead of PV(g) whenever K(g+1) has landed
      // (and PV(g-1) is done), so the next tile's scores are ready when the softmax warpgroup
      // turns to them; otherwise it follows PV(g).
      if (lane == 0) {
        auto issue_s = [&](int g, uint32_t k_addr) {
          const uint32_t q_addr = sbase + C::OFF_Q;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            mma_ss(tmem + sbuf_col(g), sdesc_sw128(q_addr + koff, 16, 1024),
                   sdesc_sw128(k_addr + koff, 16, 1024), C::IDESC_S, kk > 0);
          }
          tc_commit(BAR_SF(g & 1));
        };
        // S buffer g & 1 is free once PV(g - 2) has completed (it read the P held there)
        // (with FA_FWD_INORDER, S(g) simply follows PV(g - 2) in issue order; packed decoding
        // keeps the wait, measured 1% faster there)
        const bool inorder = FA_FWD_INORDER && !(SPLIT && p.pack > 1);
        auto sbuf_free = [&](int g, int site) -> bool {
          return inorder || g < 2 || W.wait(BAR_OD(g & 1), ((g - 2) >> 1) & 1, site);
        };
        int g = 0, kv_it = 0, kq = 0, nun = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int u = fwd_unit_of(k, cta, G, p.units);
          if (u < 0) break;
          const Unit un(u, p);
          const int J = un.J;
          if (J == 0) continue;
          const int s0 = kv_it % C::KST;
          if (!(ok = W.wait(BAR_Q, kq & 1, 10))) break;
          if (!(ok = W.wait(BAR_KF(s0), (kv_it / C::KST) & 1, 11))) break;
          if (!(ok = sbuf_free(g, 12))) break;
          tc_fence_after();
          issue_s(g, sbase + C::OFF_K + s0 * C::KVTILE_BYTES);
          tc_commit(BAR_KE(s0));
          if (J == 1) tc_commit(BAR_QE);
          for (int j = 0; ok && j < J; ++j) {
            const int gg = g + j;
            const int s = (kv_it + j) % C::VST;  // V stage of key tile j
            const int s1 = (kv_it + j + 1) % C::KST;
            const uint32_t kph1 = ((kv_it + j + 1) / C::KST) & 1;
            bool s_next = j + 1 < J;
            if (s_next && mbar_test_wait(BAR_KF(s1), kph1) &&
                (inorder || gg + 1 < 2 ||
                 mbar_test_wait(BAR_OD((gg + 1) & 1), ((gg - 1) >> 1) & 1))) {
              tc_fence_after();
              issue_s(gg + 1, sbase + C::OFF_K + s1 * C::KVTILE_BYTES);
              tc_commit(BAR_KE(s1));
              if (j + 2 == J) tc_commit(BAR_QE);  // every S of this unit is issued
              s_next = false;
            }
            if (!(ok = W.wait(BAR_VF(s), ((kv_it + j) / C::VST) & 1, 13))) break;
            if (!(ok = W.wait(BAR_PF(gg & 1), (gg >> 1) & 1, 14))) break;
            // the first PV of a unit overwrites O: the previous epilogue must have read it
            if (j == 0 && nun > 0 && !(ok = W.wait(BAR_OF(0), (nun - 1) & 1, 15))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk) {
              mma_ts(tmem + C::TMEM_O, tmem + sbuf_col(gg) + kk * 8,
                     sdesc_sw128(sbase + C::OFF_V + s * C::KVTILE_BYTES + kk * 2048,
                                 C::EXTRA ? uint32_t(C::OFF_ONES - C::OFF_V - s * C::KVTILE_BYTES)
                                          : uint32_t(C::BN * 128),
                                 1024),
                     C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(BAR_OD(gg & 1));
            tc_commit(BAR_VE(s));
            if (s_next) {
              if (!(ok = W.wait(BAR_KF(s1), kph1, 16))) break;
              if (!(ok = sbuf_free(gg + 1, 17))) break;
              tc_fence_after();
              issue_s(gg + 1, sbase + C::OFF_K + s1 * C::KVTILE_BYTES);
              tc_commit(BAR_KE(s1));
              if (j + 2 == J) tc_commit(BAR_QE);
            }
          }
          if (!ok) break;
          g += J;
          kv_it += J;
          ++kq;
          ++nun;
        }
        // every MMA issued above has completed before the tensor memory is released
        tc_commit(BAR_DRAIN);
        W.drain(BAR_DRAIN, 0);
      }
    } else if (warp == C::MMA_WARP) {
      // -------------------------------------------------------------- MMA issuer
      W.sleep = !(FA_FWD_MMA_POLL == 1 || (FA_FWD_MMA_POLL < 0 && D == 128));
      // Order per KV tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).  S_t(j+1) overwrites the
      // tensor memory that holds P_t(j); it follows PV_t(j) in issue order (FA_FWD_INORDER, else
      // it waits for PV_t(j) to complete), so softmax t starts on tile j+1 while the other query
      // tile's PV runs.
      if (lane == 0) {
        auto issue_s = [&](int t, uint32_t k_addr) {
          const uint32_t q_addr = sbase + C::OFF_Q + t * C::QTILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            mma_ss(tmem + C::TMEM_S + t * C::BN, sdesc_sw128(q_addr + koff, 16, 1024),
                   sdesc_sw128(k_addr + koff, 16, 1024), C::IDESC_S, kk > 0);
          }
          tc_commit(BAR_SF(t));
        };
        int kv_it = 0;
        int tit[NQT], tun[NQT];  // per tile: KV iterations and units processed so far
#pragma unroll
        for (int t = 0; t < NQT; ++t) tit[t] = tun[t] = 0;
        bool ok = true;
        int kq = 0;  // units with work so far (the Q barriers' phase)
        for (int k = 0; ok; ++k) {
          const int u = fwd_unit_of(k, cta, G, p.units);
          if (u < 0) break;
          const Unit un(u, p);
          const int J = un.J;
          if (J == 0) continue;  // skipped by the producer too
          const int s0 = kv_it % C::KST;
          if (!(ok = W.wait(BAR_Q, kq & 1, 10))) break;
          if (!(ok = W.wait(BAR_KF(s0), (kv_it / C::KST) & 1, 11))) break;
          for (int t = 0; t < NQT && ok; ++t) {
            if (un.nkv[t] == 0) continue;
            // S_t's columns hold P_t of the previous unit's last tile until its PV completed
            if (!FA_FWD_INORDER && tit[t] > 0 && !(ok = W.wait(BAR_OD(t), (tit[t] - 1) & 1, 12)))
              break;
            tc_fence_after();
            issue_s(t, sbase + C::OFF_K + s0 * C::KVTILE_BYTES);
          }
          if (!ok) break;
          tc_commit(BAR_KE(s0));
          if (J == 1) tc_commit(BAR_QE);  // every S of this unit is issued: Q may be replaced
          for (int j = 0; ok && j < J; ++j) {
            const int g = kv_it + j;
            const int s = g % C::VST;         // V stage of key tile j
            const int s1 = (g + 1) % C::KST;  // K stage of key tile j + 1
            const uint32_t v_addr = sbase + C::OFF_V + s * C::KVTILE_BYTES;
            const uint32_t k1_addr = sbase + C::OFF_K + s1 * C::KVTILE_BYTES;
            FA_TRACE_EV(8, j);
            if (!(ok = W.wait(BAR_VF(s), (g / C::VST) & 1, 13))) break;
            FA_TRACE_EV(9, j);
            bool k_ready = false;
            for (int t = 0; t < NQT && ok; ++t) {
              if (j >= un.nkv[t]) continue;
              FA_TRACE_EV(1 + 16 * t, j);
              if (!(ok = W.wait(BAR_PF(t), tit[t] & 1, 14))) break;
              // the first PV of a unit overwrites O_t: the previous epilogue must have read it
              if (j == 0 && tun[t] > 0 && !(ok = W.wait(BAR_OF(t), (tun[t] - 1) & 1, 15))) break;
              FA_TRACE_EV(2 + 16 * t, j);
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < C::BN / 16; ++kk) {
                // P~ is packed bf16: 16 keys = 8 columns; V rows (keys) are 128 B apart, so a
                // 16-key slice is 2048 B further on; 64-wide d blocks are BN*128 B apart.
                // with EXTRA, the second 64-wide N block of B is the ones tile, LBO bytes on
                mma_ts(tmem + C::TMEM_O + t * C::OCOLS, tmem + C::TMEM_S + t * C::BN + kk * 8,
                       sdesc_sw128(v_addr + kk * 2048,
                                   C::EXTRA ? uint32_t(C::OFF_ONES - C::OFF_V - s * C::KVTILE_BYTES)
                                            : uint32_t(C::BN * 128),
                                   1024),
                       C::IDESC_PV,
                       (j > 0 || kk > 0) ? 1u : 0u);
              }
              tc_commit(BAR_OD(t));
              FA_TRACE_EV(4 + 16 * t, j);
              if (j + 1 < un.nkv[t]) {
                if (!k_ready &&
                    !(ok = W.wait(BAR_KF(s1), ((g + 1) / C::KST) & 1, 16)))
                  break;
                k_ready = true;
                if (!FA_FWD_INORDER && !(ok = W.wait(BAR_OD(t), tit[t] & 1, 17)))
                  break;  // P_t(j) consumed
                FA_TRACE_EV(3 + 16 * t, j);
                tc_fence_after();
                issue_s(t, k1_addr);
                FA_TRACE_EV(5 + 16 * t, j);
              }
              ++tit[t];
            }
            if (!ok) break;
            tc_commit(BAR_VE(s));
            if (k_ready) tc_commit(BAR_KE(s1));
            // S MMAs of the last KV tile are issued during tile J-2: Q may then be replaced
            if (j == J - 2) tc_commit(BAR_QE);
          }
          if (!ok) break;
#pragma unroll
          for (int t = 0; t < NQT; ++t) tun[t] += (un.nkv[t] > 0);
          kv_it += J;
          ++kq;
        }
        // every MMA issued above has completed before the tensor memory is released
        tc_commit(BAR_DRAIN);
        W.drain(BAR_DRAIN, 0);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    if constexpr (C::REALLOC) regs_inc<C::SOFTMAX_REGS>();
    const int t = warp >> 2;                  // query tile of this warpgroup
    const int r = threadIdx.x & 127;          // row within the tile == TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    // key tile gi's score buffer and barrier slot / phase (see sbuf_col)
    auto tS_of = [&](int gi) -> uint32_t {
      return tmem + lane_base + (C::DBUF ? sbuf_col(gi) : uint32_t(C::TMEM_S + t * C::BN));
    };
    auto slot = [&](int gi) { return C::DBUF ? (gi & 1) : t; };
    auto sph = [&](int gi) -> uint32_t { return C::DBUF ? uint32_t((gi >> 1) & 1) : uint32_t(gi & 1); };
    const uint32_t tO = tmem + lane_base + C::TMEM_O + t * C::OCOLS;
    // m: reference max (log2 units of the scaled scores) that the exponentials and l are taken
    // against.  It only moves when a row's max grows by more than kRescale (2^8 in value): the
    // result is the same exact softmax, P~ stays <= 256, and O is rescaled far less often.
    constexpr float kRescale = FA_FWD_RESCALE;
    int tit = 0;  // KV iterations of this tile so far (barrier phases continue across units)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = fwd_unit_of(k, cta, G, p.units);
      if (u < 0) break;
      const Unit un(u, p);
      const int n = un.nkv[t];
      // this thread's query: index `row` of head `qh` (packed: tile row g * Nq + i)
      const bool packed = SPLIT && p.pack > 1;
      const int row = packed ? r % p.Nq : un.q0 + t * C::BM + r;
      const int qh = packed ? un.head + r / p.Nq : un.head;
      const bool valid = packed ? (t == 0 && r < p.pack * p.Nq) : row < p.Nq;
      if (n == 0) {
        // split mode: this tile's queries see none of the range's keys; its partials weigh 0
        if (SPLIT && valid && p.lse_part != nullptr)
          p.lse_part[(size_t(un.split) * p.BH + qh) * p.Nq + row] = -INFINITY;
        continue;
      }
      float m = -INFINITY;
      float l = 0.f;   // sum of the fp32 exponentials (for L)
      float lr = 0.f;  // sum of the bf16-rounded exponentials (divides O)
      if (SPLIT && packed && p.pack * p.Nq <= 16) {
        // ---- decoding: at most 16 valid rows, all in lanes 0-15 of the first warp.  Each row is
        // spread over four threads (the 16-lane TMEM shapes), so a row's exponentials take a
        // quarter of the time they would on one thread; the other three warps only keep the
        // barrier phases in step.  Row statistics live in the four threads of the row and are
        // combined with two shuffles; at the end they move to thread = row for the epilogue.
        const bool worker = (warp & 3) == 0;
        const bool two_sets = p.pack * p.Nq > 8;  // rows 8-15 in use (second register set)
        const int g4 = lane >> 2, c2 = 2 * (lane & 3);
        float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f, rA = 0.f, rB = 0.f;
        for (int j = 0; j < n; ++j, ++tit) {
          if (!(ok = W.wait_warp(BAR_SF(slot(tit)), sph(tit), 20))) break;
          tc_fence_after();
          float alphaA = 1.f, alphaB = 1.f;
          if (worker) {
            uint32_t sv[64];
            tmem_ld16x256b_x16(tS_of(tit), sv);
            tmem_wait_ld64(sv);
            const int key0 = (un.kt0 + j) * C::BN;
            uint32_t wd[32];
#pragma unroll
            for (int set = 0; set < 2; ++set) {
              if (set == 1 && !two_sets) {
#pragma unroll
                for (int k = 0; k < 16; ++k) wd[2 * k + 1] = 0u;
                break;
              }
              const int lrow = g4 + 8 * set;  // tile row == lane
              const int qi = lrow % p.Nq;
              const int lim = CAUSAL ? min(qi + p.off, p.Nk - 1) - key0 : (p.Nk - 1) - key0;
              float mx = -INFINITY;
#pragma unroll
              for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  if (8 * k + c2 + e > lim) sv[4 * k + 2 * set + e] = __float_as_uint(-INFINITY);
                  mx = fmaxf(mx, __uint_as_float(sv[4 * k + 2 * set + e]));
                }
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
              float& mr = set ? mB : mA;
              const float m_tile = mx * p.scale_log2;
              const float m_use = (j == 0 || m_tile > mr + kRescale) ? fmaxf(mr, m_tile) : mr;
              const float alpha = (j == 0 || m_use == mr) ? 1.f : ex2(mr - m_use);
              const float m_ref = m_use == -INFINITY ? 0.f : m_use;
              const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2);
              const uint64_t nm2 = f2pack(-m_ref, -m_ref);
              uint64_t sx = 0ull;
              float s0 = 0.f, s1 = 0.f;
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                float x0, x1;
                f2unpack(ffma2(f2pack(__uint_as_float(sv[4 * k + 2 * set]),
                                      __uint_as_float(sv[4 * k + 2 * set + 1])),
                               sc2, nm2),
                         x0, x1);
                const float p0 = ex2(x0), p1 = ex2(x1);
                const uint32_t pk = pack_bf16(p0, p1);
                wd[2 * k + set] = pk;
                sx = fadd2(sx, f2pack(p0, p1));
                if (C::EXTRA == 0) add_bf16pair_f32(pk, s0, s1);
              }
              float a0, a1;
              f2unpack(sx, a0, a1);
              float ls = a0 + a1, rs = s0 + s1;
              ls += __shfl_xor_sync(0xffffffffu, ls, 1);
              ls += __shfl_xor_sync(0xffffffffu, ls, 2);
              rs += __shfl_xor_sync(0xffffffffu, rs, 1);
              rs += __shfl_xor_sync(0xffffffffu, rs, 2);
              if (set == 0) {
                lA = lA * alpha + ls;
                rA = rA * alpha + rs;
                alphaA = alpha;
              } else {
                lB = lB * alpha + ls;
                rB = rB * alpha + rs;
                alphaB = alpha;
              }
              mr = m_use;
            }
            // P~ (bf16 pairs) over the first 64 columns of S_t, rows 0-15
            tmem_st16x128b_x16(tS_of(tit), wd);
            // the row factors to thread = row for the 32x32b rescale of O
            const float aA = __shfl_sync(0xffffffffu, alphaA, 4 * (lane & 7));
            const float aB = __shfl_sync(0xffffffffu, alphaB, 4 * (lane & 7));
            const float alpha = lane < 8 ? aA : (lane < 16 ? aB : 1.f);
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
              if (!(ok = W.wait_warp(BAR_OD(slot(tit - 1)), sph(tit - 1), 21))) {
                tmem_wait_st();
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld(o);
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st32(tO + 32 * c, o);
              }
              if constexpr (C::EXTRA > 0) {
                uint32_t o[16];
                tmem_ld16(tO + D, o);
                tmem_wait_ld16(o);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st16(tO + D, o);
              }
            }
            tmem_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR_PF(slot(tit)));
        }
        if (!ok) break;
        // row statistics to thread = row (lanes 0-15 of the first warp) for the epilogue
        const float vmA = __shfl_sync(0xffffffffu, mA, 4 * (lane & 7));
        const float vmB = __shfl_sync(0xffffffffu, mB, 4 * (lane & 7));
        const float vlA = __shfl_sync(0xffffffffu, lA, 4 * (lane & 7));
        const float vlB = __shfl_sync(0xffffffffu, lB, 4 * (lane & 7));
        const float vrA = __shfl_sync(0xffffffffu, rA, 4 * (lane & 7));
        const float vrB = __shfl_sync(0xffffffffu, rB, 4 * (lane & 7));
        m = lane < 8 ? vmA : vmB;
        l = lane < 8 ? vlA : vlB;
        lr = lane < 8 ? vrA : vrB;
      } else
      for (int j = 0; j < n; ++j, ++tit) {
        FA_TRACE_EV(10, j);
        if (!(ok = W.wait_warp(BAR_SF(slot(tit)), sph(tit), 20))) break;
        FA_TRACE_EV(11, j);
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS_of(tit) + 32 * c, s[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld(s[c]);
        FA_TRACE_EV(15, j);
        // mask keys past Nk and, on diagonal tiles, keys after the query's position (causal)
        const int key0 = (un.kt0 + j) * C::BN;
        const int lim = CAUSAL ? min(row + p.off, p.Nk - 1) - key0 : (p.Nk - 1) - key0;
        if (lim < C::BN - 1) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * c + e > lim) s[c][e] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#if FA_FWD_MAX3
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mx8[(e >> 1) & 7] = fmax3(mx8[(e >> 1) & 7], __uint_as_float(s[c][e]),
                                      __uint_as_float(s[c][e + 1]));
#else
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(s[c][e]));
#endif
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        FA_TRACE_EV(16, j);
        const float m_tile = mx * p.scale_log2;
        const float m_use = (j == 0 || m_tile > m + kRescale) ? fmaxf(m, m_tile) : m;
        const float alpha = (j == 0 || m_use == m) ? 1.f : ex2(m - m_use);
        // a row that has seen no key yet (possible only when a split starts past its last
        // visible key) keeps m = -inf; its exponentials are taken against 0 and come out 0
        const float m_ref = (SPLIT && m_use == -INFINITY) ? 0.f : m_use;
        // exact fp32 sum (for L) and the sum of the bf16-rounded weights the PV MMA uses (for
        // O's normalisation: numerator and denominator then agree, so a row dominated by one
        // key reproduces that key's V), both accumulated in paired fp32
        uint64_t sum_x[2] = {0ull, 0ull}, sum_r[2] = {0ull, 0ull};
        const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2pack(-m_ref, -m_ref);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1, p0, p1;
            f2unpack(ffma2(f2pack(__uint_as_float(s[c][2 * e]), __uint_as_float(s[c][2 * e + 1])),
                           sc2, nm2),
                     x0, x1);
            constexpr int kPoly =
                FA_FWD_POLY_MASK >= 0 ? FA_FWD_POLY_MASK : (D == 64 ? 0x11 : 0x00);
            if ((kPoly >> (e >> 1)) & 1) {
              exp2_fma2(x0, x1, p0, p1);
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            pk[e] = pack_bf16(p0, p1);
            sum_x[e & 1] = fadd2(sum_x[e & 1], f2pack(p0, p1));
#if FA_FWD_RSUM == 1
            if (C::EXTRA == 0)
              sum_r[e & 1] = fadd2(sum_r[e & 1], f2pack(__uint_as_float(pk[e] << 16),
                                                       __uint_as_float(pk[e] & 0xffff0000u)));
#elif FA_FWD_RSUM == 2
            if (C::EXTRA == 0) {
              float r0, r1;
              f2unpack(sum_r[e & 1], r0, r1);
              add_bf16pair_f32(pk[e], r0, r1);
              sum_r[e & 1] = f2pack(r0, r1);
            }
#endif
          }
          // 32 keys -> 16 packed columns; two chunks share one 32-column store
          if (c & 1) {
#pragma unroll
            for (int e = 0; e < 16; ++e) s[c - 1][16 + e] = pk[e];
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) s[c][e] = pk[e];
          }
        }
        FA_TRACE_EV(12, j);
        // P~ (bf16) over the first 64 columns of S_t
        tmem_st32(tS_of(tit) + 0, s[0]);
        tmem_st32(tS_of(tit) + 32, s[2]);
        {
          float a0, a1, b0, b1;
          f2unpack(fadd2(sum_x[0], sum_x[1]), a0, a1);
          f2unpack(fadd2(sum_r[0], sum_r[1]), b0, b1);
          l = l * alpha + (a0 + a1);
          if (C::EXTRA == 0) lr = (FA_FWD_RSUM == 0) ? l : lr * alpha + (b0 + b1);
        }
        m = m_use;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          FA_TRACE_EV(14, j);
          // O_t holds PV_t(j-1) (S_t(j) was issued only after it completed); rescale it
          if (!(ok = W.wait_warp(BAR_OD(slot(tit - 1)), sph(tit - 1), 21))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + 32 * c, o);
          }
          if constexpr (C::EXTRA > 0) {  // the row sums of the rounded weights, with O
            uint32_t o[16];
            tmem_ld16(tO + D, o);
            tmem_wait_ld16(o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tO + D, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR_PF(slot(tit)));
        FA_TRACE_EV(13, j);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> global; L = (m + log2 l) * ln 2.  O_t is released to the
      // next unit's first PV once its last chunk has been read.
      if (!(ok = W.wait_warp(BAR_OD(slot(tit - 1)), sph(tit - 1), 22))) break;
      tc_fence_after();
      // a row with no visible key in this split (split mode only) gets O = 0 and L = -inf
      if constexpr (C::EXTRA > 0) {  // the MMA's row sum of the rounded weights
        uint32_t o[16];
        tmem_ld16(tO + D, o);
        tmem_wait_ld16(o);
        lr = __uint_as_float(o[0]);
      }
      const float inv_l = (!SPLIT || lr > 0.f) ? 1.f / lr : 0.f;
      if constexpr (!SPLIT && C::TMA_EPI) {
        // O / l as bf16 into this warpgroup's staging block(s), one 64-column block at a time,
        // each written by a TMA tensor store in whole rows (rows past Nq are clipped)
        constexpr int NBUF = NQT == 2 ? 1 : 2;
        uint8_t* stg = smem + C::OFF_STG + (NQT == 2 ? t * C::STG_BLK : 0);
        const bool issuer = (warp & 3) == 0 && lane == 0;
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          uint8_t* buf = stg + (kb % NBUF) * C::STG_BLK;
          // the previous store out of this block (this unit's or the last unit's) has read it
          if (issuer) {
            if (NBUF == 1) bulk_wait_group_read<0>();
            else bulk_wait_group_read<1>();
          }
          named_bar_sync(1 + t, 128);
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int c = 2 * kb + c2;
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld(o);
            if (c == D / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(BAR_OF(t));
            }
            stage_chunk_sw128(o, inv_l, buf, r, c2);
          }
          fence_async_smem();
          named_bar_sync(1 + t, 128);
          if (issuer) {
            tma_store_3d(&tmO, smem_u32(buf), kb * 64, un.q0 + t * C::BM, un.head);
            bulk_commit_group();
          }
        }
        if (valid) p.lse[size_t(qh) * p.Nq + row] = (m + lg2(l)) * 0.69314718055994531f;
        continue;
      }
      const bool part = SPLIT && p.o_part != nullptr;
      const size_t prow = (size_t(un.split) * p.BH + qh) * p.Nq + row;
      __nv_bfloat16* orow = p.o + (size_t(qh) * p.Nq + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld(o);
        if (c == D / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR_OF(t));
        }
        if (part) {
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l,
                                   __uint_as_float(o[4 * e + 1]) * inv_l,
                                   __uint_as_float(o[4 * e + 2]) * inv_l,
                                   __uint_as_float(o[4 * e + 3]) * inv_l);
          }
          continue;
        }
        uint4 pk[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pw[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = pk[e];
        }
      }
      if (valid) {
        const float L = (!SPLIT || l > 0.f) ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
        if (part)
          p.lse_part[prow] = L;
        else
          p.lse[size_t(qh) * p.Nq + row] = L;
      }
    }
    // the last O stores have read their staging blocks before the CTA's memory goes away
    if constexpr (!SPLIT && C::TMA_EPI)
      if ((warp & 3) == 0 && lane == 0) bulk_wait_group_all();
    tc_fence_before();
  }

  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
