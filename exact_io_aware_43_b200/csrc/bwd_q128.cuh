// bwd_q128.cuh -- attention backward main kernel for d = 64 and 128 with 128-query steps (sm_100a).
//
// Same mathematics as fa_bwd_kernel (robocikowo.com "Flash Attention": the backward recomputes
// P from the saved L; the gradient formulas are those of the definition), with a different
// tiling: each step takes 128 queries instead of 64, so every one of the five GEMMs of a step is
// a 128 x 128 x 128 tcgen05.mma group.  At N = 64 the tensor core's operand fetch from shared
// memory (6 KB per 16-deep instruction) is what limits it; at N = 128 the K_j / V_j operand is
// read once per 128 queries, which cuts shared-memory bytes per FLOP by a quarter.
//
// Tensor memory (512 columns) holds, per step:
//   R1 [0,128)    S^T = K_j Q_i^T (fp32).  Each query half h (64 columns, one warpgroup) then
//                 overwrites its own columns with P^T in bf16 at [96h, 96h+32).
//   R2 [128,256)  dP^T = V_j dO_i^T (fp32); once the dS^T warps have read it, dQ_i^T =
//                 K_j^T dS^T (fp32, d on lanes, 128 query columns).
//   [256,384) dV accumulator, [384,512) dK accumulator.
// The row statistics enter through the tensor core instead of shared-memory loads: each S^T
// and dP^T group gets a ninth K = 16 step whose A operand is a constant ones block and whose B
// operand holds, per query, -L/s and -D split into three bf16 terms each (hi + mid + lo, about 24
// bits; written by the preprocess kernel in the MMA's core-matrix layout).  The MMA then leaves
// S^T - L/s and dP^T - D in tensor memory, so P^T = exp2((S^T - L/s) s log2e) and
// dS^T = P^T (dP^T - D) need no per-query value from shared memory (the broadcast loads of L and
// D cost as many shared-memory wavefronts as the MMA operands of a GEMM).
// dS^T (bf16) goes to a shared tile, from which both dQ^T and dK (dS^T Q_i, both operands in
// shared memory) read it.  Tensor memory that other warps read is reused only after their
// completion barrier: dP^T(i+1) is issued once dQ^T(i) has been read out.  S^T(i+1), which
// overwrites the P^T(i) that this thread's own dV(i) reads, follows dV(i) in issue order
// (FA_BWDQ_INORDER; else it waits for dV(i) to complete).
// (Compile-time alternatives keep dS^T in tensor memory for dK -- dQ^T then waits for dK -- or
// stage dQ in the dS^T tile's space.)
//
// Warp roles (512 threads): warps 0-7 compute P^T and dS^T (warpgroup h owns query columns
// [64h, 64h+64); thread = key row = TMEM lane), warps 8-11 drain dQ^T (TMEM -> x scale ->
// shared staging -> TMA bulk reduce-add into the fp32 accumulator),
// warp 12 issues TMA loads, warp 13 allocates tensor memory and issues the MMAs.
#pragma once

#include "bwd.cuh"

// FA_BWDQ_EARLY_S: 1 issues S^T(i+1) right after dV(i) completes (before dK(i)); 0 issues it
// after dK(i), which leaves the tensor core no gap while the MMA thread waits for dV(i).
#ifndef FA_BWDQ_EARLY_S
#define FA_BWDQ_EARLY_S 1
#endif
// FA_BWDQ_DK_SS: 1 reads dS^T for dK from the shared tile (both operands in shared memory), so
// dQ^T may overwrite R2 as soon as dS^T is ready and is issued first; 0 reads dS^T from tensor
// memory, and dQ^T then waits for dK to complete.
#ifndef FA_BWDQ_DK_SS
#define FA_BWDQ_DK_SS 1
#endif
// FA_BWDQ_INORDER: 1 issues S^T(i+1) into R1 right behind dV(i), which reads P^T(i) there,
// without waiting for dV(i) to complete: the MMAs of one issuing thread run through the tensor
// core in issue order, so dV(i) has read its operand before S^T(i+1) writes.
#ifndef FA_BWDQ_INORDER
#define FA_BWDQ_INORDER 1
#endif
// FA_BWDQ_DQ_OWN: 1 gives dQ^T its own tensor-memory columns where they are free (d = 64: dV and
// dK take 64 columns each), so dP^T(i+1) need not wait for dQ^T(i) to be drained; dQ^T(i+1)
// waits for it instead.  Needs FA_BWDQ_DK_SS (dK reading dS^T from shared memory).  d = 64
// backward, TFLOP/s: 1x16x8192 causal 596 -> 630, 4x16x2048 causal 405 -> 426.
#ifndef FA_BWDQ_DQ_OWN
#define FA_BWDQ_DQ_OWN 1
#endif

// FA_BWDQ_PIPE_LD: 1 loads the second 32 columns of S^T / dP^T while the first 32 are worked on
// (one tcgen05.wait::ld covers all of a thread's loads, so the second load is issued after the
// first wait); 0 loads both, then waits.
#ifndef FA_BWDQ_PIPE_LD
#define FA_BWDQ_PIPE_LD 0
#endif
// FA_BWDQ_POLY_MASK: bit g set computes the exponentials of query columns [8g, 8g+8) of every 64
// on the FMA pipe (exp2_fma2) instead of the MUFU unit.
#ifndef FA_BWDQ_POLY_MASK
#define FA_BWDQ_POLY_MASK 0x00
#endif

namespace fattn {

template <int D_>
struct BwdQ128Cfg {
  static constexpr int D = D_;            // 64 or 128
  static constexpr int KB = D / 64;       // 128-byte swizzle blocks across d
  static constexpr int BC = 128;          // keys per CTA
  static constexpr int BR = 128;          // queries per step
  static constexpr int BLK = 128 * 128;   // one 64-column (128-byte-row) block of a 128-row tile
  static constexpr int TILE = KB * BLK;   // a 128-row x D bf16 tile (K_j, V_j, Q_i, dO_i)
  static constexpr int DS_TILE = 2 * BLK; // dS^T: [2 query halves][128 keys][64 queries] bf16
  // dQ^T has d on its rows: M = 128 puts row 32w + i in lane i of warp w's lane quarter; M = 64
  // puts rows 16w .. 16w + 15 in lanes 0 .. 15 of it (lanes 16 .. 31 hold nothing)
  static constexpr int DW = D == 128 ? 32 : 16;  // d rows per drain warp
  static constexpr int THREADS = 512;
  static constexpr int CMP_WARPS = 8;
  static constexpr int DQ_WARP0 = 8;
  static constexpr int PRODUCER_WARP = 12;
  static constexpr int MMA_WARP = 13;
  // register split over the four warpgroups (launch: 512 threads x 128 registers)
  static constexpr int LAUNCH_REGS = 128;
#ifndef FA_BWDQ_CMP_REGS
#define FA_BWDQ_CMP_REGS 136
#endif
#ifndef FA_BWDQ_DQ_REGS
#define FA_BWDQ_DQ_REGS 144
#endif
#ifndef FA_BWDQ_CTRL_REGS
#define FA_BWDQ_CTRL_REGS 96
#endif
  static constexpr int CMP_REGS = FA_BWDQ_CMP_REGS, DQ_REGS = FA_BWDQ_DQ_REGS,
                       CTRL_REGS = FA_BWDQ_CTRL_REGS;
  static_assert(2 * 128 * CMP_REGS + 128 * DQ_REGS + 128 * CTRL_REGS <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
  // tensor memory columns
  static constexpr bool DQ_OWN = FA_BWDQ_DQ_OWN && FA_BWDQ_DK_SS && D == 64;
  static constexpr int T_S = 0, T_DP = 128, T_DQ = DQ_OWN ? 384 : 128, T_DV = 256, T_DK = 256 + D;
  static constexpr int TMEM_COLS = 512;
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;        // 2 stages
  static constexpr int DO_STAGES = 1;
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;            // dO_i
  static constexpr int OFF_DS = OFF_DO + DO_STAGES * TILE;   // dS^T [2 q halves][128 keys][64 q]
  static constexpr int OFF_STG = OFF_DS + DS_TILE;           // dQ staging: 4 x [32 q][DW d] f32
  static constexpr int STG_BYTES = 4 * 32 * DW * 4;
  // row-statistics operands of the ninth K step (no swizzle: 8-row x 16-byte core matrices,
  // 8-row groups 128 B apart, the second 8 K-elements AUG_LBO bytes on):
  //   AUG [2 stages][2 K halves: -L/s terms | -D terms][16 query groups][8 rows][8 bf16]
  //   ONES [ones | zeros | ones], each [16 groups][8 rows][1, 1, 1, 0, 0, 0, 0, 0]: the S^T step
  //   reads (ones, zeros) and so picks the -L/s terms, the dP^T step (zeros, ones) the -D terms
  static constexpr int AUG_LBO = 2048;
  static constexpr int AUG_BYTES = 2 * AUG_LBO;              // per 128-query block
  static constexpr int OFF_AUG = OFF_STG + STG_BYTES;
  static constexpr int OFF_ONES = OFF_AUG + 2 * AUG_BYTES;
  // barriers: kv, q_full[2], q_empty[2], do_full[2], do_empty[2], s_full, p_full, dp_full,
  //           ds_full, dv_done, dk_done, dq_full, dq_empty, ds_free, drain, kv_empty
  static constexpr int NBAR = 20;
  static constexpr int OFF_BAR = OFF_ONES + 3 * AUG_LBO;
  static constexpr int OFF_MISC = OFF_BAR + 160;
  static constexpr int SMEM_NEED = OFF_MISC + 16;             // from a 1024-aligned base
  static constexpr int SMEM_MAX = 227 * 1024;                 // opt-in limit per CTA on sm_100
  // up to 1 KB of slack for aligning the base; the kernel checks what it actually got
  static constexpr int SMEM_BYTES = SMEM_NEED + 1024 < SMEM_MAX ? SMEM_NEED + 1024 : SMEM_MAX;
  static_assert(NBAR * 8 <= 160, "barrier area");
  static_assert(SMEM_NEED <= SMEM_MAX, "shared memory budget");
  static constexpr uint32_t IDESC_ST = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A in TMEM)
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(D, 128, 1, 1);    // dQ^T = K^T dS^T
};

// Descriptor of a no-swizzle K-major operand (layout code 0): core matrices of 8 rows x 16
// bytes, K-adjacent ones `lbo` bytes apart, 8-row groups `sbo` bytes apart.
__device__ __forceinline__ uint64_t sdesc_interleave(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// The k-th unit of CTA c among G CTAs: rounds of G units, every other round in reverse CTA order,
// so that the heaviest units (the first of each band) are spread over the CTAs; -1 when none is
// left.
__device__ __forceinline__ int bwdq_unit_of(int k, int c, int G, int units) {
  const int u = k * G + ((k & 1) ? (G - 1 - c) : c);
  return u < units ? u : -1;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(BwdQ128Cfg<D>::THREADS, 1)
    fa_bwd_kernel_q128(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ,
                       const __grid_constant__ CUtensorMap tmdK,
                       const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using C = BwdQ128Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need a 1024-byte-aligned base; with the largest layouts there is less
  // than 1 KB of slack, so a base that cannot be aligned within it is reported, not used
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + C::SMEM_NEED > C::SMEM_BYTES) {
    if (threadIdx.x == 0 && atomicCAS(&g_status[0], 0, 2 /* FA_ERR_UNSUPPORTED */) == 0)
      g_status[1] = 90;
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FA_TRACE_DECL;
  FA_TRACE_EV(90, 0);  // CTA start

  // ---- work units: (key block j, key/value head [, share of a group's query heads]) in the
  // order of BwdUnit; for each query head of the group (see BwdGroup), query blocks i from j
  // (causal) or 0 to the last.  With a grid of G < (unit count) CTAs each CTA takes units in
  // zig-zag rounds of G (see bwdq_unit_of) and every barrier's phases run on across them (global
  // step index T); with one CTA per unit the loops below run once.
  const int units = p.BHkv * p.nkb * p.gsplit;
  const int nqb = (p.N + C::BR - 1) / C::BR;
  const int G = int(gridDim.x), cta = int(blockIdx.x);

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  const uint32_t BAR_KV = bar(0);
  auto BAR_QF = [&](int s) { return bar(1 + s); };
  auto BAR_QE = [&](int s) { return bar(3 + s); };
  auto BAR_DOF = [&](int s) { return bar(5 + s); };
  auto BAR_DOE = [&](int s) { return bar(7 + s); };
  const uint32_t BAR_SF = bar(9), BAR_PF = bar(10), BAR_DPF = bar(11), BAR_DSF = bar(12),
                 BAR_DVD = bar(13), BAR_DKD = bar(14), BAR_DQF = bar(15), BAR_DQE = bar(16),
                 BAR_DSFREE = bar(17), BAR_DRAIN = bar(18), BAR_KVE = bar(19);
  constexpr int DS_ = C::DO_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  // plain try_wait polling (no suspend hint) measured faster here than sleeping waits
  const Waiter W{abort_flag, p.limit_ns, false};

  if (threadIdx.x == 0) {
    mbar_init(BAR_KV, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR_QF(s), 1);
      mbar_init(BAR_QE(s), 1);
      mbar_init(BAR_DOF(s), 1);
      mbar_init(BAR_DOE(s), 1);
    }
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_PF, C::CMP_WARPS);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_DSF, C::CMP_WARPS);
    mbar_init(BAR_DVD, 1);
    mbar_init(BAR_DKD, 1);
    mbar_init(BAR_DQF, 1);
    mbar_init(BAR_DQE, 4);
    mbar_init(BAR_DSFREE, 1);
    mbar_init(BAR_DRAIN, 1);
    mbar_init(BAR_KVE, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  {
    // the constant A operands of the ninth K step: [ones | zeros | ones], each 128 rows of
    // [1, 1, 1, 0, 0, 0, 0, 0] (bf16) or of zeros, as 16-byte core-matrix rows
    uint4* ones = reinterpret_cast<uint4*>(smem + C::OFF_ONES);
    for (int i = threadIdx.x; i < 3 * C::AUG_LBO / 16; i += C::THREADS)
      ones[i] = (i / (C::AUG_LBO / 16)) == 1 ? make_uint4(0u, 0u, 0u, 0u)
                                             : make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    fence_async_smem();
  }
  __syncthreads();
  FA_TRACE_EV(91, 0);  // set-up done
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= C::PRODUCER_WARP) {
    // ================================================================ control warpgroup
    regs_dec<C::CTRL_REGS>();
    if (warp == C::PRODUCER_WARP && lane == 0) {
      // -------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      int tq = 0, td = 0, tkv = 0;  // Q, dO, K/V tiles issued
      bool ok = true;
      int T = 0;  // global index of the unit's first step
      for (int kc = 0; ok; ++kc) {
        const int u = bwdq_unit_of(kc, cta, G, units);
        if (u < 0) break;
        const BwdUnit unit(u, p, 1);
        const int j = unit.j, kvh = unit.kvh, k0 = j * C::BC;
        const BwdGroup grp(p, kvh, unit.gs, CAUSAL ? j : 0, nqb);
        const int nit = grp.nheads * grp.nit_h;  // >= 1
        // Q_i / dO_i of the unit's steps in order; K_j, V_j once every MMA of the previous unit
        // has completed, issued after the first step's tiles so that these load while the
        // previous unit finishes
        auto load_kv = [&]() -> bool {
          if (!W.wait(BAR_KVE, (kc & 1) ^ 1, 30)) return false;
          mbar_arrive_expect_tx(BAR_KV, 2 * C::TILE);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_3d(sbase + C::OFF_K + kb * C::BLK, &tmK, BAR_KV, kb * 64, k0, kvh);
            tma_load_3d(sbase + C::OFF_V + kb * C::BLK, &tmV, BAR_KV, kb * 64, k0, kvh);
          }
          ++tkv;
          return true;
        };
        BwdCursor cur(grp);
        for (int tl = 0; tl < nit; ++tl) {
          const int t = T + tl;
          const int i = cur.i, head = cur.head;
          cur.next();
          const int s = t & 1;
          // Q_i and its row-statistics operand into stage s once dK of step t-2 has released it
          if (!(ok = W.wait(BAR_QE(s), ((t >> 1) & 1) ^ 1, 31))) break;
          mbar_arrive_expect_tx(BAR_QF(s), C::TILE + C::AUG_BYTES);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(sbase + C::OFF_Q + s * C::TILE + kb * C::BLK, &tmQ, BAR_QF(s), kb * 64,
                        i * C::BR, head);
          const size_t aoff = (size_t(head) * (p.Npad / C::BR) + size_t(i)) * C::AUG_BYTES;
          bulk_load(sbase + C::OFF_AUG + s * C::AUG_BYTES,
                    reinterpret_cast<const uint8_t*>(p.aug) + aoff, C::AUG_BYTES, BAR_QF(s));
          ++tq;
          FA_TRACE_EV(20, t);
          // dO_i into its buffer once dP^T and dV of the step that used it last have read it
          const int sd = t % DS_;
          if (!(ok = W.wait(BAR_DOE(sd), ((t / DS_) & 1) ^ 1, 32))) break;
          mbar_arrive_expect_tx(BAR_DOF(sd), C::TILE);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(sbase + C::OFF_DO + sd * C::TILE + kb * C::BLK, &tmdO, BAR_DOF(sd),
                        kb * 64, i * C::BR, head);
          ++td;
          if (tl == 0 && !(ok = load_kv())) break;
        }
        T += nit;
      }
      if (W.aborted()) {
        // let the copies already issued land before the CTA's shared memory goes away
        if (tkv > 0) W.drain(BAR_KV, (tkv - 1) & 1);
        for (int jj = tq > 2 ? tq - 2 : 0; jj < tq; ++jj) W.drain(BAR_QF(jj & 1), (jj >> 1) & 1);
        for (int jj = td > DS_ ? td - DS_ : 0; jj < td; ++jj)
          W.drain(BAR_DOF(jj % DS_), (jj / DS_) & 1);
      }
    } else if (warp == C::MMA_WARP && lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      const uint32_t k_addr = sbase + C::OFF_K, v_addr = sbase + C::OFF_V;
      const uint32_t ds_addr = sbase + C::OFF_DS;
      auto q_addr = [&](int s) { return sbase + C::OFF_Q + s * C::TILE; };
      auto do_addr = [&](int t) { return sbase + C::OFF_DO + (t % DS_) * C::TILE; };
      // [S^T | dP^T] (128 keys x 128 queries) = A (keys x d) * B (queries x d)^T, both K-major,
      // then the ninth step adds -L/s (ones at K 0-2 of the A block) or -D (ones at K 8-10) of
      // each query from the stage's statistics operand
      auto issue_st = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base, uint32_t ones_addr,
                          uint32_t aug_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + d_col, sdesc_sw128(a_base + off, 16, 1024),
                 sdesc_sw128(b_base + off, 16, 1024), C::IDESC_ST, kk > 0 ? 1u : 0u);
        }
        mma_ss(tmem + d_col, sdesc_interleave(ones_addr, C::AUG_LBO, 128),
               sdesc_interleave(aug_addr, C::AUG_LBO, 128), C::IDESC_ST, 1u);
      };
      const uint32_t ones_s = sbase + C::OFF_ONES, ones_dp = ones_s + C::AUG_LBO;
      auto aug_addr = [&](int t) { return sbase + C::OFF_AUG + (t & 1) * C::AUG_BYTES; };
      // [dV | dK] (128 keys x 128 d) += A (TMEM, bf16 keys x queries: query half h packed at
      // columns 96h..96h+31) * B (queries x d, MN-major; the two 64-wide d blocks BLK apart)
      auto issue_kv = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + 96 * (kk >> 2) + (kk & 3) * 8,
                 sdesc_sw128(b_base + kk * 2048, C::BLK, 1024), C::IDESC_KV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // dK (128 keys x 128 d) += dS^T (keys x queries, K-major, shared) * Q_i (queries x d)
      auto issue_dk_ss = [&](uint32_t b_base, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + C::T_DK, sdesc_sw128(ds_addr + (kk >> 2) * C::BLK + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(b_base + kk * 2048, C::BLK, 1024), C::IDESC_KV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // dQ^T (128 d x 128 queries) = K^T (d x keys, MN-major) * dS^T (keys x queries, MN-major)
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + C::T_DQ, sdesc_sw128(k_addr + kk * 2048, C::BLK, 1024),
                 sdesc_sw128(ds_addr + kk * 2048, C::BLK, 1024), C::IDESC_DQ, kk > 0 ? 1u : 0u);
      };
      auto next_s = [&](int t) -> bool {  // S^T(t+1) into R1 once dV(t) has read P^T(t)
        if (!FA_BWDQ_INORDER && !W.wait(BAR_DVD, t & 1, 44)) return false;
        if (!W.wait(BAR_QF((t + 1) & 1), ((t + 1) >> 1) & 1, 45)) return false;
        FA_TRACE_EV(3, t);
        tc_fence_after();
        issue_st(C::T_S, k_addr, q_addr((t + 1) & 1), ones_s, aug_addr(t + 1));
        tc_commit(BAR_SF);
        return true;
      };
      bool ok = true;
      int T = 0;  // global index of the unit's first step
      for (int kc = 0; ok; ++kc) {
        const int u = bwdq_unit_of(kc, cta, G, units);
        if (u < 0) break;
        const BwdUnit unit(u, p, 1);
        const int j = unit.j;
        const BwdGroup grp(p, unit.kvh, unit.gs, CAUSAL ? j : 0, nqb);
        const int nit = grp.nheads * grp.nit_h;  // >= 1
        (void)j;
        if (!(ok = W.wait(BAR_KV, kc & 1, 40))) break;
        FA_TRACE_EV(92, T);  // K_j, V_j landed
        // the unit's first S^T into R1 once dV of the previous step has read P^T there, its dP^T
        // into R2 once the previous dQ^T has been drained from it
        if (!FA_BWDQ_INORDER && T > 0 && !(ok = W.wait(BAR_DVD, (T - 1) & 1, 38))) break;
        if (!C::DQ_OWN && T > 0 && !(ok = W.wait(BAR_DQE, (T - 1) & 1, 39))) break;
        if (!(ok = W.wait(BAR_QF(T & 1), (T >> 1) & 1, 41))) break;
        FA_TRACE_EV(93, T);  // first Q_i landed
        tc_fence_after();
        issue_st(C::T_S, k_addr, q_addr(T & 1), ones_s, aug_addr(T));
        tc_commit(BAR_SF);
        if (!(ok = W.wait(BAR_DOF(T % DS_), (T / DS_) & 1, 42))) break;
        tc_fence_after();
        issue_st(C::T_DP, v_addr, do_addr(T), ones_dp, aug_addr(T));
        tc_commit(BAR_DPF);
        for (int tl = 0; ok && tl < nit; ++tl) {
          const int t = T + tl;
          const int s = t & 1;
          const bool more = tl + 1 < nit;
          // dV += P^T dO_i
          FA_TRACE_EV(1, t);
          if (!(ok = W.wait(BAR_PF, t & 1, 43))) break;
          FA_TRACE_EV(2, t);
          tc_fence_after();
          issue_kv(C::T_DV, C::T_S, do_addr(t), tl > 0);
          if (!FA_BWDQ_INORDER) tc_commit(BAR_DVD);
          tc_commit(BAR_DOE(t % DS_));
          if (FA_BWDQ_EARLY_S && more && !(ok = next_s(t))) break;
          FA_TRACE_EV(4, t);
          if (!(ok = W.wait(BAR_DSF, t & 1, 46))) break;
          FA_TRACE_EV(5, t);
          tc_fence_after();
          if (FA_BWDQ_DK_SS) {
            // dQ_i^T = K_j^T dS^T into R2 (the dP^T columns, read by now), then dK += dS^T Q_i;
            // both take dS^T from the shared tile.  With its own columns, dQ^T(t) waits for the
            // previous one to be drained instead.
            if (C::DQ_OWN && t > 0 && !(ok = W.wait(BAR_DQE, (t - 1) & 1, 48))) break;
            if (C::DQ_OWN) tc_fence_after();
            issue_dq();
            tc_commit(BAR_DQF);
            issue_dk_ss(q_addr(s), tl > 0);
            tc_commit(BAR_DKD);
            tc_commit(BAR_QE(s));
            FA_TRACE_EV(6, t);
            if (!FA_BWDQ_EARLY_S && more && !(ok = next_s(t))) break;
          } else {
            // dK += dS^T Q_i (dS^T from tensor memory)
            issue_kv(C::T_DK, C::T_DP, q_addr(s), tl > 0);
            tc_commit(BAR_DKD);
            tc_commit(BAR_QE(s));
            if (!FA_BWDQ_EARLY_S && more && !(ok = next_s(t))) break;
            // dQ_i^T = K_j^T dS^T into R2 once dK has read dS^T
            if (!(ok = W.wait(BAR_DKD, t & 1, 47))) break;
            FA_TRACE_EV(6, t);
            tc_fence_after();
            issue_dq();
            tc_commit(BAR_DQF);
          }
          if (more) {
            // dP^T(t+1) into R2 once dQ^T(t) has been read out (its statistics operand came with
            // Q_{t+1}, which S^T(t+1) has already waited for)
            if (!C::DQ_OWN && !(ok = W.wait(BAR_DQE, t & 1, 48))) break;
            if (!(ok = W.wait(BAR_DOF((t + 1) % DS_), ((t + 1) / DS_) & 1, 49))) break;
            if (!FA_BWDQ_EARLY_S && !(ok = W.wait(BAR_QF((t + 1) & 1), ((t + 1) >> 1) & 1, 45)))
              break;
            FA_TRACE_EV(7, t);
            tc_fence_after();
            issue_st(C::T_DP, v_addr, do_addr(t + 1), ones_dp, aug_addr(t + 1));
            tc_commit(BAR_DPF);
          }
        }
        // K_j, V_j are read by nothing once this unit's MMAs have completed
        tc_commit(BAR_KVE);
        T += nit;
      }
      // every MMA issued above has completed before the tensor memory is released
      tc_commit(BAR_DRAIN);
      W.drain(BAR_DRAIN, 0);
    }
  } else if (warp < C::CMP_WARPS) {
    // ================================================================ P / dS warpgroups
    regs_inc<C::CMP_REGS>();
    const int h = warp >> 2;                // query half
    const int c0 = 64 * h;                  // first query column of this thread
    const int r = (warp & 3) * 32 + lane;   // key row within the block == TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    uint8_t* ds_row = smem + C::OFF_DS + h * C::BLK + r * 128;
    bool ok = true;
    int T = 0;  // global index of the unit's first step
    for (int kc = 0; ok; ++kc) {
    const int u = bwdq_unit_of(kc, cta, G, units);
    if (u < 0) break;
    const BwdUnit unit(u, p, 1);
    const int j = unit.j, kvh = unit.kvh, k0 = j * C::BC;
    const BwdGroup grp(p, kvh, unit.gs, CAUSAL ? j : 0, nqb);
    const int nit = grp.nheads * grp.nit_h;  // >= 1
    const int key = k0 + r;
    const bool key_ok = key < p.N;
    BwdCursor cur(grp);
    for (int tl = 0; tl < nit; ++tl) {
      const int t = T + tl;
      const int i = cur.i;
      cur.next();
      if (!(ok = W.wait_warp(BAR_SF, t & 1, 50))) break;
      FA_TRACE_EV(11, t);
      tc_fence_after();
      uint32_t sv[2][32];
      tmem_ld32(tmem + lane_base + C::T_S + c0, sv[0]);
      if (!FA_BWDQ_PIPE_LD) tmem_ld32(tmem + lane_base + C::T_S + c0 + 32, sv[1]);
      tmem_wait_ld(sv[0]);
      if (FA_BWDQ_PIPE_LD) tmem_ld32(tmem + lane_base + C::T_S + c0 + 32, sv[1]);
      else tmem_wait_ld(sv[1]);
      FA_TRACE_EV(15, t);
      // P^T = exp2((S^T - L/s) s log2e) (the MMA has subtracted L/s); zero for masked (causal
      // key > query) and padded keys.  Only the diagonal block (i == j) and a ragged last key
      // block need the test.
      uint32_t pk[32];
      const bool need_mask = !key_ok || (CAUSAL && i == j);
      const uint64_t sl2 = f2pack(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const int c = 2 * c2;
        // with FA_BWDQ_PIPE_LD the second 32 columns arrive while the first are worked on
        if (FA_BWDQ_PIPE_LD && c2 == 16) tmem_wait_ld(sv[1]);
        float x0, x1;
        f2unpack(fmul2(f2pack(__uint_as_float(sv[c >> 5][c & 31]),
                              __uint_as_float(sv[c >> 5][(c & 31) + 1])),
                       sl2),
                 x0, x1);
        float p0, p1;
        if ((FA_BWDQ_POLY_MASK >> (c2 >> 2)) & 1) {
          exp2_fma2(x0, x1, p0, p1);
        } else {
          p0 = ex2(x0);
          p1 = ex2(x1);
        }
        if (need_mask) {
          p0 = (key_ok && (!CAUSAL || r <= c0 + c)) ? p0 : 0.f;
          p1 = (key_ok && (!CAUSAL || r <= c0 + c + 1)) ? p1 : 0.f;
        }
        pk[c2] = pack_bf16(p0, p1);
      }
      // P^T over this thread's own S^T columns (the whole warpgroup has read them)
      FA_TRACE_EV(16, t);
      tmem_st32(tmem + lane_base + C::T_S + 96 * h, pk);
      tmem_wait_st();
      FA_TRACE_EV(17, t);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_PF);
      FA_TRACE_EV(12, t);
      // dS^T = P^T * (dP^T - D), with P^T as rounded to bf16 for the dV product
      if (!(ok = W.wait_warp(BAR_DPF, t & 1, 53))) break;
      FA_TRACE_EV(13, t);
      tc_fence_after();
      tmem_ld32(tmem + lane_base + C::T_DP + c0, sv[0]);
      if (!FA_BWDQ_PIPE_LD) tmem_ld32(tmem + lane_base + C::T_DP + c0 + 32, sv[1]);
      tmem_wait_ld(sv[0]);
      if (FA_BWDQ_PIPE_LD) tmem_ld32(tmem + lane_base + C::T_DP + c0 + 32, sv[1]);
      else tmem_wait_ld(sv[1]);
      FA_TRACE_EV(18, t);
      // the MMA has subtracted D: dS^T = P^T dP'^T, one paired multiply per two queries
      uint32_t dsk[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const int c = 2 * c2;
        if (FA_BWDQ_PIPE_LD && c2 == 16) tmem_wait_ld(sv[1]);
        const uint32_t pp = pk[c2];
        float d0, d1;
        f2unpack(fmul2(f2pack(__uint_as_float(pp << 16), __uint_as_float(pp & 0xffff0000u)),
                       f2pack(__uint_as_float(sv[c >> 5][c & 31]),
                              __uint_as_float(sv[c >> 5][(c & 31) + 1]))),
                 d0, d1);
        dsk[c2] = pack_bf16(d0, d1);
      }
      // dS^T into the shared tile (for dQ^T, and for dK when it reads shared memory) and, when dK
      // reads tensor memory, over this thread's own dP^T columns
      FA_TRACE_EV(19, t);
      if (!FA_BWDQ_DK_SS) tmem_st32(tmem + lane_base + C::T_DP + 96 * h, dsk);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = make_uint4(dsk[4 * c], dsk[4 * c + 1], dsk[4 * c + 2], dsk[4 * c + 3]);
        *reinterpret_cast<uint4*>(ds_row + ((c ^ (r & 7)) << 4)) = v;
      }
      fence_async_smem();
      FA_TRACE_EV(21, t);
      if (!FA_BWDQ_DK_SS) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DSF);
      FA_TRACE_EV(14, t);
    }
    if (ok) {
      // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (x scale), bf16
      ok = W.wait_warp(BAR_DKD, (T + nit - 1) & 1, 55);
      FA_TRACE_EV(94, 0);  // epilogue start
      if (ok) {
        tc_fence_after();
        const uint32_t col = h == 0 ? C::T_DV : C::T_DK;
        const float mul = h == 0 ? 1.f : p.scale;
        const CUtensorMap* tmo = h == 0 ? &tmdV : &tmdK;
        const bool issuer = (warp & 3) == 0 && lane == 0;
        if (p.gsplit > 1) {
          // a group's query heads split over CTAs: fp32 reduce-adds into the accumulators
          const size_t base = (size_t(kvh) * p.N + key) * C::D;
          float* acc = (h == 0 ? p.dv_acc : p.dk_acc) + base;
#pragma unroll
          for (int c = 0; c < C::D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + col + 32 * c, v);
            tmem_wait_ld(v);
            bwd_store_chunk(v, mul, key_ok, nullptr, acc + 32 * c);
          }
        } else if (bwdq_unit_of(kc + 1, cta, G, units) < 0) {
          // the CTA's last unit: staged as a swizzled tile in Q stage h (no longer read: every
          // MMA has completed and nothing is loaded after it), then written by TMA tensor stores
          // in whole rows (rows past N are clipped)
          uint8_t* tile = smem + C::OFF_Q + h * C::TILE;
#pragma unroll
          for (int c = 0; c < C::D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + col + 32 * c, v);
            tmem_wait_ld(v);
            stage_chunk_sw128(v, mul, tile, r, c);
          }
          fence_async_smem();
          named_bar_sync(1 + h, 128);
          if (issuer) {
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
              tma_store_3d(tmo, sbase + C::OFF_Q + h * C::TILE + kb * C::BLK, kb * 64, k0, kvh);
            bulk_commit_group();
            bulk_wait_group_read<0>();  // the tile is read before the CTA's memory goes away
          }
        } else {
          // another unit follows (the Q stages already hold its tiles): staged one 64-column
          // block at a time in this warpgroup's half of the dS^T tile, free until this
          // warpgroup writes the next unit's dS^T
          uint8_t* blk = smem + C::OFF_DS + h * C::BLK;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              uint32_t v[32];
              tmem_ld32(tmem + lane_base + col + 32 * (2 * kb + c2), v);
              tmem_wait_ld(v);
              stage_chunk_sw128(v, mul, blk, r, c2);
            }
            fence_async_smem();
            named_bar_sync(1 + h, 128);
            if (issuer) {
              tma_store_3d(tmo, sbase + C::OFF_DS + h * C::BLK, kb * 64, k0, kvh);
              bulk_commit_group();
              bulk_wait_group_read<0>();  // read before the block is written again
            }
            named_bar_sync(1 + h, 128);
          }
        }
      }
    }
    T += nit;
    }  // units
    tc_fence_before();
  } else {
    // ================================================================ dQ drain warpgroup
    // dQ^T (d on TMEM lanes, 128 query columns) -> x scale -> shared staging -> TMA bulk
    // reduce-add into the fp32 accumulator.  Each drain warp owns 32 d rows and its own 4 KB
    // staging block ([32 queries][32 d]); it works through the step's four 32-query quarters on
    // its own, with no barrier shared with the other drain warps: write a quarter, hand it to
    // the TMA unit, and before the next one wait until that reduce has read the block (rows past
    // N are clipped by the tensor map; quarters wholly past N are skipped).  The whole dQ^T is
    // read out of tensor memory first, so the MMA warp may reuse its columns at once.
    regs_inc<C::DQ_REGS>();
    const int wq = warp - C::DQ_WARP0;
    const bool issuer = lane == 0;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    float* wslot = reinterpret_cast<float*>(smem + C::OFF_STG) + wq * (32 * C::DW);
    if (issuer) tma_prefetch_desc(&tmdQ);
    bool ok = true;
    int T = 0;  // global index of the unit's first step
    for (int kc = 0; ok; ++kc) {
    const int u = bwdq_unit_of(kc, cta, G, units);
    if (u < 0) break;
    const BwdUnit unit(u, p, 1);
    const BwdGroup grp(p, unit.kvh, unit.gs, CAUSAL ? unit.j : 0, nqb);
    const int nit = grp.nheads * grp.nit_h;  // >= 1
    BwdCursor cur(grp);
    for (int tl = 0; tl < nit; ++tl) {
      const int t = T + tl;
      const int i = cur.i, head = cur.head;
      cur.next();
      if (!(ok = W.wait_warp(BAR_DQF, t & 1, 60))) break;
      FA_TRACE_EV(60, t);
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_base + C::T_DQ + 32 * q, v[q]);
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_wait_ld(v[q]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DQE);
      FA_TRACE_EV(61, t);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int row0 = i * C::BR + 32 * qq;
        if (row0 >= p.N) break;  // uniform over the warp
        if (issuer) bulk_wait_group_read<0>();  // this warp's previous reduce has read the block
        __syncwarp();
        if (lane < C::DW) {  // d row DW * wq + lane (see DW)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            wslot[c * C::DW + lane] = __uint_as_float(v[qq][c]) * p.scale;
        }
        fence_async_smem();
        __syncwarp();
        FA_TRACE_EV(62, t);
        if (issuer) {
          tma_reduce_add_3d(&tmdQ, smem_u32(wslot), C::DW * wq, row0, head);
          bulk_commit_group();
        }
      }
    }
    T += nit;
    }  // units
    if (issuer) bulk_wait_group_all();
    tc_fence_before();
  }

  FA_TRACE_EV(95, 0);  // role done
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
