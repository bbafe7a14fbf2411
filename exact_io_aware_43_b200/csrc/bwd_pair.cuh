// bwd_pair.cuh -- attention backward for d = 256 on pairs of CTAs (thread-block clusters of two)
// that exchange the probability and gradient tiles through distributed shared memory.
//
// The backward recomputes the attention matrix from Q, K and the saved logsumexp L instead of
// storing it (robocikowo.com "Flash Attention", the backward pass).  Per key block j (128 keys)
// and query block i (64 queries) it needs
//     S^T = K_j Q_i^T,  P^T = exp(s S^T - L_i),  dP^T = V_j dO_i^T,  dS^T = P^T * (dP^T - D_i),
//     dV_j += P^T dO_i,  dK_j += s dS^T Q_i,  dQ_i += s dS K_j       (D_i = rowsum(dO_i * O_i))
// At d = 256, dK_j and dV_j (128 x 256 fp32 each) fill the 512 columns of one SM's tensor memory
// between them, so one CTA cannot keep both beside the score tiles.  The two CTAs of a cluster
// therefore split the work by what they accumulate, and compute every product once:
//
//   CTA 0 ("S" CTA):  K_j resident, Q_i streamed.  S^T -> P^T (exponentials) -> P^T into CTA 1's
//                     shared memory;  dK_j += dS^T Q_i and dQ_i[:, 0:128] += dS K_j[:, 0:128] with
//                     the dS^T it receives.
//   CTA 1 ("dP" CTA): V_j resident in TENSOR memory (the A operand of dP^T), K_j[:, 128:256] in
//                     shared memory, dO_i streamed.  dP^T;  dS^T = P^T (dP^T - D) with the P^T it
//                     receives -> dS^T into CTA 0's shared memory and its own;  dV_j += P^T dO_i
//                     and dQ_i[:, 128:256] += dS K_j[:, 128:256].
//
// Each CTA issues five 128 x 64 x 128-equivalent GEMM units per step, ten in all, where two
// independent CTAs that each recompute S^T and dP^T for a 128-wide slice of d issue fourteen, and
// each reduces half of dQ.  Keeping V_j in tensor memory is what makes room in CTA 1's shared
// memory for K_j's upper half, two dS^T tiles and dQ staging.  The exchanged tiles (P^T and dS^T,
// 16 KB each per step) travel as asynchronous remote stores (st.async) whose bytes complete a
// transaction count on the receiver's mbarrier, so the data announces its own arrival; each side
// has two buffers, and a buffer is handed back (a remote arrival) once its last reader -- an MMA,
// and for P^T also CTA 1's dS warps -- has finished.
//
// Warp roles: warps 0-7 exponentials (CTA 0) or dS (CTA 1), thread = key row = TMEM lane, the two
// warpgroups on query columns [0, 32) and [32, 64) of every step; warps 8-11 drain this CTA's
// dQ^T half (32 d rows each, two 4 KB staging blocks each) into the fp32 accumulator with TMA
// bulk reduce-adds; warp 12 issues TMA loads; warp 13 allocates tensor memory and issues the
// MMAs as independent ready-driven streams; warp 14 of CTA 1 hands P^T tiles back.
//
// Every wait is bounded.  A CTA that gives up sets its own and its peer's abort flag, so both
// fall through to the teardown, where each sender first waits (bounded) for the hand-back of its
// last tile -- no asynchronous store is then still in flight -- and a cluster barrier keeps
// either CTA from exiting while the other may still write into its shared memory.
#pragma once

#include "bwd.cuh"

namespace fattn {

// ------------------------------------------------------------------------------------------
// cluster and distributed-shared-memory primitives
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t caddr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}
// Non-blocking probe of a phase, acquiring at cluster scope.
__device__ __forceinline__ uint32_t mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
// Asynchronous 16-byte store into another CTA's shared memory; its bytes count toward the
// transaction count of the mbarrier `cbar` in that CTA (complete_tx on arrival), so the receiver
// learns that the data has landed from the barrier itself and the sender waits for nothing.
__device__ __forceinline__ void st_async_v4(uint32_t caddr, uint4 v, uint32_t cbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(caddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(cbar)
      : "memory");
}
// Arrive on an mbarrier of another CTA and add `bytes` to the transaction count of its phase.
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   cbar),
               "r"(bytes)
               : "memory");
}
// Plain arrival on an mbarrier of another CTA (a hand-back signal that carries no data: what
// it announces -- MMA reads of a buffer -- completed before the local commit this thread waited
// on).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}
// Phase wait that acquires at cluster scope (the arrivals may come from the peer CTA).
__device__ __forceinline__ uint32_t mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
__device__ __forceinline__ uint32_t mbar_try_wait_cluster_sleep(uint32_t bar, uint32_t parity,
                                                                uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok;
}
// All threads of both CTAs.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

#ifndef FA_PAIR_HANDBACK_LIMIT_NS
#define FA_PAIR_HANDBACK_LIMIT_NS 4000000000ull
#endif

// Bounded waits for a CTA of a pair: like Waiter, with cluster-scope acquire, and giving up
// also raises the peer's abort flag.
struct PairWaiter {
  volatile int* abort_flag;
  uint32_t peer_abort;  // shared::cluster address of the peer CTA's abort flag
  uint64_t limit_ns;
  __device__ __forceinline__ void give_up(int site) const {
    *abort_flag = 1;
    st_cluster_u32(peer_abort, 1u);
    if (atomicCAS(&g_status[0], 0, 5 /* FA_ERR_TIMEOUT */) == 0) g_status[1] = site;
  }
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, int site) const {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
      if (mbar_try_wait_cluster_sleep(bar, parity, 1000000u)) return true;
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) {
        give_up(site);
        return false;
      }
    }
  }
  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, int site) const {
    const bool ok = wait(bar, parity, site);
    return __all_sync(0xffffffffu, ok);
  }
  __device__ __forceinline__ bool aborted() const { return *abort_flag != 0; }
  __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity) const {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (global_ns() - t0 > Waiter::kDrainLimitNs) return false;
    }
    return true;
  }
  // Teardown wait for the peer's hand-back of a tile this warp sent (cluster-scope acquire),
  // ignoring the abort flag.  After an abort the hand-back may never come; the bound only has to
  // exceed the landing time of the asynchronous stores (microseconds).
  static constexpr uint64_t kHandBackLimitNs = FA_PAIR_HANDBACK_LIMIT_NS;
  __device__ __forceinline__ void drain_warp(uint32_t bar, uint32_t parity) const {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
      if (global_ns() - t0 > kHandBackLimitNs) break;
    }
    __syncwarp();
  }
};

// FA_PAIR_POLL_NS: the MMA thread's pause between rounds of barrier probes that found nothing
// ready (nanoseconds).
#ifndef FA_PAIR_POLL_NS
#define FA_PAIR_POLL_NS 32
#endif

struct BwdPairCfg {
  static constexpr int D = 256;
  static constexpr int BC = 128;                 // keys per cluster (M of S^T, dP^T, dK, dV)
  static constexpr int BR = 64;                  // queries per step
  static constexpr int KV_BLK = BC * 128;        // [128 keys][64 d] bf16, 128-byte rows: 16 KB
  static constexpr int Q_BLK = BR * 128;         // [64 queries][64 d] bf16: 8 KB
  static constexpr int STAGE = 4 * Q_BLK;        // a Q_i or dO_i tile, [64][256]: 32 KB
  static constexpr int XT = BC * BR * 2;         // a P^T or dS^T tile, [128 keys][64 q]: 16 KB
  static constexpr int NS = 3;                   // Q_i (CTA 0) or dO_i (CTA 1) stages
  static constexpr int WPS = 8;                  // exponential / dS warps, all on every step
  // shared memory map (both CTAs use the same offsets; remote stores address the peer's copy)
  //   OFF_A   CTA 0: K_j (64 KB).  CTA 1: K_j[:, 128:256] (32 KB), then its two dS^T tiles.
  //   OFF_S   NS stages of Q_i (CTA 0) or dO_i (CTA 1); CTA 1 first stages V_j in the first two
  //           on its way into tensor memory
  //   OFF_X   the two tiles the peer writes: dS^T (CTA 0) / P^T (CTA 1)
  //   OFF_STG dQ staging, 2 x 4 KB per drain warp
  static constexpr int OFF_A = 0;
  static constexpr int OFF_DSL = OFF_A + 2 * KV_BLK;  // CTA 1: dS^T tiles
  static constexpr int OFF_S = OFF_A + 4 * KV_BLK;
  static constexpr int OFF_X = OFF_S + NS * STAGE;
  static constexpr int OFF_STG = OFF_X + 2 * XT;
  static constexpr int OFF_ROWS = OFF_STG + 8 * 4096;  // per stage 64 floats: L2 (CTA 0) / D (CTA 1)
  static constexpr int NBAR = 26;
  static constexpr int OFF_BAR = OFF_ROWS + NS * BR * 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 480;
  static constexpr int DQ_WARP0 = 8, PRODUCER_WARP = 12, MMA_WARP = 13, RELAY_WARP = 14;
  // tensor memory columns
  //   CTA 0: S^T buffers [0, 128), dK [128, 384), dQ^T half 0 [384, 448)
  //   CTA 1: V_j as bf16 pairs (A operand of dP^T) [0, 128), dP^T [128, 192), dQ^T half 1
  //          [192, 256), dV [256, 512)
  static constexpr int T_S = 0, T_DK = 128, T_DQ0 = 384;
  static constexpr int T_V = 0, T_DP = 128, T_DQ1 = 192, T_DV = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC_ST = idesc_bf16_f32(BC, BR, 0, 0);   // S^T, dP^T
  static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(BC, D, 0, 1);   // dK, dV (N = 256)
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, BR, 1, 1);  // a dQ^T half = K_h^T dS^T
  // barriers
  static constexpr int B_KV = 0;      // resident K_j (CTA 0) / K_j[:, 128:256] (CTA 1) landed
  static constexpr int B_VL = 1;      // CTA 1: V_j landed in the staging area
  static constexpr int B_VD = 2;      // CTA 1: V_j in tensor memory (8 warps)
  static constexpr int B_LF = 3;      // + s: stage s loaded
  static constexpr int B_LE = 6;      // + s: stage s free (MMA commit + the step's WPS warps)
  static constexpr int B_AF = 9;      // + b: S^T / dP^T buffer b computed
  static constexpr int B_AFREE = 11;  // + b: S^T / dP^T buffer b read out (WPS warps)
  static constexpr int B_XF = 13;     // + b: exchange tile b written by the peer (WPS remote warps)
  static constexpr int B_XE = 15;     // + b: the peer's exchange tile b is free (1 remote arrival)
  static constexpr int B_XR = 17;     // + b: CTA 1: P^T tile b read (MMA commit + WPS warps)
  static constexpr int B_DSL = 19;    // + b: CTA 1: own dS^T tile b written (WPS warps)
  static constexpr int B_DSLE = 21;   // + b: CTA 1: own dS^T tile b read by dQ^T (MMA commit)
  static constexpr int B_DQF = 23;    // this step's dQ^T half complete
  static constexpr int B_DQE = 24;    // dQ^T read out of tensor memory (4 drain warps)
  static constexpr int B_DRAIN = 25;
};
static_assert(BwdPairCfg::SMEM_BYTES <= 232448, "pair backward exceeds 227 KB of shared memory");

template <bool CAUSAL>
__global__ void __launch_bounds__(BwdPairCfg::THREADS, 1)
    fa_bwd_kernel_pair(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ,
                       const __grid_constant__ CUtensorMap tmdK,
                       const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using C = BwdPairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FA_TRACE_DECL;
  const uint32_t role = cluster_ctarank();  // 0: S^T, P, dK, dQ[:, :128];  1: dP^T, dS, dV, dQ[:, 128:]
  const uint32_t peer = role ^ 1u;
  const int NBA = role == 0 ? 2 : 1;  // S^T / dP^T buffers in tensor memory

  // ---- work unit (both CTAs of the cluster take the same one)
  const BwdUnit unit(int(blockIdx.x >> 1), p, 1);
  const int j = unit.j, kvh = unit.kvh;
  const int k0 = j * C::BC;
  const int nqblk = (p.N + C::BR - 1) / C::BR;
  const BwdGroup grp(p, kvh, unit.gs, CAUSAL ? (k0 / C::BR) : 0, nqblk);
  const int nit = grp.nheads * grp.nit_h;  // >= 1

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  constexpr int NS = C::NS;
  auto stage_addr = [&](int s) -> uint32_t { return sbase + C::OFF_S + s * C::STAGE; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV), 1);
    mbar_init(bar(C::B_VL), 1);
    mbar_init(bar(C::B_VD), 8);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(C::B_LF + s), 1);
      mbar_init(bar(C::B_LE + s), 1 + C::WPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::B_AF + b), 1);
      mbar_init(bar(C::B_AFREE + b), C::WPS);
      mbar_init(bar(C::B_XF + b), C::WPS);
      mbar_init(bar(C::B_XE + b), 1);
      mbar_init(bar(C::B_XR + b), 1 + C::WPS);
      mbar_init(bar(C::B_DSL + b), C::WPS);
      mbar_init(bar(C::B_DSLE + b), 1);
    }
    mbar_init(bar(C::B_DQF), 1);
    mbar_init(bar(C::B_DQE), 4);
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  // both CTAs' barriers exist before either side arrives remotely
  cluster_barrier();
  FA_TRACE_EV(98, 0);  // both CTAs leave this barrier together: aligns their clocks
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const PairWaiter W{abort_flag, mapa_shared(smem_u32(const_cast<int*>(abort_flag)), peer),
                     p.limit_ns};
  const float* rows_smem = reinterpret_cast<const float*>(smem + C::OFF_ROWS);

  if (warp == C::PRODUCER_WARP) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const CUtensorMap* tmS = role == 0 ? &tmQ : &tmdO;  // the streamed operand
      tma_prefetch_desc(tmS);
      tma_prefetch_desc(&tmK);
      bool ok = true;
      if (role == 0) {
        mbar_arrive_expect_tx(bar(C::B_KV), 4 * C::KV_BLK);
        for (int kb = 0; kb < 4; ++kb)
          tma_load_3d(sbase + C::OFF_A + kb * C::KV_BLK, &tmK, bar(C::B_KV), kb * 64, k0, kvh);
      } else {
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KV_BLK);
        for (int kb = 2; kb < 4; ++kb)
          tma_load_3d(sbase + C::OFF_A + (kb - 2) * C::KV_BLK, &tmK, bar(C::B_KV), kb * 64, k0,
                      kvh);
        // V_j through the first two stages into tensor memory; the stages stream dO_i after
        mbar_arrive_expect_tx(bar(C::B_VL), 4 * C::KV_BLK);
        for (int kb = 0; kb < 4; ++kb)
          tma_load_3d(sbase + C::OFF_S + kb * C::KV_BLK, &tmV, bar(C::B_VL), kb * 64, k0, kvh);
        ok = W.wait(bar(C::B_VD), 0, 69);
      }
      const float* rows_src = role == 0 ? p.L2 : p.Drow;
      int it = 0;
      bool starved = false;
      BwdCursor cur(grp);
      for (; ok && it < nit; ++it) {
        const int i = cur.i, head = cur.head;
        cur.next();
        const int s = it % NS;
#ifdef FA_TEST_STARVE
        // Test build only (libfattn_starve.so): CTA 1 of the first cluster never issues its second
        // dO_i tile, so the bounded waits for it run out on both CTAs of the pair, which must
        // report FA_ERR_TIMEOUT and tear down cleanly.  The loads issued so far are drained below.
        if (blockIdx.x == 1 && it == 1) {
          starved = true;
          break;
        }
#endif
        if (!W.wait(bar(C::B_LE + s), ((it / NS) & 1) ^ 1, 70)) break;
        FA_TRACE_EV(30, it);
        mbar_arrive_expect_tx(bar(C::B_LF + s), C::STAGE + C::BR * 4);
        for (int kb = 0; kb < 4; ++kb)
          tma_load_3d(stage_addr(s) + kb * C::Q_BLK, tmS, bar(C::B_LF + s), kb * 64, i * C::BR,
                      head);
        bulk_load(sbase + C::OFF_ROWS + s * C::BR * 4,
                  rows_src + size_t(head) * p.Npad + size_t(i) * C::BR, C::BR * 4,
                  bar(C::B_LF + s));
      }
      if (W.aborted() || starved) {
        W.drain(bar(C::B_KV), 0);
        if (role == 1) W.drain(bar(C::B_VL), 0);
        for (int jj = max(0, it - NS); jj < it; ++jj)
          W.drain(bar(C::B_LF + jj % NS), (jj / NS) & 1);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ================================================================ MMA issuer
    // Three independent streams, each in step order, issued as they become ready: A, S^T(t)
    // (CTA 0, two buffers) or dP^T(t) (CTA 1, one buffer; A operand V_j from tensor memory), once
    // the stage has landed and the buffer has been read out; B, dK (CTA 0) or dV (CTA 1), once
    // the peer's tile of step t has arrived -- the stage is then released; C, this CTA's dQ^T
    // half, once its dS^T tile is there (the received one on CTA 0, the CTA's own on CTA 1) and
    // the drain has read dQ^T(t-1).
    if (lane == 0) {
      const uint32_t a_addr = sbase + C::OFF_A;  // K_j (CTA 0) or K_j[:, 128:256] (CTA 1)
      bool ok = W.wait(bar(C::B_KV), 0, 71);
      if (ok && role == 1) ok = W.wait(bar(C::B_VD), 0, 78);
      int ns = 0, na = 0, nq = 0;  // next step of streams A, B, C
      uint64_t t_last = global_ns();
      const uint32_t t_dq = role == 0 ? C::T_DQ0 : C::T_DQ1;
      while (ok && (na < nit || nq < nit)) {
        bool progress = false;
        if (ns < nit && mbar_test_wait(bar(C::B_LF + ns % NS), (ns / NS) & 1) &&
            mbar_test_wait(bar(C::B_AFREE + ns % NBA), ((ns / NBA) & 1) ^ 1)) {
          tc_fence_after();
          const uint32_t st_addr = stage_addr(ns % NS);
          if (role == 0) {
            // S^T (128 x 64, K = 256) = K_j Q_i^T, both K-major in shared memory
#pragma unroll
            for (int kk = 0; kk < C::D / 16; ++kk)
              mma_ss(tmem + C::T_S + 64 * (ns & 1),
                     sdesc_sw128(a_addr + (kk >> 2) * C::KV_BLK + (kk & 3) * 32, 16, 1024),
                     sdesc_sw128(st_addr + (kk >> 2) * C::Q_BLK + (kk & 3) * 32, 16, 1024),
                     C::IDESC_ST, kk > 0);
          } else {
            // dP^T (128 x 64, K = 256) = V_j dO_i^T: A = V_j from tensor memory (bf16 pairs,
            // 8 columns per 16-deep step), B = dO_i K-major in shared memory
#pragma unroll
            for (int kk = 0; kk < C::D / 16; ++kk)
              mma_ts(tmem + C::T_DP, tmem + C::T_V + kk * 8,
                     sdesc_sw128(st_addr + (kk >> 2) * C::Q_BLK + (kk & 3) * 32, 16, 1024),
                     C::IDESC_ST, kk > 0);
          }
          tc_commit(bar(C::B_AF + ns % NBA));
          FA_TRACE_EV(1, ns);
          ++ns;
          progress = true;
        }
        if (na < ns && mbar_test_wait_cluster(bar(C::B_XF + (na & 1)), (na >> 1) & 1)) {
          FA_TRACE_EV(2, na);
          fence_async_smem();  // the tile arrived by asynchronous stores; the tensor core reads it
          tc_fence_after();
          const int b = na & 1, s = na % NS;
          const uint32_t x_addr = sbase + C::OFF_X + b * C::XT;
          // dK += dS^T Q_i (CTA 0) or dV += P^T dO_i (CTA 1): A = the received tile
          // (K-major, [128 keys][64 q]), B = Q_i / dO_i (MN-major, N = 256)
#pragma unroll
          for (int kk = 0; kk < C::BR / 16; ++kk)
            mma_ss(tmem + (role == 0 ? C::T_DK : C::T_DV), sdesc_sw128(x_addr + kk * 32, 16, 1024),
                   sdesc_sw128(stage_addr(s) + kk * 2048, C::Q_BLK, 1024), C::IDESC_ACC,
                   (na > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(C::B_LE + s));  // the MMAs are the stage's last readers
          if (role == 1) tc_commit(bar(C::B_XR + b));
          FA_TRACE_EV(4, na);
          ++na;
          progress = true;
        }
        if (nq < nit && (role == 0 ? nq < na
                                   : mbar_test_wait(bar(C::B_DSL + (nq & 1)), (nq >> 1) & 1)) &&
            (nq == 0 || mbar_test_wait(bar(C::B_DQE), (nq - 1) & 1))) {
          // dQ^T half (128 d x 64 q, K = 128 keys): A = K_j[:, half]^T (MN-major, two 64-wide d
          // blocks), B = the dS^T tile (MN-major)
          tc_fence_after();
          const uint32_t ds_addr = role == 0 ? sbase + C::OFF_X + (nq & 1) * C::XT
                                             : sbase + C::OFF_DSL + (nq & 1) * C::XT;
#pragma unroll
          for (int kk = 0; kk < C::BC / 16; ++kk)
            mma_ss(tmem + t_dq, sdesc_sw128(a_addr + kk * 2048, C::KV_BLK, 1024),
                   sdesc_sw128(ds_addr + kk * 2048, C::Q_BLK, 1024), C::IDESC_DQ, kk > 0);
          tc_commit(bar(C::B_DQF));
          if (role == 1) tc_commit(bar(C::B_DSLE + (nq & 1)));
          FA_TRACE_EV(5, nq);
          ++nq;
          progress = true;
        }
        if (progress) {
          t_last = global_ns();
        } else {
          if (W.aborted()) break;
          if (global_ns() - t_last > p.limit_ns) {
            W.give_up(72);
            break;
          }
          __nanosleep(FA_PAIR_POLL_NS);
        }
      }
      tc_commit(bar(C::B_DRAIN));
      W.drain(bar(C::B_DRAIN), 0);
    }
  } else if (warp < 8) {
    // ================================================================ exponentials / dS
    // Thread = key row = TMEM lane; both warpgroups work on every step, warpgroup h on query
    // columns [32h, 32h + 32).  (Every warp waits on every phase of the per-step barriers, so
    // no parity test can alias a phase two behind.)  Step t uses exchange tiles t & 1.
    constexpr int NCOL = 32;  // query columns per thread and step
    const int h = warp >> 2;
    const int c0 = 32 * h;
    const int r = (warp & 3) * 32 + lane;  // key row within the block == TMEM lane
    const int key = k0 + r;
    const bool key_ok = key < p.N;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t row_off = uint32_t(r) * 128;
    // the peer's exchange tiles (at this thread's row) and their barriers
    const uint32_t peer_x0 = mapa_shared(sbase + C::OFF_X, peer) + row_off;
    const uint32_t peer_x1 = mapa_shared(sbase + C::OFF_X + C::XT, peer) + row_off;
    const uint32_t peer_xf0 = mapa_shared(bar(C::B_XF + 0), peer);
    const uint32_t peer_xf1 = mapa_shared(bar(C::B_XF + 1), peer);
    bool ok = true;
    int sent = 0;  // steps whose tile this warp has sent to the peer
    if (role == 1) {
      // V_j into tensor memory as the dP^T MMA's A operand: row r (this thread's lane), d
      // columns [128h, 128h + 128) of this warpgroup, bf16 pairs (even d in the low half)
      if ((ok = W.wait_warp(bar(C::B_VL), 0, 79))) {
#pragma unroll
        for (int kb2 = 0; kb2 < 2; ++kb2) {
          const int kb = 2 * h + kb2;
          const uint8_t* vrow = smem + C::OFF_S + kb * C::KV_BLK + row_off;
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 q4 = *reinterpret_cast<const uint4*>(vrow + ((c ^ (r & 7)) << 4));
            v[4 * c] = q4.x;
            v[4 * c + 1] = q4.y;
            v[4 * c + 2] = q4.z;
            v[4 * c + 3] = q4.w;
          }
          tmem_st32(tmem + lane_base + C::T_V + 32 * kb, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_VD));
      }
    }
    BwdCursor cur(grp);
    for (int it = 0; ok && it < nit; ++it) {
      const int i = cur.i;
      cur.next();
      const int s = it % NS, b = it & 1, u = it >> 1;  // stage, exchange tile, its use
      const int ba = it % NBA, ua = it / NBA;          // S^T / dP^T buffer, its use
      if (!(ok = W.wait_warp(bar(C::B_AF + ba), ua & 1, 80))) break;
      if (!(ok = W.wait_warp(bar(C::B_LF + s), (it / NS) & 1, 81))) break;
      FA_TRACE_EV(10, it);
      tc_fence_after();
      uint32_t v[NCOL / 32][32];
      const uint32_t t_a = role == 0 ? C::T_S + 64 * ba : C::T_DP;
#pragma unroll
      for (int q = 0; q < NCOL / 32; ++q) tmem_ld32(tmem + lane_base + t_a + c0 + 32 * q, v[q]);
#pragma unroll
      for (int q = 0; q < NCOL / 32; ++q) tmem_wait_ld(v[q]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_AFREE + ba));
      FA_TRACE_EV(11, it);
      const float* rows = rows_smem + s * C::BR + c0;
      if (role == 1) {
        if (!(ok = W.wait_warp(bar(C::B_XF + b), u & 1, 82))) break;  // P^T landed
        // own dS^T tile b is free once dQ^T of its previous use has read it
        if (!(ok = W.wait_warp(bar(C::B_DSLE + b), (u & 1) ^ 1, 83))) break;
      }
      // the peer's tile b is free once it has handed back the previous use
      if (!(ok = W.wait_warp(bar(C::B_XE + b), (u & 1) ^ 1, 84))) break;
      FA_TRACE_EV(16, it);
      // this warp's 32 rows x NCOL bf16: one arrival with their byte count, then the stores
      const uint32_t pxf = b ? peer_xf1 : peer_xf0, px = b ? peer_x1 : peer_x0;
      if (lane == 0) mbar_arrive_expect_tx_cluster(pxf, 32 * NCOL * 2);
      __syncwarp();
      const int qbase = i * C::BR + c0;
      const bool need_mask = role == 0 && (!key_ok || (CAUSAL && key > qbase));
      const uint8_t* own_x = smem + C::OFF_X + b * C::XT + row_off;
      uint8_t* own_ds = smem + C::OFF_DSL + b * C::XT + row_off;
#pragma unroll
      for (int e = 0; e < NCOL / 8; ++e) {
        // columns c0 + 8e .. c0 + 8e + 7: one 16-byte chunk of the key's 128-byte tile row
        const int ch = c0 / 8 + e;
        const float4 ra = reinterpret_cast<const float4*>(rows)[2 * e];
        const float4 rb = reinterpret_cast<const float4*>(rows)[2 * e + 1];
        const float rv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
        uint32_t pk[4];
        if (role == 0) {
          // P^T = exp2(S^T s log2e - L2); zero for masked (causal: key > query) and padded keys
          float pr[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            pr[c] = ex2(fmaf(__uint_as_float(v[e >> 2][(e & 3) * 8 + c]), p.scale_log2, -rv[c]));
            if (need_mask && (!key_ok || (CAUSAL && key > qbase + 8 * e + c))) pr[c] = 0.f;
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
        } else {
          // dS^T = P^T * (dP^T - D), with P^T as CTA 0 rounded it to bf16
          const uint4 q4 = *reinterpret_cast<const uint4*>(own_x + ((ch ^ (r & 7)) << 4));
          const uint32_t pw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float p0 = __uint_as_float(pw[c] << 16);
            const float p1 = __uint_as_float(pw[c] & 0xffff0000u);
            const int cc = (e & 3) * 8 + 2 * c;
            pk[c] = pack_bf16(p0 * (__uint_as_float(v[e >> 2][cc]) - rv[2 * c]),
                              p1 * (__uint_as_float(v[e >> 2][cc + 1]) - rv[2 * c + 1]));
          }
          // and into the CTA's own dS^T tile, for its dQ^T half
          *reinterpret_cast<uint4*>(own_ds + ((ch ^ (r & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        st_async_v4(px + ((ch ^ (r & 7)) << 4), make_uint4(pk[0], pk[1], pk[2], pk[3]), pxf);
      }
      ++sent;
      if (role == 1) fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(C::B_LE + s));  // this step's row vector has been read
        if (role == 1) {
          mbar_arrive(bar(C::B_XR + b));   // its P^T tile too
          mbar_arrive(bar(C::B_DSL + b));  // and the own dS^T tile is written
        }
      }
      FA_TRACE_EV(17, it);
    }
    if (ok) {
      // ---- epilogue: dK (x scale, CTA 0) or dV (CTA 1), bf16; warpgroup h writes d columns
      // [128h, 128h + 128).  The MMA warp's final commit (a barrier with a single phase, so no
      // parity can alias) says every MMA of the CTA has completed.
      ok = W.wait_warp(bar(C::B_DRAIN), 0, 85);
      if (ok) {
        tc_fence_after();
        const float mul = role == 0 ? p.scale : 1.f;
        const uint32_t t_acc = role == 0 ? C::T_DK : C::T_DV;
        if (p.gsplit > 1) {
          // a group's query heads split over CTAs: fp32 reduce-adds into the accumulators
          const size_t base = (size_t(kvh) * p.N + key) * C::D + 128 * h;
          float* acc = (role == 0 ? p.dk_acc : p.dv_acc) + base;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t vv[32];
            tmem_ld32(tmem + lane_base + t_acc + 128 * h + 32 * c, vv);
            tmem_wait_ld(vv);
            bwd_store_chunk(vv, mul, key_ok, nullptr, acc + 32 * c);
          }
        } else {
          // staged as a swizzled tile (d columns [128h, 128h + 128): two 64-column blocks) in
          // stage h, no longer read once every MMA has completed, then written by TMA tensor
          // stores in whole rows (rows past N are clipped)
          uint8_t* tile = smem + C::OFF_S + h * C::STAGE;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t vv[32];
            tmem_ld32(tmem + lane_base + t_acc + 128 * h + 32 * c, vv);
            tmem_wait_ld(vv);
            stage_chunk_sw128(vv, mul, tile, r, c);
          }
          fence_async_smem();
          named_bar_sync(1 + h, 128);
          if ((warp & 3) == 0 && lane == 0) {
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
              tma_store_3d(role == 0 ? &tmdK : &tmdV, stage_addr(h) + kb * C::KV_BLK,
                           (2 * h + kb) * 64, k0, kvh);
            bulk_commit_group();
            bulk_wait_group_read<0>();  // the tile is read before the CTA's memory goes away
          }
        }
      }
    }
    // Before the teardown, the peer's hand-back of the last tile this warpgroup sent: it follows
    // the landing of the asynchronous stores, so none is still in flight when the cluster
    // exits.  (After an abort the peer may never hand back; the wait then ends at its own limit,
    // long after the stores have landed.)
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int n_b = (sent + 1 - b) / 2;  // uses of buffer b
      if (n_b > 0) W.drain_warp(bar(C::B_XE + b), (n_b - 1) & 1);
    }
    tc_fence_before();
  } else if (warp < C::DQ_WARP0 + 4) {
    // ================================================================ dQ drain
    // This CTA's dQ^T half (d on TMEM lanes, 64 query columns) -> x scale -> staging blocks
    // ([32 queries][32 d], two per warp) -> TMA bulk reduce-add into the fp32 accumulator (rows
    // past N are clipped by the tensor map; quarters wholly past N are skipped).  On CTA 0, once
    // dQ^T of a step has completed its dS^T tile has been consumed (dK was issued before), so
    // warp 8 hands it back to CTA 1.
    const int wq = warp - C::DQ_WARP0;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t t_dq = role == 0 ? C::T_DQ0 : C::T_DQ1;
    const int d0 = int(role) * 128 + 32 * wq;
    const uint32_t peer_xe0 = mapa_shared(bar(C::B_XE + 0), peer);
    const uint32_t peer_xe1 = mapa_shared(bar(C::B_XE + 1), peer);
    float* wslot = reinterpret_cast<float*>(smem + C::OFF_STG) + wq * 2048;
    if (lane == 0) tma_prefetch_desc(&tmdQ);
    int group = 0;
    BwdCursor cur(grp);
    for (int it = 0; it < nit; ++it) {
      const int i = cur.i, head = cur.head;
      cur.next();
      if (!W.wait_warp(bar(C::B_DQF), it & 1, 86)) break;
      FA_TRACE_EV(20, it);
      if (role == 0 && wq == 0 && lane == 0)
        mbar_arrive_cluster((it & 1) == 0 ? peer_xe0 : peer_xe1);
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(tmem + lane_base + t_dq, v[0]);
      tmem_ld32(tmem + lane_base + t_dq + 32, v[1]);
      tmem_wait_ld(v[0]);
      tmem_wait_ld(v[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DQE));
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int row0 = i * C::BR + 32 * qq;
        if (row0 >= p.N) continue;  // uniform over the warp
        float* slot = wslot + (group & 1) * 1024;
        if (lane == 0) bulk_wait_group_read<1>();  // the slot's previous reduce has read it
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 32; ++c) slot[c * 32 + lane] = __uint_as_float(v[qq][c]) * p.scale;
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmdQ, smem_u32(slot), d0, row0, head);
          bulk_commit_group();
        }
        ++group;
      }
      FA_TRACE_EV(21, it);
    }
    if (lane == 0) bulk_wait_group_all();
    tc_fence_before();
  } else if (warp == C::RELAY_WARP && role == 1) {
    // ================================================================ hand-back (CTA 1)
    // P^T tile t & 1 is free once dV(t) has completed and the dS warps have read it.
    const uint32_t peer_xe0 = mapa_shared(bar(C::B_XE + 0), peer);
    const uint32_t peer_xe1 = mapa_shared(bar(C::B_XE + 1), peer);
    for (int it = 0; it < nit; ++it) {
      if (!W.wait_warp(bar(C::B_XR + (it & 1)), (it >> 1) & 1, 87)) break;
      if (lane == 0) mbar_arrive_cluster((it & 1) == 0 ? peer_xe0 : peer_xe1);
    }
  }

  // neither CTA leaves while the other may still write into its shared memory or arrive on its
  // barriers
  __syncwarp();
  cluster_barrier();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
