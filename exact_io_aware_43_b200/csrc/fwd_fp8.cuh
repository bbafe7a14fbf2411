// fwd_fp8.cuh -- attention forward on FP8 (e4m3) inputs for sm_100a.
//
// The low-precision forward the pages attribute to FlashAttention-3 (robocikowo.com "Flash
// Attention", the FA-3 entry: "FP8"; systems-analysis.info "FlashAttention (PL)", section
// "FlashAttention-3 (2024)": about 1.2 PFLOPS in FP8; dexblog.ro, the dtype row: FA-3 adds FP8 to
// the forward).  The pages give no kernel design for it; this one keeps the bf16 forward's shape
// (fwd.cuh: persistent CTAs, TMA ring, one MMA thread, two ping-pong softmax warpgroups,
// accumulators in tensor memory) and changes what the tensor core multiplies:
//
//   Q, K, V are e4m3 codes with one scale per tensor: the attended values are q_scale * Q8,
//   k_scale * K8, v_scale * V8.  Both GEMMs run as tcgen05.mma kind::f8f6f4 (e4m3 x e4m3 ->
//   fp32 in tensor memory, 32 keys or d-elements per instruction, twice the bf16 rate):
//     S  = Q8 K8^T                               scaled by s * q_scale * k_scale in the softmax
//     P^ = e4m3(2^8 * exp2(S s' log2e - m))      written back into tensor memory (4 per column)
//     O += P^ V8                                  A = P^ from tensor memory, V8 MN-major
//   and at the end O = v_scale * O / l with l = sum 2^8 exp2(...) in fp32, L = m + ln(l / 2^8).
//
// Why the factor 2^8 and the exact rescale: P^ is rounded to e4m3 (3 mantissa bits).  The row
// reference m follows every increase of the row maximum (no lazy threshold), so the largest
// weight of a row is exactly 2^8 = 256, representable, and a row dominated by one key keeps that
// key's weight exact; weights down to 2^-14 of the maximum stay normal numbers (relative rounding
// error at most 2^-4), smaller ones round to multiples of 2^-17 of it.  l and L use the fp32
// exponentials, so L carries no fp8 rounding; O's error is the weights' rounding, bounded by
// 2^-4 of sum_j P_ij |v_j| per element (the tests state and check this bound).
#pragma once

#include <cuda_fp8.h>

#include "fwd.cuh"

namespace fattn {

// Self-test kernel for exp2_fma2 (used only by fa_selftest_exp2_fma).
__global__ void fa_selftest_exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y,
                                            int n);

// D[tmem] (+)= A[smem] * B[smem]^T with e4m3 A and B (kind::f8f6f4), fp32 accumulate.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, e4m3 A (K-major in tensor memory, 4 per 32-bit column).
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f8f6f4 with e4m3 A and B (format code 0) and fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                         // D format f32
         | (uint32_t(a_mn) << 15)          // A major
         | (uint32_t(b_mn) << 16)          // B major
         | (uint32_t(N >> 3) << 17)        // N / 8
         | (uint32_t(M >> 4) << 24);       // M / 16
}

// Shared-memory matrix descriptor with an explicit swizzle mode (layout code 2: 128-byte,
// 4: 64-byte swizzle), same fields as sdesc_sw128.
__device__ __forceinline__ uint64_t sdesc_swz(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (uint64_t(layout) << 61);
}

// FA_FP8_POLY_MASK: bit e set sends the e-th group of four scores of every 32 through exp2_fma2
// (the FMA pipe) instead of the MUFU unit; at the fp8 MMA rate the exponentials, not the tensor
// core, bound the kernel, so moving a share of them to the FMA pipe shortens each softmax step.
// Measured on the long-context causal workload (TFLOP/s): none 1128, groups 2 and 5 (a quarter)
// 1157, groups 1, 4, 7 1125, every other group 1052 (the issue slots then bind).
#ifndef FA_FP8_POLY_MASK
#define FA_FP8_POLY_MASK 0x24
#endif
// FA_FP8_INORDER: 1 issues S_t(j+1) straight behind PV_t(j) (which reads P_t(j) from the tensor
// memory S_t(j+1) overwrites) without waiting for PV_t(j) to complete: one thread's MMAs execute
// in issue order.  -1: without the causal mask only (d = 128, TFLOP/s: non-causal 1057 vs 1027,
// causal 1132 vs 1147).  FA_FP8_MMA_POLL: the MMA warp polls its barriers without a suspend hint.
#ifndef FA_FP8_INORDER
#define FA_FP8_INORDER -1
#endif
#ifndef FA_FP8_MMA_POLL
#define FA_FP8_MMA_POLL 0
#endif

// Four fp32 values -> four e4m3 codes in one 32-bit word (value k in byte k), round to nearest
// even, saturating to the finite range.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

template <int D, int NQT>
struct Fp8Cfg {
  static constexpr int BM = 128;                       // query rows per tile (MMA M)
  static constexpr int BN = 128;                       // keys per KV tile
  static constexpr int SWB = D >= 128 ? 128 : 64;      // swizzle span in bytes (= elements)
  static constexpr uint32_t LAYOUT = SWB == 128 ? 2u : 4u;
  static constexpr int KB = D / SWB;                   // swizzle blocks across d
  static constexpr int QTILE_BYTES = BM * D;
  static constexpr int KVTILE_BYTES = BN * D;
  static constexpr int STAGES = D == 256 ? 2 : 4;
  static constexpr int SOFTMAX_WARPS = 4 * NQT;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int THREADS = (SOFTMAX_WARPS + 4) * 32;
  static constexpr bool REALLOC = NQT == 2;
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int CTRL_REGS = 104;
  static constexpr int SOFTMAX_REGS = 200;
  static_assert(!REALLOC || CTRL_REGS * 128 + SOFTMAX_REGS * 256 <= LAUNCH_REGS * THREADS,
                "register split exceeds the launch allocation");
  static constexpr int TMEM_S = 0;                     // S_t at column t*BN (P^_t: first 32)
  static constexpr int TMEM_O = NQT * BN;              // O_t at TMEM_O + t*D
  static constexpr int TMEM_COLS = 512;
  static_assert(NQT * (BN + D) <= TMEM_COLS, "tensor memory budget");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQT * QTILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KVTILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KVTILE_BYTES;
  static constexpr int NBAR = 2 + 4 * STAGES + 4 * NQT + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t IDESC_S = idesc_e4m3_f32(BM, BN, 0, 0);   // Q8, K8 both K-major
  static constexpr uint32_t IDESC_PV = idesc_e4m3_f32(BM, D, 0, 1);   // P^ (tmem), V8 MN-major
};

// p.scale_log2 = s * q_scale * k_scale * log2(e); v_scale multiplies the output.
template <int D, bool CAUSAL, int NQT>
__global__ void __launch_bounds__(Fp8Cfg<D, NQT>::THREADS, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdParams p,
                      const float v_scale) {
  using C = Fp8Cfg<D, NQT>;
  using Unit = FwdUnit<NQT, CAUSAL, false>;
  constexpr bool kInorder = FA_FP8_INORDER == 1 || (FA_FP8_INORDER < 0 && !CAUSAL);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  const uint32_t BAR_Q = bar(0);
  const uint32_t BAR_QE = bar(1);
  auto BAR_KF = [&](int s) { return bar(2 + s); };
  auto BAR_KE = [&](int s) { return bar(2 + C::STAGES + s); };
  auto BAR_VF = [&](int s) { return bar(2 + 2 * C::STAGES + s); };
  auto BAR_VE = [&](int s) { return bar(2 + 3 * C::STAGES + s); };
  auto BAR_SF = [&](int t) { return bar(2 + 4 * C::STAGES + t); };
  auto BAR_PF = [&](int t) { return bar(2 + 4 * C::STAGES + NQT + t); };
  auto BAR_OD = [&](int t) { return bar(2 + 4 * C::STAGES + 2 * NQT + t); };
  auto BAR_OF = [&](int t) { return bar(2 + 4 * C::STAGES + 3 * NQT + t); };
  const uint32_t BAR_DRAIN = bar(C::NBAR - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  Waiter W{abort_flag, p.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    mbar_init(BAR_QE, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR_KF(s), 1);
      mbar_init(BAR_KE(s), 1);
      mbar_init(BAR_VF(s), 1);
      mbar_init(BAR_VE(s), 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(BAR_SF(t), 1);
      mbar_init(BAR_PF(t), 4);
      mbar_init(BAR_OD(t), 1);
      mbar_init(BAR_OF(t), 4);
    }
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

  if (warp >= C::SOFTMAX_WARPS) {
    // ================================================================ control warpgroup
    if constexpr (C::REALLOC) regs_dec<C::CTRL_REGS>();
    if (warp == C::PRODUCER_WARP) {
      // -------------------------------------------------------------- TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int kv_it = 0, kq = 0, q_n = 0;
        int k_n[C::STAGES], v_n[C::STAGES];  // loads issued per stage (one phase each)
#pragma unroll
        for (int s = 0; s < C::STAGES; ++s) k_n[s] = v_n[s] = 0;
        bool ok = true;
        for (int k = 0;; ++k) {
          const int u = fwd_unit_of(k, cta, G, p.units);
          if (u < 0) break;
          const Unit un(u, p);
          if (un.J == 0) continue;
          if (kq > 0 && !(ok = W.wait(BAR_QE, (kq - 1) & 1, 3))) break;
          int q_tiles = 0;
          for (int t = 0; t < NQT; ++t) q_tiles += (un.nkv[t] > 0);
          mbar_arrive_expect_tx(BAR_Q, q_tiles * C::QTILE_BYTES);
          for (int t = 0; t < NQT; ++t) {
            if (un.nkv[t] == 0) continue;
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_Q + t * C::QTILE_BYTES + kb * (C::BM * C::SWB), &tmQ,
                          BAR_Q, kb * C::SWB, un.q0 + t * C::BM, un.head);
          }
          ++q_n;
          for (int j = 0; j < un.J; ++j) {
            const int g = kv_it + j;
            const int s = g % C::STAGES;
            const uint32_t ph = (g / C::STAGES) & 1;
            if (!(ok = W.wait(BAR_KE(s), ph ^ 1, 1))) break;
            mbar_arrive_expect_tx(BAR_KF(s), C::KVTILE_BYTES);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_K + s * C::KVTILE_BYTES + kb * (C::BN * C::SWB), &tmK,
                          BAR_KF(s), kb * C::SWB, (un.kt0 + j) * C::BN, un.kv_head);
            ++k_n[s];
            if (!(ok = W.wait(BAR_VE(s), ph ^ 1, 2))) break;
            mbar_arrive_expect_tx(BAR_VF(s), C::KVTILE_BYTES);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_3d(sbase + C::OFF_V + s * C::KVTILE_BYTES + kb * (C::BN * C::SWB), &tmV,
                          BAR_VF(s), kb * C::SWB, (un.kt0 + j) * C::BN, un.kv_head);
            ++v_n[s];
          }
          if (!ok) break;
          kv_it += un.J;
          ++kq;
        }
        if (!ok) {
          // drain: the last phase of every barrier that has loads issued (at most that one is
          // outstanding), so every copy lands before the CTA exits
          if (q_n > 0) W.drain(BAR_Q, (q_n - 1) & 1);
#pragma unroll
          for (int s = 0; s < C::STAGES; ++s) {
            if (k_n[s] > 0) W.drain(BAR_KF(s), (k_n[s] - 1) & 1);
            if (v_n[s] > 0) W.drain(BAR_VF(s), (v_n[s] - 1) & 1);
          }
        }
      }
    } else if (warp == C::MMA_WARP) {
      // -------------------------------------------------------------- MMA issuer
      W.sleep = !FA_FP8_MMA_POLL;
      // Same order as the bf16 forward: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).
      if (lane == 0) {
        auto issue_s = [&](int t, uint32_t k_addr) {
          const uint32_t q_addr = sbase + C::OFF_Q + t * C::QTILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            // 32 e4m3 = 32 bytes of K per instruction, inside a swizzle row of SWB bytes
            const uint32_t koff = (kk * 32 / C::SWB) * (128 * C::SWB) + (kk * 32) % C::SWB;
            mma_ss_f8(tmem + C::TMEM_S + t * C::BN,
                      sdesc_swz(q_addr + koff, 16, 8 * C::SWB, C::LAYOUT),
                      sdesc_swz(k_addr + koff, 16, 8 * C::SWB, C::LAYOUT), C::IDESC_S, kk > 0);
          }
          tc_commit(BAR_SF(t));
        };
        int kv_it = 0;
        int tit[NQT], tun[NQT];
#pragma unroll
        for (int t = 0; t < NQT; ++t) tit[t] = tun[t] = 0;
        bool ok = true;
        int kq = 0;
        for (int k = 0; ok; ++k) {
          const int u = fwd_unit_of(k, cta, G, p.units);
          if (u < 0) break;
          const Unit un(u, p);
          const int J = un.J;
          if (J == 0) continue;
          const int s0 = kv_it % C::STAGES;
          if (!(ok = W.wait(BAR_Q, kq & 1, 10))) break;
          if (!(ok = W.wait(BAR_KF(s0), (kv_it / C::STAGES) & 1, 11))) break;
          for (int t = 0; t < NQT && ok; ++t) {
            if (un.nkv[t] == 0) continue;
            if (!kInorder && tit[t] > 0 && !(ok = W.wait(BAR_OD(t), (tit[t] - 1) & 1, 12)))
              break;
            tc_fence_after();
            issue_s(t, sbase + C::OFF_K + s0 * C::KVTILE_BYTES);
          }
          if (!ok) break;
          tc_commit(BAR_KE(s0));
          if (J == 1) tc_commit(BAR_QE);
          for (int j = 0; ok && j < J; ++j) {
            const int g = kv_it + j;
            const int s = g % C::STAGES;
            const int s1 = (g + 1) % C::STAGES;
            const uint32_t v_addr = sbase + C::OFF_V + s * C::KVTILE_BYTES;
            const uint32_t k1_addr = sbase + C::OFF_K + s1 * C::KVTILE_BYTES;
            if (!(ok = W.wait(BAR_VF(s), (g / C::STAGES) & 1, 13))) break;
            bool k_ready = false;
            for (int t = 0; t < NQT && ok; ++t) {
              if (j >= un.nkv[t]) continue;
              if (!(ok = W.wait(BAR_PF(t), tit[t] & 1, 14))) break;
              if (j == 0 && tun[t] > 0 && !(ok = W.wait(BAR_OF(t), (tun[t] - 1) & 1, 15))) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < C::BN / 32; ++kk) {
                // P^ packs 4 keys per column: 32 keys = 8 columns; V8 rows (keys) are SWB bytes
                // apart, so a 32-key slice is 32 * SWB bytes further on; d blocks of SWB
                // elements are BN * SWB bytes apart (LBO)
                mma_ts_f8(tmem + C::TMEM_O + t * D, tmem + C::TMEM_S + t * C::BN + kk * 8,
                          sdesc_swz(v_addr + kk * 32 * C::SWB, C::BN * C::SWB, 8 * C::SWB,
                                    C::LAYOUT),
                          C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
              }
              tc_commit(BAR_OD(t));
              if (j + 1 < un.nkv[t]) {
                if (!k_ready && !(ok = W.wait(BAR_KF(s1), ((g + 1) / C::STAGES) & 1, 16))) break;
                k_ready = true;
                if (!kInorder && !(ok = W.wait(BAR_OD(t), tit[t] & 1, 17))) break;
                tc_fence_after();
                issue_s(t, k1_addr);
              }
              ++tit[t];
            }
            if (!ok) break;
            tc_commit(BAR_VE(s));
            if (k_ready) tc_commit(BAR_KE(s1));
            if (j == J - 2) tc_commit(BAR_QE);
          }
          if (!ok) break;
#pragma unroll
          for (int t = 0; t < NQT; ++t) tun[t] += (un.nkv[t] > 0);
          kv_it += J;
          ++kq;
        }
        tc_commit(BAR_DRAIN);
        W.drain(BAR_DRAIN, 0);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    if constexpr (C::REALLOC) regs_inc<C::SOFTMAX_REGS>();
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::TMEM_S + t * C::BN;
    const uint32_t tO = tmem + lane_base + C::TMEM_O + t * D;
    int tit = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = fwd_unit_of(k, cta, G, p.units);
      if (u < 0) break;
      const Unit un(u, p);
      const int n = un.nkv[t];
      const int row = un.q0 + t * C::BM + r;
      const bool valid = row < p.Nq;
      if (n == 0) continue;
      float m = -INFINITY;  // row maximum so far (log2 units of the scaled scores)
      float l = 0.f;        // sum of 2^8 exp2(x - m) in fp32
      for (int j = 0; j < n; ++j, ++tit) {
        if (!(ok = W.wait_warp(BAR_SF(t), tit & 1, 20))) break;
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, s[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld(s[c]);
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
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(s[c][e]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        // exact rescale: the reference follows every increase of the row maximum
        const float m_new = fmaxf(m, mx * p.scale_log2);
        const float alpha = (j == 0 || m_new == m) ? 1.f : ex2(m - m_new);
        uint64_t sum2[2] = {0ull, 0ull};
        const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2pack(8.f - m_new, 8.f - m_new);  // weights scaled by 2^8
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x0, x1, x2, x3;
            f2unpack(ffma2(f2pack(__uint_as_float(s[c][4 * e]), __uint_as_float(s[c][4 * e + 1])),
                           sc2, nm2),
                     x0, x1);
            f2unpack(ffma2(f2pack(__uint_as_float(s[c][4 * e + 2]),
                                  __uint_as_float(s[c][4 * e + 3])),
                           sc2, nm2),
                     x2, x3);
            float p0, p1, p2, p3;
            if ((FA_FP8_POLY_MASK >> e) & 1) {
              exp2_fma2(x0, x1, p0, p1);
              exp2_fma2(x2, x3, p2, p3);
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
              p2 = ex2(x2);
              p3 = ex2(x3);
            }
            pk[8 * c + e] = pack_e4m3x4(p0, p1, p2, p3);
            sum2[e & 1] = fadd2(sum2[e & 1], fadd2(f2pack(p0, p1), f2pack(p2, p3)));
          }
        }
        // P^ (e4m3, 4 keys per column) over the first 32 columns of S_t
        tmem_st32(tS + 0, pk);
        {
          float a0, a1;
          f2unpack(fadd2(sum2[0], sum2[1]), a0, a1);
          l = l * alpha + (a0 + a1);
        }
        m = m_new;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O_t holds PV_t(j-1) (S_t(j) was issued only after it completed); rescale it
          if (!(ok = W.wait_warp(BAR_OD(t), (tit - 1) & 1, 21))) break;
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
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR_PF(t));
      }
      if (!ok) break;
      // ---- epilogue: O = v_scale * O / l -> bf16; L = (m + log2(l) - 8) ln 2
      if (!(ok = W.wait_warp(BAR_OD(t), (tit - 1) & 1, 22))) break;
      tc_fence_after();
      const float inv_l = v_scale / l;
      __nv_bfloat16* orow = p.o + (size_t(un.head) * p.Nq + row) * D;
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
        uint4 pkd[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pw[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = pkd[e];
        }
      }
      if (valid) p.lse[size_t(un.head) * p.Nq + row] = (m + lg2(l) - 8.f) * 0.69314718055994531f;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

__global__ void fa_selftest_exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y,
                                            int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    exp2_fma2(x[i], x[i + 1], y[i], y[i + 1]);
  } else if (i < n) {
    float d;
    exp2_fma2(x[i], x[i], y[i], d);
  }
}

}  // namespace fattn
