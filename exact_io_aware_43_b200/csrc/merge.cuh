// merge.cuh -- combine the partial results of a split-key forward (sm_100a).
//
// With the keys of a head cut into S ranges, range s gives each query row a partial output O_s
// (normalised over its own keys) and L_s = ln sum_{j in s} exp(score_j).  The exact result over
// all keys follows from the associativity of the online-softmax update (robocikowo.com "Flash
// Attention": O <- rescale(O_prev, m_old, m_new) + ...; chipfoundryservices.com glossary "Online
// Softmax Trick"):
//     L = ln sum_s exp(L_s),      O = sum_s exp(L_s - L) O_s.
// Ranges a row cannot see carry L_s = -inf and weigh 0.  One warp per query row; lane c holds
// columns c, c + 32, ... (coalesced reads of every partial row).  HBM bound: it reads S rows of
// 4*D + 4 bytes and writes 2*D + 4 per query row.
#pragma once

#include "sm100.cuh"

namespace fattn {

template <int D>
__global__ void __launch_bounds__(256)
    fa_fwd_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                        __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int splits,
                        long long rows) {
  constexpr int PER_LANE = D / 32;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = warp0; row < rows; row += nwarps) {
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, lse_part[s * rows + row]);
    float acc[PER_LANE];
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) acc[c] = 0.f;
    float L = -INFINITY;
    if (m != -INFINITY) {
      float sum = 0.f;
      for (int s = 0; s < splits; ++s) sum += expf(lse_part[s * rows + row] - m);
      L = m + logf(sum);
      for (int s = 0; s < splits; ++s) {
        const float w = expf(lse_part[s * rows + row] - L);  // 0 for an empty range
        if (w == 0.f) continue;
        const float* src = o_part + ((long long)s * rows + row) * D;
#pragma unroll
        for (int c = 0; c < PER_LANE; ++c) acc[c] = fmaf(w, src[lane + 32 * c], acc[c]);
      }
    }
    __nv_bfloat16* dst = o + row * D;
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) dst[lane + 32 * c] = __float2bfloat16_rn(acc[c]);
    if (lane == 0) lse[row] = L;
  }
}

}  // namespace fattn
