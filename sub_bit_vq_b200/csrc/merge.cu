// Split-K log-sum-exp merge of decode partials (shared by the LoopVQ and
// the bf16-KV decode kernels).
//
// Partial s of a (sequence, query head) pair holds (m_s, l_s, o_s[d]) with
// m in log2 units, l = sum 2^(x - m) and o = sum 2^(x - m) v (unnormalised).
// The merge is  M = max m_s,  L = sum l_s 2^(m_s - M),
// out = sum o_s 2^(m_s - M) / L,  lse = ln2 * (M + log2 L).

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

// One warp per pair. partials [pairs][S][d+2] -> out [pairs][d], lse [pairs].
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ partials, int pairs,
                                                    int S, int d, int out_dtype, void* out,
                                                    float* lse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x * 4 + warp;
  if (pair >= pairs) return;
  const int stride = d + 2;
  const float* P = partials + static_cast<size_t>(pair) * S * stride;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, P[s * stride]);
  M = warp_max(M);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int s = lane; s < S; s += 32) {
      const float m = P[s * stride];
      if (m != -INFINITY) L += P[s * stride + 1] * fast_exp2(m - M);
    }
  }
  L = warp_sum(L);
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  for (int ch = lane; ch < d; ch += 32) {
    float o = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float m = P[s * stride];
        if (m != -INFINITY) o = fmaf(P[s * stride + 2 + ch], fast_exp2(m - M), o);
      }
    }
    o *= inv;
    if (out_dtype == LOOPVQ_DTYPE_F32) {
      static_cast<float*>(out)[static_cast<size_t>(pair) * d + ch] = o;
    } else {
      static_cast<__nv_bfloat16*>(out)[static_cast<size_t>(pair) * d + ch] = __float2bfloat16_rn(o);
    }
  }
  if (lane == 0 && lse != nullptr)
    lse[pair] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace

loopvq_status launch_merge(const float* partials, int pairs, int splits, int d, int out_dtype,
                           void* out, float* lse, void* stream) {
  const dim3 grid((pairs + 3) / 4);
  merge_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(partials, pairs, splits, d,
                                                                     out_dtype, out, lse);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace loopvq
