// Weighted centroid update of one k-means (Lloyd) step over the LoopVQ
// codebooks (sm_100a). The assignment half of the step is the encoder
// itself, writing indices to an array instead of the pool.
//
// The codebooks are fitted offline with Fisher-weighted k-means (airadar.tv,
// opening paragraph). With the per-element weighted squared distance of the
// encoder, sum_i w_i (s_i - C[e]_i)^2, the centroid that minimises a
// cluster's distortion is, element by element, the weighted mean
//     C[e]_i = sum_{n in e} w_ni s_ni / sum_{n in e} w_ni,
// and an element whose weight sum is zero (an empty cluster, or zero
// weights) keeps its value.
//
// One CTA per codebook (channel group j, kv-head h): shared memory holds
// num[e][i] and den[e][i] in rows of D + 1 floats (so that the lanes' rows
// spread over the banks); the threads take tokens tid, tid + T, .. and add
// each sub-vector into the row of its centroid with shared-memory float
// atomics (so the float32 sums are order-dependent in their last bits); the
// CTA then rewrites its codebook in place.

#include "common.cuh"
#include "encode_common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kKmThreads = 256;

template <int C, int G>
__global__ void __launch_bounds__(kKmThreads) kmeans_update_kernel(const EncodeParams p, float* cb) {
  constexpr int D = C * G;
  constexpr int DP = D + 1;                            // padded row
  extern __shared__ float acc[];                       // num [E][DP], then den [E][DP]
  float* num = acc;
  float* den = acc + kE * DP;
  const int j = blockIdx.x, h = blockIdx.y;
  for (int i = threadIdx.x; i < 2 * kE * DP; i += kKmThreads) acc[i] = 0.f;
  __syncthreads();
  const uint8_t* as = p.assign + (static_cast<int64_t>(h) * p.J + j) * p.n_tokens;
  for (int n = threadIdx.x; n < p.n_tokens; n += kKmThreads) {
    const int e = as[n];
    float s[D], w[D];
    load_subvector<C, G>(p, n, j, h, s, w);
#pragma unroll
    for (int i = 0; i < D; ++i) {
      atomicAdd(num + e * DP + i, w[i] * s[i]);
      atomicAdd(den + e * DP + i, w[i]);
    }
  }
  __syncthreads();
  // element i = tau*C + ch of centroid e sits at cb + h*stride_head + tau*stride_loop + (j*E + e)*C + ch
  float* cbj = cb + h * p.cb_stride_head + static_cast<int64_t>(j) * kE * C;
  for (int k = threadIdx.x; k < kE * D; k += kKmThreads) {
    const int e = k / D, i = k % D;
    const float dn = den[e * DP + i];
    if (dn > 0.f) cbj[(i / C) * p.cb_stride_loop + e * C + i % C] = num[e * DP + i] / dn;
  }
}

template <int C, int G>
loopvq_status launch_update(const EncodeParams& p, float* cb, int J, int H, cudaStream_t st) {
  constexpr size_t smem = 2u * kE * (C * G + 1) * sizeof(float);
  static_assert(smem <= 227u * 1024u, "accumulators fit shared memory");
  if (smem > 48u * 1024u &&
      cudaFuncSetAttribute(kmeans_update_kernel<C, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  kmeans_update_kernel<C, G><<<dim3(J, H), kKmThreads, smem, st>>>(p, cb);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace

loopvq_status launch_kmeans_update(const EncodeArgs& a, float* codebooks) {
  const Geometry& g = *a.geo;
  const EncodeParams p = encode_params(a);
  // the same (layer, head 0, gamma, kv, tau 0) offset as p.cb, writable
  float* cb = codebooks + a.layer * g.cb_stride_layer + a.gamma * g.cb_stride_group +
              a.kv * g.cb_stride_kv;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  switch (g.c * 100 + g.g) {
    case 404: return launch_update<4, 4>(p, cb, g.J, g.Hkv, st);
    case 804: return launch_update<8, 4>(p, cb, g.J, g.Hkv, st);
    case 204: return launch_update<2, 4>(p, cb, g.J, g.Hkv, st);
    case 402: return launch_update<4, 2>(p, cb, g.J, g.Hkv, st);
    case 802: return launch_update<8, 2>(p, cb, g.J, g.Hkv, st);
    case 208: return launch_update<2, 8>(p, cb, g.J, g.Hkv, st);
    case 408: return launch_update<4, 8>(p, cb, g.J, g.Hkv, st);
    case 401: return launch_update<4, 1>(p, cb, g.J, g.Hkv, st);
    case 801: return launch_update<8, 1>(p, cb, g.J, g.Hkv, st);
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace loopvq
