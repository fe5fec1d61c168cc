// Nearest-centroid encoder, direct form (sm_100a CUDA cores), and the
// dispatch among the three encoder forms: a warp per token for the small
// batches of the window eviction, this kernel for mid-sized batches, and the
// tensor-core form (encode_tc.cu) for prefill-sized ones.
//
// One CTA = (tile of 128 tokens, channel group j, kv-head h). The CTA stages
// the E x D codebook of (layer, h, gamma, K/V, j) in shared memory as
// [E][D] (every thread then reads the same codeword: broadcast), and each
// thread encodes one token's sub-vector
//     s[tau*c + ch] = x[tau][n][h][j*c + ch],   tau < g, ch < c
// by scanning all 256 codewords with the float32 weighted squared distance
// sum_i w_i (s_i - C[e]_i)^2, keeping the first minimum (smallest index on
// exact ties). The index byte goes to the rotated slot position of the pool.

#include "common.cuh"
#include "encode_common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kEncThreads = 128;
constexpr int kEncWarpThreads = 256;    // small batches: one CTA per (group, head), a warp per token
constexpr int kEncWarpMaxTokens = 64;   // batches up to this size take the warp form
constexpr int kEncTcMinTokens = 2048;   // batches from this size take the tensor-core form

// Small batches (the tokens leaving the recent window at each decode step):
// one CTA per (group j, head h) stages the codebook of (j, h) once as
// [tau][E][c]; each warp takes tokens warp, warp+8, .., the lanes scan
// centroids lane, lane+32, .. with the same float32 weighted distance and
// term order as encode_kernel, and a shuffle argmin keeps the smallest
// index among equal distances.
// The body of the small-batch form for (group j, head h): stages the
// codebook of (j, h) once as [tau][E][c] in `cbs`; each warp takes tokens
// warp, warp+8, .., the lanes scan centroids lane, lane+32, .. with the same
// float32 weighted distance and term order as encode_kernel, and a shuffle
// argmin keeps the smallest index among equal distances.
template <int C, int G>
__device__ __forceinline__ void encode_tokens_warp(const EncodeParams& p, int j, int h, float* cbs) {
  constexpr int D = C * G;
  const float* cb = p.cb + h * p.cb_stride_head + static_cast<int64_t>(j) * kE * C;
  for (int i = threadIdx.x * 4; i < G * kE * C; i += kEncWarpThreads * 4) {
    const int tau = i / (kE * C), r = i % (kE * C);
    cp_async16(cbs + i, cb + tau * p.cb_stride_loop + r);
  }
  cp_async_wait_all();
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int n = warp; n < p.n_tokens; n += kEncWarpThreads / 32) {
    const int64_t slot = token_slot(p, n);
    if (slot < 0 || slot >= p.n_slots) continue;   // warp-uniform
    float s[D], w[D];
    load_subvector<C, G>(p, n, j, h, s, w);
    float best = INFINITY;
    int best_e = 0;
#pragma unroll 2
    for (int k = 0; k < kE / 32; ++k) {
      const int e = 32 * k + lane;
      float dist = 0.f;
#pragma unroll
      for (int tau = 0; tau < G; ++tau) {
        const float* cw = cbs + (tau * kE + e) * C;
#pragma unroll
        for (int ch = 0; ch < C; ++ch) {
          const float df = s[tau * C + ch] - cw[ch];
          dist = fmaf(w[tau * C + ch] * df, df, dist);
        }
      }
      if (dist < best) {
        best = dist;
        best_e = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, best, off);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
      if (od < best || (od == best && oe < best_e)) {
        best = od;
        best_e = oe;
      }
    }
    if (lane == 0) store_index(p, slot, j, h, best_e);
  }
}

// Small batches (the tokens leaving the recent window at each decode step):
// one CTA per (group j, head h).
template <int C, int G>
__global__ void __launch_bounds__(kEncWarpThreads) encode_warp_kernel(const EncodeParams p) {
  __shared__ __align__(16) float cbs[G * kE * C];
  encode_tokens_warp<C, G>(p, blockIdx.x, blockIdx.y, cbs);
}

// The window eviction of one decode step in one launch: CTA (j, h, z)
// encodes the tokens for (group j, head h) of combination z = (layer*G +
// gamma)*2 + kv. Combination z reads its g loop slices at x + z*x_combo
// ([g][n][Hkv][d] bf16) and writes the K or V plane of (layer, gamma).
struct EvictParams {
  EncodeParams base;            // layer 0, gamma 0, K; x of combination 0
  int64_t x_combo;              // elements between combinations
  int64_t cb_stride_layer, cb_stride_group, cb_stride_kv;
  int64_t pool_stride_layer, pool_stride_group;
  int G;
};

template <int C, int G>
__global__ void __launch_bounds__(kEncWarpThreads) encode_evict_kernel(const EvictParams e) {
  __shared__ __align__(16) float cbs[G * kE * C];
  const int z = blockIdx.z, kv = z & 1, gamma = (z >> 1) % e.G, layer = (z >> 1) / e.G;
  EncodeParams p = e.base;
  p.x = e.base.x + z * e.x_combo;
  p.cb = e.base.cb + layer * e.cb_stride_layer + gamma * e.cb_stride_group + kv * e.cb_stride_kv;
  p.pool = e.base.pool + layer * e.pool_stride_layer + gamma * e.pool_stride_group;
  p.kv = kv;
  encode_tokens_warp<C, G>(p, blockIdx.x, blockIdx.y, cbs);
}

template <int C, int G>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const EncodeParams p) {
  constexpr int D = C * G;
  __shared__ __align__(16) float cbs[kE * D];
  const int j = blockIdx.y, h = blockIdx.z;
  const float* cb = p.cb + h * p.cb_stride_head;
  for (int i = threadIdx.x; i < kE * D; i += kEncThreads) {
    const int e = i / D, k = i % D, tau = k / C, ch = k % C;
    cbs[i] = cb[tau * p.cb_stride_loop + (static_cast<int64_t>(j) * kE + e) * C + ch];
  }
  __syncthreads();
  const int n = blockIdx.x * kEncThreads + threadIdx.x;
  if (n >= p.n_tokens) return;
  const int64_t slot = token_slot(p, n);
  if (slot < 0 || slot >= p.n_slots) return;

  float s[D], w[D];
  load_subvector<C, G>(p, n, j, h, s, w);

  float best = INFINITY;
  int best_e = 0;
#pragma unroll 2
  for (int e = 0; e < kE; ++e) {
    const float4* c4 = reinterpret_cast<const float4*>(cbs + e * D);
    float dist = 0.f;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
      const float4 cw = c4[k];
      const float d0 = s[4 * k] - cw.x, d1 = s[4 * k + 1] - cw.y;
      const float d2 = s[4 * k + 2] - cw.z, d3 = s[4 * k + 3] - cw.w;
      dist = fmaf(w[4 * k] * d0, d0, dist);
      dist = fmaf(w[4 * k + 1] * d1, d1, dist);
      dist = fmaf(w[4 * k + 2] * d2, d2, dist);
      dist = fmaf(w[4 * k + 3] * d3, d3, dist);
    }
    if (dist < best) {
      best = dist;
      best_e = e;
    }
  }

  store_index(p, slot, j, h, best_e);
}

template <int C, int G>
loopvq_status launch_enc(const EncodeParams& p, int J, int H, cudaStream_t st) {
  if (p.n_tokens >= kEncTcMinTokens && encode_tc_supported(C, G)) {
    const loopvq_status r = launch_encode_tc(p, C, G, J, H, st);
    if (r != LOOPVQ_ERR_UNSUPPORTED) return r;       // else: inputs TMA cannot describe, direct form
  }
  if (p.n_tokens <= kEncWarpMaxTokens) {
    encode_warp_kernel<C, G><<<dim3(J, H), kEncWarpThreads, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
  }
  const dim3 grid((p.n_tokens + kEncThreads - 1) / kEncThreads, J, H);
  encode_kernel<C, G><<<grid, kEncThreads, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

template <int C, int G>
loopvq_status launch_evict(const EvictParams& e, int J, int H, int combos, cudaStream_t st) {
  encode_evict_kernel<C, G><<<dim3(J, H, combos), kEncWarpThreads, 0, st>>>(e);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace

loopvq_status launch_encode_evict(const EncodeArgs& a) {
  const Geometry& g = *a.geo;
  if (a.n_tokens > kEncWarpMaxTokens) return LOOPVQ_ERR_UNSUPPORTED;
  EvictParams e{};
  e.base = encode_params(a);                           // layer 0, gamma 0, K
  e.x_combo = static_cast<int64_t>(g.g) * a.n_tokens * g.Hkv * g.d;
  e.cb_stride_layer = g.cb_stride_layer;
  e.cb_stride_group = g.cb_stride_group;
  e.cb_stride_kv = g.cb_stride_kv;
  e.pool_stride_layer = g.pool_stride_layer;
  e.pool_stride_group = g.pool_stride_group;
  e.G = g.G;
  const int combos = g.L * g.G * 2;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  switch (g.c * 100 + g.g) {
    case 404: return launch_evict<4, 4>(e, g.J, g.Hkv, combos, st);
    case 804: return launch_evict<8, 4>(e, g.J, g.Hkv, combos, st);
    case 204: return launch_evict<2, 4>(e, g.J, g.Hkv, combos, st);
    case 402: return launch_evict<4, 2>(e, g.J, g.Hkv, combos, st);
    case 802: return launch_evict<8, 2>(e, g.J, g.Hkv, combos, st);
    case 208: return launch_evict<2, 8>(e, g.J, g.Hkv, combos, st);
    case 408: return launch_evict<4, 8>(e, g.J, g.Hkv, combos, st);
    case 401: return launch_evict<4, 1>(e, g.J, g.Hkv, combos, st);
    case 801: return launch_evict<8, 1>(e, g.J, g.Hkv, combos, st);
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
}

EncodeParams encode_params(const EncodeArgs& a) {
  const Geometry& g = *a.geo;
  EncodeParams p{};
  p.x = static_cast<const uint16_t*>(a.x);
  p.x_loop_stride = a.x_loop_stride;
  p.x_token_stride = a.x_token_stride;
  p.w = a.w;
  p.w_loop_stride = a.w_loop_stride;
  p.w_token_stride = a.w_token_stride;
  p.cb = a.codebooks + a.layer * g.cb_stride_layer + a.gamma * g.cb_stride_group +
         a.kv * g.cb_stride_kv;
  p.cb_stride_head = g.cb_stride_head;
  p.cb_stride_loop = g.cb_stride_loop;
  p.slot_mapping = a.slot_mapping;
  p.assign = a.assign;
  p.pool = (a.pool != nullptr) ? a.pool + a.layer * g.pool_stride_layer + a.gamma * g.pool_stride_group
                               : nullptr;
  p.pool_stride_head = g.pool_stride_head;
  p.page_bytes = g.page_bytes;
  p.plane_bytes = g.plane_bytes;
  p.n_slots = (a.assign != nullptr) ? a.n_tokens : static_cast<int64_t>(g.n_pages) * g.Pg;
  p.status = encode_status_word();
  p.n_tokens = a.n_tokens;
  p.d = g.d;
  p.Pg = g.Pg;
  p.J = g.J;
  p.LB = g.LB;
  p.GR = g.GR;
  p.kv = a.kv;
  return p;
}

loopvq_status launch_encode(const EncodeArgs& a) {
  const Geometry& g = *a.geo;
  const EncodeParams p = encode_params(a);
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  switch (g.c * 100 + g.g) {
    case 404: return launch_enc<4, 4>(p, g.J, g.Hkv, st);
    case 804: return launch_enc<8, 4>(p, g.J, g.Hkv, st);
    case 204: return launch_enc<2, 4>(p, g.J, g.Hkv, st);
    case 402: return launch_enc<4, 2>(p, g.J, g.Hkv, st);
    case 802: return launch_enc<8, 2>(p, g.J, g.Hkv, st);
    case 208: return launch_enc<2, 8>(p, g.J, g.Hkv, st);
    case 408: return launch_enc<4, 8>(p, g.J, g.Hkv, st);
    case 401: return launch_enc<4, 1>(p, g.J, g.Hkv, st);
    case 801: return launch_enc<8, 1>(p, g.J, g.Hkv, st);
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace loopvq
