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

// The window eviction of one decode step in one launch. The work is one
// unit per codebook u = (z, h, j), z = (layer*G + gamma)*2 + kv: the
// n_tokens tokens' sub-vectors of (group j, head h) in combination z (whose
// g loop slices are at x + z*x_combo, [g][n][Hkv][d] bf16) are encoded with
// that codebook and written to the K or V plane of (layer, gamma). Every
// unit reads a different 16 KB codebook once, so the kernel streams the
// model's codebooks: a persistent grid takes units u = blockIdx.x + k *
// gridDim.x, with kEvStages codebooks (and their tokens) in flight by
// cp.async. Thread t scores centroids t and t + 128 for every token, two at
// a time in packed float32x2 arithmetic in encode_kernel's term order (the
// weights are all 1); a warp's argmin takes redux.sync minima, and the four
// warps' bests meet in shared memory (smallest index on equal distances).
struct EvictParams {
  EncodeParams base;            // layer 0, gamma 0, K; x of combination 0
  int64_t x_combo;              // elements between combinations
  int64_t cb_stride_layer, cb_stride_group, cb_stride_kv;
  int64_t pool_stride_layer, pool_stride_group;
  int G, H, combos;
};

constexpr int kEvThreads = 128;
constexpr int kEvStages = 2;

template <int C, int G>
struct EvGeo {
  static constexpr int D = C * G;
  static constexpr int CBF = G * kE * C;                        // floats of one codebook
  static constexpr int CB_OFF = 0;                              // [kEvStages][CBF] float
  static constexpr int X_OFF = CB_OFF + kEvStages * CBF * 4;    // [kEvStages][64][D] bf16
  static constexpr int S_OFF = X_OFF + kEvStages * kEncWarpMaxTokens * D * 2;   // [64][D] (s, s)
  static constexpr int BEST_OFF = S_OFF + kEncWarpMaxTokens * D * 8;           // [64][4] (dist, e)
  static constexpr int SLOT_OFF = BEST_OFF + kEncWarpMaxTokens * 4 * 8;        // [64] int64
  static constexpr int SMEM = SLOT_OFF + kEncWarpMaxTokens * 8;
};

__device__ __forceinline__ void cp_async_bytes(void* smem_dst, const void* gmem_src, int bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  if (bytes == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
  else if (bytes == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(d), "l"(gmem_src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

template <int C, int G>
__global__ void __launch_bounds__(kEvThreads) encode_evict_kernel(const EvictParams ep) {
  using Geo = EvGeo<C, G>;
  constexpr int D = Geo::D, CBF = Geo::CBF;
  extern __shared__ __align__(16) unsigned char esm[];
  float* cbst = reinterpret_cast<float*>(esm + Geo::CB_OFF);
  uint16_t* xst = reinterpret_cast<uint16_t*>(esm + Geo::X_OFF);
  uint64_t* sdup = reinterpret_cast<uint64_t*>(esm + Geo::S_OFF);
  float2* wbest = reinterpret_cast<float2*>(esm + Geo::BEST_OFF);
  int64_t* slots = reinterpret_cast<int64_t*>(esm + Geo::SLOT_OFF);
  const EncodeParams& b = ep.base;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int J = b.J, H = ep.H, n = b.n_tokens;
  const int U = J * H * ep.combos;
  for (int i = tid; i < n; i += kEvThreads) slots[i] = token_slot(b, i);

  // cp.async of unit u's codebook and tokens into stage `st` (one commit group
  // per thread even when u is past the end, so that the group count stays aligned)
  auto issue = [&](int u, int st) {
    if (u < U) {
      const int jj = u % J, h = (u / J) % H, z = u / (J * H);
      const int kv = z & 1, gamma = (z >> 1) % ep.G, layer = (z >> 1) / ep.G;
      const float* cb = b.cb + layer * ep.cb_stride_layer + gamma * ep.cb_stride_group + kv * ep.cb_stride_kv +
                        h * b.cb_stride_head + static_cast<int64_t>(jj) * kE * C;
      float* dst = cbst + st * CBF;
      for (int i = tid * 4; i < CBF; i += kEvThreads * 4) {
        const int tau = i / (kE * C), r = i % (kE * C);
        cp_async16(dst + i, cb + tau * b.cb_stride_loop + r);
      }
      const uint16_t* x = b.x + z * ep.x_combo + static_cast<int64_t>(h) * b.d + jj * C;
      uint16_t* xd = xst + st * kEncWarpMaxTokens * D;
      for (int i = tid; i < n * G; i += kEvThreads) {
        const int nn = i / G, tau = i % G;
        cp_async_bytes(xd + nn * D + tau * C, x + tau * b.x_loop_stride + nn * b.x_token_stride, 2 * C);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

#pragma unroll
  for (int k = 0; k < kEvStages - 1; ++k) issue(blockIdx.x + k * gridDim.x, k);
  for (int k = 0;; ++k) {
    const int u = blockIdx.x + k * gridDim.x;
    if (u >= U) break;
    const int u_j = u % J, u_h = (u / J) % H, u_z = u / (J * H);
    issue(blockIdx.x + (k + kEvStages - 1) * gridDim.x, (k + kEvStages - 1) % kEvStages);
    asm volatile("cp.async.wait_group %0;\n" ::"n"(kEvStages - 1) : "memory");
    __syncthreads();                                   // unit u's stage complete for every thread
    const int st = k % kEvStages;
    const uint16_t* xs = xst + st * kEncWarpMaxTokens * D;
    for (int i = tid; i < n * D; i += kEvThreads) {
      const float v = __uint_as_float(static_cast<uint32_t>(xs[i]) << 16);
      sdup[i] = f2_pack(v, v);
    }
    __syncthreads();
    // centroids tid and tid + 128, element i packed as (C[tid][i], C[tid + 128][i])
    const float* cbs = cbst + st * CBF;
    uint64_t cw[D];
#pragma unroll
    for (int tau = 0; tau < G; ++tau)
#pragma unroll
      for (int ch = 0; ch < C; ++ch)
        cw[tau * C + ch] = f2_pack(cbs[(tau * kE + tid) * C + ch], cbs[(tau * kE + tid + 128) * C + ch]);
    // four tokens at a time: four independent accumulation chains
    for (int n0 = 0; n0 < n; n0 += 4) {
      uint64_t dist[4] = {0ull, 0ull, 0ull, 0ull};   // (+0, +0)
#pragma unroll
      for (int i = 0; i < D; i += 2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nn = min(n0 + q, n - 1);           // a tail lane repeats the last token
          const ulonglong2 sv = *reinterpret_cast<const ulonglong2*>(sdup + nn * D + i);
          asm("{\n .reg .b64 df;\n"
              " sub.rn.f32x2 df, %1, %2;\n fma.rn.f32x2 %0, df, df, %0;\n"
              " sub.rn.f32x2 df, %3, %4;\n fma.rn.f32x2 %0, df, df, %0;\n}\n"
              : "+l"(dist[q])
              : "l"(sv.x), "l"(cw[i]), "l"(sv.y), "l"(cw[i + 1]));
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float d0, d1;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(dist[q]));
        const float dl = d1 < d0 ? d1 : d0;            // the smaller index wins ties
        const int el = d1 < d0 ? tid + 128 : tid;
        float m;
        asm("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(dl));
        uint32_t em;
        asm("redux.sync.min.u32 %0, %1, 0xffffffff;"
            : "=r"(em) : "r"(dl == m ? static_cast<uint32_t>(el) : 0xffffffffu));
        if (lane == 0 && n0 + q < n) wbest[(n0 + q) * 4 + warp] = make_float2(m, __uint_as_float(em));
      }
    }
    __syncthreads();
    for (int nn = tid; nn < n; nn += kEvThreads) {
      const int64_t slot = slots[nn];
      if (slot < 0 || slot >= b.n_slots) continue;
      float bd = INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float2 v = wbest[nn * 4 + w];
        const int ve = static_cast<int>(__float_as_uint(v.y));
        if (v.x < bd || (v.x == bd && ve < be)) {
          bd = v.x;
          be = ve;
        }
      }
      const int jj = u_j, h = u_h, z = u_z;
      const int kv = z & 1, gamma = (z >> 1) % ep.G, layer = (z >> 1) / ep.G;
      EncodeParams p = b;
      p.pool = b.pool + layer * ep.pool_stride_layer + gamma * ep.pool_stride_group;
      p.kv = kv;
      store_index(p, slot, jj, h, be);
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");   // nothing left in flight at exit
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
loopvq_status launch_evict(const EvictParams& e, cudaStream_t st) {
  constexpr int smem = EvGeo<C, G>::SMEM;
  static_assert(smem <= 227 * 1024, "eviction shared memory above 227 KB");
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  if (cudaFuncSetAttribute(encode_evict_kernel<C, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  int per_sm = 0;                                      // persistent: every CTA resident
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_evict_kernel<C, G>, kEvThreads, smem) !=
          cudaSuccess || per_sm < 1)
    return LOOPVQ_ERR_CUDA;
  const int units = e.base.J * e.H * e.combos;
  const int grid = units < per_sm * sms ? units : per_sm * sms;
  encode_evict_kernel<C, G><<<grid, kEvThreads, smem, st>>>(e);
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
  e.H = g.Hkv;
  e.combos = g.L * g.G * 2;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  switch (g.c * 100 + g.g) {
    case 404: return launch_evict<4, 4>(e, st);
    case 804: return launch_evict<8, 4>(e, st);
    case 204: return launch_evict<2, 4>(e, st);
    case 402: return launch_evict<4, 2>(e, st);
    case 802: return launch_evict<8, 2>(e, st);
    case 208: return launch_evict<2, 8>(e, st);
    case 408: return launch_evict<4, 8>(e, st);
    case 401: return launch_evict<4, 1>(e, st);
    case 801: return launch_evict<8, 1>(e, st);
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
