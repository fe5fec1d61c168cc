// Dense bf16-KV decode attention (split-K flash-decoding), the same-shape
// comparison point for the LoopVQ kernel. Writes the same (m, l, o) split
// partials, merged by the same merge kernel.
//
// One CTA = (context split, query head, sequence), 4 warps. A token is
// handled by LPT lanes (LPT = next power of two >= d/8); each lane holds 8
// channels (one 16-byte load of K and one of V per token). A warp handles
// 32/LPT tokens per step and unrolls 4 steps so 8 independent 16-byte loads
// per lane are in flight. Online softmax in log2 units per token group,
// merged across groups by shuffles and across warps through shared memory.

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kBW = 4;  // warps per CTA
constexpr int kUnroll = 4;

struct Bf16Params {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* seq_lens;
  float* partials;
  int Hq, Hkv, ratio, max_seq_len, S, chunk;
  float scale_log2;
};

__device__ __forceinline__ void merge_state(float& m, float& l, float (&o)[8], float m2, float l2,
                                            const float (&o2)[8]) {
  const float M = fmaxf(m, m2);
  const float a = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
  const float b = (m2 == -INFINITY) ? 0.f : fast_exp2(m2 - M);
  l = a * l + b * l2;
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = a * o[i] + b * o2[i];
  m = M;
}

template <int D>
__global__ void __launch_bounds__(kBW * 32) bf16_decode_kernel(const Bf16Params p) {
  constexpr int NL = D / 8;                                  // lanes with channels
  constexpr int LPT = NL <= 1 ? 1 : NL <= 2 ? 2 : NL <= 4 ? 4 : NL <= 8 ? 8 : NL <= 16 ? 16 : 32;
  constexpr int TPW = 32 / LPT;
  __shared__ float s_m[kBW], s_l[kBW];
  __shared__ __align__(16) float s_o[kBW][D];

  const int split = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPT, tsub = lane / LPT;
  const bool active = sub < NL;
  const int hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int tok_lo = split * p.chunk;
  const int tok_hi = min(N, tok_lo + p.chunk);

  float q[8];
  {
    const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * D + sub * 8;
    uint4 qr = make_uint4(0, 0, 0, 0);
    if (active) qr = *reinterpret_cast<const uint4*>(qp);
    const uint32_t w[4] = {qr.x, qr.y, qr.z, qr.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = bf16x2_to_float2(w[i]);
      q[2 * i] = f.x * p.scale_log2;
      q[2 * i + 1] = f.y * p.scale_log2;
    }
  }
  const size_t head_off = (static_cast<size_t>(b) * p.Hkv + hkv) * p.max_seq_len;
  const uint16_t* kbase = p.k + head_off * D + sub * 8;
  const uint16_t* vbase = p.v + head_off * D + sub * 8;

  float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;

  constexpr int STEP = kBW * TPW;
  // The loop bound is warp-uniform (base0 does not depend on the lane), so
  // every lane runs the same trip count and reaches every full-mask shuffle.
  for (int base0 = tok_lo + warp * TPW; base0 < tok_hi; base0 += STEP * kUnroll) {
    const int base = base0 + tsub;
    uint4 kr[kUnroll], vr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = base + u * STEP;
      if (active && t < tok_hi) {
        kr[u] = __ldcs(reinterpret_cast<const uint4*>(kbase + static_cast<size_t>(t) * D));
        vr[u] = __ldcs(reinterpret_cast<const uint4*>(vbase + static_cast<size_t>(t) * D));
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = base + u * STEP;
      const uint32_t kw[4] = {kr[u].x, kr[u].y, kr[u].z, kr[u].w};
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_float2(kw[i]);
        dot = fmaf(q[2 * i], f.x, dot);
        dot = fmaf(q[2 * i + 1], f.y, dot);
      }
#pragma unroll
      for (int off = LPT / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (t < tok_hi) {                 // no shuffle inside this branch
        const float mn = fmaxf(m, dot);
        const float sc = (m == mn) ? 1.f : fast_exp2(m - mn);
        const float pr = fast_exp2(dot - mn);
        l = fmaf(l, sc, pr);
        const uint32_t vw[4] = {vr[u].x, vr[u].y, vr[u].z, vr[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf16x2_to_float2(vw[i]);
          o[2 * i] = fmaf(o[2 * i], sc, pr * f.x);
          o[2 * i + 1] = fmaf(o[2 * i + 1], sc, pr * f.y);
        }
        m = mn;
      }
    }
  }
  // merge token groups of the warp
#pragma unroll
  for (int off = LPT; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
    float o2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o2[i] = __shfl_xor_sync(0xffffffffu, o[i], off);
    merge_state(m, l, o, m2, l2, o2);
  }
  if (tsub == 0) {
    if (lane == 0) {
      s_m[warp] = m;
      s_l[warp] = l;
    }
    if (active) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s_o[warp][sub * 8 + i] = o[i];
    }
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kBW; ++w) M = fmaxf(M, s_m[w]);
  float* part = p.partials + (static_cast<size_t>(b * p.Hq + hq) * p.S + split) * (D + 2);
  float f[kBW];
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kBW; ++w) {
    f[w] = (s_m[w] == -INFINITY) ? 0.f : fast_exp2(s_m[w] - M);
    L += f[w] * s_l[w];
  }
  for (int c = threadIdx.x; c < D; c += kBW * 32) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kBW; ++w) acc = fmaf(f[w], s_o[w][c], acc);
    part[2 + c] = (M == -INFINITY) ? 0.f : acc;
  }
  if (threadIdx.x == 0) {
    part[0] = M;
    part[1] = (M == -INFINITY) ? 0.f : L;
  }
}

template <int D>
loopvq_status launch_bf16(const Bf16Params& p, dim3 grid, cudaStream_t st) {
  bf16_decode_kernel<D><<<grid, kBW * 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace

loopvq_status launch_bf16_decode(const Bf16DecodeArgs& a) {
  Bf16Params p{};
  p.q = static_cast<const uint16_t*>(a.q);
  p.k = static_cast<const uint16_t*>(a.k);
  p.v = static_cast<const uint16_t*>(a.v);
  p.seq_lens = a.seq_lens;
  p.partials = static_cast<float*>(a.workspace);
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.ratio = a.Hq / a.Hkv;
  p.max_seq_len = a.max_seq_len;
  p.S = a.splits;
  p.chunk = a.max_seq_len > 0 ? (a.max_seq_len + a.splits - 1) / a.splits : 1;
  p.scale_log2 = a.sm_scale * kLog2e;
  const dim3 grid(a.splits, a.Hq, a.batch);
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  loopvq_status s;
  switch (a.d) {
    case 64: s = launch_bf16<64>(p, grid, st); break;
    case 96: s = launch_bf16<96>(p, grid, st); break;
    case 128: s = launch_bf16<128>(p, grid, st); break;
    case 256: s = launch_bf16<256>(p, grid, st); break;
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
  if (s != LOOPVQ_OK) return s;
  return launch_merge(p.partials, a.batch * a.Hq, a.splits, a.d, a.out_dtype, a.out, a.lse,
                      a.stream);
}

}  // namespace loopvq
