// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// One CTA = one (sequence b, query head hq, context split). Per CTA:
//   1. q (bf16) -> shared, pre-scaled by sm_scale*log2(e) so scores live in
//      log2 units and every exponential is a single ex2.
//   2. Key lookup table LUT[e][col] = q_j . C_K[j][e][tau][:] for the
//      loop-tau codebook slice ([E][32] float, column = replica*J + j).
//   3. Each warp streams whole index pages. One lane owns one token slot:
//      it loads its token's rotated row of J key bytes and J value bytes
//      (16-, 8- or 4-byte granules), sums J LUT entries to get the score,
//      and adds p = 2^(x - m) into its warp's private value histogram
//      W[e][col]. Because rows are rotated by the slot's lane, the 32 lanes
//      of a warp touch 32 distinct columns at every step: no bank conflicts
//      and no two lanes on one histogram word.
//   4. The window tokens (bf16 prefix + recent) are scored densely by
//      split 0.
//   5. Warps are merged, the histogram is contracted with the loop-tau value
//      codebook slice (o[j*c+ch] = sum_e W[e][j] C_V[j][e][tau][ch]) and the
//      split writes (m, l, o[d]) to the workspace.
// A second kernel merges the splits (log-sum-exp merge) into out and lse.

#include <math.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kNW = 4;                  // warps per CTA, each with its own histogram
constexpr int kThreads = kNW * 32;
constexpr float kRescaleSlack = 8.0f;   // log2 units a new maximum may exceed m before rescaling

struct DecodeParams {
  const uint16_t* q;                // bf16 bits [B][Hq][d]
  const uint8_t* pool_lg;           // pool at (layer, gamma, head 0)
  int64_t pool_stride_head;
  const float* cb_k;                // codebooks at (layer, head 0, gamma, K, tau): [J][E][c]
  const float* cb_v;                // same for V
  int64_t cb_stride_head;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint16_t* win_k;            // bf16 bits [B][Hkv][W][d]
  const uint16_t* win_v;
  float* partials;                  // [B*Hq][S][d+2]
  int Hq, Hkv, ratio, W, Pg, n_pages, max_pages_per_seq, max_seq_len;
  int64_t page_bytes, plane_bytes;
  int S, pps;
  float scale_log2;
};

// Loads the rotated row (J bytes) of `row` (this lane's slot) from a block
// of LB slots stored as [J/GR][LB][GR] bytes. `words[k]` = row bytes 4k..4k+3.
template <int J, int GR, int LB>
__device__ __forceinline__ void load_row(const uint8_t* block, int row, bool live,
                                         uint32_t (&words)[J / 4]) {
  constexpr int NG = J / GR;
  if (!live) {
#pragma unroll
    for (int k = 0; k < J / 4; ++k) words[k] = 0u;
    return;
  }
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    const uint8_t* src = block + gi * LB * GR + row * GR;
    if constexpr (GR == 16) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src));
      words[gi * 4 + 0] = v.x;
      words[gi * 4 + 1] = v.y;
      words[gi * 4 + 2] = v.z;
      words[gi * 4 + 3] = v.w;
    } else if constexpr (GR == 8) {
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(src));
      words[gi * 2 + 0] = v.x;
      words[gi * 2 + 1] = v.y;
    } else {
      words[gi] = __ldcs(reinterpret_cast<const unsigned int*>(src));
    }
  }
}

template <int J, int C>
__global__ void __launch_bounds__(kThreads, 1) vq_decode_kernel(const DecodeParams p) {
  constexpr int d = J * C;
  constexpr int R = 32 / J;                  // replicas of each column per row
  constexpr int LB = R * J;                  // slots per rotation block
  constexpr int GR = (J % 16 == 0) ? 16 : (J % 8 == 0) ? 8 : 4;
  constexpr int NWORD = J / 4;

  extern __shared__ __align__(16) float smem[];
  float* lut = smem;                                   // [E][32]
  float* hist = lut + kE * kRowStride;                 // [kNW][E][32]
  float* qs = hist + kNW * kE * kRowStride;            // [256]
  float* xwin = qs + 256;                              // [256]
  float* owin = xwin + 256;                            // [256]
  float* wstat = owin + 256;                           // [2*kNW]

  const int split = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_vq = max(0, N - p.W);
  const int n_pg = min((n_vq + p.Pg - 1) / p.Pg, p.max_pages_per_seq);
  const int pg_lo = split * p.pps;
  const int pg_hi = min(n_pg, pg_lo + p.pps);
  const int n_win = (split == 0) ? min(N, p.W) : 0;

  const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * d;
  for (int i = tid; i < d; i += kThreads) qs[i] = bf16_bits_to_float(qp[i]) * p.scale_log2;
  __syncthreads();

  const float* cbk = p.cb_k + hkv * p.cb_stride_head;
  const float* cbv = p.cb_v + hkv * p.cb_stride_head;

  // ---- key lookup table and histogram reset ----------------------------
  {
    const int j = lane % J;
    const bool live = lane < LB;
    float qj[C];
#pragma unroll
    for (int ch = 0; ch < C; ++ch) qj[ch] = qs[j * C + ch];
    const float* src = cbk + static_cast<size_t>(j) * kE * C;
    constexpr int EPW = kE / kNW;
    for (int e = warp * EPW; e < (warp + 1) * EPW; ++e) {
      float v = 0.f;
      if constexpr (C % 4 == 0) {
#pragma unroll
        for (int ch = 0; ch < C; ch += 4) {
          const float4 cw = __ldg(reinterpret_cast<const float4*>(src + e * C + ch));
          v = fmaf(qj[ch], cw.x, v);
          v = fmaf(qj[ch + 1], cw.y, v);
          v = fmaf(qj[ch + 2], cw.z, v);
          v = fmaf(qj[ch + 3], cw.w, v);
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < C; ++ch) v = fmaf(qj[ch], __ldg(src + e * C + ch), v);
      }
      lut[e * kRowStride + lane] = live ? v : 0.f;
    }
    float4* h4 = reinterpret_cast<float4*>(hist + warp * kE * kRowStride);
    for (int i = lane; i < kE * kRowStride / 4; i += 32) h4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();

  // ---- stream index pages -----------------------------------------------
  const bool lane_live = lane < LB;
  const int c0 = lane % J;
  const int rbase = lane - c0;
  float* my_hist = hist + warp * kE * kRowStride;
  float m_w = -INFINITY;
  float l_lane = 0.f;
  const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;

  for (int pg = pg_lo + warp; pg < pg_hi; pg += kNW) {
    const int phys = bt[pg];
    if (phys < 0 || phys >= p.n_pages) continue;     // absent page: warp-uniform skip
    const uint8_t* kpl = pool_h + static_cast<int64_t>(phys) * p.page_bytes;
    const uint8_t* vpl = kpl + p.plane_bytes;
    const int valid_in_page = min(p.Pg, n_vq - pg * p.Pg);
    const int nblk = (valid_in_page + LB - 1) / LB;
    for (int blk = 0; blk < nblk; ++blk) {
      const bool valid = lane_live && (blk * LB + lane) < valid_in_page;
      uint32_t kw[NWORD], vw[NWORD];
      load_row<J, GR, LB>(kpl + blk * LB * J, lane, lane_live, kw);
      load_row<J, GR, LB>(vpl + blk * LB * J, lane, lane_live, vw);
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int s = 0; s < J; s += 2) {
        const uint32_t e0 = byte_of(kw[s >> 2], s & 3);
        const uint32_t e1 = byte_of(kw[(s + 1) >> 2], (s + 1) & 3);
        const int col0 = lane_live ? rbase + ((c0 + s) % J) : lane;
        const int col1 = lane_live ? rbase + ((c0 + s + 1) % J) : lane;
        x0 += lut[e0 * kRowStride + col0];
        x1 += lut[e1 * kRowStride + col1];
      }
      const float x = valid ? x0 + x1 : -INFINITY;
      const float xm = warp_max(x);                  // finite: slot 0 of the block is valid
      if (xm > m_w + kRescaleSlack) {
        if (m_w != -INFINITY) {
          const float f = fast_exp2(m_w - xm);
          __syncwarp();
          float4* h4 = reinterpret_cast<float4*>(my_hist);
          for (int i = lane; i < kE * kRowStride / 4; i += 32) {
            float4 t = h4[i];
            t.x *= f; t.y *= f; t.z *= f; t.w *= f;
            h4[i] = t;
          }
          __syncwarp();
          l_lane *= f;
        }
        m_w = xm;
      }
      const float pr = valid ? fast_exp2(x - m_w) : 0.f;
      l_lane += pr;
      // The J steps of one slot touch J distinct columns, hence J distinct
      // words: issue every load before any store so the loads overlap.
      int ha[J];
      float hv[J];
#pragma unroll
      for (int s = 0; s < J; ++s) {
        const uint32_t e = byte_of(vw[s >> 2], s & 3);
        const int col = lane_live ? rbase + ((c0 + s) % J) : lane;
        ha[s] = e * kRowStride + col;
        hv[s] = my_hist[ha[s]];
      }
#pragma unroll
      for (int s = 0; s < J; ++s) my_hist[ha[s]] = hv[s] + pr;
      __syncwarp();
    }
  }
  const float l_w = warp_sum(l_lane);
  if (lane == 0) {
    wstat[warp] = m_w;
    wstat[kNW + warp] = l_w;
  }

  // ---- bf16 window tokens (split 0) -----------------------------------
  if (n_win > 0) {
    const uint16_t* wk =
        p.win_k + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * d;
    for (int t = warp; t < n_win; t += kNW) {
      float acc = 0.f;
      for (int ch = lane; ch < d; ch += 32) acc = fmaf(qs[ch], bf16_bits_to_float(wk[t * d + ch]), acc);
      acc = warp_sum(acc);
      if (lane == 0) xwin[t] = acc;
    }
  }
  __syncthreads();
  float m_win = -INFINITY;
  float l_win = 0.f;
  if (n_win > 0) {
    for (int t = 0; t < n_win; ++t) m_win = fmaxf(m_win, xwin[t]);
    for (int t = 0; t < n_win; ++t) l_win += fast_exp2(xwin[t] - m_win);
    const uint16_t* wv =
        p.win_v + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * d;
    for (int ch = tid; ch < d; ch += kThreads) {
      float o = 0.f;
      for (int t = 0; t < n_win; ++t)
        o = fmaf(fast_exp2(xwin[t] - m_win), bf16_bits_to_float(wv[t * d + ch]), o);
      owin[ch] = o;
    }
  }

  // ---- merge warps, contract the histogram -----------------------------
  float M = m_win;
#pragma unroll
  for (int w = 0; w < kNW; ++w) M = fmaxf(M, wstat[w]);
  float* part = p.partials + (static_cast<size_t>(b * p.Hq + hq) * p.S + split) * (d + 2);
  if (M == -INFINITY) {                               // no token in this split
    for (int i = tid; i < d + 2; i += kThreads) part[i] = (i == 0) ? -INFINITY : 0.f;
    return;
  }
  float f[kNW];
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kNW; ++w) {
    f[w] = (wstat[w] == -INFINITY) ? 0.f : fast_exp2(wstat[w] - M);
    L += f[w] * wstat[kNW + w];
  }
  const float f_win = (m_win == -INFINITY) ? 0.f : fast_exp2(m_win - M);
  L += f_win * l_win;
  {
    float4* h0 = reinterpret_cast<float4*>(hist);
    for (int i = tid; i < kE * kRowStride / 4; i += kThreads) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float4 t = reinterpret_cast<const float4*>(hist + w * kE * kRowStride)[i];
        acc.x = fmaf(f[w], t.x, acc.x);
        acc.y = fmaf(f[w], t.y, acc.y);
        acc.z = fmaf(f[w], t.z, acc.z);
        acc.w = fmaf(f[w], t.w, acc.w);
      }
      h0[i] = acc;
    }
  }
  __syncthreads();
  for (int o = tid; o < d; o += kThreads) {
    const int j = o / C, ch = o % C;
    const float* src = cbv + static_cast<size_t>(j) * kE * C + ch;
    float acc = 0.f;
#pragma unroll 8
    for (int e = 0; e < kE; ++e) {
      float wsum = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) wsum += hist[e * kRowStride + r * J + j];
      acc = fmaf(wsum, __ldg(src + e * C), acc);
    }
    part[2 + o] = acc + ((n_win > 0) ? f_win * owin[o] : 0.f);
  }
  if (tid == 0) {
    part[0] = M;
    part[1] = L;
  }
}

// (m, l, o) partials [pairs][S][d+2] -> out [pairs][d], lse [pairs].
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

constexpr size_t decode_smem_bytes() {
  return (static_cast<size_t>(kE) * kRowStride * (1 + kNW) + 256 * 3 + 2 * kNW) * sizeof(float);
}

template <int J, int C>
loopvq_status launch_vq(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  const size_t smem = decode_smem_bytes();
  // The attribute belongs to (function, device); remember which devices have it.
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit == 0 || !(configured.load(std::memory_order_relaxed) & bit)) {
    if (cudaFuncSetAttribute(vq_decode_kernel<J, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return LOOPVQ_ERR_CUDA;
    configured.fetch_or(bit, std::memory_order_relaxed);
  }
  vq_decode_kernel<J, C><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace

loopvq_status launch_merge(const float* partials, int pairs, int splits, int d, int out_dtype,
                           void* out, float* lse, void* stream) {
  const dim3 grid((pairs + 3) / 4);
  merge_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(partials, pairs, splits, d,
                                                                     out_dtype, out, lse);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

loopvq_status launch_decode(const DecodeArgs& a) {
  const Geometry& g = *a.geo;
  const int gamma = a.loop_step / g.g, tau = a.loop_step % g.g;
  DecodeParams p{};
  p.q = static_cast<const uint16_t*>(a.q);
  p.pool_lg = a.pool + a.layer * g.pool_stride_layer + gamma * g.pool_stride_group;
  p.pool_stride_head = g.pool_stride_head;
  const float* cb_l = a.codebooks + a.layer * g.cb_stride_layer + gamma * g.cb_stride_group +
                      tau * g.cb_stride_loop;
  p.cb_k = cb_l;
  p.cb_v = cb_l + g.cb_stride_kv;
  p.cb_stride_head = g.cb_stride_head;
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.win_k = static_cast<const uint16_t*>(a.win_k);
  p.win_v = static_cast<const uint16_t*>(a.win_v);
  p.partials = static_cast<float*>(a.workspace);
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.ratio = g.Hq / g.Hkv;
  p.W = g.W;
  p.Pg = g.Pg;
  p.n_pages = g.n_pages;
  p.max_pages_per_seq = g.max_pages_per_seq;
  p.max_seq_len = a.max_seq_len;
  p.page_bytes = g.page_bytes;
  p.plane_bytes = g.plane_bytes;
  const int n_vq = a.max_seq_len > g.W ? a.max_seq_len - g.W : 0;
  const int pages = (n_vq + g.Pg - 1) / g.Pg;
  p.S = a.splits;
  p.pps = pages > 0 ? (pages + a.splits - 1) / a.splits : 1;
  p.scale_log2 = a.sm_scale * kLog2e;
  const dim3 grid(a.splits, g.Hq, a.batch);
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  loopvq_status s;
  switch (g.J * 100 + g.c) {
    case 1604: s = launch_vq<16, 4>(p, grid, st); break;
    case 3204: s = launch_vq<32, 4>(p, grid, st); break;
    case 1208: s = launch_vq<12, 8>(p, grid, st); break;
    case 3202: s = launch_vq<32, 2>(p, grid, st); break;
    case 1608: s = launch_vq<16, 8>(p, grid, st); break;
    case 2404: s = launch_vq<24, 4>(p, grid, st); break;
    case 3208: s = launch_vq<32, 8>(p, grid, st); break;
    case 804:  s = launch_vq<8, 4>(p, grid, st); break;
    case 808:  s = launch_vq<8, 8>(p, grid, st); break;
    case 1202: s = launch_vq<12, 2>(p, grid, st); break;
    case 1602: s = launch_vq<16, 2>(p, grid, st); break;
    case 2402: s = launch_vq<24, 2>(p, grid, st); break;
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
  if (s != LOOPVQ_OK) return s;
  return launch_merge(p.partials, a.batch * g.Hq, a.splits, g.d, a.out_dtype, a.out, a.lse,
                      a.stream);
}

}  // namespace loopvq
