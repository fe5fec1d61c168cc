// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// One CTA = one (sequence b, query head hq, context split), 5 warps, one CTA
// per SM (the per-warp value histograms fill shared memory). Per CTA:
//   1. The first index blocks of every warp are requested (register ring),
//      then the loop-tau key codebook slice is staged into shared memory
//      with cp.async while q is pre-scaled by sm_scale*log2(e) (scores live
//      in log2 units: every exponential is one ex2).
//   2. Key lookup table LUT[e][k] = q_j . C_K[j][e][tau][:] with j = k % J,
//      [E][64] float (every group repeated along the row so that a lane's
//      column lane + step never wraps), built from shared memory.
//   3. Split 0 scores the bf16 window tokens (prefix + recent) densely and
//      keeps them as a (m, l, o) partial.
//   4. Each warp streams blocks of LB token slots. Key pass: lane = slot;
//      the slot's rotated row of J key bytes gives J LUT reads that hit J
//      distinct columns across the warp (no bank conflicts); the score is a
//      per-lane sum. Value pass: lane = (replica, channel group) and owns
//      one column of its warp's private histogram W[e][col]; it adds
//      p = 2^(x - m) of its J slots at the rows given by the group-major
//      value bytes, two slots per step with an equality check so that two
//      updates of one word in a step merge. No lane writes another lane's
//      column, so no atomics and no warp-level ordering are needed. Index
//      bytes are prefetched kDepth blocks ahead into registers.
//   5. Warps are merged, the loop-tau value codebook slice is staged into
//      the freed histogram space and contracted with the histogram
//      (o[j*c+ch] = sum_e W[e][j] C_V[j][e][tau][ch]); the split writes
//      (m, l, o[d]) to the workspace. merge.cu combines the splits.

#include <math.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kNW = 5;                  // warps per CTA, one value histogram each
constexpr int kThreads = kNW * 32;
constexpr int kDepth = 4;               // blocks in flight per warp
constexpr int kRegion = kE * kRowStride;  // floats in one [E][32] table (32 KB)
constexpr int kLutRow = 64;             // LUT row: 64 columns, column k holds group k % J
constexpr int kLutFloats = kE * kLutRow;  // 64 KB
constexpr int kStageRegions = 4;        // histogram regions 1..4 double as codebook staging
constexpr int kWinChunk = 12;           // window tokens per warp per round of loads
constexpr int kPrefetchPages = 8;       // pages a warp asks L2 to fetch ahead of its loads
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

template <int J>
struct Traits {
  static constexpr int R = 32 / J;      // replicas of each column per table row
  static constexpr int LB = R * J;      // slots per block
  static constexpr int GR = (J % 16 == 0) ? 16 : (J % 8 == 0) ? 8 : 4;   // granule
  static constexpr int NWORD = J / 4;   // words per lane per plane and block
};

template <int J>
struct BlockRegs {
  uint32_t k[J / 4];   // this lane's rotated key row (lane = slot)
  uint32_t v[J / 4];   // this lane's value bytes: group j, J consecutive slots
  bool ok;             // page present (same value in every lane)
};

template <int GR>
__device__ __forceinline__ void load_words(const uint8_t* src, uint32_t* w, int nwords) {
#pragma unroll
  for (int i = 0; i < nwords; i += GR / 4) {
    if constexpr (GR == 16) {
      const uint4 t = __ldcs(reinterpret_cast<const uint4*>(src + 4 * i));
      w[i] = t.x; w[i + 1] = t.y; w[i + 2] = t.z; w[i + 3] = t.w;
    } else if constexpr (GR == 8) {
      const uint2 t = __ldcs(reinterpret_cast<const uint2*>(src + 4 * i));
      w[i] = t.x; w[i + 1] = t.y;
    } else {
      w[i] = __ldcs(reinterpret_cast<const unsigned int*>(src + 4 * i));
    }
  }
}

// Loads block `blk` of the page at `kpl` (K plane; the V plane follows).
template <int J>
__device__ __forceinline__ void load_block(const uint8_t* kpl, int64_t plane_bytes, int Pg, int blk,
                                           int lane, BlockRegs<J>& r) {
  using T = Traits<J>;
  if (lane < T::LB) {
#pragma unroll
    for (int gi = 0; gi < J / T::GR; ++gi)
      load_words<T::GR>(kpl + blk * T::LB * J + gi * T::LB * T::GR + lane * T::GR,
                        r.k + gi * (T::GR / 4), T::GR / 4);
    const int rr = lane / J, j = lane % J;
    load_words<T::GR>(kpl + plane_bytes + static_cast<int64_t>(j) * Pg + blk * T::LB + rr * J, r.v,
                      T::NWORD);
  } else {
#pragma unroll
    for (int i = 0; i < T::NWORD; ++i) {
      r.k[i] = 0u;
      r.v[i] = 0u;
    }
  }
}

// Copies `nfloats` (multiple of 4) from global to shared with cp.async.
__device__ __forceinline__ void stage_async(float* dst, const float* src, int nfloats, int tid) {
  for (int i = tid * 4; i < nfloats; i += kThreads * 4) cp_async16(dst + i, src + i);
}

// sum_ch a[ch] * b[ch] for C channels held contiguously (16-byte aligned
// when C % 4 == 0).
template <int C>
__device__ __forceinline__ float dot_c(const float* a, const float* b) {
  float v = 0.f;
  if constexpr (C % 4 == 0) {
#pragma unroll
    for (int ch = 0; ch < C; ch += 4) {
      const float4 x = *reinterpret_cast<const float4*>(a + ch);
      const float4 y = *reinterpret_cast<const float4*>(b + ch);
      v = fmaf(x.x, y.x, v);
      v = fmaf(x.y, y.y, v);
      v = fmaf(x.z, y.z, v);
      v = fmaf(x.w, y.w, v);
    }
  } else {
#pragma unroll
    for (int ch = 0; ch < C; ++ch) v = fmaf(a[ch], b[ch], v);
  }
  return v;
}

template <int J, int C>
__global__ void __launch_bounds__(kThreads, 1) vq_decode_kernel(const DecodeParams p) {
  using T = Traits<J>;
  constexpr int d = J * C;
  constexpr int R = T::R, LB = T::LB;
  constexpr int OPT = (d + kThreads - 1) / kThreads;   // output channels per thread
  constexpr int NPL = (d / 2 + 31) / 32;               // bf16 channel pairs per lane (window)
  // channel groups per staging chunk: a [JC][E][C] slice fits regions 1..4
  constexpr int JC = (J * kE * C <= kStageRegions * kRegion) ? J : (kStageRegions * kRegion) / (kE * C);
  static_assert(J % JC == 0, "staging chunks must tile the channel groups");

  extern __shared__ __align__(16) float smem[];
  float* lut = smem;                                   // [E][64]
  float* hist = lut + kLutFloats;                      // [kNW][E][32]
  float* pbuf = hist + kNW * kRegion;                  // [kNW][32]
  float* wstat = pbuf + kNW * 32;                      // [2*kNW]
  float* stage = hist + kRegion;                       // regions 1..4
  // scratch inside region 0 until the histograms are zeroed
  float* qs = hist;                                    // [256]
  float* xwin = hist + 256;                            // [256]
  float* opart = hist + 512;                           // [kNW][256]

  const int split = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_vq = max(0, N - p.W);
  const int n_pg = min((n_vq + p.Pg - 1) / p.Pg, p.max_pages_per_seq);
  const int pg_lo = split * p.pps;
  const int pg_hi = min(n_pg, pg_lo + p.pps);
  const int n_win = (split == 0) ? min(N, p.W) : 0;
  const float* cbk = p.cb_k + hkv * p.cb_stride_head;
  const float* cbv = p.cb_v + hkv * p.cb_stride_head;

  // ---- 1. request the first index blocks of this warp ---------------------
  const bool lane_live = lane < LB;
  const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
  const int my_first = pg_lo + warp;
  const int n_my_pages = (pg_hi > my_first) ? (pg_hi - my_first + kNW - 1) / kNW : 0;
  const int bpp = p.Pg / LB;                            // blocks per page
  const int n_blocks = n_my_pages * bpp;
  // page table window: lane l holds the physical page of this warp's page
  // index i0 + l (cur) and i0 + 32 + l (nxt)
  int i0 = 0;
  auto bt_entry = [&](int i) -> int { return (i < n_my_pages) ? bt[my_first + i * kNW] : -1; };
  int bt_cur = bt_entry(lane);
  int bt_nxt = bt_entry(32 + lane);
  // L2 prefetch of this warp's first pages (lane l: page index l)
  if (lane < kPrefetchPages && lane < n_my_pages && bt_cur >= 0 && bt_cur < p.n_pages)
    prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_cur) * p.page_bytes,
                     static_cast<uint32_t>(p.page_bytes));
  const uint32_t bpp_magic = 0xFFFFFFFFu / static_cast<uint32_t>(bpp) + 1u;   // k / bpp = umulhi
  BlockRegs<J> ring[kDepth];
  auto issue = [&](int k, BlockRegs<J>& r) {
    const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(k), bpp_magic));
    const int blk = k - pi * bpp;
    if (pi >= i0 + 32) {                                // warp-uniform
      bt_cur = bt_nxt;
      i0 += 32;
      bt_nxt = bt_entry(i0 + 32 + lane);
    }
    if (blk == 0) {                                     // first block of a page: prefetch ahead
      const int tgt = pi + kPrefetchPages;              // tgt - i0 < 64: inside cur or nxt
      const int src = (tgt - i0 < 32) ? bt_cur : bt_nxt;
      const int pf = __shfl_sync(0xffffffffu, src, (tgt - i0) & 31);
      if (lane == 0 && tgt < n_my_pages && pf >= 0 && pf < p.n_pages)
        prefetch_l2_bulk(pool_h + static_cast<int64_t>(pf) * p.page_bytes,
                         static_cast<uint32_t>(p.page_bytes));
    }
    const int phys = __shfl_sync(0xffffffffu, bt_cur, pi - i0);
    r.ok = phys >= 0 && phys < p.n_pages;
    if (!r.ok) {                                        // absent page: read nothing
#pragma unroll
      for (int i = 0; i < T::NWORD; ++i) {
        r.k[i] = 0u;
        r.v[i] = 0u;
      }
      return;
    }
    load_block<J>(pool_h + static_cast<int64_t>(phys) * p.page_bytes, p.plane_bytes, p.Pg, blk,
                  lane, r);
  };
#pragma unroll
  for (int u = 0; u < kDepth - 1; ++u)
    if (u < n_blocks) issue(u, ring[u]);

  // ---- 2. key lookup table (codebook staged in regions 1..4) ---------------
  stage_async(stage, cbk, JC * kE * C, tid);
  const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * d;
  for (int i = tid; i < d; i += kThreads) qs[i] = bf16_bits_to_float(qp[i]) * p.scale_log2;

  // ---- 3. window keys: one round of loads per kWinChunk tokens per warp ---
  uint32_t wv_reg[kWinChunk][NPL];                      // first chunk of window values
  const uint16_t* wkb = p.win_k + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * d;
  const uint16_t* wvb = p.win_v + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * d;
  if (n_win > 0) {
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      const int t = warp + i * kNW;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;                   // channel pair index
        wv_reg[i][k] = (t < n_win && pc < d / 2)
                           ? __ldg(reinterpret_cast<const unsigned int*>(wvb + t * d) + pc) : 0u;
      }
    }
  }
  __syncthreads();                                      // qs visible
  for (int t0 = warp; t0 < n_win; t0 += kNW * kWinChunk) {
    uint32_t kr[kWinChunk][NPL];
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      const int t = t0 + i * kNW;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;
        kr[i][k] = (t < n_win && pc < d / 2)
                       ? __ldg(reinterpret_cast<const unsigned int*>(wkb + t * d) + pc) : 0u;
      }
    }
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;
        if (pc < d / 2) {
          const float2 kv = bf16x2_to_float2(kr[i][k]);
          acc = fmaf(qs[2 * pc], kv.x, fmaf(qs[2 * pc + 1], kv.y, acc));
        }
      }
      acc = warp_sum(acc);
      const int t = t0 + i * kNW;
      if (lane == 0 && t < n_win) xwin[t] = acc;
    }
  }

  // ---- LUT from the staged key codebook ----------------------------------
  for (int j0 = 0; j0 < J; j0 += JC) {
    if (j0 > 0) {
      __syncthreads();                                  // previous chunk consumed
      stage_async(stage, cbk + static_cast<size_t>(j0) * kE * C, JC * kE * C, tid);
    }
    cp_async_wait_all();
    __syncthreads();
    // item = (e-tile of 32, step s): lane -> e = tile*32 + lane, group
    // j0 + (lane + s) % JC; rotating the group keeps the table writes on
    // distinct banks.
    for (int item = warp; item < (kE / 32) * JC; item += kNW) {
      const int tile = item / JC, s = item % JC;
      const int e = tile * 32 + lane;
      const int jj = (lane + s) % JC;
      const int j = j0 + jj;
      const float v = dot_c<C>(qs + j * C, stage + (static_cast<size_t>(jj) * kE + e) * C);
#pragma unroll
      for (int k = j; k < kLutRow; k += J) lut[e * kLutRow + k] = v;
    }
  }
  __syncthreads();                                      // xwin complete, LUT complete

  // ---- window partial -----------------------------------------------------
  float m_win = -INFINITY, l_win = 0.f;
  float owin[OPT];
#pragma unroll
  for (int k = 0; k < OPT; ++k) owin[k] = 0.f;
  if (n_win > 0) {
    for (int t = 0; t < n_win; ++t) m_win = fmaxf(m_win, xwin[t]);
    for (int t = 0; t < n_win; ++t) l_win += fast_exp2(xwin[t] - m_win);
    float oacc[NPL][2];
#pragma unroll
    for (int k = 0; k < NPL; ++k) oacc[k][0] = oacc[k][1] = 0.f;
    for (int t0 = warp; t0 < n_win; t0 += kNW * kWinChunk) {
      uint32_t vr[kWinChunk][NPL];
#pragma unroll
      for (int i = 0; i < kWinChunk; ++i) {
        const int t = t0 + i * kNW;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const int pc = lane + 32 * k;
          vr[i][k] = (t0 == warp) ? wv_reg[i][k]
                     : ((t < n_win && pc < d / 2)
                            ? __ldg(reinterpret_cast<const unsigned int*>(wvb + t * d) + pc) : 0u);
        }
      }
#pragma unroll
      for (int i = 0; i < kWinChunk; ++i) {
        const int t = t0 + i * kNW;
        const float w = (t < n_win) ? fast_exp2(xwin[t] - m_win) : 0.f;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const float2 vv = bf16x2_to_float2(vr[i][k]);
          oacc[k][0] = fmaf(w, vv.x, oacc[k][0]);
          oacc[k][1] = fmaf(w, vv.y, oacc[k][1]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int pc = lane + 32 * k;
      if (pc < d / 2) {
        opart[warp * 256 + 2 * pc] = oacc[k][0];
        opart[warp * 256 + 2 * pc + 1] = oacc[k][1];
      }
    }
  }
  __syncthreads();
  if (n_win > 0) {
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
      const int ch = tid + k * kThreads;
      if (ch < d) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) o += opart[w * 256 + ch];
        owin[k] = o;
      }
    }
  }
  __syncthreads();                                      // scratch in region 0 no longer read
  {
    float4* h4 = reinterpret_cast<float4*>(hist + warp * kRegion);
    for (int i = lane; i < kRegion / 4; i += 32) h4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncwarp();

  // ---- 4. stream index blocks --------------------------------------------
  float* my_hist = hist + warp * kRegion;
  float* my_p = pbuf + warp * 32;
  const char* lut_bytes = reinterpret_cast<const char*>(lut);
  char* hist_bytes = reinterpret_cast<char*>(my_hist);
  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;   // fits one byte
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;   // fits one byte
  float m_w = -INFINITY;
  float l_lane = 0.f;

  auto process = [&](int k, const BlockRegs<J>& r) {
    const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(k), bpp_magic));
    const int blk = k - pi * bpp;
    const int pg = my_first + pi * kNW;
    const int valid_in_page = min(p.Pg, n_vq - pg * p.Pg);
    const int base = blk * LB;
    if (base >= valid_in_page || !r.ok) return;         // warp-uniform
    // key pass: lane = slot. Row byte s holds the index of group
    // (lane + s) % J, which LUT column lane + s holds: one byte permute
    // forms (e << 8) | lane*4 and the step goes into the load's offset.
    float xa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < J; ++s) {
      const uint32_t off = __byte_perm(r.k[s >> 2], lane4, 0x5504u | (uint32_t(s & 3) << 4));
      xa[s & 3] += *reinterpret_cast<const float*>(lut_bytes + off + 4 * s);
    }
    const bool valid = lane_live && (base + lane) < valid_in_page;
    const float x = valid ? (xa[0] + xa[1]) + (xa[2] + xa[3]) : -INFINITY;
    const float xm = warp_max(x);                       // finite: slot 0 of the block is valid
    if (xm > m_w + kRescaleSlack) {                     // warp-uniform
      if (m_w != -INFINITY) {
        const float f = fast_exp2(m_w - xm);
#pragma unroll 8
        for (int e = 0; e < kE; ++e) my_hist[e * kRowStride + lane] *= f;   // own column
        l_lane *= f;
      }
      m_w = xm;
    }
    const float pr = valid ? fast_exp2(x - m_w) : 0.f;
    l_lane += pr;
    my_p[lane] = pr;
    __syncwarp();
    // value pass: lane = (replica, group) owns column `lane`; slots rr*J + i
    if (lane_live) {
      const float* pp = my_p + (lane / J) * J;
#pragma unroll
      for (int i = 0; i < J; i += 2) {
        // (e << 8 | lane*8) >> 1 = e*128 + lane*4: the byte offset of W[e][lane]
        const uint32_t oa = __byte_perm(r.v[i >> 2], lane8, 0x5504u | (uint32_t(i & 3) << 4)) >> 1;
        const uint32_t ob =
            __byte_perm(r.v[(i + 1) >> 2], lane8, 0x5504u | (uint32_t((i + 1) & 3) << 4)) >> 1;
        const float2 pab = *reinterpret_cast<const float2*>(pp + i);
        float* wa = reinterpret_cast<float*>(hist_bytes + oa);
        float* wb = reinterpret_cast<float*>(hist_bytes + ob);
        const float va = *wa, vb = *wb;
        const bool same = (oa == ob);
        const float na = va + (same ? pab.x + pab.y : pab.x);
        const float nb = same ? na : vb + pab.y;
        *wa = na;
        *wb = nb;
      }
    }
    __syncwarp();                                       // my_p is rewritten by the next block
  };

  for (int k0 = 0; k0 < n_blocks; k0 += kDepth) {
#pragma unroll
    for (int u = 0; u < kDepth; ++u) {
      const int k = k0 + u;
      if (k + kDepth - 1 < n_blocks) issue(k + kDepth - 1, ring[(u + kDepth - 1) % kDepth]);
      if (k < n_blocks) process(k, ring[u]);
    }
  }
  const float l_w = warp_sum(l_lane);
  if (lane == 0) {
    wstat[warp] = m_w;
    wstat[kNW + warp] = l_w;
  }
  __syncthreads();

  // ---- 5. merge warps, contract the histogram -----------------------------
  float M = m_win;
#pragma unroll
  for (int w = 0; w < kNW; ++w) M = fmaxf(M, wstat[w]);
  float* part = p.partials + (static_cast<size_t>(b * p.Hq + hq) * p.S + split) * (d + 2);
  if (M == -INFINITY) {                                 // no token in this split
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
    for (int i = tid; i < kRegion / 4; i += kThreads) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float4 t = reinterpret_cast<const float4*>(hist + w * kRegion)[i];
        acc.x = fmaf(f[w], t.x, acc.x);
        acc.y = fmaf(f[w], t.y, acc.y);
        acc.z = fmaf(f[w], t.z, acc.z);
        acc.w = fmaf(f[w], t.w, acc.w);
      }
      h0[i] = acc;
    }
  }
  for (int j0 = 0; j0 < J; j0 += JC) {
    __syncthreads();                                    // histogram merged / previous chunk used
    stage_async(stage, cbv + static_cast<size_t>(j0) * kE * C, JC * kE * C, tid);
    cp_async_wait_all();
    __syncthreads();
    // thread -> (group jj, channel ch); rows visited from e = jj so that the
    // threads of a warp read different banks of the staged slice
    for (int t = tid; t < JC * C; t += kThreads) {
      const int jj = t / C, ch = t % C, j = j0 + jj;
      const float* cv = stage + static_cast<size_t>(jj) * kE * C + ch;
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < kE; ++i) {
        const int e = (i + jj) & (kE - 1);
        float wsum = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) wsum += hist[e * kRowStride + r * J + j];
        acc = fmaf(wsum, cv[e * C], acc);
      }
      const int o = j * C + ch;
      // the window part of channel o lives in thread o % kThreads, slot o / kThreads
      part[2 + o] = acc;
    }
  }
  __syncthreads();                                      // every part[2 + o] written
#pragma unroll
  for (int k = 0; k < OPT; ++k) {
    const int o = tid + k * kThreads;
    if (o < d && f_win != 0.f) part[2 + o] += f_win * owin[k];
  }
  if (tid == 0) {
    part[0] = M;
    part[1] = L;
  }
}

constexpr size_t decode_smem_bytes() {
  return (static_cast<size_t>(kLutFloats) + static_cast<size_t>(kRegion) * kNW + kNW * 32 + 2 * kNW) *
         sizeof(float);
}
static_assert(decode_smem_bytes() <= 227 * 1024, "decode kernel shared memory above 227 KB");

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
