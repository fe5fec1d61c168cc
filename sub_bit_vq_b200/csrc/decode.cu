// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// Two kernels per call.
//
// vq_stream_kernel: a persistent grid (at most one CTA per SM, 5 warps) over
// the quantised tokens of every (sequence, query head) pair. The work is
// counted in pages; all pages of all pairs form one list, and CTA c takes
// the contiguous range [U*c/n, U*(c+1)/n) of it, so every CTA streams the
// same number of pages and touches one or two pairs ("segments"). Per
// segment:
//   1. The first index blocks of every warp are requested (register ring),
//      then the loop-tau key codebook slice is staged into shared memory
//      with cp.async while q is pre-scaled by sm_scale*log2(e) (scores live
//      in log2 units: every exponential is one ex2).
//   2. Key lookup table LUT[e][k] = q_j . C_K[j][e][tau][:] with j = k % J,
//      [E][64] float: every group is repeated along the row so that a
//      lane's column lane + step never wraps.
//   3. Each warp streams blocks of LB token slots, two blocks per step. Key
//      pass: lane = slot; the slot's rotated row of J key bytes gives J LUT
//      reads on J distinct columns across the warp (no bank conflicts); one
//      byte permute forms the address and the step is the load's offset.
//      Value pass: lane = (replica, channel group) owns one column of its
//      warp's private histogram W[e][col]; it adds p = 2^(x - m) of its
//      slots at the rows given by the group-major value bytes, two slots per
//      step with one equality check so that two updates of one word merge.
//      No lane writes another lane's column: no atomics, no warp ordering.
//      Index bytes are prefetched two blocks ahead into registers and pages
//      further ahead into L2.
//   4. Warps are merged, the loop-tau value codebook slice is staged into
//      the freed histogram space and contracted with the histogram
//      (o[j*c+ch] = sum_e W[e][j] C_V[j][e][tau][ch]); the segment writes
//      (m, l, o[d]) to record slot (pair + cta).
//
// vq_finish_kernel: one CTA per pair. It scores the bf16 window tokens
// (prefix + recent) densely and merges that partial with the pair's segment
// records (log-sum-exp merge) into out and lse.

#include <math.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kNW = 5;                  // warps per CTA, one value histogram each
constexpr int kThreads = kNW * 32;
constexpr int kRing = 4;                // blocks in registers: the pair in use + the next pair
constexpr int kRegion = kE * kRowStride;  // floats in one [E][32] table (32 KB)
constexpr int kLutRow = 64;             // LUT row: 64 columns, column k holds group k % J
constexpr int kLutFloats = kE * kLutRow;  // 64 KB
constexpr int kStageRegions = 4;        // histogram regions 1..4 double as codebook staging
constexpr int kPrefetchPages = 8;       // pages a warp asks L2 to fetch ahead of its loads
constexpr float kRescaleSlack = 8.0f;   // log2 units a new maximum may exceed m before rescaling
constexpr int kFinishThreads = 128;
constexpr int kWinChunk = 8;            // window tokens per warp per round of loads (finish)

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
  float* records;                   // [pairs + n_cta][d+2]
  void* out;
  float* lse;
  int B, Hq, Hkv, ratio, W, Pg, n_pages, max_pages_per_seq, max_seq_len;
  int64_t page_bytes, plane_bytes;
  int n_cta, out_dtype;
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
  int base;            // first slot of the block inside its page, or -1: no block
  int valid;           // valid slots in the page (same value in every lane)
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
template <int NT>
__device__ __forceinline__ void stage_async(float* dst, const float* src, int nfloats, int tid) {
  for (int i = tid * 4; i < nfloats; i += NT * 4) cp_async16(dst + i, src + i);
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

// Quantised-token pages of sequence b.
__device__ __forceinline__ int seq_pages(const DecodeParams& p, int b) {
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_vq = max(0, N - p.W);
  return min((n_vq + p.Pg - 1) / p.Pg, p.max_pages_per_seq);
}

// Inclusive warp prefix sum.
__device__ __forceinline__ long long warp_incl_scan(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Walks sequences 0..B-1 (a warp at a time) to find the sequence whose
// units [Hq*pre, Hq*(pre + pages)) contain unit `u` (or, with u < 0, just
// the total). Returns the total number of units; *b_out, *pre_out describe
// the hit (b_out = -1 if none).
__device__ long long find_unit(const DecodeParams& p, long long u, int lane, int* b_out,
                               long long* pre_out) {
  long long acc = 0;                                   // units before sequence b0
  *b_out = -1;
  *pre_out = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const long long units = (b < p.B) ? static_cast<long long>(p.Hq) * seq_pages(p, b) : 0;
    const long long incl = warp_incl_scan(units, lane);
    const long long excl = incl - units;
    const bool hit = units > 0 && acc + excl <= u && u < acc + incl;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m != 0u && *b_out < 0) {
      const int src = __ffs(m) - 1;
      *b_out = b0 + src;
      *pre_out = (acc + __shfl_sync(0xffffffffu, excl, src)) / p.Hq;
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  return acc;
}

template <int J, int C>
__global__ void __launch_bounds__(kThreads, 1) vq_stream_kernel(const DecodeParams p) {
  using T = Traits<J>;
  constexpr int d = J * C;
  constexpr int R = T::R, LB = T::LB;
  // channel groups per staging chunk: a [JC][E][C] slice fits regions 1..4
  constexpr int JC = (J * kE * C <= kStageRegions * kRegion) ? J : (kStageRegions * kRegion) / (kE * C);
  static_assert(J % JC == 0, "staging chunks must tile the channel groups");

  extern __shared__ __align__(16) float smem[];
  float* lut = smem;                                   // [E][64]
  float* hist = lut + kLutFloats;                      // [kNW][E][32]
  float* pbuf = hist + kNW * kRegion;                  // [kNW][64]
  float* wstat = pbuf + kNW * 64;                      // [2*kNW]
  float* stage = hist + kRegion;                       // regions 1..4
  float* qs = hist;                                    // scratch in region 0 before zeroing

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool lane_live = lane < LB;
  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;   // fits one byte
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;   // fits one byte
  const char* lut_bytes = reinterpret_cast<const char*>(lut);
  float* my_hist = hist + warp * kRegion;
  char* hist_bytes = reinterpret_cast<char*>(my_hist);
  float* my_p = pbuf + warp * 64;
  const int bpp = p.Pg / LB;                           // blocks per page
  const uint32_t bpp_magic = 0xFFFFFFFFu / static_cast<uint32_t>(bpp) + 1u;   // k / bpp = umulhi

  // ---- this CTA's range of units (pages) ---------------------------------
  int b_first;
  long long pre_first;
  const long long U = find_unit(p, -1, lane, &b_first, &pre_first);
  const long long u_lo = U * blockIdx.x / p.n_cta;
  const long long u_hi = U * (blockIdx.x + 1) / p.n_cta;
  if (u_lo >= u_hi) return;                            // CTA-uniform
  int b;
  long long pre;
  find_unit(p, u_lo, lane, &b, &pre);
  int pages_b = seq_pages(p, b);
  long long off = u_lo - static_cast<long long>(p.Hq) * pre;   // unit offset inside sequence b
  int hq = static_cast<int>(off / pages_b);
  int pg_start = static_cast<int>(off % pages_b);
  long long u = u_lo;

  while (u < u_hi && b < p.B) {                        // one segment per iteration
    const int seg_pages = static_cast<int>(min(static_cast<long long>(pages_b - pg_start), u_hi - u));
    const int pg_lo = pg_start, pg_hi = pg_start + seg_pages;
    const int hkv = hq / p.ratio;
    const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
    const int n_vq = max(0, N - p.W);
    const float* cbk = p.cb_k + hkv * p.cb_stride_head;
    const float* cbv = p.cb_v + hkv * p.cb_stride_head;
    __syncthreads();                                   // previous segment done with shared memory

    // ---- 1. request the first index blocks of this warp ------------------
    const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
    const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
    const int my_first = pg_lo + warp;
    const int n_my_pages = (pg_hi > my_first) ? (pg_hi - my_first + kNW - 1) / kNW : 0;
    const int n_blocks = n_my_pages * bpp;
    int i0 = 0;
    auto bt_entry = [&](int i) -> int { return (i < n_my_pages) ? bt[my_first + i * kNW] : -1; };
    int bt_cur = bt_entry(lane);
    int bt_nxt = bt_entry(32 + lane);
    if (lane < kPrefetchPages && lane < n_my_pages && bt_cur >= 0 && bt_cur < p.n_pages)
      prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_cur) * p.page_bytes,
                       static_cast<uint32_t>(p.page_bytes));
    BlockRegs<J> ring[kRing];
    auto clear = [&](BlockRegs<J>& r) {
      r.base = -1;
#pragma unroll
      for (int i = 0; i < T::NWORD; ++i) {
        r.k[i] = 0u;
        r.v[i] = 0u;
      }
    };
    auto issue = [&](int k, BlockRegs<J>& r) {
      if (k >= n_blocks) {                              // warp-uniform
        clear(r);
        return;
      }
      const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(k), bpp_magic));
      const int blk = k - pi * bpp;
      if (pi >= i0 + 32) {                              // warp-uniform
        bt_cur = bt_nxt;
        i0 += 32;
        bt_nxt = bt_entry(i0 + 32 + lane);
      }
      if (blk == 0) {                                   // first block of a page: prefetch ahead
        const int tgt = pi + kPrefetchPages;            // tgt - i0 < 64: inside cur or nxt
        const int src = (tgt - i0 < 32) ? bt_cur : bt_nxt;
        const int pf = __shfl_sync(0xffffffffu, src, (tgt - i0) & 31);
        if (lane == 0 && tgt < n_my_pages && pf >= 0 && pf < p.n_pages)
          prefetch_l2_bulk(pool_h + static_cast<int64_t>(pf) * p.page_bytes,
                           static_cast<uint32_t>(p.page_bytes));
      }
      const int phys = __shfl_sync(0xffffffffu, bt_cur, pi - i0);
      const int pg = my_first + pi * kNW;
      r.valid = min(p.Pg, n_vq - pg * p.Pg);
      r.base = blk * LB;
      if (phys < 0 || phys >= p.n_pages || r.base >= r.valid) {   // nothing to read
        clear(r);
        return;
      }
      load_block<J>(pool_h + static_cast<int64_t>(phys) * p.page_bytes, p.plane_bytes, p.Pg, blk,
                    lane, r);
    };
#pragma unroll
    for (int u2 = 0; u2 < kRing; ++u2) issue(u2, ring[u2]);

    // ---- 2. key lookup table (codebook staged in regions 1..4) -------------
    stage_async<kThreads>(stage, cbk, JC * kE * C, tid);
    const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * d;
    for (int i = tid; i < d; i += kThreads) qs[i] = bf16_bits_to_float(qp[i]) * p.scale_log2;
    for (int j0 = 0; j0 < J; j0 += JC) {
      if (j0 > 0) {
        __syncthreads();                                // previous chunk consumed
        stage_async<kThreads>(stage, cbk + static_cast<size_t>(j0) * kE * C, JC * kE * C, tid);
      }
      cp_async_wait_all();
      __syncthreads();
      // item = (e-tile of 32, step s): lane -> e = tile*32 + lane, group
      // j0 + (lane + s) % JC; rotating the group spreads the table writes
      // over distinct banks.
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
    __syncthreads();                                    // LUT complete; scratch no longer read
    {
      float4* h4 = reinterpret_cast<float4*>(my_hist);
      for (int i = lane; i < kRegion / 4; i += 32) h4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncwarp();

    // ---- 3. stream index blocks, two per step ------------------------------
    float m_w = -INFINITY;
    float l_lane = 0.f;

    auto key_scores = [&](const BlockRegs<J>& r) -> float {
      // Row byte s holds the index of group (lane + s) % J, which LUT column
      // lane + s holds: one byte permute forms (e << 8) | lane*4 and the
      // step goes into the load's offset.
      float xa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < J; ++s) {
        const uint32_t o = __byte_perm(r.k[s >> 2], lane4, 0x5504u | (uint32_t(s & 3) << 4));
        xa[s & 3] += *reinterpret_cast<const float*>(lut_bytes + o + 4 * s);
      }
      const bool valid = r.base >= 0 && lane_live && (r.base + lane) < r.valid;
      return valid ? (xa[0] + xa[1]) + (xa[2] + xa[3]) : -INFINITY;
    };
    auto value_pass = [&](const BlockRegs<J>& r, const float* pp) {
      // lane = (replica, group) owns column `lane`; slots rr*J + i of the block
      if (r.base < 0 || !lane_live) return;
      pp += (lane / J) * J;
#pragma unroll
      for (int i = 0; i < J; i += 2) {
        // (e << 8 | lane*8) >> 1 = e*128 + lane*4: the byte offset of W[e][lane]
        const uint32_t oa = __byte_perm(r.v[i >> 2], lane8, 0x5504u | (uint32_t(i & 3) << 4)) >> 1;
        const uint32_t ob =
            __byte_perm(r.v[(i + 1) >> 2], lane8, 0x5504u | (uint32_t((i + 1) & 3) << 4)) >> 1;
        const float2 pab = *reinterpret_cast<const float2*>(pp + i);
        float* wa = reinterpret_cast<float*>(hist_bytes + oa);
        float* wb = reinterpret_cast<float*>(hist_bytes + ob);
        const float na = *wa + pab.x;
        const float vb = (oa == ob) ? na : *wb;         // second update of the same word
        *wa = na;
        *wb = vb + pab.y;
      }
    };
    auto process_pair = [&](const BlockRegs<J>& ra, const BlockRegs<J>& rb) {
      const float xa = key_scores(ra);
      const float xb = key_scores(rb);
      const float xm = warp_max(fmaxf(xa, xb));
      if (xm == -INFINITY) return;                      // both blocks empty: warp-uniform
      if (xm > m_w + kRescaleSlack) {                   // warp-uniform
        if (m_w != -INFINITY) {
          const float f = fast_exp2(m_w - xm);
#pragma unroll 8
          for (int e = 0; e < kE; ++e) my_hist[e * kRowStride + lane] *= f;   // own column
          l_lane *= f;
        }
        m_w = xm;
      }
      const float pa = (xa == -INFINITY) ? 0.f : fast_exp2(xa - m_w);
      const float pb = (xb == -INFINITY) ? 0.f : fast_exp2(xb - m_w);
      l_lane += pa + pb;
      my_p[lane] = pa;
      my_p[32 + lane] = pb;
      __syncwarp();
      value_pass(ra, my_p);
      value_pass(rb, my_p + 32);
      __syncwarp();                                     // my_p is rewritten by the next step
    };

    for (int k0 = 0; k0 < n_blocks; k0 += kRing) {
      process_pair(ring[0], ring[1]);
      issue(k0 + kRing, ring[0]);
      issue(k0 + kRing + 1, ring[1]);
      if (k0 + 2 >= n_blocks) break;
      process_pair(ring[2], ring[3]);
      issue(k0 + kRing + 2, ring[2]);
      issue(k0 + kRing + 3, ring[3]);
    }
    const float l_w = warp_sum(l_lane);
    if (lane == 0) {
      wstat[warp] = m_w;
      wstat[kNW + warp] = l_w;
    }
    __syncthreads();

    // ---- 4. merge warps, contract the histogram ----------------------------
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, wstat[w]);
    float* rec = p.records + static_cast<size_t>(b * p.Hq + hq + blockIdx.x) * (d + 2);
    if (M == -INFINITY) {                               // only absent pages: empty record
      for (int i = tid; i < d + 2; i += kThreads) rec[i] = (i == 0) ? -INFINITY : 0.f;
    } else {
      float f[kNW];
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        f[w] = (wstat[w] == -INFINITY) ? 0.f : fast_exp2(wstat[w] - M);
        L += f[w] * wstat[kNW + w];
      }
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
        __syncthreads();                                // histogram merged / previous chunk used
        stage_async<kThreads>(stage, cbv + static_cast<size_t>(j0) * kE * C, JC * kE * C, tid);
        cp_async_wait_all();
        __syncthreads();
        // thread -> (group jj, channel ch); rows visited from e = jj so that
        // the threads of a warp read different banks of the staged slice
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
          rec[2 + j * C + ch] = acc;
        }
      }
      if (tid == 0) {
        rec[0] = M;
        rec[1] = L;
      }
    }

    // ---- next segment ------------------------------------------------------
    u += seg_pages;
    pg_start = 0;
    if (++hq == p.Hq) {
      hq = 0;
      do {
        ++b;
      } while (b < p.B && u < u_hi && (pages_b = seq_pages(p, b)) == 0);
    }
  }
}

// ---------------------------------------------------------------------------
// Value path by explicit dequantisation (used when the loop-tau value
// codebook slice fits in shared memory next to the key LUT).
//
// Same partition, segment walk, index stream and key pass as
// vq_stream_kernel. The value slice is staged once per segment as
// [E][C/CW][JP][CW] floats (JP = J rounded up so that the 16-byte reads of
// the lanes of a warp fall on distinct bank groups). In the value pass a
// lane = (replica, group j) accumulates o[j*c..j*c+c) += p * C_V[e][j] in
// registers, one 16-byte shared read per slot: no read-modify-write, no
// per-warp histogram, so the CTA runs kDqWarps warps and an online-softmax
// rescale only touches registers.
// ---------------------------------------------------------------------------

constexpr int kDqWarps = 8;
constexpr int kDqThreads = kDqWarps * 32;

template <int J, int C>
struct DqGeo {
  static constexpr int CW = (C >= 4) ? 4 : C;          // floats per shared read
  static constexpr int NH = C / CW;                    // reads per codeword slice
  static constexpr int JP = (CW == 4) ? ((J + 7) / 8) * 8 : ((J + 15) / 16) * 16;
  static constexpr int CV_FLOATS = kE * NH * JP * CW;  // [E][NH][JP][CW]
  static constexpr int CK_FLOATS = J * kE * C;         // staged key slice [J][E][C]
  static constexpr int STAGE_FLOATS = CV_FLOATS > CK_FLOATS ? CV_FLOATS : CK_FLOATS;
  static constexpr int RSB = NH * JP * CW * 4;         // bytes per centroid row of the value slice
};

template <int J, int C>
constexpr size_t dq_smem_bytes() {
  return (static_cast<size_t>(kLutFloats) + DqGeo<J, C>::STAGE_FLOATS + kDqWarps * 32 * C +
          kDqWarps * 64 + 2 * kDqWarps) *
         sizeof(float);
}

template <int J, int C>
constexpr bool dq_fits() {
  return dq_smem_bytes<J, C>() <= 227 * 1024 && C % 2 == 0;
}

template <int J, int C>
__global__ void __launch_bounds__(kDqThreads, 1) vq_stream_dq_kernel(const DecodeParams p) {
  using T = Traits<J>;
  using G = DqGeo<J, C>;
  constexpr int d = J * C;
  constexpr int LB = T::LB;
  constexpr int NW = kDqWarps;

  extern __shared__ __align__(16) float smem[];
  float* lut = smem;                                   // [E][64]
  float* stage = lut + kLutFloats;                     // key slice, then value slice
  float* obuf = stage + G::STAGE_FLOATS;               // [NW][32][C] end-of-segment partials
  float* pbuf = obuf + NW * 32 * C;                    // [NW][64]
  float* wstat = pbuf + NW * 64;                       // [2*NW]
  float* qs = obuf;                                    // q scratch (d floats) before the stream

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool lane_live = lane < LB;
  const int vj = lane % J;                             // value pass: this lane's group
  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
  const char* lut_bytes = reinterpret_cast<const char*>(lut);
  const char* cv_bytes = reinterpret_cast<const char*>(stage) + vj * G::CW * 4;
  float* my_p = pbuf + warp * 64;
  const int bpp = p.Pg / LB;
  const uint32_t bpp_magic = 0xFFFFFFFFu / static_cast<uint32_t>(bpp) + 1u;

  int b_first;
  long long pre_first;
  const long long U = find_unit(p, -1, lane, &b_first, &pre_first);
  const long long u_lo = U * blockIdx.x / p.n_cta;
  const long long u_hi = U * (blockIdx.x + 1) / p.n_cta;
  if (u_lo >= u_hi) return;
  int b;
  long long pre;
  find_unit(p, u_lo, lane, &b, &pre);
  int pages_b = seq_pages(p, b);
  const long long off = u_lo - static_cast<long long>(p.Hq) * pre;
  int hq = static_cast<int>(off / pages_b);
  int pg_start = static_cast<int>(off % pages_b);
  long long u = u_lo;

  while (u < u_hi && b < p.B) {
    const int seg_pages = static_cast<int>(min(static_cast<long long>(pages_b - pg_start), u_hi - u));
    const int pg_lo = pg_start, pg_hi = pg_start + seg_pages;
    const int hkv = hq / p.ratio;
    const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
    const int n_vq = max(0, N - p.W);
    const float* cbk = p.cb_k + hkv * p.cb_stride_head;
    const float* cbv = p.cb_v + hkv * p.cb_stride_head;
    __syncthreads();                                   // previous segment done with shared memory

    // ---- index ring prologue ------------------------------------------------
    const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
    const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
    const int my_first = pg_lo + warp;
    const int n_my_pages = (pg_hi > my_first) ? (pg_hi - my_first + NW - 1) / NW : 0;
    const int n_blocks = n_my_pages * bpp;
    int i0 = 0;
    auto bt_entry = [&](int i) -> int { return (i < n_my_pages) ? bt[my_first + i * NW] : -1; };
    int bt_cur = bt_entry(lane);
    int bt_nxt = bt_entry(32 + lane);
    if (lane < kPrefetchPages && lane < n_my_pages && bt_cur >= 0 && bt_cur < p.n_pages)
      prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_cur) * p.page_bytes,
                       static_cast<uint32_t>(p.page_bytes));
    BlockRegs<J> ring[kRing];
    auto clear = [&](BlockRegs<J>& r) {
      r.base = -1;
#pragma unroll
      for (int i = 0; i < T::NWORD; ++i) {
        r.k[i] = 0u;
        r.v[i] = 0u;
      }
    };
    auto issue = [&](int k, BlockRegs<J>& r) {
      if (k >= n_blocks) {
        clear(r);
        return;
      }
      const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(k), bpp_magic));
      const int blk = k - pi * bpp;
      if (pi >= i0 + 32) {
        bt_cur = bt_nxt;
        i0 += 32;
        bt_nxt = bt_entry(i0 + 32 + lane);
      }
      if (blk == 0) {
        const int tgt = pi + kPrefetchPages;
        const int src = (tgt - i0 < 32) ? bt_cur : bt_nxt;
        const int pf = __shfl_sync(0xffffffffu, src, (tgt - i0) & 31);
        if (lane == 0 && tgt < n_my_pages && pf >= 0 && pf < p.n_pages)
          prefetch_l2_bulk(pool_h + static_cast<int64_t>(pf) * p.page_bytes,
                           static_cast<uint32_t>(p.page_bytes));
      }
      const int phys = __shfl_sync(0xffffffffu, bt_cur, pi - i0);
      const int pg = my_first + pi * NW;
      r.valid = min(p.Pg, n_vq - pg * p.Pg);
      r.base = blk * LB;
      if (phys < 0 || phys >= p.n_pages || r.base >= r.valid) {
        clear(r);
        return;
      }
      load_block<J>(pool_h + static_cast<int64_t>(phys) * p.page_bytes, p.plane_bytes, p.Pg, blk,
                    lane, r);
    };
#pragma unroll
    for (int u2 = 0; u2 < kRing; ++u2) issue(u2, ring[u2]);

    // ---- key LUT from the staged key slice ---------------------------------
    stage_async<kDqThreads>(stage, cbk, G::CK_FLOATS, tid);
    const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * d;
    for (int i = tid; i < d; i += kDqThreads) qs[i] = bf16_bits_to_float(qp[i]) * p.scale_log2;
    cp_async_wait_all();
    __syncthreads();
    for (int item = warp; item < (kE / 32) * J; item += NW) {
      const int tile = item / J, s = item % J;
      const int e = tile * 32 + lane;
      const int j = (lane + s) % J;
      const float v = dot_c<C>(qs + j * C, stage + (static_cast<size_t>(j) * kE + e) * C);
#pragma unroll
      for (int k = j; k < kLutRow; k += J) lut[e * kLutRow + k] = v;
    }
    __syncthreads();                                   // LUT done; key slice no longer read
    // ---- value slice [E][NH][JP][CW] ----------------------------------------
    for (int idx = tid; idx < J * kE * G::NH; idx += kDqThreads) {
      const int j = idx / (kE * G::NH), rem = idx % (kE * G::NH);
      const int e = rem / G::NH, h = rem % G::NH;
      const float* src = cbv + (static_cast<size_t>(j) * kE + e) * C + h * G::CW;
      float* dst = stage + ((e * G::NH + h) * G::JP + j) * G::CW;
      if constexpr (G::CW == 4)
        cp_async16(dst, src);
      else
        cp_async8(dst, src);
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- stream -------------------------------------------------------------
    float m_w = -INFINITY;
    float l_lane = 0.f;
    float o[C];
#pragma unroll
    for (int c = 0; c < C; ++c) o[c] = 0.f;

    auto key_scores = [&](const BlockRegs<J>& r) -> float {
      float xa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < J; ++s) {
        const uint32_t ob = __byte_perm(r.k[s >> 2], lane4, 0x5504u | (uint32_t(s & 3) << 4));
        xa[s & 3] += *reinterpret_cast<const float*>(lut_bytes + ob + 4 * s);
      }
      const bool valid = r.base >= 0 && lane_live && (r.base + lane) < r.valid;
      return valid ? (xa[0] + xa[1]) + (xa[2] + xa[3]) : -INFINITY;
    };
    auto value_pass = [&](const BlockRegs<J>& r, const float* pp) {
      if (r.base < 0 || !lane_live) return;
      pp += (lane / J) * J;
#pragma unroll
      for (int i = 0; i < J; i += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(pp + i);
        const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t e = byte_of(r.v[i >> 2], k);
          const char* row = cv_bytes + e * G::RSB;
#pragma unroll
          for (int h = 0; h < G::NH; ++h) {
            if constexpr (G::CW == 4) {
              const float4 cw = *reinterpret_cast<const float4*>(row + h * G::JP * 16);
              o[4 * h] = fmaf(pv[k], cw.x, o[4 * h]);
              o[4 * h + 1] = fmaf(pv[k], cw.y, o[4 * h + 1]);
              o[4 * h + 2] = fmaf(pv[k], cw.z, o[4 * h + 2]);
              o[4 * h + 3] = fmaf(pv[k], cw.w, o[4 * h + 3]);
            } else {
              const float2 cw = *reinterpret_cast<const float2*>(row + h * G::JP * 8);
              o[2 * h] = fmaf(pv[k], cw.x, o[2 * h]);
              o[2 * h + 1] = fmaf(pv[k], cw.y, o[2 * h + 1]);
            }
          }
        }
      }
    };
    auto process_pair = [&](const BlockRegs<J>& ra, const BlockRegs<J>& rb) {
      const float xa = key_scores(ra);
      const float xb = key_scores(rb);
      const float xm = warp_max(fmaxf(xa, xb));
      if (xm == -INFINITY) return;
      if (xm > m_w + kRescaleSlack) {
        if (m_w != -INFINITY) {
          const float f = fast_exp2(m_w - xm);
#pragma unroll
          for (int c = 0; c < C; ++c) o[c] *= f;
          l_lane *= f;
        }
        m_w = xm;
      }
      const float pa = (xa == -INFINITY) ? 0.f : fast_exp2(xa - m_w);
      const float pb = (xb == -INFINITY) ? 0.f : fast_exp2(xb - m_w);
      l_lane += pa + pb;
      my_p[lane] = pa;
      my_p[32 + lane] = pb;
      __syncwarp();
      value_pass(ra, my_p);
      value_pass(rb, my_p + 32);
      __syncwarp();                                    // my_p is rewritten by the next step
    };

    for (int k0 = 0; k0 < n_blocks; k0 += kRing) {
      process_pair(ring[0], ring[1]);
      issue(k0 + kRing, ring[0]);
      issue(k0 + kRing + 1, ring[1]);
      if (k0 + 2 >= n_blocks) break;
      process_pair(ring[2], ring[3]);
      issue(k0 + kRing + 2, ring[2]);
      issue(k0 + kRing + 3, ring[3]);
    }
    const float l_w = warp_sum(l_lane);
    if (lane == 0) {
      wstat[warp] = m_w;
      wstat[NW + warp] = l_w;
    }
#pragma unroll
    for (int c = 0; c < C; ++c) obuf[(warp * 32 + lane) * C + c] = lane_live ? o[c] : 0.f;
    __syncthreads();

    // ---- merge warps into the segment record --------------------------------
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wstat[w]);
    float* rec = p.records + static_cast<size_t>(b * p.Hq + hq + blockIdx.x) * (d + 2);
    if (M == -INFINITY) {
      for (int i = tid; i < d + 2; i += kDqThreads) rec[i] = (i == 0) ? -INFINITY : 0.f;
    } else {
      float L = 0.f;
      float f[NW];
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        f[w] = (wstat[w] == -INFINITY) ? 0.f : fast_exp2(wstat[w] - M);
        L += f[w] * wstat[NW + w];
      }
      for (int oi = tid; oi < d; oi += kDqThreads) {
        const int j = oi / C, c = oi % C;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          float s = 0.f;
#pragma unroll
          for (int r = 0; r < T::R; ++r) s += obuf[(w * 32 + r * J + j) * C + c];
          acc = fmaf(f[w], s, acc);
        }
        rec[2 + oi] = acc;
      }
      if (tid == 0) {
        rec[0] = M;
        rec[1] = L;
      }
    }

    u += seg_pages;
    pg_start = 0;
    if (++hq == p.Hq) {
      hq = 0;
      do {
        ++b;
      } while (b < p.B && u < u_hi && (pages_b = seq_pages(p, b)) == 0);
    }
  }
}

// One CTA per (sequence, query head): the bf16 window partial, merged with
// the pair's segment records into out and lse.
template <int D>
__global__ void __launch_bounds__(kFinishThreads) vq_finish_kernel(const DecodeParams p) {
  constexpr int NW = kFinishThreads / 32;
  constexpr int NPL = (D / 2 + 31) / 32;               // bf16 channel pairs per lane
  __shared__ float qs[D];
  __shared__ float xwin[256];
  __shared__ float opart[NW][D];
  __shared__ float sstat[5];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x;
  const int b = pair / p.Hq, hq = pair % p.Hq, hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_win = min(N, p.W);

  const uint16_t* qp = p.q + static_cast<size_t>(pair) * D;
  for (int i = tid; i < D; i += kFinishThreads) qs[i] = bf16_bits_to_float(qp[i]) * p.scale_log2;
  __syncthreads();

  // window scores: warp w takes tokens w, w + NW, ...; lane = channel pairs
  const uint16_t* wkb = p.win_k + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * D;
  const uint16_t* wvb = p.win_v + (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * D;
  for (int t0 = warp; t0 < n_win; t0 += NW * kWinChunk) {
    uint32_t kr[kWinChunk][NPL];
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      const int t = t0 + i * NW;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;
        kr[i][k] = (t < n_win && pc < D / 2)
                       ? __ldg(reinterpret_cast<const unsigned int*>(wkb + t * D) + pc) : 0u;
      }
    }
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;
        if (pc < D / 2) {
          const float2 kv = bf16x2_to_float2(kr[i][k]);
          acc = fmaf(qs[2 * pc], kv.x, fmaf(qs[2 * pc + 1], kv.y, acc));
        }
      }
      acc = warp_sum(acc);
      const int t = t0 + i * NW;
      if (lane == 0 && t < n_win) xwin[t] = acc;
    }
  }
  __syncthreads();
  float m_win = -INFINITY, l_win = 0.f;
  for (int t = 0; t < n_win; ++t) m_win = fmaxf(m_win, xwin[t]);
  for (int t = 0; t < n_win; ++t) l_win += fast_exp2(xwin[t] - m_win);
  {
    float oacc[NPL][2];
#pragma unroll
    for (int k = 0; k < NPL; ++k) oacc[k][0] = oacc[k][1] = 0.f;
    for (int t0 = warp; t0 < n_win; t0 += NW * kWinChunk) {
      uint32_t vr[kWinChunk][NPL];
#pragma unroll
      for (int i = 0; i < kWinChunk; ++i) {
        const int t = t0 + i * NW;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const int pc = lane + 32 * k;
          vr[i][k] = (t < n_win && pc < D / 2)
                         ? __ldg(reinterpret_cast<const unsigned int*>(wvb + t * D) + pc) : 0u;
        }
      }
#pragma unroll
      for (int i = 0; i < kWinChunk; ++i) {
        const int t = t0 + i * NW;
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
      if (pc < D / 2) {
        opart[warp][2 * pc] = oacc[k][0];
        opart[warp][2 * pc + 1] = oacc[k][1];
      }
    }
  }

  // the pair's segment records: slots pair + c for the CTAs c that own its units
  if (warp == 0) {
    int bb;
    long long pre;
    const long long U = find_unit(p, -1, lane, &bb, &pre);
    // units before this pair: Hq * (pages of sequences < b) + hq * pages_b
    long long before = 0;
    for (int b0 = 0; b0 < b; b0 += 32) {
      const int bi = b0 + lane;
      long long v = (bi < b) ? static_cast<long long>(seq_pages(p, bi)) : 0;
      v = warp_incl_scan(v, lane);
      before += __shfl_sync(0xffffffffu, v, 31);
    }
    const int pages_b = seq_pages(p, b);
    const long long u0 = before * p.Hq + static_cast<long long>(hq) * pages_b;
    int c_first = 0, c_last = -1;
    if (pages_b > 0 && U > 0) {
      c_first = static_cast<int>(((u0 + 1) * p.n_cta - 1) / U);
      c_last = static_cast<int>(((u0 + pages_b) * p.n_cta - 1) / U);
    }
    // a CTA whose unit range is empty wrote no record
    auto has_units = [&](int c) { return U * c / p.n_cta < U * (c + 1) / p.n_cta; };
    float M = m_win;
    for (int c = c_first + lane; c <= c_last; c += 32)
      if (has_units(c)) M = fmaxf(M, p.records[static_cast<size_t>(pair + c) * (D + 2)]);
    M = warp_max(M);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int c = c_first + lane; c <= c_last; c += 32) {
        if (!has_units(c)) continue;
        const float* rec = p.records + static_cast<size_t>(pair + c) * (D + 2);
        if (rec[0] != -INFINITY) L += rec[1] * fast_exp2(rec[0] - M);
      }
    }
    L = warp_sum(L);
    if (lane == 0) {
      L += (m_win == -INFINITY) ? 0.f : l_win * fast_exp2(m_win - M);
      sstat[0] = M;
      sstat[1] = L;
      sstat[2] = __int_as_float(c_first);
      sstat[3] = __int_as_float(c_last);
      sstat[4] = __int_as_float(static_cast<int>(U));   // units fit in 31 bits
    }
  }
  __syncthreads();
  const float M = sstat[0], L = sstat[1];
  const int c_first = __float_as_int(sstat[2]), c_last = __float_as_int(sstat[3]);
  const long long U = __float_as_int(sstat[4]);
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  const float f_win = (m_win == -INFINITY || M == -INFINITY) ? 0.f : fast_exp2(m_win - M);
  for (int ch = tid; ch < D; ch += kFinishThreads) {
    float o = 0.f;
    if (M != -INFINITY) {
      for (int c = c_first; c <= c_last; ++c) {
        if (U * c / p.n_cta == U * (c + 1) / p.n_cta) continue;   // no record
        const float* rec = p.records + static_cast<size_t>(pair + c) * (D + 2);
        if (rec[0] != -INFINITY) o = fmaf(rec[2 + ch], fast_exp2(rec[0] - M), o);
      }
      if (f_win != 0.f) {
        float ow = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) ow += opart[w][ch];
        o = fmaf(f_win, ow, o);
      }
    }
    o *= inv;
    if (p.out_dtype == LOOPVQ_DTYPE_F32)
      static_cast<float*>(p.out)[static_cast<size_t>(pair) * D + ch] = o;
    else
      static_cast<__nv_bfloat16*>(p.out)[static_cast<size_t>(pair) * D + ch] = __float2bfloat16_rn(o);
  }
  if (tid == 0 && p.lse != nullptr)
    p.lse[pair] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
}

constexpr size_t stream_smem_bytes() {
  return (static_cast<size_t>(kLutFloats) + static_cast<size_t>(kRegion) * kNW + kNW * 64 + 2 * kNW) *
         sizeof(float);
}
static_assert(stream_smem_bytes() <= 227 * 1024, "stream kernel shared memory above 227 KB");

template <typename K>
loopvq_status set_smem(K kernel, size_t smem, std::atomic<uint64_t>& configured) {
  // The attribute belongs to (function, device); remember which devices have it.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit == 0 || !(configured.load(std::memory_order_relaxed) & bit)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return LOOPVQ_ERR_CUDA;
    configured.fetch_or(bit, std::memory_order_relaxed);
  }
  return LOOPVQ_OK;
}

template <int J, int C>
loopvq_status launch_vq(const DecodeParams& p, cudaStream_t st, bool run_stream) {
  constexpr int d = J * C;
  if (run_stream && dq_fits<J, C>()) {
    static std::atomic<uint64_t> configured{0};
    const size_t smem = dq_smem_bytes<J, C>();
    if (set_smem(vq_stream_dq_kernel<J, C>, smem, configured) != LOOPVQ_OK) return LOOPVQ_ERR_CUDA;
    vq_stream_dq_kernel<J, C><<<p.n_cta, kDqThreads, smem, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  } else if (run_stream) {
    const size_t smem = stream_smem_bytes();
    // The attribute belongs to (function, device); remember which devices have it.
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit == 0 || !(configured.load(std::memory_order_relaxed) & bit)) {
      if (cudaFuncSetAttribute(vq_stream_kernel<J, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess)
        return LOOPVQ_ERR_CUDA;
      configured.fetch_or(bit, std::memory_order_relaxed);
    }
    vq_stream_kernel<J, C><<<p.n_cta, kThreads, smem, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  }
  vq_finish_kernel<d><<<p.B * p.Hq, kFinishThreads, 0, st>>>(p);
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
  p.records = static_cast<float*>(a.workspace);
  p.out = a.out;
  p.lse = a.lse;
  p.B = a.batch;
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
  p.n_cta = a.n_cta;
  p.out_dtype = a.out_dtype;
  p.scale_log2 = a.sm_scale * kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  const bool run = a.n_cta > 0;
  if (!run) p.n_cta = 1;
  switch (g.J * 100 + g.c) {
    case 1604: return launch_vq<16, 4>(p, st, run);
    case 3204: return launch_vq<32, 4>(p, st, run);
    case 1208: return launch_vq<12, 8>(p, st, run);
    case 3202: return launch_vq<32, 2>(p, st, run);
    case 1608: return launch_vq<16, 8>(p, st, run);
    case 2404: return launch_vq<24, 4>(p, st, run);
    case 3208: return launch_vq<32, 8>(p, st, run);
    case 804:  return launch_vq<8, 4>(p, st, run);
    case 808:  return launch_vq<8, 8>(p, st, run);
    case 1202: return launch_vq<12, 2>(p, st, run);
    case 1602: return launch_vq<16, 2>(p, st, run);
    case 2402: return launch_vq<24, 2>(p, st, run);
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace loopvq
