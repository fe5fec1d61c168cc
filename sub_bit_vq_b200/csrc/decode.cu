// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// Two kernels per call.
//
// vq_stream_kernel: a persistent grid (at most one CTA per SM, sixteen warps)
// over the quantised tokens of every (sequence, query head) pair. All pages
// of all pairs form one list and CTA c takes the contiguous range
// [U*c/n, U*(c+1)/n) of it, so every CTA streams the same number of pages and
// touches one or a few pairs ("segments"). Per segment:
//   1. The key codebook slice of the pair's kv-head and loop step is staged
//      into the (empty) histogram window with cp.async while the warps
//      request their first index blocks (a register ring); the key lookup
//      table LUT[e][col] = s*log2(e) * q_j . C_K[j][e][tau] (column col holds
//      group j = col % J) is built from it and the window is zeroed.
//   2. Streaming, in chunks of kChunkBlocks blocks per warp. Key phase:
//      lane = slot; byte s of the slot's rotated row is group (lane+s) % J,
//      held by LUT column lane+s (the LUT repeats its J columns over 64), and
//      the scores x (log2 units) stay in registers.
//      The warps' maxima meet at a barrier; the segment's reference maximum
//      m becomes the integer ceil(max x) so far (when it rises, the histogram
//      is shifted right by the difference, which is exact in fixed point).
//      Value phase, lane = slot again: the slot's weight 2^(x - m) <= 1
//      becomes the integer w = rn(2^(x - m) * 2^kFixBits) and is added, for
//      each byte s of the slot's rotated value row, to the shared histogram
//      cell H[idx][(lane + s) % LB] by a 32-bit shared-memory atomic add on
//      the low word of a 64-bit cell, with the carry added to the high word.
//      Integer atomics run at full shared-memory rate on sm_100 and need no
//      turn taking, so all warps update the one histogram concurrently.
//   3. The histogram, converted to float, is contracted with the value
//      codebook slice, o_j = sum_e W[e][j] C_V[j][e][tau], and the segment
//      record (m, l = sum_e W[e][j], o[d]) goes to slot (pair + cta).
//
// vq_finish_kernel: one CTA per pair scores the bf16 window tokens (prefix +
// recent), merges them with the pair's segment records (log-sum-exp
// weights) and writes out and lse.
//
// The hot loops address shared memory by absolute shared-window address, so
// that one byte permute of an index byte gives a complete address: the LUT
// sits in a 64 KB-aligned window with 256-byte rows (64 columns) and the
// histogram in the next 64 KB window with 256-byte rows (low words in bytes
// 0..127 of a row, high words in bytes 128..255). Both windows are placed at run time
// above the dynamic allocation's base; a CTA whose allocation cannot hold
// them writes NaN records and flags the call's status word instead of
// running.

#include <math.h>

#include <atomic>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kNW = 16;                   // warps of the streaming kernel
constexpr int kThreads = kNW * 32;
constexpr int kRing = 4;                  // index blocks in registers
constexpr int kChunkBlocks = 4;           // blocks per warp per chunk (key phase, then value phase)
constexpr int kPrefetchPages = 4;         // pages a warp asks L2 to fetch ahead of its loads
constexpr int kFixBits = 30;              // fixed-point weight: w = rn(p * 2^kFixBits), p <= 1
constexpr float kFixScale = 1073741824.0f;          // 2^kFixBits
constexpr float kFixInv = 1.0f / 1073741824.0f;     // 2^-kFixBits
constexpr int kFinishThreads = 256;
constexpr int kWinChunk = 9;              // window tokens per warp per round of loads (72 = 8 warps x 9)
constexpr int kSegmentUnits = 16;         // work units (pages) charged for a segment's setup

// Small area at the start of the dynamic allocation (byte offsets).
constexpr uint32_t kWmaxOff = 0;                                  // [2][kNW] chunk maxima
constexpr uint32_t kQsOff = kWmaxOff + 2 * kNW * 4;               // [256] scaled q
constexpr uint32_t kSmallBytes = kQsOff + 256 * 4;
constexpr uint32_t kLutBytes = 0x10000u;  // [E][64] floats: column c holds group c % J
constexpr uint32_t kHistBytes = 0x10000u; // [E][64] words: 32 low, 32 high
// From any base b with b + kSmallBytes <= 0x10000 the LUT window starts at
// 0x10000 and the histogram window at 0x20000, so the allocation must reach
// 0x30000 - b; asking for 0x30000 bytes covers every such base.
constexpr uint32_t kDynBytes = 0x30000u;

// Groups of a [J][E][C] float codebook slice staged at once into the
// histogram window: the largest divisor of J whose slice part fits.
constexpr int stage_groups(int J, int C) {
  int jc = J;
  while (jc > 1 && (J % jc != 0 || jc * 256 * C * 4 > static_cast<int>(kHistBytes))) --jc;
  return jc;
}

// Bits of the status word (see loopvq.h).
constexpr int kStatusBadPage = 1;
constexpr int kStatusSharedBase = 2;

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
  float* records;                   // [pairs + n_cta][4 + d]: m, l, -, -, o[d]
  int* status;                      // status word (bit flags), never cleared by the kernels
  void* out;
  float* lse;
  int B, Hq, Hkv, ratio, W, Pg, n_pages, max_pages_per_seq, max_seq_len;
  int64_t page_bytes, plane_bytes;
  int n_cta, out_dtype;
  float scale_log2;
};

template <int J>
struct Traits {
  static constexpr int R = 32 / J;      // replicas of each group per block
  static constexpr int LB = R * J;      // slots per block
  static constexpr int GR = (J % 16 == 0) ? 16 : (J % 8 == 0) ? 8 : 4;   // granule
  static constexpr int NWORD = J / 4;   // words per lane and block
};

// One index block in registers: the rotated row of slot `lane` of the K
// plane (a key item) or of the V plane (a value item).
template <int J>
struct BlockRegs {
  uint32_t w[J / 4];
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

// Loads block `blk` of a page's K plane (kv = 0) or V plane (kv = 1): both
// planes hold rotated slot rows in granules, so lane = slot reads its row.
template <int J>
__device__ __forceinline__ void load_block(const uint8_t* kpl, int64_t plane_bytes, int blk, int kv,
                                           int lane, BlockRegs<J>& r) {
  using T = Traits<J>;
  if (lane < T::LB) {
    const uint8_t* src = kpl + kv * plane_bytes + blk * T::LB * J + lane * T::GR;
#pragma unroll
    for (int gi = 0; gi < J / T::GR; ++gi)
      load_words<T::GR>(src + gi * T::LB * T::GR, r.w + gi * (T::GR / 4), T::GR / 4);
  } else {
#pragma unroll
    for (int i = 0; i < T::NWORD; ++i) r.w[i] = 0u;
  }
}

// C consecutive floats from global memory (16-byte aligned when C % 4 == 0,
// 8-byte aligned when C == 2).
template <int C>
__device__ __forceinline__ void load_cw(const float* src, float (&v)[C]) {
  if constexpr (C % 4 == 0) {
#pragma unroll
    for (int i = 0; i < C; i += 4) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(src + i));
      v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < C; i += 2) {
      const float2 t = __ldg(reinterpret_cast<const float2*>(src + i));
      v[i] = t.x; v[i + 1] = t.y;
    }
  }
}

// sum_ch a[ch] * b[ch] for C channels held contiguously in shared memory
// (16-byte aligned when C % 4 == 0).
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

// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1 (compile-time i).
template <int N, typename F, int... I>
__device__ __forceinline__ void constexpr_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void constexpr_for(F&& f) {
  constexpr_for_impl<N>(f, std::make_integer_sequence<int, N>{});
}

// ---- shared memory by absolute shared-window address ------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

// LUT word at address a + OFF: not written while it is read.
template <int OFF>
__device__ __forceinline__ float lds_lut(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
// Histogram update: low word += w; on a carry out of the low word, the high
// word (128 bytes further along the row) += 1.
// Histogram updates of four cells by the same weight w: the low words at
// a0..a3 get w added and their old values come back in o0..o3.
__device__ __forceinline__ void hist_add4(const uint32_t (&a)[4], uint32_t w, uint32_t (&o)[4]) {
  asm volatile(
      "atom.shared.add.u32 %0, [%4], %8;\n"
      "atom.shared.add.u32 %1, [%5], %8;\n"
      "atom.shared.add.u32 %2, [%6], %8;\n"
      "atom.shared.add.u32 %3, [%7], %8;\n"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(w));
}
// The carries of those four updates: where an old low word exceeded
// nw = ~w (the sum wrapped), the high word 128 bytes further along the row
// gets 1.
__device__ __forceinline__ void hist_carry4(const uint32_t (&a)[4], const uint32_t (&o)[4],
                                            uint32_t nw) {
  asm volatile(
      "{\n .reg .pred P<4>;\n"
      " setp.gt.u32 P0, %4, %8;\n setp.gt.u32 P1, %5, %8;\n"
      " setp.gt.u32 P2, %6, %8;\n setp.gt.u32 P3, %7, %8;\n"
      " @P0 red.shared.add.u32 [%0+128], 1;\n @P1 red.shared.add.u32 [%1+128], 1;\n"
      " @P2 red.shared.add.u32 [%2+128], 1;\n @P3 red.shared.add.u32 [%3+128], 1;\n}\n"
      ::"r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]),
      "r"(nw));
}

// Quantised-token pages of sequence b.
__device__ __forceinline__ int seq_pages(const DecodeParams& p, int b) {
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_vq = max(0, N - p.W);
  return min((n_vq + p.Pg - 1) / p.Pg, p.max_pages_per_seq);
}

// Work units of one (sequence, head) pair: its quantised pages, led by
// kSegmentUnits units that stand for the setup of a segment. A CTA whose
// range reaches into a second pair so takes fewer pages.
__device__ __forceinline__ int pair_units(int pages) { return pages > 0 ? pages + kSegmentUnits : 0; }

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
// units [Hq*pre, Hq*(pre + pair_units)) contain unit `u` (or, with u < 0,
// just the total). Returns the total number of units; *b_out, *pre_out describe
// the hit (b_out = -1 if none).
__device__ long long find_unit(const DecodeParams& p, long long u, int lane, int* b_out,
                               long long* pre_out) {
  long long acc = 0;                                   // units before sequence b0
  *b_out = -1;
  *pre_out = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const long long units = (b < p.B) ? static_cast<long long>(p.Hq) * pair_units(seq_pages(p, b)) : 0;
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

// Window partial of one pair over its n_win bf16 window tokens:
// x_t = q . K_win[t] (log2 units), m = max x, l = sum 2^(x-m),
// o = sum 2^(x-m) V_win[t]; written to res[0], res[1], res[2..2+D).
// Every thread of the CTA (NWARPS warps) calls it. Warp w takes tokens
// w, w + NWARPS, ..: it requests the key and value rows of up to kWinChunk
// tokens at once, keeps its own running (m, l, o) and leaves it in
// wstat[2w..2w+1] and wpart[w][D]; the warp partials are then merged.
// Ends with a barrier.
template <int D, int NWARPS>
__device__ void window_partial(const DecodeParams& p, int b, int hkv, const uint16_t* qp,
                               int n_win, float* wstat, float* wpart, float* res) {
  constexpr int NPL = (D / 2 + 31) / 32;               // bf16 channel pairs per lane
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (n_win <= 0) {                                    // CTA-uniform
    for (int i = tid; i < D + 2; i += NWARPS * 32) res[i] = (i == 0) ? -INFINITY : 0.f;
    __syncthreads();
    return;
  }
  float qf[NPL][2];
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    const int pc = lane + 32 * k;
    const uint32_t w = (pc < D / 2) ? reinterpret_cast<const unsigned int*>(qp)[pc] : 0u;
    const float2 f = bf16x2_to_float2(w);
    qf[k][0] = f.x * p.scale_log2;
    qf[k][1] = f.y * p.scale_log2;
  }
  const size_t head = (static_cast<size_t>(b) * p.Hkv + hkv) * static_cast<size_t>(p.W) * D;
  const unsigned int* wk = reinterpret_cast<const unsigned int*>(p.win_k + head);
  const unsigned int* wv = reinterpret_cast<const unsigned int*>(p.win_v + head);
  float m = -INFINITY, l = 0.f;
  float oacc[NPL][2];
#pragma unroll
  for (int k = 0; k < NPL; ++k) oacc[k][0] = oacc[k][1] = 0.f;
  for (int t0 = warp; t0 < n_win; t0 += NWARPS * kWinChunk) {
    uint32_t kr[kWinChunk][NPL], vr[kWinChunk][NPL];
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      const int t = t0 + i * NWARPS;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int pc = lane + 32 * k;
        const bool ok = t < n_win && pc < D / 2;
        kr[i][k] = ok ? __ldg(wk + static_cast<size_t>(t) * (D / 2) + pc) : 0u;
        vr[i][k] = ok ? __ldg(wv + static_cast<size_t>(t) * (D / 2) + pc) : 0u;
      }
    }
    float x[kWinChunk];
    float mc = -INFINITY;
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const float2 kv = bf16x2_to_float2(kr[i][k]);
        acc = fmaf(qf[k][0], kv.x, fmaf(qf[k][1], kv.y, acc));
      }
      x[i] = (t0 + i * NWARPS < n_win) ? warp_sum(acc) : -INFINITY;
      mc = fmaxf(mc, x[i]);
    }
    if (mc > m) {                                      // warp-uniform
      const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - mc);
      l *= f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        oacc[k][0] *= f;
        oacc[k][1] *= f;
      }
      m = mc;
    }
#pragma unroll
    for (int i = 0; i < kWinChunk; ++i) {
      const float w = fast_exp2(x[i] - m);             // 0 past the window
      l += w;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const float2 vv = bf16x2_to_float2(vr[i][k]);
        oacc[k][0] = fmaf(w, vv.x, oacc[k][0]);
        oacc[k][1] = fmaf(w, vv.y, oacc[k][1]);
      }
    }
  }
  if (lane == 0) {
    wstat[2 * warp] = m;
    wstat[2 * warp + 1] = l;
  }
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    const int pc = lane + 32 * k;
    if (pc < D / 2) {
      wpart[warp * D + 2 * pc] = oacc[k][0];
      wpart[warp * D + 2 * pc + 1] = oacc[k][1];
    }
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) M = fmaxf(M, wstat[2 * w]);
  float f[NWARPS];
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) f[w] = (wstat[2 * w] == -INFINITY) ? 0.f : fast_exp2(wstat[2 * w] - M);
  for (int ch = tid; ch < D; ch += NWARPS * 32) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) o = fmaf(f[w], wpart[w * D + ch], o);
    res[2 + ch] = o;
  }
  if (tid == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) L = fmaf(f[w], wstat[2 * w + 1], L);
    res[0] = M;
    res[1] = L;
  }
  __syncthreads();
}


template <int J, int C>
__global__ void __launch_bounds__(kThreads, 1) vq_stream_kernel(const DecodeParams p) {
  using T = Traits<J>;
  constexpr int d = J * C;
  constexpr int LB = T::LB;
  constexpr int KB = kChunkBlocks;                     // blocks per warp per chunk
  constexpr int RS = 4 + d;                            // record floats
  constexpr int EP = kE + 1;                           // padded row of the transposed merged histogram
  static_assert(J * EP * 4 <= static_cast<int>(kHistBytes), "merged histogram fits the window");
  static_assert((2 * KB) % kRing == 0, "a chunk's items map onto fixed ring slots");
  // groups of the key slice staged at once in the (empty) histogram window
  constexpr int JC = stage_groups(J, C);
  static_assert(JC >= 1 && J % JC == 0, "staging chunks tile the groups");
  static_assert(d <= 256, "q fits its buffer");

  extern __shared__ __align__(16) unsigned char smem_u8[];
  const uint32_t sbase = smem_addr(smem_u8);
  float* wmax = reinterpret_cast<float*>(smem_u8 + kWmaxOff);
  float* qs = reinterpret_cast<float*>(smem_u8 + kQsOff);
  // the LUT and histogram windows, aligned above the small area
  const uint32_t lut_abs = (sbase + kSmallBytes + kLutBytes - 1u) & ~(kLutBytes - 1u);
  const uint32_t hist_abs = lut_abs + kLutBytes;
  const bool bad_base = hist_abs + kHistBytes > sbase + kDynBytes;
  float* lut = reinterpret_cast<float*>(smem_u8 + (bad_base ? 0u : lut_abs - sbase));
  float* stage = reinterpret_cast<float*>(smem_u8 + (bad_base ? 0u : hist_abs - sbase));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool lane_live = lane < LB;
  // Byte permutes that put an index byte into byte 1 of these give addresses.
  // Key lookup s of slot `lane` reads LUT column lane + s (the replicated
  // columns make the modulo unnecessary): the address of lookup s is
  // perm(lxb) + 4s. Value update s goes to histogram column (lane + s) % LB.
  const uint32_t lxb = lut_abs | static_cast<uint32_t>(lane * 4);
  uint32_t hx[J];
#pragma unroll
  for (int s = 0; s < J; ++s) hx[s] = hist_abs | (4u * static_cast<uint32_t>((lane + s) % LB));
  const int bpp = p.Pg / LB;
  const uint32_t bpp_magic = 0xFFFFFFFFu / static_cast<uint32_t>(bpp) + 1u;

  int b_first;
  long long pre_first;
  const long long U = find_unit(p, -1, lane, &b_first, &pre_first);
  const long long u_lo = U * blockIdx.x / p.n_cta;
  const long long u_hi = U * (blockIdx.x + 1) / p.n_cta;
  // the finish kernel may start its window work as SMs free up; it waits for
  // this grid before it reads the records
  asm volatile("griddepcontrol.launch_dependents;");
  if (u_lo >= u_hi) return;                            // CTA-uniform
  int b;
  long long pre;
  find_unit(p, u_lo, lane, &b, &pre);
  int units_b = pair_units(seq_pages(p, b));
  const long long off = u_lo - static_cast<long long>(p.Hq) * pre;
  int hq = static_cast<int>(off / units_b);
  int pu_start = static_cast<int>(off % units_b);     // unit offset inside the pair
  long long u = u_lo;
  if (bad_base && tid == 0 && p.status != nullptr) atomicOr(p.status, kStatusSharedBase);

  while (u < u_hi && b < p.B) {
    const int seg_units = static_cast<int>(min(static_cast<long long>(units_b - pu_start), u_hi - u));
    // pages of this segment: its units past the pair's leading setup units
    const int pg_lo = max(pu_start - kSegmentUnits, 0);
    const int pg_hi = max(pu_start + seg_units - kSegmentUnits, 0);
    const int hkv = hq / p.ratio;
    const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
    const int n_vq = max(0, N - p.W);
    float* rec = p.records + static_cast<size_t>(b * p.Hq + hq + blockIdx.x) * RS;
    if (bad_base) {
      if (tid == 0) {
        rec[0] = NAN;
        rec[1] = 1.f;
      }
    } else if (pg_hi <= pg_lo) {                       // setup units only: an empty record
      if (tid == 0) {
        rec[0] = -INFINITY;
        rec[1] = 0.f;
      }
    } else {
      const float* cbk = p.cb_k + hkv * p.cb_stride_head;
      const uint16_t* qp = p.q + (static_cast<size_t>(b) * p.Hq + hq) * d;
      __syncthreads();                                 // previous segment done with LUT, histogram, q
      // the first chunk of the key slice goes out before anything that waits
      for (int i = tid * 4; i < JC * kE * C; i += kThreads * 4) cp_async16(stage + i, cbk + i);
      const float* cbv = p.cb_v + hkv * p.cb_stride_head;
      if (warp == kNW - 1) {                           // the value slice, into L2 for the contraction
        constexpr uint32_t kSlice = kE * J * C * 4, kPiece = kSlice / 32;
        static_assert(kSlice % (32 * 16) == 0, "prefetch pieces are 16-byte multiples");
        prefetch_l2_bulk(reinterpret_cast<const char*>(cbv) + lane * kPiece, kPiece);
      }
      const float qv = (tid < d) ? bf16_bits_to_float(qp[tid]) * p.scale_log2 : 0.f;

      // ---- this warp's pages and the index ring --------------------------------
      // warp w streams the segment's pages pg_lo + w + k*kNW (k = 0, 1, ..), each
      // as bpp blocks; its t-th block is block t % bpp of its page t / bpp.
      // Chunk ch holds blocks [ch*KB, (ch+1)*KB) of every warp; its items are
      // the KB key blocks, then the same KB value blocks.
      const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
      const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
      auto pages_of = [&](int w) { return (pg_hi > pg_lo + w) ? (pg_hi - pg_lo - w + kNW - 1) / kNW : 0; };
      const int my_first = pg_lo + warp;
      const int n_my_pages = pages_of(warp);
      const int n_blocks = n_my_pages * bpp;
      const int n_chunks = (pages_of(0) * bpp + KB - 1) / KB;   // CTA-uniform (warp 0 has the most)
      int i0 = 0;                                      // page-table window: pages [i0, i0 + 64)
      auto bt_entry = [&](int i) -> int { return (i < n_my_pages) ? bt[my_first + i * kNW] : -1; };
      int bt_cur = bt_entry(lane);                     // requested now, used after the slice lands
      int bt_nxt = bt_entry(32 + lane);
      // L2 prefetch of pages [k0, k1) of this warp's list
      auto prefetch_pages = [&](int k0, int k1) {
        k1 = min(k1, n_my_pages);
        const int a = lane + i0, c = lane + i0 + 32;
        if (a >= k0 && a < k1 && bt_cur >= 0 && bt_cur < p.n_pages)
          prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_cur) * p.page_bytes,
                           static_cast<uint32_t>(p.page_bytes));
        if (c >= k0 && c < k1 && bt_nxt >= 0 && bt_nxt < p.n_pages)
          prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_nxt) * p.page_bytes,
                           static_cast<uint32_t>(p.page_bytes));
      };
      BlockRegs<J> ring[kRing];
#pragma unroll
      for (int k = 0; k < kRing; ++k) ring[k].base = -1;
      // a cleared block keeps whatever bytes it held: every byte value
      // addresses a valid row, and base = -1 masks and skips it
      auto issue = [&](int i, BlockRegs<J>& r) {
        const int ch = i / (2 * KB);
        const int pos = i - ch * 2 * KB;
        const int kv = pos >= KB ? 1 : 0;
        const int t = ch * KB + (pos - kv * KB);
        if (pos == 0) {                                  // first item of a chunk (warp-uniform)
          const int kmin = static_cast<int>(__umulhi(static_cast<uint32_t>(ch * KB), bpp_magic));
          if (kmin >= i0 + 32) {                         // slide the page-table window
            bt_cur = bt_nxt;
            i0 += 32;
            bt_nxt = bt_entry(i0 + 32 + lane);
          }
          const int knext = static_cast<int>(__umulhi(static_cast<uint32_t>((ch + 1) * KB), bpp_magic));
          prefetch_pages(kmin + kPrefetchPages, knext + kPrefetchPages);
        }
        if (t >= n_blocks) {                             // warp-uniform
          r.base = -1;
          return;
        }
        const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(t), bpp_magic));
        const int blk = t - pi * bpp;
        const int src = (pi - i0 < 32) ? bt_cur : bt_nxt;
        const int phys = __shfl_sync(0xffffffffu, src, (pi - i0) & 31);
        const int pg = my_first + pi * kNW;
        r.valid = min(p.Pg, n_vq - pg * p.Pg);
        r.base = blk * LB;
        if (phys < 0 || phys >= p.n_pages) {             // a page-table entry outside the pool
          if (lane == 0 && p.status != nullptr) atomicOr(p.status, kStatusBadPage);
          r.base = -1;
          return;
        }
        if (r.base >= r.valid) {                         // past the sequence's last token
          r.base = -1;
          return;
        }
        load_block<J>(pool_h + static_cast<int64_t>(phys) * p.page_bytes, p.plane_bytes, blk, kv, lane,
                      r);
      };

      // ---- key LUT from the key slice staged in the histogram window ----------
      if (tid < d) qs[tid] = qv;
#pragma unroll 1
      for (int j0 = 0; j0 < J; j0 += JC) {
        if (j0 > 0) {
          __syncthreads();                             // previous chunk consumed
          const float* src = cbk + static_cast<size_t>(j0) * kE * C;
          for (int i = tid * 4; i < JC * kE * C; i += kThreads * 4) cp_async16(stage + i, src + i);
        }
        cp_async_wait_all();
        __syncthreads();
        if (j0 == 0) {                                 // the page table has landed: first index blocks
          prefetch_pages(0, kPrefetchPages);
#pragma unroll
          for (int k = 0; k < kRing; ++k) issue(k, ring[k]);
        }
        // item = (tile of 32 rows, step): lane -> row tile*32 + lane, group
        // j0 + (step + lane) % JC, so the lanes' table stores hit distinct banks
#pragma unroll 4
        for (int it = warp; it < (kE / 32) * JC; it += kNW) {
          const int e = (it / JC) * 32 + lane, jj = (it % JC + lane) % JC, j = j0 + jj;
          const float v = dot_c<C>(qs + j * C, stage + (static_cast<size_t>(jj) * kE + e) * C);
#pragma unroll
          for (int c = j; c < 64; c += J) lut[e * 64 + c] = v;   // every column holding group j
        }
      }
      __syncthreads();                                 // LUT complete; staging area free
      for (uint32_t a = hist_abs + 16u * tid; a < hist_abs + kHistBytes; a += 16u * kThreads)
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
      __syncthreads();                                 // histogram zero

      // ---- stream -------------------------------------------------------------
      auto key_scores = [&](const BlockRegs<J>& r) -> float {
        if (r.base < 0) return -INFINITY;              // warp-uniform
        float xa[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t ad[J];
#pragma unroll
        for (int s = 0; s < J; ++s) ad[s] = __byte_perm(r.w[s >> 2], lxb, 0x7604u | (uint32_t(s & 3) << 4));
        constexpr_for<J>([&](auto S) { xa[S.value & 3] += lds_lut<4 * S.value>(ad[S.value]); });
        const bool valid = lane_live && (r.base + lane) < r.valid;
        return valid ? (xa[0] + xa[1]) + (xa[2] + xa[3]) : -INFINITY;
      };
      // histogram updates of one value block, lane = slot: the slot's weight
      // w = rn(2^(x - m) * 2^kFixBits) goes to row idx_V[slot][j] of column
      // (lane + s) % LB for each byte s of its rotated row; carries out of a low
      // word go to its high word
      auto value_pass = [&](const BlockRegs<J>& r, float x, float m) {
        if (r.base < 0) return;                        // warp-uniform
        if constexpr (LB < 32) {
          if (!lane_live) return;
        }
        uint32_t w = __float2uint_rn(fast_exp2(x - m) * kFixScale);   // 0 for x = -inf
        w = min(w, 1u << kFixBits);
        const uint32_t nw = ~w;
        uint32_t a[4], o[4];
#pragma unroll
        for (int i = 0; i < J / 4; ++i) {
          uint32_t an[4], on[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) an[k] = __byte_perm(r.w[i], hx[4 * i + k], 0x7604u | (uint32_t(k) << 4));
          hist_add4(an, w, on);
          if (i > 0) hist_carry4(a, o, nw);            // the previous four, whose old words are back
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            a[k] = an[k];
            o[k] = on[k];
          }
        }
        hist_carry4(a, o, nw);
      };
      // exact rescale of the 64-bit cells by 2^-sh when the reference maximum rises
      auto rescale = [&](int sh) {
        for (int cell = tid; cell < kE * 32; cell += kThreads) {
          const uint32_t ad = hist_abs + (static_cast<uint32_t>(cell >> 5) << 8) +
                              (static_cast<uint32_t>(cell & 31) << 2);
          uint32_t lo = lds_u32(ad), hi = lds_u32(ad + 128u);
          if (sh >= 64) {
            lo = 0u;
            hi = 0u;
          } else if (sh >= 32) {
            lo = hi >> (sh - 32);
            hi = 0u;
          } else {
            lo = __funnelshift_r(lo, hi, sh);
            hi >>= sh;
          }
          sts_u32(ad, lo);
          sts_u32(ad + 128u, hi);
        }
      };

      float m_cur = -INFINITY;                         // integer reference maximum (CTA-uniform)
#pragma unroll 1
      for (int ch = 0; ch < n_chunks; ++ch) {
        const int ib = ch * 2 * KB;
        float xs[KB];
        float cm = -INFINITY;
#pragma unroll
        for (int q = 0; q < KB; ++q) {                 // key phase
          xs[q] = key_scores(ring[q % kRing]);
          cm = fmaxf(cm, xs[q]);
          issue(ib + q + kRing, ring[q % kRing]);
        }
        cm = warp_max(cm);
        if (lane == 0) wmax[(ch & 1) * kNW + warp] = cm;
        __syncthreads();                               // every warp's chunk maximum
        float cmax = (lane < kNW) ? wmax[(ch & 1) * kNW + lane] : -INFINITY;
        cmax = warp_max(cmax);
        if (cmax != -INFINITY) {                       // CTA-uniform
          const float m_new = fmaxf(m_cur, ceilf(cmax));
          if (m_cur != -INFINITY && m_new > m_cur) {   // earlier chunks' weights shrink by 2^-(m_new - m_cur)
            rescale(static_cast<int>(fminf(m_new - m_cur, 64.f)));
            __syncthreads();
          }
          m_cur = m_new;
        }
#pragma unroll
        for (int q = 0; q < KB; ++q) {                 // value phase
          if (m_cur != -INFINITY) value_pass(ring[(KB + q) % kRing], xs[q], m_cur);   // CTA-uniform
          issue(ib + KB + q + kRing, ring[(KB + q) % kRing]);
        }
      }
      __syncthreads();                                 // every update landed

      // ---- histogram to float, contraction with the value slice ---------------
      if (m_cur == -INFINITY) {                        // nothing valid: an empty record
        if (tid == 0) {
          rec[0] = -INFINITY;
          rec[1] = 0.f;
        }
      } else {
        // W[e][j]: lane = column, rows warp + kNW*k; replicas of a group are summed
        constexpr int NR = kE / kNW;                   // rows per warp
        float wv[NR];
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          const int e = warp + kNW * k;
          float v = 0.f;
          if (lane_live) {
            const uint32_t ad = hist_abs + (static_cast<uint32_t>(e) << 8) + 4u * lane;
            const uint32_t lo = lds_u32(ad), hi = lds_u32(ad + 128u);
            v = (__uint2float_rn(hi) * 4294967296.0f + __uint2float_rn(lo)) * kFixInv;
          }
#pragma unroll
          for (int o = (T::R / 2) * J; o >= J; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
          wv[k] = v;
        }
        __syncthreads();                               // every histogram word read
        // transposed, padded: wt[j*EP + e] (lanes of a row and of a column hit distinct banks)
        float* wt = stage;
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          const int e = warp + kNW * k;
          if (lane < J) wt[lane * EP + e] = wv[k];
        }
        __syncthreads();
        // o[j*C + ch] = sum_e W[e][j] C_V[j][e][ch]: warp -> groups, lane -> rows lane + 32 i
        constexpr int JPW = (J + kNW - 1) / kNW;
#pragma unroll 1
        for (int jw = 0; jw < JPW; ++jw) {
          const int j = warp + kNW * jw;
          if (j >= J) break;                           // warp-uniform
          float cv[kE / 32][C];
#pragma unroll
          for (int i = 0; i < kE / 32; ++i)
            load_cw<C>(cbv + (static_cast<size_t>(j) * kE + lane + 32 * i) * C, cv[i]);
          float acc[C];
#pragma unroll
          for (int ch = 0; ch < C; ++ch) acc[ch] = 0.f;
#pragma unroll
          for (int i = 0; i < kE / 32; ++i) {
            const float h = wt[j * EP + lane + 32 * i];
#pragma unroll
            for (int ch = 0; ch < C; ++ch) acc[ch] = fmaf(h, cv[i][ch], acc[ch]);
          }
#pragma unroll
          for (int ch = 0; ch < C; ++ch) {
            const float t = warp_sum(acc[ch]);
            if (lane == ch) rec[4 + j * C + ch] = t;
          }
        }
        if (warp == kNW - 1) {                         // l = sum_e W[e][j], the same for every group j
          float l = 0.f;
#pragma unroll
          for (int i = 0; i < kE / 32; ++i) l += wt[lane + 32 * i];
          l = warp_sum(l);
          if (lane == 0) {
            rec[0] = m_cur;
            rec[1] = l;
          }
        }
      }
    }

    u += seg_units;
    pu_start = 0;
    if (++hq == p.Hq) {
      hq = 0;
      do {
        ++b;
      } while (b < p.B && u < u_hi && (units_b = pair_units(seq_pages(p, b))) == 0);
    }
  }
}

// One CTA per (sequence, query head): the bf16 window partial and the merge
// of the pair's segment records (log-sum-exp weights); writes out and lse.
template <int J, int C>
__global__ void __launch_bounds__(kFinishThreads) vq_finish_kernel(const DecodeParams p) {
  constexpr int D = J * C;
  constexpr int NW = kFinishThreads / 32;
  constexpr int RS = 4 + D;                            // record floats
  __shared__ float wst[2 * NW];
  __shared__ float wpart[NW * D];
  __shared__ float wres[D + 2];
  __shared__ float fc[kMaxStreamCtas];
  __shared__ float sstat[4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x;
  const int b = pair / p.Hq, hq = pair % p.Hq, hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int pages_b = seq_pages(p, b);                 // CTA-uniform
  window_partial<D, NW>(p, b, hkv, p.q + static_cast<size_t>(pair) * D, min(N, p.W), wst, wpart, wres);

  // the pair's segment records: slots pair + c for the CTAs c that own its units
  int c_first = 0, c_last = -1;
  long long U = 1;
  if (pages_b > 0) {
    int bb;
    long long pre;
    U = find_unit(p, -1, lane, &bb, &pre);
    long long before = 0;                              // units of one head of sequences < b
    for (int b0 = 0; b0 < b; b0 += 32) {
      const int bi = b0 + lane;
      long long v = (bi < b) ? static_cast<long long>(pair_units(seq_pages(p, bi))) : 0;
      v = warp_incl_scan(v, lane);
      before += __shfl_sync(0xffffffffu, v, 31);
    }
    const int units_b = pair_units(pages_b);
    const long long u0 = before * p.Hq + static_cast<long long>(hq) * units_b;
    c_first = static_cast<int>(((u0 + 1) * p.n_cta - 1) / U);
    c_last = static_cast<int>(((u0 + units_b) * p.n_cta - 1) / U);
  }
  // everything above reads only inputs; the segment records need the
  // streaming kernel to be complete
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // a CTA whose unit range is empty wrote no record
  auto rec_of = [&](int c) -> const float* {
    return (U * c / p.n_cta < U * (c + 1) / p.n_cta)
               ? p.records + static_cast<size_t>(pair + c) * RS : nullptr;
  };
  if (warp == 0) {
    float M = wres[0];
    for (int c = c_first + lane; c <= c_last; c += 32) {
      const float* rec = rec_of(c);
      if (rec != nullptr) M = fmaxf(M, __ldcg(rec));
    }
    M = warp_max(M);
    float L = 0.f;
    for (int c = c_first + lane; c <= c_last; c += 32) {
      const float* rec = rec_of(c);
      float f = 0.f;
      if (rec != nullptr) {
        const float m = __ldcg(rec);
        if (m != -INFINITY) {
          f = fast_exp2(m - M);                          // NaN m (a timed-out turn) poisons M and L
          L += __ldcg(rec + 1) * f;
        }
      }
      fc[c - c_first] = f;
    }
    L = warp_sum(L);
    if (lane == 0) {
      const float f_win = (wres[0] == -INFINITY) ? 0.f : fast_exp2(wres[0] - M);
      sstat[0] = M;
      sstat[1] = L + f_win * wres[1];
      sstat[2] = f_win;
    }
  }
  __syncthreads();
  const float M = sstat[0], L = sstat[1], f_win = sstat[2];
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  for (int ch = tid; ch < D; ch += kFinishThreads) {
    float o = (f_win != 0.f) ? f_win * wres[2 + ch] : 0.f;
    for (int c = c_first; c <= c_last; ++c) {
      const float f = fc[c - c_first];
      if (f != 0.f) o = fmaf(f, __ldcg(p.records + static_cast<size_t>(pair + c) * RS + 4 + ch), o);
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
  static_assert(kDynBytes <= 227 * 1024, "streaming kernel shared memory above 227 KB");
  if (run_stream) {
    static std::atomic<uint64_t> configured{0};
    if (set_smem(vq_stream_kernel<J, C>, kDynBytes, configured) != LOOPVQ_OK) return LOOPVQ_ERR_CUDA;
    vq_stream_kernel<J, C><<<p.n_cta, kThreads, kDynBytes, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  }
  // programmatic dependent launch: the finish kernel's CTAs may start while
  // the streaming kernel's last CTAs still run (griddepcontrol.wait inside)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.B * p.Hq));
  cfg.blockDim = dim3(kFinishThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, vq_finish_kernel<J, C>, p) != cudaSuccess) return LOOPVQ_ERR_CUDA;
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
  p.status = static_cast<int*>(a.workspace);
  p.records = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + kStatusBytes);
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
