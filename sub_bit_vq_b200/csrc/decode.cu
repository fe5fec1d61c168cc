// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// Two kernels per call, the second a programmatic dependent of the first.
//
// vq_pair_kernel: per (sequence, query head) pair, one CTA scores the bf16
// window tokens (prefix + recent) into a window partial (and, for a pair
// without quantised tokens, writes the result), and J/4 CTAs build the
// pair's key lookup table
//     LUT[e][j] = s*log2(e) * q_j . C_K[j][e][tau]
// (E x J floats) into the workspace.
//
// vq_stream_kernel: a persistent grid (at most one CTA per SM, sixteen warps)
// over the quantised tokens of every pair. All pages of all pairs form one
// list and CTA c takes the contiguous range [U*c/n, U*(c+1)/n) of it, so
// every CTA streams the same number of pages and touches one or a few pairs
// ("segments"). Per segment:
//   1. The pair's LUT is copied into shared memory with its J columns
//      repeated over 64 (column c holds group c % J), and the value histogram
//      H[e][c] (64 columns of 32-bit words) is zeroed.
//   2. Streaming, in chunks of kChunkBlocks index blocks (LB slots each) per
//      warp. Key phase, lane = slot: byte s of the slot's rotated K row is
//      group (lane+s) % J, held by LUT column lane+s, so the lookup address is
//      one byte permute plus the immediate 4s; the scores x (log2 units) stay
//      in registers. The warps' maxima and weight sums meet at a barrier,
//      which fixes the segment's integer reference maximum m (raised to
//      ceil(max x) + 1 when a chunk passes it) and its fixed-point exponent
//      S. Value phase, lane = slot again: the slot's weight
//      w = rn(2^(x - cm) * 2^(cm - m + S)) = rn(2^(x - m + S)) (cm: the
//      warp's chunk maximum, whose powers 2^(x - cm) also gave the weight
//      sums) is added to cell
//      H[idx][lane + s] for each byte s of its rotated V row by a 32-bit
//      shared-memory reduction (red.shared.add.u32: integer reductions run
//      at full shared-memory rate on sm_100, so all warps update the one
//      histogram without taking turns).
//      Overflow: every cell is a sum of weights of distinct tokens, so it
//      never exceeds the total weight of the segment, which the barrier
//      knows exactly. S starts at kFixMax and is lowered whenever that total
//      would pass 2^31 (the total then lands below 2^29); m rises only when
//      a chunk's maximum passes it. Either change is an exact right shift of
//      every cell by the bits lost.
//   3. The histogram, converted to float (W[e][j] = 2^-S sum of the columns
//      of group j), is contracted with the value codebook slice,
//      o_j = sum_e W[e][j] C_V[j][e][tau], and the segment record
//      (m, l = sum_e W[e][j], o[d]) goes to slot (pair + cta).
//   4. The CTA counts its record on the pair's counter; the CTA that writes
//      the pair's last record merges the window partial with every record
//      (log-sum-exp weights, one round of loads per channel) and writes out
//      and lse. No CTA waits on another.
//
// The hot loops address shared memory by absolute shared-window address: a
// byte permute puts an index byte into byte 1 of (lane * 4), and the window
// base plus 4s is the instruction's immediate offset. That needs the dynamic
// allocation to start at kSBase, which the host checks before launching (the
// device's reserved shared memory per block) and every CTA checks again; a
// CTA that finds another base writes NaN records and flags the status word.

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
constexpr int kPrefetchPages = 2;         // pages a warp asks L2 to fetch ahead of its loads
constexpr int kFixMax = 30;               // largest fixed-point exponent: w = rn(2^(x - m) * 2^S)
constexpr float kMassHigh = 2147483648.0f;  // 2^31: lower S before a segment's total passes this
constexpr int kMassLandLog2 = 29;         // after lowering S the total sits below 2^29
constexpr int kPairThreads = 256;         // window partial: 8 warps; lookup table: one thread per centroid
constexpr int kWinChunk = 9;              // window tokens per warp per round of loads (72 = 8 warps x 9)
constexpr int kSegmentUnits = 16;         // work units (pages) charged for a segment's setup
constexpr int kCols = 64;                 // columns of the shared LUT and histogram
constexpr float kMHead = 1.f;             // headroom of the reference maximum, log2 units
constexpr int kPsBits = 24;               // fixed-point bits of a warp's chunk weight sum
constexpr int kAddBits = 20;              // fixed-point bits of the CTA's chunk weight sum
constexpr float kPsScale = 16777216.0f;   // 2^kPsBits

// Shared memory, by absolute shared-window address. The dynamic allocation
// starts at kSBase (the reserved shared memory of a block on sm_100).
constexpr uint32_t kSBase = 0x400u;
constexpr uint32_t kStatOff = 0;          // [2][kNW][2] per-warp chunk maximum and weight sum
constexpr uint32_t kFlagOff = 0x200u;     // int: last-writer flag
constexpr uint32_t kSmallBytes = 0x400u;
constexpr uint32_t kLutAbs = kSBase + kSmallBytes;        // [E][64] floats, 256-byte rows
constexpr uint32_t kHistAbs = kLutAbs + kE * kCols * 4;   // [E][64] 32-bit words, 256-byte rows
constexpr uint32_t kDynBytes = kHistAbs + kE * kCols * 4 - kSBase;

// A build with LOOPVQ_RANGE_CHECK defined checks, before each access that
// the partition's arithmetic keeps in range, that it is in range, and
// flags LOOPVQ_DECODE_STATUS_RANGE (skipping the access) if it is not.
#ifdef LOOPVQ_RANGE_CHECK
constexpr bool kRangeCheck = true;
#else
constexpr bool kRangeCheck = false;
#endif

// Bits of the status word (see loopvq.h).
constexpr int kStatusBadPage = LOOPVQ_DECODE_STATUS_BAD_PAGE;
constexpr int kStatusSharedBase = LOOPVQ_DECODE_STATUS_SHARED_BASE;

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
  float* luts;                      // [pairs][E][J] key lookup tables
  float* wrecs;                     // [pairs][4 + d]: the bf16 window partial of each pair
  unsigned* counts;                 // [pairs] segment records written so far (zeroed by the pair kernel)
  int* status;                      // status word (bit flags), never cleared by the kernels
  void* out;
  float* lse;
  // B counts virtual sequences: sequence b / Q with its query b % Q (Q = 1
  // for decode); inputs of a sequence (seq_lens, block_table, windows) are
  // indexed by b / Q, those of a query (q, out, lse) by b.
  int B, Q, Hq, Hkv, ratio, W, Pg, n_pages, max_pages_per_seq, max_seq_len;
  int64_t page_bytes, plane_bytes;
  int n_cta, out_dtype, log2_bpp;
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
};

// Where a block lives: this lane's row in the K plane (the V plane follows
// at +plane_bytes) and the number of valid slots (0: no block).
struct BlockInfo {
  const uint8_t* row;
  int nv;
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

// Loads this lane's rotated row of a block whose row starts at `row` (both
// planes hold rotated slot rows in granules [J/GR][LB][GR]).
template <int J>
__device__ __forceinline__ void load_row(const uint8_t* row, int lane, BlockRegs<J>& r) {
  using T = Traits<J>;
  if (lane < T::LB) {
#pragma unroll
    for (int gi = 0; gi < J / T::GR; ++gi)
      load_words<T::GR>(row + gi * T::LB * T::GR, r.w + gi * (T::GR / 4), T::GR / 4);
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

// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1 (compile-time i).
template <typename F, int... I>
__device__ __forceinline__ void constexpr_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void constexpr_for(F&& f) {
  constexpr_for_impl(f, std::make_integer_sequence<int, N>{});
}

// ---- shared memory by absolute shared-window address ------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

// Shared word at a + OFF (OFF a compile-time window offset).
template <uint32_t OFF>
__device__ __forceinline__ float lds_at(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}
template <uint32_t OFF>
__device__ __forceinline__ void red_at(uint32_t a, uint32_t w) {
  asm volatile("red.shared.add.u32 [%0+%1], %2;" ::"r"(a), "n"(OFF), "r"(w));
}

// Warp-wide maximum (NaN ignored) and unsigned sum, one instruction each.
__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint32_t redux_add_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.add.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}
// Two floats packed in 64 bits (low first), and their lane-wise sum.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// x * 2^k for -126 <= k <= 127, by an exact power-of-two factor.
__device__ __forceinline__ float ldexp_pos(float x, int k) { return x * __int_as_float((127 + k) << 23); }

// Quantised-token pages of sequence b.
__device__ __forceinline__ int seq_pages(const DecodeParams& p, int b) {
  const int N = max(0, min(p.seq_lens[b / p.Q], p.max_seq_len));
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
  const size_t head = (static_cast<size_t>(b / p.Q) * p.Hkv + hkv) * static_cast<size_t>(p.W) * D;
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



// Merges a pair's window partial with its segment records (slots pair + c
// for the CTAs c in [c_first, c_last] whose unit range is not empty: CTA c
// of n_cta owns units [U*c/n_cta, U*(c+1)/n_cta)) and writes out and lse.
// Every thread of the CTA (NT threads) calls it. Thread ch owns output
// channel ch: it loads (m, l, o[ch]) of the window partial and of up to
// kMergeBatch records at once and folds them in with log-sum-exp weights,
// so that one round of loads serves every pair that spans at most
// kMergeBatch CTAs (all but the smallest batches). m in log2 units; a record
// with m = -inf is empty, a NaN m poisons the result.
template <int D, int NT>
__device__ void merge_pair(const DecodeParams& p, int pair, int c_first, int c_last, long long U) {
  constexpr int RS = 4 + D;
  constexpr int kMergeBatch = 8;
  const float* wr = p.wrecs + static_cast<size_t>(pair) * RS;
  const bool every = U >= p.n_cta;                     // then no CTA's range is empty
  auto written = [&](int c) { return every || U * c / p.n_cta < U * (c + 1) / p.n_cta; };
  for (int ch = threadIdx.x; ch < D; ch += NT) {
    const float m_win = __ldcg(wr), l_win = __ldcg(wr + 1), o_win = __ldcg(wr + 4 + ch);
    float m = m_win, l = 0.f, o = 0.f;
    if (m_win != -INFINITY) {
      l = l_win;
      o = o_win;
    }
    for (int c0 = c_first; c0 <= c_last; c0 += kMergeBatch) {
      float mc[kMergeBatch], lc[kMergeBatch], oc[kMergeBatch];
#pragma unroll
      for (int r = 0; r < kMergeBatch; ++r) {
        const int c = c0 + r;
        mc[r] = -INFINITY;
        lc[r] = oc[r] = 0.f;
        if (c <= c_last && written(c)) {
          const float* rc = p.records + static_cast<size_t>(pair + c) * RS;
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(rc));
          mc[r] = ml.x;
          lc[r] = ml.y;
          oc[r] = __ldcg(rc + 4 + ch);
        }
      }
#pragma unroll
      for (int r = 0; r < kMergeBatch; ++r) {
        if (mc[r] == -INFINITY) continue;              // empty record
        const float mn = fmaxf(m, mc[r]);              // a NaN mc gives NaN factors below
        const float f0 = (m == -INFINITY) ? 0.f : fast_exp2(m - mn);
        const float f1 = fast_exp2(mc[r] - mn);
        l = fmaf(l, f0, lc[r] * f1);
        o = fmaf(o, f0, oc[r] * f1);
        m = mn;
      }
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    const float v = o * inv;
    if (p.out_dtype == LOOPVQ_DTYPE_F32)
      static_cast<float*>(p.out)[static_cast<size_t>(pair) * D + ch] = v;
    else
      static_cast<__nv_bfloat16*>(p.out)[static_cast<size_t>(pair) * D + ch] = __float2bfloat16_rn(v);
    if (ch == 0 && p.lse != nullptr) p.lse[pair] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

// The per-pair work that needs no index stream, before the streaming
// kernel: CTA (pair, 0) scores the pair's bf16 window tokens (prefix +
// recent) and writes the window partial (m, l, -, -, o[d]) to wrecs[pair];
// CTA (pair, 1 + g) writes groups 4g .. 4g+3 of the pair's key lookup table
// LUT[e][j] = s*log2(e) * sum_ch q[j*C + ch] * C_K[j][e][tau][ch] into
// luts[pair][e][j] (thread e owns centroid e; its loads of C_K[j][e][.] are
// consecutive across the warp).
template <int J, int C>
__global__ void __launch_bounds__(kPairThreads) vq_pair_kernel(const DecodeParams p) {
  constexpr int D = J * C;
  constexpr int NW = kPairThreads / 32;
  constexpr int RS = 4 + D;
  static_assert(kPairThreads == kE, "one thread per centroid");
  __shared__ float wst[2 * NW];
  __shared__ float wpart[NW * D > 8 ? NW * D : 8];
  __shared__ float wres[D + 2];
  const int pair = blockIdx.x, part = blockIdx.y;
  const int b = pair / p.Hq, hq = pair % p.Hq, hkv = hq / p.ratio;
  // the streaming kernel may start now; it waits for this grid before it
  // reads a table
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x;
  if (part == 0) {
    const int N = max(0, min(p.seq_lens[b / p.Q], p.max_seq_len));
    window_partial<D, NW>(p, b, hkv, p.q + static_cast<size_t>(pair) * D, min(N, p.W), wst, wpart, wres);
    float* wr = p.wrecs + static_cast<size_t>(pair) * RS;
    for (int i = tid; i < D + 2; i += kPairThreads) wr[i < 2 ? i : i + 2] = wres[i];
    if (tid == 0) p.counts[pair] = 0u;
    if (seq_pages(p, b) == 0) {                        // window tokens only: the result is final here
      __syncthreads();
      merge_pair<D, kPairThreads>(p, pair, 0, -1, 1);
    }
    return;
  }
  if (seq_pages(p, b) == 0) return;                    // CTA-uniform: no quantised tokens
  const int j0 = (part - 1) * 4, e = tid;
  const float* cbk = p.cb_k + hkv * p.cb_stride_head;  // [J][E][C]
  const uint16_t* qp = p.q + static_cast<size_t>(pair) * D + j0 * C;
  float cw[4][C];
#pragma unroll
  for (int k = 0; k < 4; ++k) load_cw<C>(cbk + (static_cast<size_t>(j0 + k) * kE + e) * C, cw[k]);
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float acc = 0.f;
#pragma unroll
    for (int ch = 0; ch < C; ++ch) acc = fmaf(bf16_bits_to_float(qp[k * C + ch]) * p.scale_log2, cw[k][ch], acc);
    v[k] = acc;
  }
  *reinterpret_cast<float4*>(p.luts + (static_cast<size_t>(pair) * kE + e) * J + j0) =
      make_float4(v[0], v[1], v[2], v[3]);
}

template <int J, int C>
__global__ void __launch_bounds__(kThreads, 1) vq_stream_kernel(const DecodeParams p) {
  using T = Traits<J>;
  constexpr int d = J * C;
  constexpr int LB = T::LB;
  constexpr int KB = kChunkBlocks;                     // blocks per warp per chunk
  constexpr int RS = 4 + d;                            // record floats
  constexpr int EP = kE + 1;                           // padded row of the transposed merged histogram
  static_assert(KB == kRing, "a chunk's block q lives in ring slot q");
  static_assert(LB + J - 1 <= kCols, "lookup columns lane + s stay inside the 64 columns");
  static_assert(J * EP * 4 <= kE * kCols * 4, "merged histogram fits the LUT window");

  extern __shared__ __align__(16) unsigned char smem_u8[];
  const uint32_t sbase = smem_addr(smem_u8);
  float* stat = reinterpret_cast<float*>(smem_u8 + kStatOff);
  float* lut = reinterpret_cast<float*>(smem_u8 + (kLutAbs - kSBase));
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_u8 + (kHistAbs - kSBase));
  const bool bad_base = sbase != kSBase;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;   // byte 0 of every table address
  const int bpp = p.Pg / LB;                           // blocks per page, a power of two
  const int lbpp = p.log2_bpp;

  int b_first;
  long long pre_first;
  const long long U = find_unit(p, -1, lane, &b_first, &pre_first);
  const long long u_lo = U * blockIdx.x / p.n_cta;
  const long long u_hi = U * (blockIdx.x + 1) / p.n_cta;
  // the finish kernel may start its window work as SMs free up; it waits for
  // this grid before it reads the records
  asm volatile("griddepcontrol.launch_dependents;");
  if (u_lo >= u_hi) {                                  // CTA-uniform
    asm volatile("griddepcontrol.wait;" ::: "memory");   // this grid completes after the one before
    return;
  }
  int b;
  long long pre;                                       // units of one head of the sequences before b
  find_unit(p, u_lo, lane, &b, &pre);
  int units_b = pair_units(seq_pages(p, b));
  const long long off = u_lo - static_cast<long long>(p.Hq) * pre;
  int hq = static_cast<int>(off / units_b);
  int pu_start = static_cast<int>(off % units_b);     // unit offset inside the pair
  long long u = u_lo;
  if (bad_base && tid == 0 && p.status != nullptr) atomicOr(p.status, kStatusSharedBase);
  bool tables_ready = false;
  // the pair kernel's tables, window partials and zeroed counters
  auto ensure_ready = [&]() {
    if (!tables_ready) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      tables_ready = true;
    }
  };
  int* s_last = reinterpret_cast<int*>(smem_u8 + kFlagOff);   // this CTA wrote a pair's last record

  while (u < u_hi && b < p.B) {
    const int seg_units = static_cast<int>(min(static_cast<long long>(units_b - pu_start), u_hi - u));
    // pages of this segment: its units past the pair's leading setup units
    const int pg_lo = max(pu_start - kSegmentUnits, 0);
    const int pg_hi = max(pu_start + seg_units - kSegmentUnits, 0);
    const int hkv = hq / p.ratio;
    const int N = max(0, min(p.seq_lens[b / p.Q], p.max_seq_len));
    const int n_vq = max(0, N - p.W);
    const int pair = b * p.Hq + hq;
    float* rec = p.records + static_cast<size_t>(pair + blockIdx.x) * RS;
    if (kRangeCheck && (pair + static_cast<int>(blockIdx.x) >= p.B * p.Hq + kMaxStreamCtas ||
                        static_cast<int>(blockIdx.x) >= kMaxStreamCtas)) {
      if (tid == 0 && p.status != nullptr) atomicOr(p.status, LOOPVQ_DECODE_STATUS_RANGE);
      return;                                          // CTA-uniform
    }
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
      __syncthreads();                                 // previous segment done with LUT and histogram
      const float* cbv = p.cb_v + hkv * p.cb_stride_head;
      if (warp == kNW - 1) {                           // the value slice, into L2 for the contraction
        constexpr uint32_t kSlice = kE * J * C * 4, kPiece = kSlice / 32;
        static_assert(kSlice % (32 * 16) == 0, "prefetch pieces are 16-byte multiples");
        prefetch_l2_bulk(reinterpret_cast<const char*>(cbv) + lane * kPiece, kPiece);
      }

      // ---- this warp's pages and blocks ----------------------------------------
      // Warp w streams the segment's pages pg_lo + w + k*kNW (k = 0, 1, ..), each
      // as bpp blocks; its t-th block is block t % bpp of its page t / bpp.
      // Chunk ch holds blocks [ch*KB, (ch+1)*KB) of every warp: their key rows,
      // then their value rows.
      const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
      const int32_t* bt = p.block_table + static_cast<size_t>(b / p.Q) * p.max_pages_per_seq;
      auto pages_of = [&](int w) { return (pg_hi > pg_lo + w) ? (pg_hi - pg_lo - w + kNW - 1) / kNW : 0; };
      const int my_first = pg_lo + warp;
      const int n_my_pages = pages_of(warp);
      const int n_blocks = n_my_pages << lbpp;
      const int n_chunks = ((pages_of(0) << lbpp) + KB - 1) / KB;   // CTA-uniform (warp 0 has the most)
      int i0 = 0;                                      // page-table window: this warp's pages [i0, i0 + 64)
      // page-table entry of this warp's page i, or -1 past its pages; an entry
      // outside the pool flags the status word and reads as -1 (its blocks are
      // skipped)
      auto bt_entry = [&](int i) -> int {
        int v = (i < n_my_pages) ? bt[my_first + i * kNW] : -1;
        if (i < n_my_pages && (v < 0 || v >= p.n_pages)) {
          if (p.status != nullptr) atomicOr(p.status, kStatusBadPage);
          v = -1;
        }
        return v;
      };
      int bt_cur = bt_entry(lane);
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
      BlockInfo info[KB];
      // Locates block t of this warp (its key row is loaded by the caller).
      // No branch: a block past this warp's list or on a skipped page gets
      // nv = 0 and the row of page 0 (in the pool, never read for nv = 0).
      auto locate = [&](int t, BlockInfo& bi) {
        const int pi = t >> lbpp, blk = t & (bpp - 1);
        const int src = (pi - i0 < 32) ? bt_cur : bt_nxt;
        const int phys = __shfl_sync(0xffffffffu, src, (pi - i0) & 31);
        const int pg = my_first + pi * kNW;
        bool ok = t < n_blocks && phys >= 0;
        if (kRangeCheck && ok && (pg < 0 || pg >= p.max_pages_per_seq || blk >= bpp)) {
          if (lane == 0 && p.status != nullptr) atomicOr(p.status, LOOPVQ_DECODE_STATUS_RANGE);
          ok = false;
        }
        bi.nv = ok ? max(0, min(LB, n_vq - pg * p.Pg - blk * LB)) : 0;
        bi.row = pool_h + (ok ? static_cast<int64_t>(phys) * p.page_bytes + blk * (LB * J) : 0) + lane * T::GR;
      };
      // the key rows of chunk ch into the ring (and their locations into info)
      auto issue_keys = [&](int ch) {
        const int kmin = (ch * KB) >> lbpp;            // first page of the chunk
        if (kmin >= i0 + 32) {                         // slide the page-table window
          bt_cur = bt_nxt;
          i0 += 32;
          bt_nxt = bt_entry(i0 + 32 + lane);
        }
        prefetch_pages(kmin + kPrefetchPages, (((ch + 1) * KB) >> lbpp) + kPrefetchPages);
      };
      auto issue_key = [&](int ch, int q) {
        locate(ch * KB + q, info[q]);
        if (info[q].nv > 0) load_row<J>(info[q].row, lane, ring[q]);
      };
      auto issue_value = [&](int q) {
        if (info[q].nv > 0) load_row<J>(info[q].row + p.plane_bytes, lane, ring[q]);
      };

      // ---- first key rows, then the pair's LUT and a zero histogram --------------
      prefetch_pages(0, kPrefetchPages);
      issue_keys(0);
#pragma unroll
      for (int q = 0; q < KB; ++q) issue_key(0, q);
      ensure_ready();
      {
        constexpr int NF = kE * J / 4;                 // float4s of the table
        constexpr int PER = (NF + kThreads - 1) / kThreads;
        const float4* src = reinterpret_cast<const float4*>(p.luts + static_cast<size_t>(pair) * kE * J);
        float4 v[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k)
          if (tid + k * kThreads < NF) v[k] = __ldcg(src + tid + k * kThreads);
#pragma unroll
        for (int i = tid * 4; i < kE * kCols; i += kThreads * 4)
          *reinterpret_cast<uint4*>(hist + i) = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int f = tid + k * kThreads;
          if (f < NF) {
            const int e = f / (J / 4), c0 = (f - e * (J / 4)) * 4;
#pragma unroll
            for (int c = c0; c + 4 <= kCols; c += J) *reinterpret_cast<float4*>(lut + e * kCols + c) = v[k];
          }
        }
      }
      __syncthreads();                                 // LUT and histogram ready, staging area free
      // ---- stream -------------------------------------------------------------
      // every block is scored (a block with nv = 0 holds stale or zero bytes,
      // which address cells inside the table) and masked afterwards
      auto key_score = [&](const BlockRegs<J>& r, int nv) -> float {
        uint32_t ad[J];
#pragma unroll
        for (int s = 0; s < J; ++s) ad[s] = __byte_perm(r.w[s >> 2], lane4, 0x7604u | (uint32_t(s & 3) << 4));
        uint64_t xa[2] = {0ull, 0ull};                 // two packed pairs of partial sums
        constexpr_for<J / 2>([&](auto P) {
          constexpr int s = 2 * P.value;
          xa[P.value & 1] = add_f32x2(xa[P.value & 1], f2_pack(lds_at<kLutAbs + 4u * s>(ad[s]),
                                                                  lds_at<kLutAbs + 4u * (s + 1)>(ad[s + 1])));
        });
        const float2 a = f2_unpack(xa[0]), b = f2_unpack(xa[1]);
        return lane < nv ? (a.x + a.y) + (b.x + b.y) : -INFINITY;
      };
      // histogram updates of one value block, lane = slot: the slot's weight
      // w = rn(2^(x - m + S)) goes to cell [idx][lane + s] for each byte s of its
      // rotated value row (w = 0 for an invalid slot)
      auto value_pass = [&](const BlockRegs<J>& r, float ex, float factor) {
        const uint32_t w = __float2uint_rn(ex * factor);
        uint32_t ad[J];
#pragma unroll
        for (int s = 0; s < J; ++s) ad[s] = __byte_perm(r.w[s >> 2], lane4, 0x7604u | (uint32_t(s & 3) << 4));
        constexpr_for<J>([&](auto S) { red_at<kHistAbs + 4u * S.value>(ad[S.value], w); });
      };
      // every cell >>= sh (an exact rescale of the fixed-point weights)
      auto rescale = [&](int sh) {
        for (int i = tid * 4; i < kE * kCols; i += kThreads * 4) {
          uint4 v = *reinterpret_cast<uint4*>(hist + i);
          if (sh >= 32) {
            v = make_uint4(0u, 0u, 0u, 0u);
          } else {
            v.x >>= sh; v.y >>= sh; v.z >>= sh; v.w >>= sh;
          }
          *reinterpret_cast<uint4*>(hist + i) = v;
        }
      };

      float m_cur = -INFINITY;                         // integer reference maximum (CTA-uniform)
      int S = kFixMax;                                 // fixed-point exponent (CTA-uniform)
      float mass = 0.f;                                // sum of weights so far, units of 2^(m_cur) (CTA-uniform)
#pragma unroll 1
      for (int ch = 0; ch < n_chunks; ++ch) {
        // A chunk whose last block is past this warp's pages (the last chunk
        // of a warp with fewer pages than warp 0) skips its empty blocks;
        // every other chunk runs without a branch per block (an empty block
        // there, on a skipped page, is reduced with weight 0).
        const bool tail = !__all_sync(0xffffffffu, info[KB - 1].nv > 0);   // warp-uniform
        float xs[KB];
        float cm = -INFINITY;
        if (!tail) {
#pragma unroll
          for (int q = 0; q < KB; ++q) {               // key phase
            xs[q] = key_score(ring[q], info[q].nv);
            cm = fmaxf(cm, xs[q]);
            issue_value(q);
          }
        } else {
#pragma unroll
          for (int q = 0; q < KB; ++q) {
            xs[q] = (info[q].nv > 0) ? key_score(ring[q], info[q].nv) : -INFINITY;
            cm = fmaxf(cm, xs[q]);
            issue_value(q);
          }
        }
        cm = redux_max(cm);
        // xs[q] becomes 2^(x - cm) (0 for an invalid slot, and for every slot
        // of a warp without a valid one); ps sums them over the warp in units
        // of 2^-kPsBits (a lane's share is at most KB, so the sum fits 32 bits)
        float ps = 0.f;
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          xs[q] = (cm == -INFINITY) ? 0.f : fast_exp2(xs[q] - cm);
          ps += xs[q];
        }
        ps = ldexp_pos(redux_add_u32(__float2uint_rn(ps * kPsScale)), -kPsBits);
        float* st = stat + (ch & 1) * 2 * kNW;
        if (lane == 0) {
          st[2 * warp] = cm;
          st[2 * warp + 1] = ps;
        }
        __syncthreads();                               // every warp's chunk maximum and sum
        const float cmw = (lane < kNW) ? st[2 * lane] : -INFINITY;
        const float cmax = redux_max(cmw);
        if (cmax != -INFINITY) {                       // CTA-uniform
          // m rises to ceil(max) + kMHead, so that a later chunk passes it (and
          // costs a rescale) only when its maximum is a whole unit higher
          const float m_new = (cmax > m_cur) ? ceilf(cmax) + kMHead : m_cur;
          // the chunk's weights in units of 2^m_new, summed in fixed point (a
          // warp's share is at most 32 * KB)
          const float psw = (lane < kNW && cmw != -INFINITY) ? st[2 * lane + 1] * fast_exp2(cmw - m_new) : 0.f;
          const float add = ldexp_pos(redux_add_u32(__float2uint_rn(ldexp_pos(psw, kAddBits))), -kAddBits);
          const float kept = (m_cur == -INFINITY) ? 0.f : mass * fast_exp2(m_cur - m_new);
          const float total = kept + add;
          int S_new = S;
          if (ldexp_pos(total, S) + static_cast<float>(kThreads * KB) > kMassHigh) {
            int ex;
            frexpf(total, &ex);                        // total < 2^ex
            S_new = min(S, kMassLandLog2 - ex);
          }
          const int sh = ((m_cur == -INFINITY) ? 0 : static_cast<int>(m_new - m_cur)) + (S - S_new);
          if (m_cur != -INFINITY && sh > 0) {          // earlier weights shrink by 2^-sh
            rescale(sh);
            __syncthreads();
          }
          m_cur = m_new;
          S = S_new;
          mass = total;
        }
        // w = rn(2^(x - m + S)) = rn(2^(x - cm) * 2^(cm - m + S)); 0 for an invalid slot
        const float factor = (cm == -INFINITY || m_cur == -INFINITY) ? 0.f : fast_exp2(cm - m_cur + static_cast<float>(S));
        if (!tail) {
#pragma unroll
          for (int q = 0; q < KB; ++q) {               // value phase
            value_pass(ring[q], xs[q], factor);
            if (q == 0) issue_keys(ch + 1);
            issue_key(ch + 1, q);
          }
        } else {
#pragma unroll
          for (int q = 0; q < KB; ++q) {
            if (info[q].nv > 0) value_pass(ring[q], xs[q], factor);
            if (q == 0) issue_keys(ch + 1);
            issue_key(ch + 1, q);
          }
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
        // this warp's groups j = warp + kNW*jw of the value slice, requested
        // before the histogram is read so that the loads land meanwhile
        constexpr int JPW = (J + kNW - 1) / kNW;
        float cv[JPW][kE / 32][C];
#pragma unroll
        for (int jw = 0; jw < JPW; ++jw) {
          const int j = warp + kNW * jw;
          if (j < J) {
#pragma unroll
            for (int i = 0; i < kE / 32; ++i)
              load_cw<C>(cbv + (static_cast<size_t>(j) * kE + lane + 32 * i) * C, cv[jw][i]);
          }
        }
        // W[e][j] = 2^-S * sum of the columns c = j (mod J): lane = group, rows warp + kNW*k
        constexpr int NR = kE / kNW;                   // rows per warp
        const float inv = ldexpf(1.f, -S);
        float* wt = lut;                               // transposed, padded: wt[j*EP + e]
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          const int e = warp + kNW * k;
          if (lane < J) {
            unsigned long long v = 0ull;
#pragma unroll
            for (int c = lane; c < kCols; c += J) v += hist[e * kCols + c];
            wt[lane * EP + e] = static_cast<float>(v) * inv;
          }
        }
        __syncthreads();
        // o[j*C + ch] = sum_e W[e][j] C_V[j][e][ch]: warp -> groups, lane -> rows lane + 32 i
#pragma unroll
        for (int jw = 0; jw < JPW; ++jw) {
          const int j = warp + kNW * jw;
          if (j >= J) break;                           // warp-uniform
          float acc[C];
#pragma unroll
          for (int ch = 0; ch < C; ++ch) acc[ch] = 0.f;
#pragma unroll
          for (int i = 0; i < kE / 32; ++i) {
            const float h = wt[j * EP + lane + 32 * i];
#pragma unroll
            for (int ch = 0; ch < C; ++ch) acc[ch] = fmaf(h, cv[jw][i][ch], acc[ch]);
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

    // ---- publish the record; the pair's last writer merges ------------------
    {
      // the CTAs whose unit ranges meet the pair's units [u0, u0 + units_b)
      const long long u0 = pre * p.Hq + static_cast<long long>(hq) * units_b;
      const int c_first = static_cast<int>(((u0 + 1) * p.n_cta - 1) / U);
      const int c_last = static_cast<int>(((u0 + units_b) * p.n_cta - 1) / U);
      if (kRangeCheck && (c_first < 0 || c_last >= p.n_cta || c_first > static_cast<int>(blockIdx.x) ||
                          c_last < static_cast<int>(blockIdx.x))) {
        if (tid == 0 && p.status != nullptr) atomicOr(p.status, LOOPVQ_DECODE_STATUS_RANGE);
        return;                                        // CTA-uniform
      }
      ensure_ready();                                  // the counter was zeroed by the pair kernel
      __threadfence();                                 // this thread's record writes, device-wide
      __syncthreads();
      if (tid == 0) {
        int n = c_last - c_first + 1;                  // writers: the CTAs of the range with units
        if (U < p.n_cta)
          for (int c = c_first; c <= c_last; ++c) n -= (U * c / p.n_cta < U * (c + 1) / p.n_cta) ? 0 : 1;
        *s_last = atomicAdd(p.counts + pair, 1u) == static_cast<unsigned>(n - 1);
      }
      __syncthreads();
      if (*s_last) {                                   // CTA-uniform: every record of the pair is written
        __threadfence();
        merge_pair<d, kThreads>(p, pair, c_first, c_last, U);
      }
    }

    u += seg_units;
    pu_start = 0;
    if (++hq == p.Hq) {
      hq = 0;
      do {
        pre += units_b;
        ++b;
      } while (b < p.B && u < u_hi && (units_b = pair_units(seq_pages(p, b))) == 0);
    }
  }
  // every CTA waits once, so that this grid completes after the pair kernel
  ensure_ready();
}

template <typename K>
loopvq_status set_smem(K kernel, size_t smem, std::atomic<uint64_t>& configured) {
  // The attribute belongs to (function, device); remember which devices have
  // it. The streaming kernel's shared-memory addresses assume its dynamic
  // allocation starts at kSBase: right after the block's reserved shared
  // memory, with no static shared memory before it.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit == 0 || !(configured.load(std::memory_order_relaxed) & bit)) {
    int reserved = -1;
    if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
      return LOOPVQ_ERR_CUDA;
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return LOOPVQ_ERR_CUDA;
    if (reserved != static_cast<int>(kSBase) || fa.sharedSizeBytes != 0) return LOOPVQ_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return LOOPVQ_ERR_CUDA;
    configured.fetch_or(bit, std::memory_order_relaxed);
  }
  return LOOPVQ_OK;
}

// Launches `kernel` as a programmatic dependent of the previous kernel on
// the stream: its CTAs may start while that kernel's last CTAs still run
// (griddepcontrol.wait inside orders the reads that need its results).
template <typename K>
loopvq_status launch_dependent(K kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                               const DecodeParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, p) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

template <int J, int C>
loopvq_status launch_vq(const DecodeParams& p, cudaStream_t st, bool run_stream) {
  static_assert(kDynBytes <= 227 * 1024, "streaming kernel shared memory above 227 KB");
  const unsigned pairs = static_cast<unsigned>(p.B * p.Hq);
  // window partials, and the key tables when anything streams
  vq_pair_kernel<J, C><<<dim3(pairs, run_stream ? 1 + J / 4 : 1), kPairThreads, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (run_stream) {
    static std::atomic<uint64_t> configured{0};
    const loopvq_status s = set_smem(vq_stream_kernel<J, C>, kDynBytes, configured);
    if (s != LOOPVQ_OK) return s;
    return launch_dependent(vq_stream_kernel<J, C>, static_cast<unsigned>(p.n_cta), kThreads, kDynBytes, st,
                            p);
  }
  return LOOPVQ_OK;
}

}  // namespace

size_t decode_workspace_bytes(int pairs, int J, int d) {
  const size_t rec = (4 + static_cast<size_t>(d)) * sizeof(float);
  return kStatusBytes + (static_cast<size_t>(pairs) + kMaxStreamCtas) * rec +   // segment records
         static_cast<size_t>(pairs) * rec +                                     // window partials
         static_cast<size_t>(pairs) * kE * J * sizeof(float) +                  // key lookup tables
         (static_cast<size_t>(pairs) * sizeof(unsigned) + 15) / 16 * 16;        // record counters
}

loopvq_status launch_decode(const DecodeArgs& a) {
  const Geometry& g = *a.geo;
  const int gamma = a.loop_step / g.g, tau = a.loop_step % g.g;
  const int bpp = g.Pg / g.LB;
  int log2_bpp = 0;
  while ((1 << log2_bpp) < bpp) ++log2_bpp;
  if ((1 << log2_bpp) != bpp) return LOOPVQ_ERR_UNSUPPORTED;
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
  // workspace: status word, segment records, key lookup tables
  char* ws = static_cast<char*>(a.workspace);
  const size_t pairs = static_cast<size_t>(a.batch) * a.n_queries * g.Hq;
  p.status = reinterpret_cast<int*>(ws);
  const size_t rec = (4 + static_cast<size_t>(g.d)) * sizeof(float);
  p.records = reinterpret_cast<float*>(ws + kStatusBytes);
  p.wrecs = reinterpret_cast<float*>(ws + kStatusBytes + (pairs + kMaxStreamCtas) * rec);
  p.luts = reinterpret_cast<float*>(ws + kStatusBytes + (2 * pairs + kMaxStreamCtas) * rec);
  p.counts = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(p.luts) + pairs * kE * g.J * sizeof(float));
  p.out = a.out;
  p.lse = a.lse;
  p.B = a.batch * a.n_queries;
  p.Q = a.n_queries;
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
  p.log2_bpp = log2_bpp;
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
