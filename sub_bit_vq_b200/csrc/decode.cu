// Fused LoopVQ decode attention over the packed index cache (sm_100a).
//
// Two kernels per call.
//
// vq_stream_kernel: a persistent grid (at most one CTA per SM, twelve warps)
// over the quantised tokens of every (sequence, query head) pair. All pages
// of all pairs form one list and CTA c takes the contiguous range
// [U*c/n, U*(c+1)/n) of it, so every CTA streams the same number of pages and
// touches one or a few pairs ("segments"). Per segment:
//   1. The key codebook slice of the pair's kv-head and loop step is staged
//      into the (empty) histogram windows with cp.async while the warps
//      request their first index blocks (a register ring); the key lookup
//      table LUT[e][col] = s*log2(e) * q_j . C_K[j][e][tau] (column col holds
//      group j = col % J) is built from it and the windows are zeroed.
//   2. Streaming. Warp w takes pages w, w+12, ...; a block is LB token slots
//      (LB = floor(32/J)*J), two blocks per round. Key pass: lane = slot;
//      byte s of the slot's rotated row is group (lane+s) % J, held by LUT
//      column (lane+s) % LB. Value pass: the weights p = 2^(x - m) are added
//      into a histogram W[e][col]: lane = (replica, group) owns column
//      `lane`, rows come from the group-major value bytes, four slots at a
//      time; a weight whose row repeats later among the four is folded into
//      that later update, so the last store of a row carries all of them.
//      Three warps (w, w+4, w+8: one scheduler) share a histogram and take
//      turns through bounded mbarrier waits; a warp computes its key scores
//      and weights before its turn and only the histogram updates inside it.
//      Each histogram keeps one running maximum m, raised only when a vote
//      finds a score above m + kRescaleSlack.
//   3. The four histograms are merged with log-sum-exp weights into W[E][J],
//      which is contracted with the value codebook slice,
//      o_j = sum_e W[e][j] C_V[j][e][tau]; the segment record (m, l, o[d]) goes
//      to slot (pair + cta).
//
// vq_finish_kernel: one CTA per pair scores the bf16 window tokens (prefix +
// recent), merges them with the pair's segment records (log-sum-exp
// weights) and writes out and lse.
//
// The hot loops address shared memory by absolute shared-window address, so
// that one byte permute of an index word gives a complete address: the
// histograms occupy the 64 KB-aligned windows [0x10000, 0x30000) (row e at
// byte e*256 of its window, two histograms per window) and the LUT the
// window [0x8000, 0x10000) with 128-byte rows. The dynamic allocation starts
// at a small base (the CTA's reserved bytes) and is sized to cover both; a
// CTA whose base leaves no room below the LUT writes NaN records instead of
// running.

#include <math.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kNHist = 4;                 // value histograms
constexpr int kPerHist = 3;               // warps taking turns on one histogram
constexpr int kNW = kNHist * kPerHist;    // warps of the streaming kernel
constexpr int kThreads = kNW * 32;
constexpr int kRing = kPerHist >= 3 ? 2 : 4;   // index blocks in registers (rounds of two ahead)
constexpr int kPrefetchPages = 8;         // pages a warp asks L2 to fetch ahead of its loads
constexpr float kRescaleSlack = 8.0f;     // log2 units a score may exceed m before m is raised
constexpr int kFinishThreads = 256;
constexpr int kWinChunk = 9;              // window tokens per warp per round of loads (72 = 8 warps x 9)
constexpr int kSegmentUnits = 16;        // work units (pages) charged for a segment's setup
constexpr int kSpinLimit = 1 << 14;       // bounded mbarrier waits (each try sleeps up to kSuspendNs)
constexpr uint32_t kSuspendNs = 65536u;

constexpr uint32_t kLutAbs = 0x8000u;     // LUT [E][32] floats, 128-byte rows
constexpr uint32_t kHistAbs = 0x10000u;   // histogram h: window 1 + h/2, bytes (h%2)*128 .. of each row
constexpr uint32_t kHistEnd = 0x30000u;   // (the key slice is staged here before a segment streams)
constexpr uint32_t kDynBytes = kHistEnd;  // covers every window from any base >= 0

// Small area at the start of the dynamic allocation (byte offsets).
constexpr uint32_t kPbufOff = 0;                                  // [kNW][64] slot weights
constexpr uint32_t kWstatOff = kPbufOff + kNW * 64 * 4;           // [2*kNW] per-warp m, l
constexpr uint32_t kHmOff = kWstatOff + 2 * kNW * 4;              // [kNHist] running maxima
constexpr uint32_t kFlagOff = kHmOff + kNHist * 4;                // [4] ints
constexpr uint32_t kMbarOff = (kFlagOff + 16 + 7) & ~7u;          // [kNHist][kPerHist] mbarriers
constexpr uint32_t kSmallBytes = kMbarOff + kNHist * kPerHist * 8;

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

// ---- shared memory by absolute shared-window address ------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

// Histogram words: ordered among themselves and against other memory
// accesses (read-modify-write chains depend on it).
__device__ __forceinline__ float lds_h(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts_h(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
// LUT words: not written while they are read, so no ordering against stores.
__device__ __forceinline__ float lds_lut(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, P;\n}\n"
      : "=r"(done)
      : "r"(a), "r"(parity), "n"(kSuspendNs)
      : "memory");
  return done != 0u;
}
// Waits for the phase of parity `parity` to complete (each try sleeps until
// the phase completes or kSuspendNs pass); gives up (false) after kSpinLimit
// tries instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
  for (int i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    __nanosleep(64);                                   // leave the issue slots to the working warps
  }
  return false;
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
  constexpr int RS = 4 + d;                            // record floats
  constexpr int EP = kE + 1;                           // padded row of the transposed merged histogram
  static_assert(J * EP * 4 <= static_cast<int>(kHistEnd - kHistAbs), "merged histogram fits the windows");
  // groups of the key slice staged at once in the (empty) histogram windows
  constexpr int JC = (J * kE * C * 4 <= static_cast<int>(kHistEnd - kHistAbs))
                         ? J : static_cast<int>(kHistEnd - kHistAbs) / (kE * C * 4);
  static_assert(J % JC == 0, "staging chunks tile the groups");
  static_assert(d <= kNW * 64 && d <= kThreads, "q fits the weight buffer");

  extern __shared__ __align__(16) unsigned char smem_u8[];
  const uint32_t sbase = smem_addr(smem_u8);
  float* pbuf = reinterpret_cast<float*>(smem_u8 + kPbufOff);
  float* wstat = reinterpret_cast<float*>(smem_u8 + kWstatOff);
  float* hm = reinterpret_cast<float*>(smem_u8 + kHmOff);
  int* flags = reinterpret_cast<int*>(smem_u8 + kFlagOff);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem_u8 + kMbarOff);
  // a base that leaves no room below the LUT window: poison records, do nothing else
  const bool bad_base = sbase + kSmallBytes > kLutAbs;
  float* lut = reinterpret_cast<float*>(smem_u8 + (bad_base ? 0u : kLutAbs - sbase));
  float* stage = reinterpret_cast<float*>(smem_u8 + (bad_base ? 0u : kHistAbs - sbase));
  float* qs = pbuf;                                    // scaled q while the LUT is built

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // warps w, w+4, .. share histogram w % 4: one scheduler serves all turns on it
  const int hidx = warp % kNHist, role = warp / kNHist;
  const bool lane_live = lane < LB;
  float* my_p = pbuf + warp * 64;
  // byte permutes that put an index byte into byte 1 of these give addresses
  const uint32_t hx = ((1u + static_cast<uint32_t>(hidx >> 1)) << 16) |
                      static_cast<uint32_t>((hidx & 1) * 128 + lane * 4);
  uint32_t lx[J];                                      // (value >> 1) = LUT word of lookup s
#pragma unroll
  for (int s = 0; s < J; ++s) lx[s] = 0x10000u | (8u * static_cast<uint32_t>((lane + s) % LB));
  // turns on histogram hidx run role 0, 1, .., kPerHist-1, 0, ..
  const uint32_t bar_wait = smem_addr(mbar + hidx * kPerHist + role);
  const uint32_t bar_give = smem_addr(mbar + hidx * kPerHist + (role + 1) % kPerHist);
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

  if (!bad_base) {
    if (tid < kNHist * kPerHist) mbar_init(smem_addr(mbar + tid), 32u);
    if (tid == 0) flags[0] = 0;
    __syncthreads();
    if (role == kPerHist - 1) mbar_arrive(bar_give);   // the first turn is role 0's
  }
  uint32_t rnd = 0;                                    // rounds taken (same count in all warps of a histogram)
  bool wait_failed = false;

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
      __syncthreads();                                 // previous segment done with LUT and histograms
      // the first chunk of the key slice goes out before anything that waits
      for (int i = tid * 4; i < JC * kE * C; i += kThreads * 4) cp_async16(stage + i, cbk + i);
      const float* cbv = p.cb_v + hkv * p.cb_stride_head;
      if (warp == kNW - 1) {                           // the value slice, into L2 for the contraction
        constexpr uint32_t kSlice = kE * J * C * 4, kPiece = kSlice / 32;
        static_assert(kSlice % (32 * 16) == 0, "prefetch pieces are 16-byte multiples");
        prefetch_l2_bulk(reinterpret_cast<const char*>(cbv) + lane * kPiece, kPiece);
      }
      const float qv = (tid < d) ? bf16_bits_to_float(qp[tid]) * p.scale_log2 : 0.f;

      // ---- index ring prologue ----------------------------------------------
      const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
      const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
      auto pages_of = [&](int w) { return (pg_hi > pg_lo + w) ? (pg_hi - pg_lo - w + kNW - 1) / kNW : 0; };
      const int my_first = pg_lo + warp;
      const int n_my_pages = pages_of(warp);
      const int n_blocks = n_my_pages * bpp;
      // rounds of two blocks; all warps of a histogram take the largest count
      int most_pages = 0;
#pragma unroll
      for (int k = 0; k < kPerHist; ++k) most_pages = max(most_pages, pages_of(hidx + kNHist * k));
      const int n_rounds = (most_pages * bpp + 1) / 2;
      int i0 = 0;
      auto bt_entry = [&](int i) -> int { return (i < n_my_pages) ? bt[my_first + i * kNW] : -1; };
      int bt_cur = bt_entry(lane);                     // requested now, used after the slice lands
      int bt_nxt = bt_entry(32 + lane);
      BlockRegs<J> ring[kRing] = {};
      // a cleared block keeps whatever bytes it held: every byte value
      // addresses a valid row, and base = -1 masks its scores and skips it
      auto clear = [&](BlockRegs<J>& r) { r.base = -1; };
      auto issue = [&](int k, BlockRegs<J>& r) {
        if (k >= n_blocks) {                             // warp-uniform
          clear(r);
          return;
        }
        const int pi = static_cast<int>(__umulhi(static_cast<uint32_t>(k), bpp_magic));
        const int blk = k - pi * bpp;
        if (pi >= i0 + 32) {                             // warp-uniform
          bt_cur = bt_nxt;
          i0 += 32;
          bt_nxt = bt_entry(i0 + 32 + lane);
        }
        if (blk == 0) {                                  // first block of a page: prefetch ahead
          const int tgt = pi + kPrefetchPages;           // tgt - i0 < 64: inside cur or nxt
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

      // ---- key LUT from the key slice staged in the histogram windows ----------
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
          if (lane < kPrefetchPages && lane < n_my_pages && bt_cur >= 0 && bt_cur < p.n_pages)
            prefetch_l2_bulk(pool_h + static_cast<int64_t>(bt_cur) * p.page_bytes,
                             static_cast<uint32_t>(p.page_bytes));
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
          for (int r = 0; r < T::R; ++r) lut[e * 32 + j + r * J] = v;
        }
      }
      __syncthreads();                                 // LUT complete; staging area free
      for (uint32_t a = kHistAbs + 16u * tid; a < kHistEnd; a += 16u * kThreads)
        asm volatile("st.shared.v4.f32 [%0], {%1, %1, %1, %1};" ::"r"(a), "f"(0.f) : "memory");
      if (tid < kNHist) hm[tid] = -INFINITY;
      __syncthreads();                                 // histograms zero, maxima reset

      // ---- stream -------------------------------------------------------------
      float m_seen = -INFINITY;                        // pair maximum this warp's l refers to
      float l_lane = 0.f;
      auto key_scores = [&](const BlockRegs<J>& r) -> float {
        float xa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < J; ++s)
          xa[s & 3] += lds_lut(__byte_perm(r.k[s >> 2], lx[s], 0x7604u | (uint32_t(s & 3) << 4)) >> 1);
        const bool valid = r.base >= 0 && lane_live && (r.base + lane) < r.valid;
        return valid ? (xa[0] + xa[1]) + (xa[2] + xa[3]) : -INFINITY;
      };
      auto value_pass = [&](const BlockRegs<J>& r, const float* pp) {
        if (r.base < 0) return;                        // warp-uniform
        if constexpr (LB < 32) {
          if (!lane_live) return;
        }
        pp += (lane / J) * J;
        float4 p4 = *reinterpret_cast<const float4*>(pp);
#pragma unroll
        for (int i = 0; i < J; i += 4) {
          const uint32_t w = r.v[i >> 2];
          const uint32_t a0 = __byte_perm(w, hx, 0x7604u), a1 = __byte_perm(w, hx, 0x7614u);
          const uint32_t a2 = __byte_perm(w, hx, 0x7624u), a3 = __byte_perm(w, hx, 0x7634u);
          // fold each weight into the last slot of the four with the same row
          float q1 = p4.y, q2 = p4.z, q3 = p4.w;
          if (a1 == a0) q1 += p4.x;
          if (a2 == a0) q2 += p4.x;
          if (a2 == a1) q2 += p4.y;
          if (a3 == a0) q3 += p4.x;
          if (a3 == a1) q3 += p4.y;
          if (a3 == a2) q3 += p4.z;
          const float o0 = lds_h(a0), o1 = lds_h(a1), o2 = lds_h(a2), o3 = lds_h(a3);
          // the next batch's weights (never written during the pass) before this batch's stores
          const float4 p4n = (i + 4 < J) ? *reinterpret_cast<const float4*>(pp + i + 4) : p4;
          sts_h(a0, o0 + p4.x);
          sts_h(a1, o1 + q1);
          sts_h(a2, o2 + q2);
          sts_h(a3, o3 + q3);
          p4 = p4n;
        }
      };
      // One round: key scores and (against the maximum this warp saw last)
      // weights outside the turn, the histogram updates inside.
      auto round = [&](const BlockRegs<J>& ra, const BlockRegs<J>& rb) {
        const float xa = key_scores(ra);
        const float xb = key_scores(rb);
        const float xl = fmaxf(xa, xb);
        const bool spec = m_seen != -INFINITY &&
                          __all_sync(0xffffffffu, !(xl > m_seen + kRescaleSlack));
        float pa = 0.f, pb = 0.f;
        if (spec) {                                    // warp-uniform
          pa = fast_exp2(xa - m_seen);
          pb = fast_exp2(xb - m_seen);
          my_p[lane] = pa;
          my_p[32 + lane] = pb;
        }
        if (!wait_failed && !mbar_wait(bar_wait, rnd & 1u)) wait_failed = true;
        ++rnd;
        float m = hm[hidx];
        const bool keep = spec && m == m_seen;         // warp-uniform
        if (m != m_seen) {                             // another warp raised the maximum
          if (m_seen != -INFINITY) l_lane *= fast_exp2(m_seen - m);
          m_seen = m;
        }
        if (!keep && __any_sync(0xffffffffu, xl > m + kRescaleSlack)) {   // warp-uniform, rare
          const float xm = warp_max(xl);
          if (m != -INFINITY) {
            const float f = fast_exp2(m - xm);
            if (lane_live) {
              for (int e = 0; e < kE; ++e) {
                const uint32_t a = hx | (static_cast<uint32_t>(e) << 8);
                sts_h(a, lds_h(a) * f);
              }
            }
            l_lane *= f;
          }
          m = xm;
          m_seen = xm;
          if (lane == 0) hm[hidx] = xm;
        }
        if (m != -INFINITY) {                          // warp-uniform
          if (!keep) {
            pa = fast_exp2(xa - m);                    // 0 for xa = -inf
            pb = fast_exp2(xb - m);
            my_p[lane] = pa;
            my_p[32 + lane] = pb;
          }
          l_lane += pa + pb;
          __syncwarp();
          value_pass(ra, my_p);
          value_pass(rb, my_p + 32);
          __syncwarp();                                // my_p is rewritten next round
        }
        mbar_arrive(bar_give);                         // all lanes: releases this turn's writes
      };

      for (int r0 = 0; r0 < n_rounds; r0 += kRing / 2) {
#pragma unroll
        for (int h = 0; h < kRing / 2; ++h) {
          if (r0 + h < n_rounds) {                     // warp-uniform
            round(ring[2 * h], ring[2 * h + 1]);
            issue(2 * (r0 + h) + kRing, ring[2 * h]);
            issue(2 * (r0 + h) + kRing + 1, ring[2 * h + 1]);
          }
        }
      }
      const float l_w = warp_sum(l_lane);
      if (lane == 0) {
        wstat[warp] = m_seen;
        wstat[kNW + warp] = l_w;
        if (wait_failed) atomicOr(flags, 1);
      }
      __syncthreads();

      // ---- merge the histograms, contract with the value slice -------------------
      float Mh = -INFINITY;
#pragma unroll
      for (int h = 0; h < kNHist; ++h) Mh = fmaxf(Mh, hm[h]);
      if (Mh == -INFINITY) {                           // nothing valid: an empty record
        if (tid == 0) {
          rec[0] = (flags[0] != 0) ? NAN : -INFINITY;
          rec[1] = 0.f;
        }
      } else {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w)
          if (wstat[w] != -INFINITY) L += wstat[kNW + w] * fast_exp2(wstat[w] - Mh);
        float fh[kNHist];
#pragma unroll
        for (int h = 0; h < kNHist; ++h) fh[h] = (hm[h] == -INFINITY) ? 0.f : fast_exp2(hm[h] - Mh);
        // W[e][j]: lane = column, rows warp + kNW*k; replicas of a group are summed
        constexpr int NR = (kE + kNW - 1) / kNW;       // rows per warp
        const float* hist = stage;                     // the histogram windows as floats
        float wv[NR];
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          const int e = warp + kNW * k;
          float v = 0.f;
          if (e < kE && lane_live) {
#pragma unroll
            for (int h = 0; h < kNHist; ++h)
              v = fmaf(fh[h], hist[(h >> 1) * 16384 + e * 64 + (h & 1) * 32 + lane], v);
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
          if (e < kE && lane < J) wt[lane * EP + e] = wv[k];
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
        if (tid == 0) {
          rec[0] = (flags[0] != 0) ? NAN : Mh;         // a turn that timed out poisons the pair
          rec[1] = L;
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
