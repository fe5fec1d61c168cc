// Attention of a chunk of queries over the VQ cache on the tensor cores
// (sm_100a): the prefill form for many queries per sequence.
//
// With Q queries per (sequence, query head) the key lookup tables of the
// streaming decode would be built and read Q times; here the quantised
// tokens are dequantised once per tile instead and both products run as
// dense contractions on tcgen05:
//   S = Q_tile . K_tile^T      (M = 128 queries, N = 64 tokens, K = d)
//   O += P . V_tile            (M = 128 queries, N = d, K = 64 tokens)
// with an online softmax between them, as in flash attention.
//
// Work unit: (sequence b, query head hq, tile of 128 queries, token chunk).
// Chunks 0 .. S-2 cover the quantised tokens [c*CH, (c+1)*CH); chunk S-1 is
// the bf16 window (prefix + recent). One CTA per unit, 256 threads: query
// row r (TMEM lane r) is served by a thread of warp r / 32 and one of warp
// r / 32 + 4, each holding half of the row's S, P and O columns:
//   1. Q tile (bf16, K-major, no swizzle) into shared memory; the (layer,
//      kv-head, gamma, tau) key codebook slice, split by prefill_cb_kernel
//      into bf16 high and low parts (128 KB), by bulk copy into shared
//      memory. The value slice, rounded to bf16, stays in global memory (L2)
//      and is gathered.
//   2. Per tile of 64 tokens: the key indices of the tile (rotated rows of the
//      pool's K plane) select codewords, split into bf16 high and low parts,
//      into K_hi and K_lo [64][d]; the value indices select bf16 codewords
//      into V_tile^T [d][64] (the transposed tile is the K-major B operand of
//      the second product). Tokens past the chunk are zero and masked.
//   3. One thread issues S = Q K_hi^T + Q K_lo^T into TMEM (q is bf16, so the
//      scores keep the codewords' float32 precision to about 2^-17); each
//      thread reads its row,
//      x = s * scale * log2(e), keeps a running reference m (raised only when
//      a tile's maximum passes it by more than 8, so that P = 2^(x - m) stays
//      below 2^8; O and l are then rescaled in TMEM), writes P as bf16 into
//      shared memory and adds the rounded P to l; one thread issues O += P V.
//   4. The unit's record (m, l, o[d]) per query row goes to the workspace; a
//      split merge (merge.cu) combines the chunks and the window per query.
//
// Rounding: the value codewords and P are bf16 operands with fp32
// accumulation (relative error about 2^-9 in the output), so this form
// serves bf16 outputs; the streaming form, exact in fp32, serves fp32
// outputs and short chunks. l sums the unrounded P, so lse keeps float32
// precision.

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace loopvq {
namespace {

constexpr int kPfRows = 128;              // queries per tile (MMA M)
constexpr int kPfTok = 64;                // tokens per tile
constexpr int kPfThreads = 256;            // two threads per query row (column halves)
constexpr int kPfD = 128;                 // head_dim of this form
constexpr int kPfJ = 32;                  // channel groups (c = 4)
constexpr int kPfC = 4;
constexpr float kPfLazy = 8.f;            // raise m only when a tile passes it by this (log2)
#ifndef LOOPVQ_TC_SPIN
#define LOOPVQ_TC_SPIN (1 << 20)
#endif
constexpr int kPfSpin = LOOPVQ_TC_SPIN;
constexpr int kPfDrainSpin = 1 << 24;

// Shared memory (bytes).
constexpr int kQsOff = 0;                                  // [128][128] bf16, K-major
constexpr int kKsOff = kQsOff + kPfRows * kPfD * 2;        // [2 (hi, lo)][64 tokens][128] bf16
constexpr int kKsBytes = kPfTok * kPfD * 2;
constexpr int kVsOff = kKsOff + 2 * kKsBytes;              // [128 dims][64 tokens] bf16
constexpr int kPsOff = kVsOff + kPfD * kPfTok * 2;         // [128][64] bf16
constexpr int kCbOff = kPsOff + kPfRows * kPfTok * 2;      // key slice [J][E][C] fp32
constexpr int kCbBytes = kPfJ * kE * kPfC * 4;             // 128 KB
constexpr int kCb16Elems = kPfJ * kE * kPfC;               // one bf16 value slice, elements
constexpr int kVixOff = kCbOff + kCbBytes;                 // [64 tokens][32] value index bytes
constexpr int kBarOff = kVixOff + kPfTok * kPfJ;           // mbarriers: S, O, codebooks
constexpr int kTmemOff = kBarOff + 32;
constexpr int kPfSmem = kTmemOff + 16;
constexpr uint32_t kTmemS = 0, kTmemO = 128;               // TMEM columns of S (64) and O (128)

struct PrefillParams {
  const uint16_t* q;              // bf16 [B][Q][Hq][d]
  const uint8_t* pool_lg;         // pool at (layer, gamma, head 0)
  int64_t pool_stride_head, page_bytes, plane_bytes;
  const uint16_t* cbk16;          // bf16 key slices split high/low [Hkv][J][E][2][C]
  const uint16_t* cbv16;          // bf16 value slices [Hkv][J][E][C]
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint16_t* win_k;          // bf16 [B][Hkv][W][d]
  const uint16_t* win_v;
  float* records;                 // [B*Q*Hq][S][d + 2]
  int* status;
  int B, Q, Hq, ratio, W, Pg, LB, n_pages, max_pages_per_seq, max_seq_len;
  int S, CH, QT;                  // units per (b, hq, query tile), chunk tokens, query tiles
  float scale_log2;
};

__device__ __forceinline__ uint32_t u32s(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (r, k) of a K-major operand with KP columns
// (8-row x 16-byte core matrices, K halves 128 bytes apart).
template <int KP>
__device__ __forceinline__ uint32_t kmaj(int r, int k) {
  return static_cast<uint32_t>((r >> 3) * (KP / 8) * 128 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, int kp) {
  const uint64_t lbo = 128u >> 4, sbo = static_cast<uint64_t>(kp * 16) >> 4;
  return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) | (lbo << 16) | (sbo << 32) | (1ull << 46);
}

// bf16 x bf16 -> fp32, K-major A and B, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(n) >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ bool pf_wait(uint32_t bar, uint32_t parity, int spin) {
  for (int it = 0; it < spin; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n"
        " selp.u32 %0, 1, 0, P;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    if (ok != 0u) return true;
  }
  return false;
}

__device__ __forceinline__ void tld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tst32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
        "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// The codebook slices of every kv-head at loop offset tau in bf16: the value
// slice rounded, cbv16[h][j][e][ch], and the key slice split into high and
// low parts, cbk16[h][j][e][hi 0..3, lo 0..3] (16 bytes per codeword).
__global__ void __launch_bounds__(256) prefill_cb_kernel(const float* cb_k, const float* cb_v,
                                                         int64_t cb_stride_head, int Hkv, uint16_t* cbv16,
                                                         uint16_t* cbk16) {
  constexpr int N = kCb16Elems;
  const int64_t total = static_cast<int64_t>(Hkv) * N;
  for (int64_t i = (blockIdx.x * 256 + threadIdx.x) * 4ll; i < total; i += gridDim.x * 256ll * 4) {
    const int h = static_cast<int>(i / N), r = static_cast<int>(i % N);
    const float4 v = *reinterpret_cast<const float4*>(cb_v + h * cb_stride_head + r);
    *reinterpret_cast<uint2*>(cbv16 + i) = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    const float4 k = *reinterpret_cast<const float4*>(cb_k + h * cb_stride_head + r);
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(k.x, k.y), h23 = __floats2bfloat162_rn(k.z, k.w);
    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
    const __nv_bfloat162 l01 = __floats2bfloat162_rn(k.x - f01.x, k.y - f01.y);
    const __nv_bfloat162 l23 = __floats2bfloat162_rn(k.z - f23.x, k.w - f23.y);
    *reinterpret_cast<uint4*>(cbk16 + 2 * i) =
        make_uint4(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23),
                   *reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
  }
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_tc_kernel(const PrefillParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* Qs = sm + kQsOff;
  unsigned char* Ks = sm + kKsOff;
  unsigned char* Vs = sm + kVsOff;
  unsigned char* Ps = sm + kPsOff;
  const uint4* cbk = reinterpret_cast<const uint4*>(sm + kCbOff);   // [J][E] (hi, lo) codewords
  uint8_t* vix = sm + kVixOff;
  float* xch = reinterpret_cast<float*>(sm + kVixOff);   // [2][128] row partials (vix is free then)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kTmemOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = ((warp & 3) << 5) | lane;            // query row of the tile = TMEM lane
  const int colh = warp >> 2;                          // half of the S, P and O columns

  // ---- the unit -----------------------------------------------------------------
  int x = blockIdx.x;
  const int c = x % p.S;
  x /= p.S;
  const int qt = x % p.QT;
  x /= p.QT;
  const int hq = x % p.Hq, b = x / p.Hq;
  const int hkv = hq / p.ratio;
  const int N = max(0, min(p.seq_lens[b], p.max_seq_len));
  const int n_vq = max(0, N - p.W);
  const bool window = c == p.S - 1;
  const int k0 = window ? 0 : c * p.CH;
  const int k1 = window ? min(N, p.W) : min(n_vq, (c + 1) * p.CH);   // tokens [k0, k1)
  const int row_q = qt * kPfRows + row;                // this thread's query
  const bool row_ok = row_q < p.Q;
  float* rec = p.records + ((static_cast<size_t>(b) * p.Q + row_q) * p.Hq + hq) * p.S * (kPfD + 2) +
               static_cast<size_t>(c) * (kPfD + 2);
  if (k1 <= k0) {                                      // CTA-uniform: an empty record
    if (row_ok && colh == 0) {
      rec[0] = -INFINITY;
      rec[1] = 0.f;
    }
    return;
  }

  // ---- setup: barriers, TMEM, key codebook, Q tile ---------------------------------
  const uint32_t bar_s = u32s(bars), bar_o = u32s(bars + 1), bar_cb = u32s(bars + 2);
  if (tid == 0) {
    for (int i = 0; i < 3; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(u32s(bars + i)), "r"(1u) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(u32s(tmem_slot)),
                 "r"(256u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0 && !window) {                           // the key slice: two bulk copies of 64 KB
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_cb), "r"(kCbBytes)
                 : "memory");
    const uint16_t* src = p.cbk16 + static_cast<size_t>(hkv) * (kCbBytes / 2);
    for (int part = 0; part < 2; ++part)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(u32s(sm + kCbOff + part * (kCbBytes / 2))), "l"(src + part * (kCbBytes / 4)),
                   "r"(kCbBytes / 2), "r"(bar_cb) : "memory");
  }
  {                                                    // the query rows, bf16, zero past Q
    const uint16_t* qr = p.q + ((static_cast<size_t>(b) * p.Q + row_q) * p.Hq + hq) * kPfD + colh * 64;
#pragma unroll
    for (int k = 0; k < 64; k += 8) {
      const uint4 v = row_ok ? *reinterpret_cast<const uint4*>(qr + k) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(Qs + kmaj<kPfD>(row, colh * 64 + k)) = v;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t my_s = lane_base + kTmemS + colh * 32, my_o = lane_base + kTmemO + colh * 64;
  bool failed = !window && !pf_wait(bar_cb, 0, kPfSpin);
  failed = __syncthreads_or(failed);

  const uint8_t* pool_h = p.pool_lg + hkv * p.pool_stride_head;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages_per_seq;
  const uint16_t* wk = p.win_k + (static_cast<size_t>(b) * (p.Hq / p.ratio) + hkv) * p.W * kPfD;
  const uint16_t* wv = p.win_v + (static_cast<size_t>(b) * (p.Hq / p.ratio) + hkv) * p.W * kPfD;
  const uint32_t qs_a = u32s(Qs), ks_a = u32s(Ks), vs_a = u32s(Vs), ps_a = u32s(Ps);
  const uint16_t* cbv = p.cbv16 + static_cast<size_t>(hkv) * kCb16Elems;   // bf16, in L2
  float m_run = -INFINITY, l_run = 0.f;                // l_run: this thread's half of the row
  bool o_live = false;                                 // an O product has been issued
  int n_tiles_done = 0;
  int pending_o = -1;                                  // parity of an O commit not yet waited for

  // Index bytes of this thread's token (t & 63) and quarter (t >> 6) of the
  // tile at token tt, requested one tile ahead; its page entry two tiles ahead.
  uint2 nx_k = make_uint2(0u, 0u), nx_v = make_uint2(0u, 0u);
  bool nx_ok = false;
  int ph_a = -1, ph_b = -1;                            // page entries of my token in the next two tiles
  auto page_of = [&](int tt) -> int {                  // block-table entry of my token at tile tt
    const int kq = tt + (tid & 63);
    return (tt < k1 && kq < k1) ? bt[kq / p.Pg] : -1;
  };
  auto fetch_rows = [&](int tt) {                      // rows of tile tt (page entry ph_a); shift the entries
    const int kq = tt + (tid & 63), quarter = tid >> 6;
    const bool tok = tt < k1 && kq < k1;
    nx_ok = tok && ph_a >= 0 && ph_a < p.n_pages;
    if (tok && !nx_ok && quarter == 0 && p.status != nullptr) atomicOr(p.status, LOOPVQ_DECODE_STATUS_BAD_PAGE);
    nx_k = make_uint2(0u, 0u);
    nx_v = make_uint2(0u, 0u);
    if (nx_ok) {
      const int slot = kq % p.Pg, blk = slot / p.LB, rot = slot % p.LB;
      const uint8_t* rowp = pool_h + static_cast<int64_t>(ph_a) * p.page_bytes + blk * (p.LB * kPfJ) +
                            (quarter >> 1) * (p.LB * 16) + rot * 16 + (quarter & 1) * 8;
      nx_k = *reinterpret_cast<const uint2*>(rowp);
      nx_v = *reinterpret_cast<const uint2*>(rowp + p.plane_bytes);
    }
    ph_a = ph_b;
    ph_b = page_of(tt + 2 * kPfTok);
  };
  if (!window) {
    ph_a = page_of(k0);
    ph_b = page_of(k0 + kPfTok);
    fetch_rows(k0);                                    // tile 0 now, entries of tiles 1 and 2 in flight
  }

  for (int t0 = k0; t0 < k1 && !failed; t0 += kPfTok) {
    const int nt = min(kPfTok, k1 - t0);               // valid tokens of this tile

    // ---- index bytes of this tile (prefetched a tile ago) and the next tile's ---------
    const int n = tid & 63, quarter = tid >> 6;        // token of the tile, quarter of its 32 groups
    const bool tok_ok = n < nt;
    uint2 kidx = make_uint2(0u, 0u);
    bool page_ok = false;
    if (!window) {
      kidx = nx_k;
      page_ok = nx_ok;
      *reinterpret_cast<uint2*>(vix + n * kPfJ + quarter * 8) = nx_v;   // value bytes by position
      fetch_rows(t0 + kPfTok);                         // tile t + 1: lands during this tile
    }
    if (!window) __syncthreads();                      // value index bytes staged
    // ---- value codewords of this tile: task (group j, token octet o) gathers dims
    // 4j .. 4j+3 of tokens 8o .. 8o+7 (from L2; they land while K is dequantised)
    const int vj = tid & (kPfJ - 1), vo = tid >> 5;
    uint32_t vlo[8], vhi[8];                           // token q: dims (4j, 4j+1) and (4j+2, 4j+3)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int tn = vo * 8 + q;
      uint2 cw = make_uint2(0u, 0u);
      if (tn < nt) {
        if (window) {
          cw = *reinterpret_cast<const uint2*>(wv + static_cast<size_t>(t0 + tn) * kPfD + vj * kPfC);
        } else {
          const int rot = ((t0 + tn) % p.Pg) % p.LB;
          const int pos = (vj - rot) & (kPfJ - 1);
          const uint32_t idx = vix[tn * kPfJ + pos];
          cw = *reinterpret_cast<const uint2*>(cbv + (vj * kE + idx) * kPfC);
        }
      }
      vlo[q] = cw.x;
      vhi[q] = cw.y;
    }
    // ---- K tile [64][128] (hi, lo); the previous S product is done with Ks ------------
    if (window) {
      const uint16_t* kr = wk + static_cast<size_t>(t0 + n) * kPfD + quarter * 32;
#pragma unroll
      for (int k = 0; k < 32; k += 8) {
        const uint4 v = tok_ok ? *reinterpret_cast<const uint4*>(kr + k) : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(Ks + kmaj<kPfD>(n, quarter * 32 + k)) = v;               // exact in bf16
        *reinterpret_cast<uint4*>(Ks + kKsBytes + kmaj<kPfD>(n, quarter * 32 + k)) = make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      const int rot = ((t0 + n) % p.Pg) % p.LB;
      const uint32_t kw[2] = {kidx.x, kidx.y};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int pos = quarter * 8 + q;
        const int j = (pos + rot) & (kPfJ - 1);        // group of this byte of the rotated row
        const uint32_t idx = (kw[q >> 2] >> (8 * (q & 3))) & 0xffu;
        const uint4 cw = page_ok ? cbk[j * kE + idx] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint2*>(Ks + kmaj<kPfD>(n, j * kPfC)) = make_uint2(cw.x, cw.y);
        *reinterpret_cast<uint2*>(Ks + kKsBytes + kmaj<kPfD>(n, j * kPfC)) = make_uint2(cw.z, cw.w);
      }
    }
    // the previous tile's O product has read Ps and Vs (and O may be rescaled)
    if (pending_o >= 0) {
      const bool ok = pf_wait(bar_o, static_cast<uint32_t>(pending_o), kPfSpin);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      pending_o = -1;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    }
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {                   // V^T row 4j + ch: 8 tokens, 16 bytes
      const uint32_t* src = ch < 2 ? vlo : vhi;
      const uint32_t sel = (ch & 1) ? 0x7632u : 0x5410u;   // high or low bf16 of each word
      uint4 v;
      v.x = __byte_perm(src[0], src[1], sel);
      v.y = __byte_perm(src[2], src[3], sel);
      v.z = __byte_perm(src[4], src[5], sel);
      v.w = __byte_perm(src[6], src[7], sel);
      *reinterpret_cast<uint4*>(Vs + kmaj<kPfTok>(4 * vj + ch, vo * 8)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();

    // ---- S = Q K_hi^T + Q K_lo^T -------------------------------------------------------
    const int tile = n_tiles_done;
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; ++kk)
          mma_bf16(tmem + kTmemS, sdesc(qs_a + kk * 256, kPfD), sdesc(ks_a + part * kKsBytes + kk * 256, kPfD),
                   idesc_bf16(kPfTok), (part > 0 || kk > 0) ? 1u : 0u);
      mma_commit(bar_s);
    }
    {
      const bool ok = pf_wait(bar_s, static_cast<uint32_t>(tile & 1), kPfSpin);
      if (__syncthreads_or(!ok)) {
        failed = true;
        pending_o = -2;                                // the S product may still write TMEM
        break;
      }
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    // ---- softmax: this thread's 32 columns of its row; P into shared memory ------------
    uint32_t sv[32];
    tld32(my_s, sv);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    float mt = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float a = colh * 32 + i < nt ? __uint_as_float(sv[i]) * p.scale_log2 : -INFINITY;
      sv[i] = __float_as_uint(a);
      mt = fmaxf(mt, a);
    }
    xch[colh * kPfRows + row] = mt;
    __syncthreads();
    mt = fmaxf(xch[row], xch[kPfRows + row]);          // the row's maximum over both halves
    const bool raise = m_run == -INFINITY || mt > m_run + kPfLazy;
    if (__any_sync(0xffffffffu, raise)) {              // warp-uniform; the partner warp decides alike
      const float m_new = raise ? fmaxf(m_run, mt) : m_run;
      const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
      if (o_live) {
#pragma unroll 1
        for (int cc = 0; cc < 64; cc += 32) {
          uint32_t o[32];
          tld32(my_o + cc, o);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tst32(my_o + cc, o);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      l_run *= alpha;
      m_run = m_new;
    }
#pragma unroll
    for (int k = 0; k < 32; k += 8) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p0 = fast_exp2(__uint_as_float(sv[k + 2 * e]) - m_run);
        const float p1 = fast_exp2(__uint_as_float(sv[k + 2 * e + 1]) - m_run);
        l_run += p0 + p1;                              // unrounded: lse keeps float32 precision
        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        w[e] = *reinterpret_cast<const uint32_t*>(&pb);
      }
      *reinterpret_cast<uint4*>(Ps + kmaj<kPfTok>(row, colh * 32 + k)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();

    // ---- O += P V ---------------------------------------------------------------------
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int kk = 0; kk < kPfTok / 16; ++kk)
        mma_bf16(tmem + kTmemO, sdesc(ps_a + kk * 256, kPfTok), sdesc(vs_a + kk * 256, kPfTok),
                 idesc_bf16(kPfD), (o_live || kk > 0) ? 1u : 0u);
      mma_commit(bar_o);
    }
    o_live = true;
    pending_o = tile & 1;
    ++n_tiles_done;
  }

  // ---- the record (m, l, o) of every row ------------------------------------------------
  if (!failed && pending_o >= 0) {
    const bool ok = pf_wait(bar_o, static_cast<uint32_t>(pending_o), kPfSpin);
    failed = __syncthreads_or(!ok);
    if (!failed) pending_o = -1;
  }
  if (!failed) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
    for (int cc = 0; cc < 64; cc += 32) {
      uint32_t o[32];
      tld32(my_o + cc, o);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 32; i += 2)                // records are 8-byte aligned
          *reinterpret_cast<float2*>(rec + 2 + colh * 64 + cc + i) =
              make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1]));
      }
    }
    xch[colh * kPfRows + row] = l_run;
    __syncthreads();
    if (row_ok && colh == 0) {
      rec[0] = m_run;
      rec[1] = xch[row] + xch[kPfRows + row];
    }
  } else {
    // a bounded wait gave up: drain what the tensor cores and the bulk copy
    // may still write, flag the status word, poison the record
    if (tid == 0) {
      bool drained = true;
      if (pending_o >= 0) drained = pf_wait(bar_o, static_cast<uint32_t>(pending_o), kPfDrainSpin) && drained;
      if (pending_o == -2) drained = pf_wait(bar_s, static_cast<uint32_t>(n_tiles_done & 1), kPfDrainSpin) && drained;
      if (!window) drained = pf_wait(bar_cb, 0, kPfDrainSpin) && drained;
      if (p.status != nullptr) atomicOr(p.status, drained ? LOOPVQ_DECODE_STATUS_TIMEOUT
                                                          : (LOOPVQ_DECODE_STATUS_TIMEOUT | LOOPVQ_DECODE_STATUS_UNDRAINED));
    }
    if (row_ok && colh == 0) {
      rec[0] = NAN;
      rec[1] = 1.f;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u) : "memory");
  }
}

}  // namespace

bool prefill_tc_supported(const Geometry& g, int n_queries, int out_dtype) {
  return out_dtype == LOOPVQ_DTYPE_BF16 && n_queries >= kPrefillTcMinQueries && g.d == kPfD &&
         g.c == kPfC && g.J == kPfJ && g.LB == 32 && g.GR == 16 && g.Pg % g.LB == 0;
}

size_t prefill_tc_workspace_bytes(const Geometry& g, int batch, int n_queries, int max_seq_len, int* S,
                                  int* CH) {
  const int n_vq_max = max_seq_len > g.W ? max_seq_len - g.W : 0;
  // chunks of at least 2048 tokens, at most 32 of them
  int ch = 2048;
  while ((n_vq_max + ch - 1) / ch > 32) ch *= 2;
  const int s = (n_vq_max + ch - 1) / ch + 1;
  if (S != nullptr) *S = s;
  if (CH != nullptr) *CH = ch;
  const size_t rows = static_cast<size_t>(batch) * n_queries * g.Hq;
  const size_t rec = rows * s * (g.d + 2) * sizeof(float);
  const size_t cb = static_cast<size_t>(g.Hkv) * kCb16Elems * 2 * 3;   // value bf16, key hi/lo
  return kStatusBytes + ((rec + 255) / 256) * 256 + cb;
}

loopvq_status launch_prefill_tc(const DecodeArgs& a, size_t workspace_bytes) {
  const Geometry& g = *a.geo;
  int S = 0, CH = 0;
  const size_t need = prefill_tc_workspace_bytes(g, a.batch, a.n_queries, a.max_seq_len, &S, &CH);
  if (need > workspace_bytes) return LOOPVQ_ERR_UNSUPPORTED;   // the streaming form takes it
  const int gamma = a.loop_step / g.g, tau = a.loop_step % g.g;
  PrefillParams p{};
  p.q = static_cast<const uint16_t*>(a.q);
  p.pool_lg = a.pool + a.layer * g.pool_stride_layer + gamma * g.pool_stride_group;
  p.pool_stride_head = g.pool_stride_head;
  p.page_bytes = g.page_bytes;
  p.plane_bytes = g.plane_bytes;
  const float* cb_l = a.codebooks + a.layer * g.cb_stride_layer + gamma * g.cb_stride_group + tau * g.cb_stride_loop;
  char* ws = static_cast<char*>(a.workspace);
  p.status = reinterpret_cast<int*>(ws);
  p.records = reinterpret_cast<float*>(ws + kStatusBytes);
  const size_t rows = static_cast<size_t>(a.batch) * a.n_queries * g.Hq;
  const size_t rec = rows * S * (g.d + 2) * sizeof(float);
  uint16_t* cb16 = reinterpret_cast<uint16_t*>(ws + kStatusBytes + ((rec + 255) / 256) * 256);
  p.cbv16 = cb16;
  p.cbk16 = cb16 + static_cast<size_t>(g.Hkv) * kCb16Elems;
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.win_k = static_cast<const uint16_t*>(a.win_k);
  p.win_v = static_cast<const uint16_t*>(a.win_v);
  p.B = a.batch;
  p.Q = a.n_queries;
  p.Hq = g.Hq;
  p.ratio = g.Hq / g.Hkv;
  p.W = g.W;
  p.Pg = g.Pg;
  p.LB = g.LB;
  p.n_pages = g.n_pages;
  p.max_pages_per_seq = g.max_pages_per_seq;
  p.max_seq_len = a.max_seq_len;
  p.S = S;
  p.CH = CH;
  p.QT = (a.n_queries + kPfRows - 1) / kPfRows;
  p.scale_log2 = a.sm_scale * kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  prefill_cb_kernel<<<g.Hkv * 2, 256, 0, st>>>(cb_l, cb_l + g.cb_stride_kv, g.cb_stride_head, g.Hkv, cb16,
                                               cb16 + static_cast<size_t>(g.Hkv) * kCb16Elems);
  if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  static_assert(kPfSmem <= 227 * 1024, "prefill shared memory above 227 KB");
  if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmem) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  const long long units = static_cast<long long>(a.batch) * g.Hq * p.QT * S;
  if (units > 0x7fffffffLL) return LOOPVQ_ERR_UNSUPPORTED;
  prefill_tc_kernel<<<static_cast<unsigned>(units), kPfThreads, kPfSmem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return LOOPVQ_ERR_CUDA;
  return launch_merge(p.records, static_cast<int>(rows), S, g.d, a.out_dtype, a.out, a.lse, a.stream);
}

}  // namespace loopvq
