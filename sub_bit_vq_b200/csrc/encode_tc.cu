// Nearest-centroid encoder on the tensor cores (tcgen05), for prefill-sized
// batches (sm_100a).
//
// For a token's sub-vector s (D values) with weights w, the weighted squared
// distance to centroid e is
//     d_e = sum_i w_i s_i^2 - 2 sum_i (w_i s_i) C_ei + sum_i w_i C_ei^2,
// so the nearest centroid minimises S_e = a . b_e with a = [w*s, w] and
// b_e = [-2 C_e, C_e*C_e] (K = 2D): one dense [tokens x 2D] x [2D x 256]
// contraction per (head, channel group).
//
// One CTA per (channel group j, kv-head h) keeps B = [b_e] for the 256
// centroids in shared memory and walks the tokens in tiles of 128. The x and
// w rows of a tile arrive by TMA (one 3-d box per tensor: the group's
// channels, rounded out to 16 bytes, x 128 tokens x g loop steps) into one
// of three staging buffers, three tiles ahead, so that the per-token 8- and
// 16-byte pieces never occupy the load/store unit. Two threads serve each
// tile row, one per half of the 256 centroid columns (the 256 threads read
// TMEM as two warps per 32-lane quarter). Per tile: both threads of a row
// compute the row's scale and margin and write their half of the row of A;
// one thread issues the tcgen05.mma chain that leaves S (128 x 256, fp32) in
// tensor memory; each thread reads its 128 columns back with tcgen05.ld,
// the halves exchange minima, and each marks its columns within the margin.
// Each warp then lists its (row, column) candidates and its lanes score
// the list round-robin.
//
// Operands are fp16, scaled by powers of two so that each operand uses the
// top of fp16's range: the -2C half of B by 2^beta1 and the C*C half by
// 2^beta2 (fixed per codebook), a row of A by 2^(rho - beta) per half (rho
// per row). Every product of a row is then a_k b_ek 2^rho, so S' = 2^rho S
// has S's argmin. fp16 x fp16 products are exact in the fp32 accumulator,
// so with alpha = scaled a and beta' = scaled b, each S'_e is off by at most
//     2^-9.98 sum_k |alpha_k| |beta'_ek| + 2^-24.9 (sum_k |alpha_k| + sum_k |beta'_ek|)
// (the two fp16 roundings, 2^-11 each, the float32 rounding of w*s and C*C,
// fp16's subnormal spacing and the fp32 accumulation over K). Every centroid
// within
//     margin = 2^-8.5 2^rho sum_k |a_k| max_e |b_ek| + 2^-17 2^rho sum_i w_i s_i^2
//              + 2^-23 (sum_k |alpha_k| + sum_k max_e |beta'_ek|)
// of the row's smallest S'_e is rescored with the float32 direct form and
// term order of encode_kernel (the margin covers twice the error above plus
// the direct form's own rounding); the first minimum of those (smallest
// index on equal distances) is the index encode_kernel chooses. A row whose
// minimum or margin is not finite rescores all 256 centroids.
//
// Shared operands use the K-major layout without swizzle: 8-row x 16-byte
// core matrices, the two 8-element halves of a 16-wide K step 128 bytes
// apart (leading byte offset) and consecutive 8-row groups KP*16 bytes
// apart (stride byte offset).

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "encode_common.cuh"

namespace loopvq {

// Encoder status word of this device (flag bits, LOOPVQ_ENCODE_STATUS_*),
// set by the kernels and read (and cleared) by loopvq_encode_status.
__device__ int g_encode_status = 0;

namespace {

constexpr int kTcRows = 128;              // tokens per tile (MMA M)
constexpr int kTcThreads = 256;           // two threads per tile row, one per half of the 256 columns
constexpr int kListCap = 256;             // rescoring list entries per warp
constexpr int kStages = 3;                // TMA staging buffers (tiles in flight)
#ifndef LOOPVQ_TC_SPIN
#define LOOPVQ_TC_SPIN (1 << 20)
#endif
constexpr int kTcSpin = LOOPVQ_TC_SPIN;   // bounded mbarrier wait (tries) for a tile's MMA
constexpr int kTcDrainSpin = 1 << 24;     // bounded wait for the last MMA before TMEM is freed
constexpr int kTopExp = 13;               // scaled operands lie in [2^13, 2^14) at their largest
constexpr float kMarginRel = 0.0027621358640099515f;    // 2^-8.5
constexpr float kMarginWss = 7.62939453125e-06f;        // 2^-17
constexpr float kMarginAbs = 1.1920928955078125e-07f;   // 2^-23

template <int C, int G>
struct TcGeo {
  static constexpr int D = C * G;
  static constexpr int K2 = 2 * D;                      // [w*s, w] . [-2C, C*C]
  static constexpr int KP = ((K2 + 15) / 16) * 16;      // padded to the MMA K step
  static constexpr int A_BYTES = kTcRows * KP * 2;
  static constexpr int B_BYTES = kE * KP * 2;
  static constexpr int CB_FLOATS = G * kE * C;          // fp32 codebook [tau][E][c] for rescoring
  static constexpr int XIN = 8;                         // x box: 8 bf16 channels (16 bytes)
  static constexpr int WIN = C > 4 ? C : 4;             // w box: at least 4 floats (16 bytes)
  static constexpr int XBOX = XIN * kTcRows * G * 2;    // [G][128][XIN] bf16
  static constexpr int WBOX = WIN * kTcRows * G * 4;    // [G][128][WIN] float
  static constexpr int STAGE = ((XBOX + WBOX + 127) / 128) * 128;
  static constexpr int STG_OFF = 0;                     // kStages staging buffers
  static constexpr int A_OFF = STG_OFF + kStages * STAGE;
  static constexpr int B_OFF = A_OFF + A_BYTES;
  static constexpr int CB_OFF = B_OFF + B_BYTES;
  static constexpr int BMAX_OFF = CB_OFF + CB_FLOATS * 4;   // [K2] uint: max_e |b_ek| (float bits)
  static constexpr int WSH_OFF = BMAX_OFF + K2 * 4;         // [D] float: weights shared by all tokens
  static constexpr int PMIN_OFF = WSH_OFF + D * 4;          // [2][kTcRows] float: minimum of each half
  static constexpr int PBEST_OFF = PMIN_OFF + 2 * kTcRows * 4;   // [2][kTcRows] (float, int): best of each half
  static constexpr int LIST_OFF = PBEST_OFF + 2 * kTcRows * 8;   // [8 warps][kListCap] uint16 (row lane, column)
  static constexpr int DLIST_OFF = LIST_OFF + 8 * kListCap * 2;  // [8 warps][kListCap] float distances
  static constexpr int MBAR_OFF = (DLIST_OFF + 8 * kListCap * 4 + 7) & ~7;   // MMA, then one per stage
  static constexpr int TMEM_OFF = MBAR_OFF + 8 * (1 + kStages);
  static constexpr int SMEM = TMEM_OFF + 16;
};

// Byte offset of element (r, k) of a K-major operand with KP columns.
template <int KP>
__device__ __forceinline__ uint32_t op_off(int r, int k) {
  return static_cast<uint32_t>((r >> 3) * (KP / 8) * 128 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

// Shared-memory matrix descriptor: K-major, no swizzle, leading byte offset
// 128 (next 8-element K half), stride byte offset kp*16 (next 8-row group).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, int kp) {
  const uint64_t lbo = 128u >> 4, sbo = static_cast<uint64_t>(kp * 16) >> 4;
  return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) | (lbo << 16) | (sbo << 32) | (1ull << 46);
}

// Instruction descriptor: f16 x f16 -> fp32, both operands K-major,
// M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ uint32_t u32_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// floor(log2 m) for a normal m > 0 (-127 for zero or subnormal m).
__device__ __forceinline__ int exp_of(float m) {
  return static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127;
}

// 2^e for e in [-126, 127] (clamped), exactly.
__device__ __forceinline__ float pow2(int e) {
  e = max(-126, min(127, e));
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

// (d0, d1) = bits of (a.lo - b0, a.hi - b1), rounded to nearest.
__device__ __forceinline__ void sub_f32x2(uint64_t a, uint32_t b0, uint32_t b1, uint32_t& d0, uint32_t& d1) {
  uint64_t b, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "r"(b0), "r"(b1));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(d0), "=r"(d1) : "l"(d));
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Writes row r of an fp16 operand with KP columns: v[k] rounded to nearest,
// zero past K2.
template <int KP, int K2>
__device__ __forceinline__ void write_row_f16(unsigned char* base, int r, const float (&v)[K2]) {
#pragma unroll
  for (int k0 = 0; k0 < KP; k0 += 8) {
    uint32_t u[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int k = k0 + 2 * t;
      const float lo = k < K2 ? v[k] : 0.f, hi = k + 1 < K2 ? v[k + 1] : 0.f;
      const __half2 h2 = __floats2half2_rn(lo, hi);
      u[t] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(base + op_off<KP>(r, k0)) = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

// Row r of an fp16 operand with KP columns: the N values v, rounded to
// nearest, into columns [col0, col0 + N) (N and col0 multiples of 8); only
// v[k_begin, k_end) is written.
template <int KP, int N>
__device__ __forceinline__ void write_row_f16_range(unsigned char* base, int r, const float (&v)[N],
                                                    int k_begin, int k_end, int col0) {
#pragma unroll
  for (int k0 = 0; k0 < N; k0 += 8) {
    if (k0 < k_begin || k0 >= k_end) continue;
    uint32_t u[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __half2 h2 = __floats2half2_rn(v[k0 + 2 * t], v[k0 + 2 * t + 1]);
      u[t] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(base + op_off<KP>(r, col0 + k0)) = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

// Token n's sub-vector of (group j, head h) and its weights (1 when no
// weights are given), with one vector load per loop step for each.
template <int C, int G>
__device__ __forceinline__ void load_subvector_vec(const EncodeParams& p, int n, int j, int h,
                                                   float (&s)[C * G], float (&w)[C * G]) {
#pragma unroll
  for (int tau = 0; tau < G; ++tau) {
    const uint16_t* xr = p.x + tau * p.x_loop_stride + n * p.x_token_stride +
                         static_cast<int64_t>(h) * p.d + j * C;
    uint32_t u[C / 2];
    if constexpr (C == 8) {
      const uint4 t = *reinterpret_cast<const uint4*>(xr);
      u[0] = t.x; u[1] = t.y; u[2] = t.z; u[3] = t.w;
    } else if constexpr (C == 4) {
      const uint2 t = *reinterpret_cast<const uint2*>(xr);
      u[0] = t.x; u[1] = t.y;
    } else {
      u[0] = *reinterpret_cast<const uint32_t*>(xr);
    }
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      s[tau * C + 2 * i] = __uint_as_float(u[i] << 16);
      s[tau * C + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
    if (p.w != nullptr) {
      const float* wr = p.w + tau * p.w_loop_stride + n * p.w_token_stride +
                        static_cast<int64_t>(h) * p.d + j * C;
      if constexpr (C == 2) {
        const float2 t = *reinterpret_cast<const float2*>(wr);
        w[tau * C] = t.x; w[tau * C + 1] = t.y;
      } else {
#pragma unroll
        for (int i = 0; i < C; i += 4) {
          const float4 t = *reinterpret_cast<const float4*>(wr + i);
          w[tau * C + i] = t.x; w[tau * C + i + 1] = t.y; w[tau * C + i + 2] = t.z; w[tau * C + i + 3] = t.w;
        }
      }
    } else {
#pragma unroll
      for (int ch = 0; ch < C; ++ch) w[tau * C + ch] = 1.f;
    }
  }
}

// Byte of (slot, group j, head h) in the pool, or in assign[h][j][slot], for
// slot < 2^31: one 32-bit division by the block size (page_tokens is a
// power-of-two multiple of it, and the granule a power of two).
__device__ __forceinline__ void store_index_u32(const EncodeParams& p, uint32_t slot, int j, int h, int e,
                                                int pg_shift, int gr_shift) {
  if (p.assign != nullptr) {
    p.assign[(static_cast<int64_t>(h) * p.J + j) * p.n_tokens + slot] = static_cast<uint8_t>(e);
    return;
  }
  const uint32_t lb = static_cast<uint32_t>(p.LB), jj = static_cast<uint32_t>(p.J);
  const uint32_t q = slot / lb;                      // block index over the pool
  const uint32_t rot = slot - q * lb;                // row in the block
  const uint32_t page = q >> pg_shift, blk = q & ((1u << pg_shift) - 1u);
  int pos = j - static_cast<int>(rot % jj);
  if (pos < 0) pos += p.J;
  const uint32_t off = blk * lb * jj + ((static_cast<uint32_t>(pos) >> gr_shift) * lb << gr_shift) +
                       (rot << gr_shift) + (static_cast<uint32_t>(pos) & ((1u << gr_shift) - 1u));
  p.pool[h * p.pool_stride_head + static_cast<int64_t>(page) * p.page_bytes + p.kv * p.plane_bytes + off] =
      static_cast<uint8_t>(e);
}

// 32 consecutive TMEM columns of this warp's 32 lanes, one per register
// (tcgen05_wait_ld makes them usable).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
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
__device__ __forceinline__ void tcgen05_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Bounded wait for phase `parity` of the mbarrier at shared address `bar`.
__device__ __forceinline__ bool wait_parity(uint32_t bar, uint32_t parity, int spin) {
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

// One 3-d TMA box of `map` at coordinates (c0, c1, c2) into shared memory at
// `dst`, counted on the mbarrier at `bar` (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Row `r` of tile staging buffer `stg`: the token's sub-vector s and, for
// per-token weights (w_mode 2), its weights w.
template <int C, int G>
__device__ __forceinline__ void staged_row(const unsigned char* stg, int r, int x_off, int w_off, int w_mode,
                                           const float* w_shared, float (&s)[C * G], float (&w)[C * G]) {
  using Geo = TcGeo<C, G>;
#pragma unroll
  for (int tau = 0; tau < G; ++tau) {
    const uint16_t* xr = reinterpret_cast<const uint16_t*>(stg) + (tau * kTcRows + r) * Geo::XIN + x_off;
    uint32_t u[C / 2];
    if constexpr (C == 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr);
      u[0] = v.x; u[1] = v.y; u[2] = v.z; u[3] = v.w;
    } else if constexpr (C == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(xr);
      u[0] = v.x; u[1] = v.y;
    } else {
      u[0] = *reinterpret_cast<const uint32_t*>(xr);
    }
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      s[tau * C + 2 * i] = __uint_as_float(u[i] << 16);
      s[tau * C + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
    if (w_mode == 2) {
      const float* wr = reinterpret_cast<const float*>(stg + Geo::XBOX) + (tau * kTcRows + r) * Geo::WIN + w_off;
      if constexpr (C == 2) {
        const float2 v = *reinterpret_cast<const float2*>(wr);
        w[tau * C] = v.x; w[tau * C + 1] = v.y;
      } else {
#pragma unroll
        for (int i = 0; i < C; i += 4) {
          const float4 v = *reinterpret_cast<const float4*>(wr + i);
          w[tau * C + i] = v.x; w[tau * C + i + 1] = v.y; w[tau * C + i + 2] = v.z; w[tau * C + i + 3] = v.w;
        }
      }
    } else {
#pragma unroll
      for (int ch = 0; ch < C; ++ch) w[tau * C + ch] = w_shared[tau * C + ch];
    }
  }
}

// encode_kernel's float32 distance of (s, w) to codeword e, in its term order.
template <int C, int G>
__device__ __forceinline__ float direct_dist(const float* cbs, int e, const float (&s)[C * G],
                                             const float (&w)[C * G]) {
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
  return dist;
}

template <int C, int G>
__global__ void __launch_bounds__(kTcThreads, 2) encode_tc_kernel(const EncodeParams p,
                                                                   const __grid_constant__ CUtensorMap tmx,
                                                                   const __grid_constant__ CUtensorMap tmw) {
  using Geo = TcGeo<C, G>;
  constexpr int D = Geo::D, K2 = Geo::K2, KP = Geo::KP;
  extern __shared__ __align__(128) unsigned char tsm[];
  unsigned char* As = tsm + Geo::A_OFF;
  unsigned char* Bs = tsm + Geo::B_OFF;
  float* cbs = reinterpret_cast<float*>(tsm + Geo::CB_OFF);
  unsigned int* bmax = reinterpret_cast<unsigned int*>(tsm + Geo::BMAX_OFF);
  float* pmin = reinterpret_cast<float*>(tsm + Geo::PMIN_OFF);
  float2* pbest = reinterpret_cast<float2*>(tsm + Geo::PBEST_OFF);
  uint16_t* list = reinterpret_cast<uint16_t*>(tsm + Geo::LIST_OFF);
  float* dlist = reinterpret_cast<float*>(tsm + Geo::DLIST_OFF);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(tsm + Geo::MBAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tsm + Geo::TMEM_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = warp >> 2;                        // this thread's columns: [128 half, 128 half + 128)
  const int row = ((warp & 3) << 5) | lane;          // this thread's tile row (its warp's TMEM lanes)
  const int j = blockIdx.x, h = blockIdx.y;

  // ---- codebook of (j, h): fp32 copy for rescoring, scaled fp16 B operand ---
  const float* cb = p.cb + h * p.cb_stride_head + static_cast<int64_t>(j) * kE * C;
  for (int i = tid * 4; i < G * kE * C; i += kTcThreads * 4) {
    const int tau = i / (kE * C), r = i % (kE * C);
    cp_async16(cbs + i, cb + tau * p.cb_stride_loop + r);
  }
  if (tid < K2) bmax[tid] = 0u;
  if (tid == 0) {                                    // MMA commits, then the staging buffers
    for (int i = 0; i < 1 + kStages; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(u32_smem(mbar + i)), "r"(1u) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {                                   // 256 TMEM columns: one fp32 per centroid
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(u32_smem(tmem_slot)), "r"(256u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  cp_async_wait_all();
  __syncthreads();
  auto b_row = [&](int e, float (&b)[K2]) {
#pragma unroll
    for (int tau = 0; tau < G; ++tau) {
#pragma unroll
      for (int ch = 0; ch < C; ++ch) {
        const float c = cbs[(tau * kE + e) * C + ch];
        b[tau * C + ch] = -2.f * c;
        b[D + tau * C + ch] = c * c;
      }
    }
  };
  for (int e = tid; e < kE; e += kTcThreads) {
    float b[K2];
    b_row(e, b);
#pragma unroll
    for (int i = 0; i < K2; ++i) atomicMax(bmax + i, __float_as_uint(fabsf(b[i])));
  }
  __syncthreads();
  // column scales: the largest |b| of each half lands in [2^13, 2^14)
  const float* bm = reinterpret_cast<const float*>(bmax);   // max_e |b_ek|, read from shared memory
  float m_lo = 0.f, m_hi = 0.f;
#pragma unroll
  for (int i = 0; i < K2; ++i) {
    if (i < D) m_lo = fmaxf(m_lo, bm[i]); else m_hi = fmaxf(m_hi, bm[i]);
  }
  const int beta1 = m_lo > 0.f ? kTopExp - exp_of(m_lo) : 0;
  const int beta2 = m_hi > 0.f ? kTopExp - exp_of(m_hi) : 0;
  const float fb1 = pow2(beta1), fb2 = pow2(beta2);
  float q_abs = 0.f;                                 // sum_k max_e |beta'_ek|
#pragma unroll
  for (int i = 0; i < K2; ++i) q_abs += bm[i] * (i < D ? fb1 : fb2);
  // rho keeps 2^rho, 2^(rho - beta1) and 2^(rho - beta2) exact
  const int rho_lo = max(-126, max(-126 + beta1, -126 + beta2));
  const int rho_hi = min(127, min(127 + beta1, 127 + beta2));
  for (int e = tid; e < kE; e += kTcThreads) {
    float b[K2];
    b_row(e, b);
#pragma unroll
    for (int i = 0; i < K2; ++i) b[i] *= (i < D ? fb1 : fb2);
    write_row_f16<KP, K2>(Bs, e, b);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // B visible to the tensor cores
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  const uint32_t a_base = u32_smem(As), b_base = u32_smem(Bs), mbar_a = u32_smem(mbar);
  const uint32_t my_tmem = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + half * 128;
  const int n_tiles = (p.n_tokens + kTcRows - 1) / kTcRows;
  const bool slot_u32 = p.n_slots <= 0x7fffffffLL;
  const int pg_shift = __ffs(p.Pg / p.LB) - 1, gr_shift = __ffs(p.GR) - 1;
  bool failed = false;
  int last_phase = 0;                                // parity of the MMA commit a failed wait left behind
  int last_tile = 0;                                 // the tile of that MMA
  // x and w of tile t arrive by TMA in staging buffer t % kStages, issued by
  // thread 0 when tile t - kStages is finished (a tile's rows are read until
  // its rescoring)
  const int cx = h * p.d + j * C;                    // first channel of (h, j)
  const int x_off = cx & (Geo::XIN - 1), w_off = cx & 3;
  const int w_mode = p.w == nullptr ? 0 : (p.w_token_stride == 0 ? 1 : 2);   // none, shared, per token
  const uint32_t stage_bytes = Geo::XBOX + (w_mode == 2 ? Geo::WBOX : 0);
  auto issue_tile = [&](int t) {                     // thread 0
    const uint32_t bar = u32_smem(mbar + 1 + t % kStages);
    const uint32_t dst = u32_smem(tsm + Geo::STG_OFF + (t % kStages) * Geo::STAGE);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(stage_bytes)
                 : "memory");
    tma_load_3d(dst, &tmx, cx - x_off, t * kTcRows, 0, bar);
    if (w_mode == 2) tma_load_3d(dst + Geo::XBOX, &tmw, cx - w_off, t * kTcRows, 0, bar);
  };
  float* w_shared = reinterpret_cast<float*>(tsm + Geo::WSH_OFF);   // weights shared by all tokens (or all 1)
  if (tid < D) w_shared[tid] = w_mode == 1 ? p.w[(tid / C) * p.w_loop_stride + cx + tid % C] : 1.f;
  int issued = 0;                                    // tiles whose TMA thread 0 has issued
  if (tid == 0) {
    for (; issued < kStages && issued < n_tiles; ++issued) issue_tile(issued);
  }
  int64_t slot_nx = -1;                              // slot of this thread's token, one tile ahead
  auto fetch_slot = [&](int t) {
    const int n = t * kTcRows + row;
    // the slot's range check waits for the load, so it is made at use
    slot_nx = (t < n_tiles && n < p.n_tokens)
                  ? (p.slot_mapping != nullptr ? p.slot_mapping[n] : static_cast<int64_t>(n))
                  : -1;
  };
  fetch_slot(0);
  int tma_failed_tile = -1;                          // tile whose staging wait gave up
  uint16_t* my_list = list + warp * kListCap;
  float* my_dlist = dlist + warp * kListCap;

  // A of tile u from its staging buffer (waited for here); margin and
  // liveness of this thread's row come back for the tile's passes
  auto build_a = [&](int u, int64_t slot, float& margin, bool& live) -> bool {
    const unsigned char* stg = tsm + Geo::STG_OFF + (u % kStages) * Geo::STAGE;
    const bool staged = wait_parity(u32_smem(mbar + 1 + u % kStages), (u / kStages) & 1, kTcSpin);
    margin = 0.f;
    if (half == 0 && slot >= p.n_slots && p.status != nullptr) atomicOr(p.status, LOOPVQ_ENCODE_STATUS_BAD_SLOT);
    live = slot >= 0 && slot < p.n_slots;
    {
      // the row's scale and margin from scalars of the whole row; each half
      // then scales and writes only its own D columns of A
      float v[D];
      if (live) {
        float s[D], w[D];
        staged_row<C, G>(stg, row, x_off, w_off, w_mode, w_shared, s, w);
        float m1 = 0.f, m2 = 0.f, wss = 0.f, pu = 0.f, sws = 0.f, sw = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) {
          const float ws = w[i] * s[i];
          m1 = fmaxf(m1, fabsf(ws));
          m2 = fmaxf(m2, fabsf(w[i]));
          wss = fmaf(ws, s[i], wss);
          pu = fmaf(fabsf(ws), bm[i], pu);
          pu = fmaf(fabsf(w[i]), bm[D + i], pu);
          sws += fabsf(ws);
          sw += fabsf(w[i]);
          v[i] = half == 0 ? ws : w[i];
        }
        const int e1 = m1 > 0.f ? exp_of(m1) - beta1 : -100000;
        const int e2 = m2 > 0.f ? exp_of(m2) - beta2 : -100000;
        const int er = max(e1, e2);
        const int rho = max(rho_lo, min(rho_hi, er == -100000 ? 0 : kTopExp - er));
        const float f1 = pow2(rho - beta1), f2 = pow2(rho - beta2), fr = pow2(rho);
        const float fh = half == 0 ? f1 : f2;
#pragma unroll
        for (int i = 0; i < D; ++i) v[i] *= fh;
        margin = fr * fmaf(kMarginRel, pu, kMarginWss * wss) + kMarginAbs * (fmaf(f1, sws, f2 * sw) + q_abs);
        if (rho_lo > rho_hi) margin = INFINITY;    // no exact scaling: rescore everything
      } else {
#pragma unroll
        for (int i = 0; i < D; ++i) v[i] = 0.f;
      }
      write_row_f16_range<KP, D>(As + 0, row, v, 0, D, half * D);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    return staged;
  };
  auto issue_mma = [&]() {                           // thread 0, after the barrier that follows build_a
    {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int kk = 0; kk < KP / 16; ++kk) {
        const uint64_t ad = smem_desc(a_base + kk * 256, KP), bd = smem_desc(b_base + kk * 256, KP);
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
            ::"r"(tmem), "l"(ad), "l"(bd), "r"(kIdesc), "r"(kk) : "memory");
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                   ::"r"(mbar_a) : "memory");
    }
  };

  for (int t = 0; t < n_tiles; ++t) {
    const unsigned char* stg = tsm + Geo::STG_OFF + (t % kStages) * Geo::STAGE;
    const int64_t slot = slot_nx;
    float margin;
    bool live;
    const bool staged = build_a(t, slot, margin, live);
    if (__syncthreads_or(!staged)) {                 // CTA-uniform: a staging wait gave up
      failed = true;
      tma_failed_tile = t;
      break;
    }
    if (tid == 0) issue_mma();
    fetch_slot(t + 1);
    const bool done = wait_parity(mbar_a, static_cast<uint32_t>(t & 1), kTcSpin);
    if (__syncthreads_or(!done)) {                   // CTA-uniform: a thread gave up on this tile
      failed = true;
      last_phase = t & 1;
      last_tile = t;
      break;                                         // nothing of this tile or later is stored
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    // ---- the row's minimum over both halves --------------------------------------
    float m0 = INFINITY, mA = INFINITY, mB = INFINITY, mC = INFINITY;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t r[32];
      tmem_ld32_async(my_tmem + c0, r);
      tcgen05_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        m0 = min3f(m0, __uint_as_float(r[q]), __uint_as_float(r[q + 1]));
        mA = min3f(mA, __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]));
        mB = min3f(mB, __uint_as_float(r[q + 4]), __uint_as_float(r[q + 5]));
        mC = min3f(mC, __uint_as_float(r[q + 6]), __uint_as_float(r[q + 7]));
      }
    }
    pmin[half * kTcRows + row] = fminf(min3f(m0, mA, mB), mC);
    __syncthreads();
    const float smin = fminf(pmin[row], pmin[kTcRows + row]);
    float thr = smin + margin;
    if (!(fabsf(smin) < INFINITY) || !(margin < INFINITY)) thr = INFINITY;

    // ---- this half's columns within the margin -----------------------------------
    // thr - v has the sign of the exact difference (IEEE subtraction never
    // rounds a nonzero difference to zero), so its sign bit marks v > thr; a
    // NaN difference (positive on this GPU) keeps the column
    uint32_t cand[4];
    const uint64_t thr2 = pack_f32x2(thr, thr);
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t r[32];
      tmem_ld32_async(my_tmem + c0, r);
      tcgen05_wait_ld();
      uint32_t above = 0u;                           // column q's bit at 31 - q
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        uint32_t d0, d1;
        sub_f32x2(thr2, r[q], r[q + 1], d0, d1);
        above = __funnelshift_l(d0, above, 1);
        above = __funnelshift_l(d1, above, 1);
      }
      cand[c0 >> 5] = live ? ~__brev(above) : 0u;    // ascending columns within the margin
    }

    // ---- exact rescoring, shared by the warp's lanes ---------------------------------
    // The warp lists its candidates (row lane, column) lane by lane in
    // ascending columns, the lanes score the list round-robin, and each lane
    // takes the first minimum of its own entries.
    const int cnt = __popc(cand[0]) + __popc(cand[1]) + __popc(cand[2]) + __popc(cand[3]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int off = incl - cnt;
    float best = INFINITY;
    int best_e = 0;
    if (total <= kListCap) {
      int k = off;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t mm = cand[c];
        while (mm != 0u) {
          const int b = __ffs(mm) - 1;
          mm &= mm - 1u;
          my_list[k++] = static_cast<uint16_t>((lane << 8) | (c * 32 + b));
        }
      }
      __syncwarp();
      for (int i = lane; i < total; i += 32) {
        const int ent = my_list[i];
        float s2[D], w2[D];
        staged_row<C, G>(stg, ((warp & 3) << 5) | (ent >> 8), x_off, w_off, w_mode, w_shared, s2, w2);
        my_dlist[i] = direct_dist<C, G>(cbs, half * 128 + (ent & 255), s2, w2);
      }
      __syncwarp();
      for (int i = off; i < off + cnt; ++i) {
        const float dd = my_dlist[i];
        if (dd < best) {
          best = dd;
          best_e = half * 128 + (my_list[i] & 255);
        }
      }
    } else {                                         // a crowded warp: every lane its own rows
      float s2[D], w2[D];
      staged_row<C, G>(stg, row, x_off, w_off, w_mode, w_shared, s2, w2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t mm = cand[c];
        while (mm != 0u) {
          const int e = half * 128 + c * 32 + __ffs(mm) - 1;
          mm &= mm - 1u;
          const float dd = direct_dist<C, G>(cbs, e, s2, w2);
          if (dd < best) {
            best = dd;
            best_e = e;
          }
        }
      }
    }
    pbest[half * kTcRows + row] = make_float2(best, __int_as_float(best_e));
    __syncthreads();
    if (half == 0 && live) {                         // half 0 holds the smaller indices: it wins ties
      const float2 o = pbest[kTcRows + row];
      const int e = o.x < best ? __float_as_int(o.y) : best_e;
      if (slot_u32)
        store_index_u32(p, static_cast<uint32_t>(slot), j, h, e, pg_shift, gr_shift);
      else
        store_index(p, slot, j, h, e);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();                                 // TMEM, A and the staging buffer of tile t free
    if (tid == 0 && issued < n_tiles) issue_tile(issued++);
  }
  if (failed) {
    // the abandoned tile's MMAs still write TMEM and the issued TMA boxes
    // still land in shared memory: wait (bounded) for both before TMEM is
    // freed and the CTA exits, and report the failure
    if (tid == 0) {
      bool done = true;
      if (tma_failed_tile < 0) done = wait_parity(mbar_a, static_cast<uint32_t>(last_phase), kTcDrainSpin);
      // tiles issued but not consumed: the failed staging tile, or the one after the failed MMA
      for (int u = tma_failed_tile >= 0 ? tma_failed_tile : last_tile + 1; u < issued; ++u)
        done = wait_parity(u32_smem(mbar + 1 + u % kStages), (u / kStages) & 1, kTcDrainSpin) && done;
      if (p.status != nullptr)
        atomicOr(p.status, done ? LOOPVQ_ENCODE_STATUS_TIMEOUT
                                : (LOOPVQ_ENCODE_STATUS_TIMEOUT | LOOPVQ_ENCODE_STATUS_UNDRAINED));
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
  }
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u) : "memory");
  }
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A 3-d map over [g][n_tokens][H*d] (innermost last) with a box of
// `box_inner` channels x 128 tokens x g loop steps; strides in elements.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, int channels,
              int n_tokens, int g, int64_t token_stride, int64_t loop_stride, int box_inner) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(channels), static_cast<cuuint64_t>(n_tokens),
                              static_cast<cuuint64_t>(g)};
  const int64_t ls = loop_stride > 0 ? loop_stride * esize : 16;   // unused when g == 1
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(token_stride * esize), static_cast<cuuint64_t>(ls)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(kTcRows),
                             static_cast<cuuint32_t>(g)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int C, int G>
loopvq_status launch_tc(const EncodeParams& p, int J, int H, cudaStream_t st) {
  using Geo = TcGeo<C, G>;
  // at least 80 KB, so that at most two CTAs (2 x 256 TMEM columns) share an SM
  constexpr int smem = Geo::SMEM > 80 * 1024 ? Geo::SMEM : 80 * 1024;
  static_assert(smem <= 227 * 1024, "encoder shared memory above 227 KB");
  // TMA wants 16-byte strides; a token stride of 0 (one x row for all
  // tokens) is not a tensor either
  if (p.x_token_stride <= 0 || (p.x_token_stride * 2) % 16 != 0 || (p.x_loop_stride * 2) % 16 != 0 ||
      (G > 1 && p.x_loop_stride <= 0))
    return LOOPVQ_ERR_UNSUPPORTED;
  const bool w_tok = p.w != nullptr && p.w_token_stride != 0;
  if (w_tok && ((p.w_token_stride * 4) % 16 != 0 || (p.w_loop_stride * 4) % 16 != 0 ||
                (G > 1 && p.w_loop_stride <= 0)))
    return LOOPVQ_ERR_UNSUPPORTED;
  CUtensorMap tmx, tmw;
  if (!make_map(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, H * p.d, p.n_tokens, G, p.x_token_stride,
                p.x_loop_stride, Geo::XIN))
    return LOOPVQ_ERR_UNSUPPORTED;
  if (w_tok) {
    if (!make_map(&tmw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.w, H * p.d, p.n_tokens, G, p.w_token_stride,
                  p.w_loop_stride, Geo::WIN))
      return LOOPVQ_ERR_UNSUPPORTED;
  } else {
    tmw = tmx;                                       // not read
  }
  if (cudaFuncSetAttribute(encode_tc_kernel<C, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  encode_tc_kernel<C, G><<<dim3(J, H), kTcThreads, smem, st>>>(p, tmx, tmw);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

}  // namespace

int* encode_status_word() {
  static std::mutex mu;
  static int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_encode_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(a);
  }
  return addr[dev];
}

loopvq_status encode_status(int* flags, int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_encode_status, sizeof(int)) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_encode_status, &zero, sizeof(int)) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  }
  *flags = v;
  return LOOPVQ_OK;
}

bool encode_tc_supported(int c, int g) {
  const int d = c * g;
  return d == 8 || d == 16 || d == 32;
}

loopvq_status launch_encode_tc(const EncodeParams& p, int c, int g, int J, int H, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (c * 100 + g) {
    case 404: return launch_tc<4, 4>(p, J, H, st);
    case 804: return launch_tc<8, 4>(p, J, H, st);
    case 204: return launch_tc<2, 4>(p, J, H, st);
    case 402: return launch_tc<4, 2>(p, J, H, st);
    case 802: return launch_tc<8, 2>(p, J, H, st);
    case 208: return launch_tc<2, 8>(p, J, H, st);
    case 408: return launch_tc<4, 8>(p, J, H, st);
    case 801: return launch_tc<8, 1>(p, J, H, st);
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace loopvq
