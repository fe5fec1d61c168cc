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
// centroids in shared memory and walks the tokens in tiles of 128. For each
// tile every thread writes its token's row of A, one thread issues the
// tcgen05.mma chain that leaves S (128 x 256, fp32) in tensor memory, and
// each thread reads its row back with tcgen05.ld. Operands are bf16 split
// into high and low parts, a.b ~= a_hi.b_hi + a_hi.b_lo + a_lo.b_hi (K' =
// 6D): each S_e is off by at most about 2^-14.3 * sum_i |a_i b_ei| (the
// dropped lo*lo terms, the split residuals, fp32 accumulation over K'), so
// twice that, plus the direct form's own rounding, stays below
//     margin = 2^-12 * (sum_i |a_i| max_e |b_ei| + sum_i w_i s_i^2).
// Every centroid whose S_e is within the margin of the row's minimum is
// rescored with the float32 direct form and term order of encode_kernel;
// the first minimum of those (smallest index on equal distances) is the
// index encode_kernel chooses.
//
// Shared operands use the K-major layout without swizzle: 8-row x 16-byte
// core matrices, the two 8-element halves of a 16-wide K step 128 bytes
// apart (leading byte offset) and consecutive 8-row groups KP*16 bytes
// apart (stride byte offset).

#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "encode_common.cuh"

namespace loopvq {

// Encoder status word of this device (flag bits, LOOPVQ_ENCODE_STATUS_*),
// set by the kernels and read (and cleared) by loopvq_encode_status.
__device__ int g_encode_status = 0;

namespace {

constexpr int kTcRows = 128;              // tokens per tile (MMA M)
constexpr int kTcThreads = 128;           // one thread per tile row
#ifndef LOOPVQ_TC_SPIN
#define LOOPVQ_TC_SPIN (1 << 20)
#endif
constexpr int kTcSpin = LOOPVQ_TC_SPIN;   // bounded mbarrier wait (tries) for a tile's MMA
constexpr int kTcDrainSpin = 1 << 24;     // bounded wait for the last MMA before TMEM is freed

template <int C, int G>
struct TcGeo {
  static constexpr int D = C * G;
  static constexpr int K2 = 2 * D;                      // [w*s, w] . [-2C, C*C]
  static constexpr int KP = ((3 * K2 + 15) / 16) * 16;  // split operands, padded to the MMA K step
  static constexpr int A_BYTES = kTcRows * KP * 2;
  static constexpr int B_BYTES = kE * KP * 2;
  static constexpr int CB_FLOATS = G * kE * C;          // fp32 codebook [tau][E][c] for rescoring
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + A_BYTES;
  static constexpr int CB_OFF = B_OFF + B_BYTES;
  static constexpr int BMAX_OFF = CB_OFF + CB_FLOATS * 4;   // [K2] uint (float bits)
  static constexpr int MBAR_OFF = (BMAX_OFF + K2 * 4 + 7) & ~7;
  static constexpr int TMEM_OFF = MBAR_OFF + 8;
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

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major,
// M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ uint32_t u32_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Writes 8 bf16 values (one 16-byte core-matrix row) at byte offset `off`.
__device__ __forceinline__ void st_row8(unsigned char* base, uint32_t off, const __nv_bfloat16 (&v)[8]) {
  uint4 u;
  u.x = static_cast<uint32_t>(__bfloat16_as_ushort(v[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(v[1])) << 16);
  u.y = static_cast<uint32_t>(__bfloat16_as_ushort(v[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(v[3])) << 16);
  u.z = static_cast<uint32_t>(__bfloat16_as_ushort(v[4])) | (static_cast<uint32_t>(__bfloat16_as_ushort(v[5])) << 16);
  u.w = static_cast<uint32_t>(__bfloat16_as_ushort(v[6])) | (static_cast<uint32_t>(__bfloat16_as_ushort(v[7])) << 16);
  *reinterpret_cast<uint4*>(base + off) = u;
}

// Row r of a split operand: v holds K2 values; the row is
// [hi(v), second(v), third(v), 0...] where the thirds are chosen by the caller.
template <int KP, int K2>
__device__ __forceinline__ void write_split_row(unsigned char* base, int r, const float (&v)[K2],
                                                bool a_side) {
  // element k of the row: part = k / K2 (0, 1, 2), i = k % K2
  // A side: [hi, hi, lo]; B side: [hi, lo, hi]
#pragma unroll
  for (int k0 = 0; k0 < KP; k0 += 8) {
    __nv_bfloat16 row[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int k = k0 + t;
      if (k < 3 * K2) {
        const int part = k / K2, i = k % K2;
        __nv_bfloat16 hi, lo;
        split_bf16(v[i], hi, lo);
        const bool take_lo = a_side ? (part == 2) : (part == 1);
        row[t] = take_lo ? lo : hi;
      } else {
        row[t] = __float2bfloat16_rn(0.f);
      }
    }
    st_row8(base, op_off<KP>(r, k0), row);
  }
}

template <int C, int G>
__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(const EncodeParams p) {
  using Geo = TcGeo<C, G>;
  constexpr int D = Geo::D, K2 = Geo::K2, KP = Geo::KP;
  extern __shared__ __align__(128) unsigned char tsm[];
  unsigned char* As = tsm + Geo::A_OFF;
  unsigned char* Bs = tsm + Geo::B_OFF;
  float* cbs = reinterpret_cast<float*>(tsm + Geo::CB_OFF);
  unsigned int* bmax = reinterpret_cast<unsigned int*>(tsm + Geo::BMAX_OFF);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(tsm + Geo::MBAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tsm + Geo::TMEM_OFF);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int j = blockIdx.x, h = blockIdx.y;

  // ---- codebook of (j, h): fp32 copy for rescoring, split B operand -------
  const float* cb = p.cb + h * p.cb_stride_head + static_cast<int64_t>(j) * kE * C;
  for (int i = tid * 4; i < G * kE * C; i += kTcThreads * 4) {
    const int tau = i / (kE * C), r = i % (kE * C);
    cp_async16(cbs + i, cb + tau * p.cb_stride_loop + r);
  }
  if (tid < K2) bmax[tid] = 0u;
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(u32_smem(mbar)), "r"(1u) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {                                   // 256 TMEM columns: one fp32 per centroid
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(u32_smem(tmem_slot)), "r"(256u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  cp_async_wait_all();
  __syncthreads();
  for (int e = tid; e < kE; e += kTcThreads) {
    float b[K2];
#pragma unroll
    for (int tau = 0; tau < G; ++tau) {
#pragma unroll
      for (int ch = 0; ch < C; ++ch) {
        const float c = cbs[(tau * kE + e) * C + ch];
        b[tau * C + ch] = -2.f * c;
        b[D + tau * C + ch] = c * c;
      }
    }
#pragma unroll
    for (int i = 0; i < K2; ++i) atomicMax(bmax + i, __float_as_uint(fabsf(b[i])));
    write_split_row<KP, K2>(Bs, e, b, false);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // B visible to the tensor cores
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  float bm[K2];
#pragma unroll
  for (int i = 0; i < K2; ++i) bm[i] = __uint_as_float(bmax[i]);

  const uint32_t a_base = u32_smem(As), b_base = u32_smem(Bs), mbar_a = u32_smem(mbar);
  const uint32_t my_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int n_tiles = (p.n_tokens + kTcRows - 1) / kTcRows;
  bool failed = false;
  int last_phase = 0;                                // parity of the MMA commit a failed wait left behind
  // this thread's token of the next tile, requested one tile ahead
  float s_nx[D], w_nx[D];
  int64_t slot_nx = -1;
  auto fetch = [&](int t) {
    const int n = t * kTcRows + tid;
    slot_nx = (t < n_tiles && n < p.n_tokens) ? token_slot(p, n) : -1;
    if (slot_nx >= 0 && slot_nx < p.n_slots) load_subvector<C, G>(p, n, j, h, s_nx, w_nx);
  };
  fetch(0);
  for (int t = 0; t < n_tiles; ++t) {
    // ---- this thread's row of A ----------------------------------------------
    const int64_t slot = slot_nx;
    float s[D], w[D];
#pragma unroll
    for (int i = 0; i < D; ++i) {
      s[i] = s_nx[i];
      w[i] = w_nx[i];
    }
    float a[K2];
    float margin = 0.f;
    const bool live = slot >= 0 && slot < p.n_slots;
    if (live) {
      float ms = 0.f, wss = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) {
        a[i] = w[i] * s[i];
        a[D + i] = w[i];
        wss = fmaf(w[i] * s[i], s[i], wss);
      }
#pragma unroll
      for (int i = 0; i < K2; ++i) ms = fmaf(fabsf(a[i]), bm[i], ms);
      margin = ldexpf(ms + wss, -12);
    } else {
#pragma unroll
      for (int i = 0; i < K2; ++i) a[i] = 0.f;
    }
    write_split_row<KP, K2>(As, tid, a, true);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();

    // ---- S = A . B^T into tensor memory ----------------------------------------
    if (tid == 0) {
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
    fetch(t + 1);                                    // lands while the tensor cores work
    bool done = false;
    for (int it = 0; it < kTcSpin && !done; ++it) {
      uint32_t ok;
      asm volatile(
          "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n"
          " selp.u32 %0, 1, 0, P;\n}\n"
          : "=r"(ok) : "r"(mbar_a), "r"(static_cast<uint32_t>(t & 1)) : "memory");
      done = ok != 0u;
    }
    if (__syncthreads_or(!done)) {                   // CTA-uniform: a thread gave up on this tile
      failed = true;
      last_phase = t & 1;
      break;                                         // nothing of this tile or later is stored
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    // ---- this row's minimum, then the exact rescore within the margin ----------
    float smin = INFINITY;
#pragma unroll 1
    for (int c0 = 0; c0 < kE; c0 += 32) {
      uint32_t r[32];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
          "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
          "%30, %31}, [%32];"
          : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
            "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
            "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
            "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
            "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
          : "r"(my_tmem + c0));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int q = 0; q < 32; ++q) smin = fminf(smin, __uint_as_float(r[q]));
    }
    const float thr = smin + margin;
    float best = INFINITY;
    int best_e = 0;
#pragma unroll 1
    for (int c0 = 0; c0 < kE; c0 += 32) {
      uint32_t r[32];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
          "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
          "%30, %31}, [%32];"
          : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
            "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
            "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
            "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
            "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
          : "r"(my_tmem + c0));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (!live) continue;
      uint32_t cand = 0u;                            // columns within the margin, ascending
#pragma unroll
      for (int q = 0; q < 32; ++q) cand |= (__uint_as_float(r[q]) <= thr ? 1u : 0u) << q;
      while (cand != 0u) {
        const int e = c0 + __ffs(cand) - 1;
        cand &= cand - 1u;
        float dist = 0.f;                            // encode_kernel's terms, in its order
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
    }
    if (live) store_index(p, slot, j, h, best_e);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();                                 // TMEM read, A free for the next tile
  }
  if (failed) {
    // the abandoned tile's MMAs still write TMEM: wait (bounded) for their
    // commit before TMEM is freed, and report the failure
    if (tid == 0) {
      bool done = false;
      for (int it = 0; it < kTcDrainSpin && !done; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n"
            " selp.u32 %0, 1, 0, P;\n}\n"
            : "=r"(ok) : "r"(mbar_a), "r"(static_cast<uint32_t>(last_phase)) : "memory");
        done = ok != 0u;
      }
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

template <int C, int G>
loopvq_status launch_tc(const EncodeParams& p, int J, int H, cudaStream_t st) {
  // at least 80 KB, so that at most two CTAs (2 x 256 TMEM columns) share an SM
  constexpr int smem = TcGeo<C, G>::SMEM > 80 * 1024 ? TcGeo<C, G>::SMEM : 80 * 1024;
  static_assert(smem <= 227 * 1024, "encoder shared memory above 227 KB");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (cudaFuncSetAttribute(encode_tc_kernel<C, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  encode_tc_kernel<C, G><<<dim3(J, H), kTcThreads, smem, st>>>(p);
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
