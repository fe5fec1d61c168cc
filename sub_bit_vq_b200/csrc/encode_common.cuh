// Pieces shared by the encoder kernels (direct form and tensor-core form).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "internal.h"
#include "loopvq.h"

namespace loopvq {

struct EncodeParams {
  const uint16_t* x;            // bf16 bits
  int64_t x_loop_stride, x_token_stride;
  const float* w;               // nullable
  int64_t w_loop_stride, w_token_stride;
  const float* cb;              // codebooks at (layer, head 0, gamma, kv, tau 0)
  int64_t cb_stride_head, cb_stride_loop;
  const int64_t* slot_mapping;  // null: token n is slot n
  uint8_t* pool;                // pool at (layer, head 0, gamma)
  uint8_t* assign;              // or null: indices [H][J][n_tokens] instead of the pool
  int64_t pool_stride_head, page_bytes, plane_bytes;
  int64_t n_slots;              // n_pages * Pg
  int* status;                  // the device's encoder status word
  int n_tokens, d, Pg, J, LB, GR, kv;
};

// Device address of this device's encoder status word (looked up once per
// device with that device current); null if the runtime fails.
int* encode_status_word();

// Slot of token n: its pool slot, or n itself when indices go to `assign`.
// A slot at or past n_slots is not written and flags the encoder status word
// (a negative one only means "skip this token").
__device__ __forceinline__ int64_t token_slot(const EncodeParams& p, int n) {
  const int64_t s = p.slot_mapping != nullptr ? p.slot_mapping[n] : static_cast<int64_t>(n);
  if (s >= p.n_slots && p.status != nullptr) atomicOr(p.status, LOOPVQ_ENCODE_STATUS_BAD_SLOT);
  return s;
}

// Writes index `e` of (slot, group j, head h) to its byte in the pool, or to
// assign[h][j][slot].
__device__ __forceinline__ void store_index(const EncodeParams& p, int64_t slot, int j, int h, int e) {
  if (p.assign != nullptr) {
    p.assign[(static_cast<int64_t>(h) * p.J + j) * p.n_tokens + slot] = static_cast<uint8_t>(e);
    return;
  }
  const int64_t page = slot / p.Pg;
  const int sl = static_cast<int>(slot % p.Pg);
  // both planes: rotated slot rows in granules
  const int blk = sl / p.LB, rot = sl % p.LB;
  int pos = j - rot % p.J;
  if (pos < 0) pos += p.J;
  const int64_t off = static_cast<int64_t>(blk) * p.LB * p.J + (pos / p.GR) * p.LB * p.GR +
                      rot * p.GR + pos % p.GR;
  p.pool[h * p.pool_stride_head + page * p.page_bytes + p.kv * p.plane_bytes + off] =
      static_cast<uint8_t>(e);
}

// Loads token n's sub-vector of (group j, head h) and its weights (1 when
// no weights are given).
template <int C, int G>
__device__ __forceinline__ void load_subvector(const EncodeParams& p, int n, int j, int h,
                                               float (&s)[C * G], float (&w)[C * G]) {
#pragma unroll
  for (int tau = 0; tau < G; ++tau) {
    const uint16_t* xr = p.x + tau * p.x_loop_stride + n * p.x_token_stride +
                         static_cast<int64_t>(h) * p.d + j * C;
#pragma unroll
    for (int ch = 0; ch < C; ++ch) s[tau * C + ch] = bf16_bits_to_float(xr[ch]);
    if (p.w != nullptr) {
      const float* wr = p.w + tau * p.w_loop_stride + n * p.w_token_stride +
                        static_cast<int64_t>(h) * p.d + j * C;
#pragma unroll
      for (int ch = 0; ch < C; ++ch) w[tau * C + ch] = wr[ch];
    } else {
#pragma unroll
      for (int ch = 0; ch < C; ++ch) w[tau * C + ch] = 1.f;
    }
  }
}

// Kernel parameters of an encode (or k-means) call; see encode.cu.
EncodeParams encode_params(const EncodeArgs& a);

// Launches the tensor-core encoder (D = c*g in {8, 16, 32}); see encode_tc.cu.
bool encode_tc_supported(int c, int g);
loopvq_status launch_encode_tc(const EncodeParams& p, int c, int g, int J, int H, void* stream);

}  // namespace loopvq
