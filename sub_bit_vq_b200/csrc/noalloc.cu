// Decode attention for callers that cannot hand the library a workspace.
//
// The split-K partials that loopvq_decode_attn keeps in caller-provided
// scratch live here in one file-scope device array instead. Every device
// that loads the library holds this array until the process exits; every
// call on a device shares it.

#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "loopvq.h"

namespace loopvq {
namespace {

constexpr size_t kStaticScratchBytes = LOOPVQ_STATIC_SCRATCH_BYTES;   // 32 MiB per device

__device__ __align__(256) float g_decode_scratch[kStaticScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and remembered.
loopvq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return LOOPVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return LOOPVQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LOOPVQ_OK;
}

}  // namespace
}  // namespace loopvq

extern "C" loopvq_status loopvq_decode_attn_noalloc(
    const loopvq_config* cfg, int layer, int loop_step, int batch, int max_seq_len, const void* q,
    const uint8_t* pool, const float* codebooks, const int32_t* block_table,
    const int32_t* seq_lens, const void* win_k, const void* win_v, float sm_scale, int out_dtype,
    void* out, float* lse, void* stream) {
  const size_t need = loopvq_decode_workspace_bytes(cfg, batch, max_seq_len);
  if (need > loopvq::kStaticScratchBytes) return LOOPVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const loopvq_status st = loopvq::scratch_address(&scratch);
  if (st != LOOPVQ_OK) return st;
  // The partials need no initial contents: every split writes its record.
  return loopvq_decode_attn(cfg, layer, loop_step, batch, max_seq_len, q, pool, codebooks,
                            block_table, seq_lens, win_k, win_v, sm_scale, out_dtype, out, lse,
                            scratch, loopvq::kStaticScratchBytes, stream);
}
