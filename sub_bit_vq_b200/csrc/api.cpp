// extern "C" entry points of libloopvq: argument checks, layout, planning.
// Every check runs on the host before any launch.

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstring>

#include "internal.h"
#include "loopvq.h"

namespace loopvq {

namespace {

constexpr int kMaxCtas = 4096;    // upper bound on decode CTAs the planner targets
constexpr int kCentroids = 256;   // 8-bit index

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

int pages_for(const Geometry& g, int seq_len) {
  const int n_vq = seq_len > g.W ? seq_len - g.W : 0;
  return (n_vq + g.Pg - 1) / g.Pg;
}

}  // namespace

loopvq_status make_geometry(const loopvq_config* cfg, Geometry* geo) {
  if (cfg == nullptr || geo == nullptr) return LOOPVQ_ERR_INVALID_ARG;
  if (cfg->struct_size != sizeof(loopvq_config)) return LOOPVQ_ERR_INVALID_ARG;
  Geometry g{};
  g.L = cfg->n_layers;
  g.Hkv = cfg->n_kv_heads;
  g.Hq = cfg->n_q_heads;
  g.d = cfg->head_dim;
  g.T = cfg->n_loops;
  g.g = cfg->loop_group;
  g.c = cfg->chan_group;
  g.E = cfg->n_centroids;
  g.P = cfg->prefix_tokens;
  g.R = cfg->recent_tokens;
  g.Pg = cfg->page_tokens;
  g.n_pages = cfg->n_pages;
  g.max_batch = cfg->max_batch;
  g.max_pages_per_seq = cfg->max_pages_per_seq;
  if (g.L <= 0 || g.Hkv <= 0 || g.Hq <= 0 || g.d <= 0 || g.T <= 0 || g.g <= 0 || g.c <= 0 ||
      g.E <= 0 || g.Pg <= 0 || g.n_pages <= 0 || g.max_batch <= 0 ||
      g.max_pages_per_seq <= 0 || g.P < 0 || g.R < 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (g.d % g.c != 0 || g.T % g.g != 0 || g.Hq % g.Hkv != 0) return LOOPVQ_ERR_INVALID_ARG;
  g.J = g.d / g.c;
  g.D = g.c * g.g;
  g.G = g.T / g.g;
  g.W = g.P + g.R;
  // What the kernels implement.
  if (g.E != kCentroids) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.d % 8 != 0 || g.d > 256) return LOOPVQ_ERR_UNSUPPORTED;
  if (!(g.c == 1 || g.c == 2 || g.c == 4 || g.c == 8 || g.c == 16)) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.J % 4 != 0 || g.J > 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.D > 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.W > 256) return LOOPVQ_ERR_UNSUPPORTED;
  g.GR = (g.J % 16 == 0) ? 16 : (g.J % 8 == 0) ? 8 : 4;
  g.LB = (32 / g.J) * g.J;
  if (g.Pg % g.LB != 0 || g.Pg % 16 != 0 || g.Pg > 256) return LOOPVQ_ERR_UNSUPPORTED;
  if (((g.Pg / g.LB) & (g.Pg / g.LB - 1)) != 0) return LOOPVQ_ERR_UNSUPPORTED;   // blocks per page: 2^k
  g.plane_bytes = static_cast<int64_t>(g.Pg) * g.J;
  g.page_bytes = 2 * g.plane_bytes;
  if (!mul_ok(g.page_bytes, g.n_pages, &g.pool_stride_group)) return LOOPVQ_ERR_INVALID_ARG;
  if (!mul_ok(g.pool_stride_group, g.G, &g.pool_stride_head)) return LOOPVQ_ERR_INVALID_ARG;
  if (!mul_ok(g.pool_stride_head, g.Hkv, &g.pool_stride_layer)) return LOOPVQ_ERR_INVALID_ARG;
  int64_t pool_bytes;
  if (!mul_ok(g.pool_stride_layer, g.L, &pool_bytes)) return LOOPVQ_ERR_INVALID_ARG;
  g.cb_stride_loop = static_cast<int64_t>(g.J) * g.E * g.c;
  g.cb_stride_kv = g.cb_stride_loop * g.g;
  g.cb_stride_group = 2 * g.cb_stride_kv;
  g.cb_stride_head = g.cb_stride_group * g.G;
  g.cb_stride_layer = g.cb_stride_head * g.Hkv;
  int64_t cb_floats;
  if (!mul_ok(g.cb_stride_layer, g.L, &cb_floats)) return LOOPVQ_ERR_INVALID_ARG;
  *geo = g;
  return LOOPVQ_OK;
}

int max_decode_splits(int pairs, int pages) {
  if (pairs <= 0) return 1;
  int s = (kMaxCtas + pairs - 1) / pairs;
  if (s > pages) s = pages;
  return s < 1 ? 1 : s;
}

int current_sm_count(loopvq_status* err) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *err = LOOPVQ_ERR_CUDA;
    return 0;
  }
  if (dev >= 0 && dev < 64) {
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    *err = LOOPVQ_ERR_CUDA;
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace loopvq

using loopvq::Geometry;

extern "C" {

const char* loopvq_status_string(loopvq_status s) {
  switch (s) {
    case LOOPVQ_OK: return "ok";
    case LOOPVQ_ERR_INVALID_ARG: return "invalid argument";
    case LOOPVQ_ERR_UNSUPPORTED: return "unsupported shape";
    case LOOPVQ_ERR_WORKSPACE: return "workspace too small";
    case LOOPVQ_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

loopvq_status loopvq_cache_layout(const loopvq_config* cfg, loopvq_layout* out) {
  if (out == nullptr) return LOOPVQ_ERR_INVALID_ARG;
  Geometry g;
  loopvq_status st = loopvq::make_geometry(cfg, &g);
  if (st != LOOPVQ_OK) return st;
  loopvq_layout L;
  std::memset(&L, 0, sizeof(L));
  L.struct_size = sizeof(loopvq_layout);
  L.J = g.J;
  L.D = g.D;
  L.n_loop_groups = g.G;
  L.granule = g.GR;
  L.rot_block = g.LB;
  L.window_tokens = g.W;
  L.plane_bytes = static_cast<size_t>(g.plane_bytes);
  L.page_bytes = static_cast<size_t>(g.page_bytes);
  L.pool_bytes = static_cast<size_t>(g.pool_stride_layer) * g.L;
  L.pool_stride_layer = g.pool_stride_layer;
  L.pool_stride_head = g.pool_stride_head;
  L.pool_stride_group = g.pool_stride_group;
  L.codebook_bytes = static_cast<size_t>(g.cb_stride_layer) * g.L * sizeof(float);
  L.cb_stride_layer = g.cb_stride_layer;
  L.cb_stride_head = g.cb_stride_head;
  L.cb_stride_group = g.cb_stride_group;
  L.cb_stride_kv = g.cb_stride_kv;
  L.cb_stride_loop = g.cb_stride_loop;
  L.window_bytes = static_cast<size_t>(g.max_batch) * g.Hkv * g.W * g.d * 2;
  L.bits_per_element = 8.0 / (static_cast<double>(g.c) * g.g);
  *out = L;
  return LOOPVQ_OK;
}

size_t loopvq_decode_workspace_bytes(const loopvq_config* cfg, int batch, int max_seq_len) {
  Geometry g;
  if (loopvq::make_geometry(cfg, &g) != LOOPVQ_OK || batch <= 0 || max_seq_len < 0) return 0;
  // record slots pair + cta of the (pair, streaming CTA) segments never
  // collide, so pairs + CTAs slots suffice
  return loopvq::decode_workspace_bytes(batch * g.Hq, g.J, g.d);
}

loopvq_status loopvq_encode(const loopvq_config* cfg, int layer, int loop_group_idx, int kv,
                            int n_tokens, const void* x, int64_t x_loop_stride,
                            int64_t x_token_stride, const float* w, int64_t w_loop_stride,
                            int64_t w_token_stride, const float* codebooks,
                            const int64_t* slot_mapping, uint8_t* pool, void* stream) {
  Geometry g;
  loopvq_status st = loopvq::make_geometry(cfg, &g);
  if (st != LOOPVQ_OK) return st;
  if (layer < 0 || layer >= g.L || loop_group_idx < 0 || loop_group_idx >= g.G) return LOOPVQ_ERR_INVALID_ARG;
  if (kv != 0 && kv != 1) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  if (x == nullptr || codebooks == nullptr || slot_mapping == nullptr || pool == nullptr)
    return LOOPVQ_ERR_INVALID_ARG;
  // x rows (c bf16 of one group) are read as whole rows of d values.
  if (!loopvq::aligned(x, 16) || x_loop_stride < 0 || x_token_stride < 0 ||
      (x_loop_stride % 8) != 0 || (x_token_stride % 8) != 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (w != nullptr && (!loopvq::aligned(w, 16) || w_loop_stride < 0 || w_token_stride < 0 ||
                       (w_loop_stride % 4) != 0 || (w_token_stride % 4) != 0))
    return LOOPVQ_ERR_INVALID_ARG;
  if (!loopvq::aligned(codebooks, 16) || !loopvq::aligned(slot_mapping, 8))
    return LOOPVQ_ERR_INVALID_ARG;
  loopvq::EncodeArgs a{&g, layer, loop_group_idx, kv, n_tokens, x, x_loop_stride, x_token_stride,
                       w, w_loop_stride, w_token_stride, codebooks, slot_mapping, pool, nullptr, stream};
  return loopvq::launch_encode(a);
}

loopvq_status loopvq_encode_status(int* flags, int clear) {
  if (flags == nullptr) return LOOPVQ_ERR_INVALID_ARG;
  return loopvq::encode_status(flags, clear);
}

loopvq_status loopvq_encode_evict(const loopvq_config* cfg, int n_tokens, const void* x,
                                  const float* codebooks, const int64_t* slot_mapping,
                                  uint8_t* pool, void* stream) {
  Geometry g;
  loopvq_status st = loopvq::make_geometry(cfg, &g);
  if (st != LOOPVQ_OK) return st;
  if (n_tokens < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  if (n_tokens > 64) return LOOPVQ_ERR_UNSUPPORTED;
  if (x == nullptr || codebooks == nullptr || slot_mapping == nullptr || pool == nullptr)
    return LOOPVQ_ERR_INVALID_ARG;
  if (!loopvq::aligned(x, 16) || !loopvq::aligned(codebooks, 16) || !loopvq::aligned(slot_mapping, 8))
    return LOOPVQ_ERR_INVALID_ARG;
  const int64_t n_tok = n_tokens;
  loopvq::EncodeArgs a{&g, 0, 0, 0, n_tokens, x, n_tok * g.Hkv * g.d, static_cast<int64_t>(g.Hkv) * g.d,
                       nullptr, 0, 0, codebooks, slot_mapping, pool, nullptr, stream};
  return loopvq::launch_encode_evict(a);
}

size_t loopvq_kmeans_assign_bytes(const loopvq_config* cfg, int n_tokens) {
  Geometry g;
  if (loopvq::make_geometry(cfg, &g) != LOOPVQ_OK || n_tokens < 0) return 0;
  return static_cast<size_t>(g.Hkv) * g.J * static_cast<size_t>(n_tokens);
}

loopvq_status loopvq_kmeans_step(const loopvq_config* cfg, int layer, int loop_group_idx, int kv,
                                 int n_tokens, const void* x, int64_t x_loop_stride,
                                 int64_t x_token_stride, const float* w, int64_t w_loop_stride,
                                 int64_t w_token_stride, float* codebooks, uint8_t* assign,
                                 size_t assign_bytes, void* stream) {
  Geometry g;
  loopvq_status st = loopvq::make_geometry(cfg, &g);
  if (st != LOOPVQ_OK) return st;
  if (layer < 0 || layer >= g.L || loop_group_idx < 0 || loop_group_idx >= g.G) return LOOPVQ_ERR_INVALID_ARG;
  if (kv != 0 && kv != 1) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  if (x == nullptr || codebooks == nullptr || assign == nullptr) return LOOPVQ_ERR_INVALID_ARG;
  if (!loopvq::aligned(x, 16) || x_loop_stride < 0 || x_token_stride < 0 ||
      (x_loop_stride % 8) != 0 || (x_token_stride % 8) != 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (w != nullptr && (!loopvq::aligned(w, 16) || w_loop_stride < 0 || w_token_stride < 0 ||
                       (w_loop_stride % 4) != 0 || (w_token_stride % 4) != 0))
    return LOOPVQ_ERR_INVALID_ARG;
  if (!loopvq::aligned(codebooks, 16)) return LOOPVQ_ERR_INVALID_ARG;
  if (assign_bytes < loopvq_kmeans_assign_bytes(cfg, n_tokens)) return LOOPVQ_ERR_WORKSPACE;
  loopvq::EncodeArgs a{&g, layer, loop_group_idx, kv, n_tokens, x, x_loop_stride, x_token_stride,
                       w, w_loop_stride, w_token_stride, codebooks, nullptr, nullptr, assign, stream};
  st = loopvq::launch_encode(a);                       // assignment under the current codebooks
  if (st != LOOPVQ_OK) return st;
  return loopvq::launch_kmeans_update(a, codebooks);   // weighted means, in place
}

}  // extern "C"

namespace loopvq {
namespace {

// Checks and launches a decode of n_queries queries per sequence (decode:
// 1; prefill over the cache: a chunk of queries).
loopvq_status decode_common(const loopvq_config* cfg, int layer, int loop_step, int batch,
                            int n_queries, int max_seq_len, const void* q, const uint8_t* pool,
                            const float* codebooks, const int32_t* block_table,
                            const int32_t* seq_lens, const void* win_k, const void* win_v,
                            float sm_scale, int out_dtype, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Geometry g;
  loopvq_status st = make_geometry(cfg, &g);
  if (st != LOOPVQ_OK) return st;
  if (layer < 0 || layer >= g.L || loop_step < 0 || loop_step >= g.T) return LOOPVQ_ERR_INVALID_ARG;
  if (batch <= 0 || batch > g.max_batch || max_seq_len < 0 || n_queries <= 0) return LOOPVQ_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * n_queries * g.Hq > (1ll << 30)) return LOOPVQ_ERR_UNSUPPORTED;
  if (out_dtype != LOOPVQ_DTYPE_BF16 && out_dtype != LOOPVQ_DTYPE_F32) return LOOPVQ_ERR_INVALID_ARG;
  if (!(sm_scale > 0.0f) || sm_scale > 1e30f) return LOOPVQ_ERR_INVALID_ARG;
  if (q == nullptr || pool == nullptr || codebooks == nullptr || block_table == nullptr ||
      seq_lens == nullptr || out == nullptr || workspace == nullptr)
    return LOOPVQ_ERR_INVALID_ARG;
  if (g.W > 0 && (win_k == nullptr || win_v == nullptr)) return LOOPVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(pool, 16) || !aligned(codebooks, 16) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(workspace, 16) ||
      !aligned(out, 16) || (lse != nullptr && !aligned(lse, 4)))
    return LOOPVQ_ERR_INVALID_ARG;
  if (g.W > 0 && (!aligned(win_k, 16) || !aligned(win_v, 16))) return LOOPVQ_ERR_INVALID_ARG;
  const int pages = pages_for(g, max_seq_len);
  if (pages > g.max_pages_per_seq) return LOOPVQ_ERR_INVALID_ARG;
  const size_t need = decode_workspace_bytes(batch * n_queries * g.Hq, g.J, g.d);
  if (workspace_bytes < need) return LOOPVQ_ERR_WORKSPACE;
  loopvq_status err = LOOPVQ_OK;
  const int sms = current_sm_count(&err);
  if (err != LOOPVQ_OK) return err;
  // persistent streaming grid: one CTA per SM, never more CTAs than pages
  const long long units_max = static_cast<long long>(batch) * n_queries * g.Hq * pages;
  int n_cta = sms < kMaxStreamCtas ? sms : kMaxStreamCtas;
  if (units_max < n_cta) n_cta = static_cast<int>(units_max);
  DecodeArgs a{&g,        layer,       loop_step, batch, n_queries, max_seq_len, q,        pool,
               codebooks, block_table, seq_lens,  win_k, win_v,     sm_scale,    out_dtype, out,
               lse,       workspace,   n_cta,     stream};
  if (prefill_tc_supported(g, n_queries, out_dtype)) {
    const loopvq_status r = launch_prefill_tc(a, workspace_bytes);
    if (r != LOOPVQ_ERR_UNSUPPORTED) return r;     // else the streaming form below
  }
  return launch_decode(a);
}

}  // namespace
}  // namespace loopvq

extern "C" {

loopvq_status loopvq_decode_attn(const loopvq_config* cfg, int layer, int loop_step, int batch,
                                 int max_seq_len, const void* q, const uint8_t* pool,
                                 const float* codebooks, const int32_t* block_table,
                                 const int32_t* seq_lens, const void* win_k, const void* win_v,
                                 float sm_scale, int out_dtype, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return loopvq::decode_common(cfg, layer, loop_step, batch, 1, max_seq_len, q, pool, codebooks,
                               block_table, seq_lens, win_k, win_v, sm_scale, out_dtype, out, lse,
                               workspace, workspace_bytes, stream);
}

size_t loopvq_prefill_workspace_bytes(const loopvq_config* cfg, int batch, int n_queries,
                                      int max_seq_len) {
  Geometry g;
  if (loopvq::make_geometry(cfg, &g) != LOOPVQ_OK || batch <= 0 || n_queries <= 0 || max_seq_len < 0)
    return 0;
  return loopvq::decode_workspace_bytes(batch * n_queries * g.Hq, g.J, g.d);
}

loopvq_status loopvq_prefill_attn(const loopvq_config* cfg, int layer, int loop_step, int batch,
                                  int n_queries, int max_seq_len, const void* q,
                                  const uint8_t* pool, const float* codebooks,
                                  const int32_t* block_table, const int32_t* seq_lens,
                                  const void* win_k, const void* win_v, float sm_scale,
                                  int out_dtype, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return loopvq::decode_common(cfg, layer, loop_step, batch, n_queries, max_seq_len, q, pool,
                               codebooks, block_table, seq_lens, win_k, win_v, sm_scale, out_dtype,
                               out, lse, workspace, workspace_bytes, stream);
}

size_t loopvq_bf16_decode_workspace_bytes(int batch, int n_q_heads, int head_dim,
                                          int max_seq_len) {
  if (batch <= 0 || n_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0) return 0;
  const int pairs = batch * n_q_heads;
  const int chunks = (max_seq_len + 255) / 256;
  const int s = loopvq::max_decode_splits(pairs, chunks);
  return static_cast<size_t>(pairs) * s * (head_dim + 2) * sizeof(float);
}

loopvq_status loopvq_bf16_decode_attn(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                      int max_seq_len, const void* q, const void* k,
                                      const void* v, const int32_t* seq_lens, float sm_scale,
                                      int out_dtype, void* out, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || max_seq_len < 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0) return LOOPVQ_ERR_INVALID_ARG;
  if (head_dim % 8 != 0 || head_dim > 256) return LOOPVQ_ERR_UNSUPPORTED;
  if (out_dtype != LOOPVQ_DTYPE_BF16 && out_dtype != LOOPVQ_DTYPE_F32) return LOOPVQ_ERR_INVALID_ARG;
  if (!(sm_scale > 0.0f) || sm_scale > 1e30f) return LOOPVQ_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || seq_lens == nullptr || out == nullptr ||
      workspace == nullptr)
    return LOOPVQ_ERR_INVALID_ARG;
  if (!loopvq::aligned(q, 16) || !loopvq::aligned(k, 16) || !loopvq::aligned(v, 16) ||
      !loopvq::aligned(seq_lens, 4) || !loopvq::aligned(out, 16) || !loopvq::aligned(workspace, 16) ||
      (lse != nullptr && !loopvq::aligned(lse, 4)))
    return LOOPVQ_ERR_INVALID_ARG;
  const size_t need = loopvq_bf16_decode_workspace_bytes(batch, n_q_heads, head_dim, max_seq_len);
  if (workspace_bytes < need) return LOOPVQ_ERR_WORKSPACE;
  loopvq_status err = LOOPVQ_OK;
  const int sms = loopvq::current_sm_count(&err);
  if (err != LOOPVQ_OK) return err;
  const int pairs = batch * n_q_heads;
  const int chunks = (max_seq_len + 255) / 256;
  int splits = (4 * sms + pairs - 1) / pairs;
  const int smax = loopvq::max_decode_splits(pairs, chunks);
  if (splits > smax) splits = smax;
  if (splits < 1) splits = 1;
  loopvq::Bf16DecodeArgs a{batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, q,   k,
                           v,     seq_lens,  sm_scale,   out_dtype, out,       lse, workspace,
                           splits, stream};
  return loopvq::launch_bf16_decode(a);
}

}  // extern "C"
