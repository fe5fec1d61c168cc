// Host-side declarations shared by the translation units of libloopvq.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "loopvq.h"

namespace loopvq {

// Everything derived from a validated loopvq_config.
struct Geometry {
  int L, Hkv, Hq, d, T, g, c, E, P, R, Pg, n_pages, max_batch, max_pages_per_seq;
  int J, D, G, GR, LB, W;        // W = P + R window slots
  int64_t plane_bytes, page_bytes;
  int64_t pool_stride_group, pool_stride_head, pool_stride_layer;
  int64_t cb_stride_loop, cb_stride_kv, cb_stride_group, cb_stride_head, cb_stride_layer;
};

// Validates `cfg` and fills `geo`. Pure host code.
loopvq_status make_geometry(const loopvq_config* cfg, Geometry* geo);

// Largest number of context splits the bf16-KV planner may use.
int max_decode_splits(int pairs, int pages);

// Most CTAs the persistent LoopVQ streaming kernel is launched with (one per
// SM up to this many); the decode workspace holds (pairs + kMaxStreamCtas)
// segment records of 4 + d floats.
constexpr int kMaxStreamCtas = 256;

// Bytes at the start of the decode workspace that hold the status word (an
// int32 of flag bits).
constexpr size_t kStatusBytes = 256;

// Decode workspace of `pairs` (sequence, query head) pairs: the status word,
// (pairs + kMaxStreamCtas) segment records and `pairs` window partials of
// 4 + d floats, one key lookup table of E x J floats per pair, and one
// 32-bit record counter per pair.
size_t decode_workspace_bytes(int pairs, int J, int d);

// Number of multiprocessors of the current device (cached per device).
// Returns 0 and sets *err when the runtime fails.
int current_sm_count(loopvq_status* err);

// Launchers (defined in the .cu files). All arguments are validated.
struct DecodeArgs {
  const Geometry* geo;
  int layer, loop_step, batch, n_queries, max_seq_len;
  const void* q;
  const uint8_t* pool;
  const float* codebooks;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const void* win_k;
  const void* win_v;
  float sm_scale;
  int out_dtype;
  void* out;
  float* lse;
  void* workspace;
  int n_cta;             // persistent streaming CTAs (0: nothing to stream)
  void* stream;
};
loopvq_status launch_decode(const DecodeArgs& a);

// The tensor-core form of attention over the cache for chunks of at least
// kPrefillTcMinQueries queries per sequence (prefill_tc.cu): bf16 outputs,
// head_dim 128 at c = 4. It keeps split records of (d + 2) floats per
// query row and token chunk, and the key and value codebook slices in bf16,
// in the workspace; when `workspace_bytes` cannot hold them it returns
// LOOPVQ_ERR_UNSUPPORTED and launches nothing.
constexpr int kPrefillTcMinQueries = 64;
bool prefill_tc_supported(const Geometry& g, int n_queries, int out_dtype);
size_t prefill_tc_workspace_bytes(const Geometry& g, int batch, int n_queries, int max_seq_len, int* S,
                                  int* CH);
loopvq_status launch_prefill_tc(const DecodeArgs& a, size_t workspace_bytes);

struct EncodeArgs {
  const Geometry* geo;
  int layer, gamma, kv, n_tokens;
  const void* x;
  int64_t x_loop_stride, x_token_stride;
  const float* w;
  int64_t w_loop_stride, w_token_stride;
  const float* codebooks;
  const int64_t* slot_mapping;   // null: token n is slot n of `assign`
  uint8_t* pool;                 // null when `assign` is given
  uint8_t* assign;               // or null: indices [Hkv][J][n_tokens] instead of the pool
  void* stream;
};
loopvq_status launch_encode(const EncodeArgs& a);

// Reads (and optionally clears) the encoder status word of the current
// device; synchronous.
loopvq_status encode_status(int* flags, int clear);

// The window eviction of one decode step: every (layer, loop group, K/V)
// of the config in one launch; x of combination z = (layer*G + gamma)*2 + kv
// at a.x + z * g*n*Hkv*d elements, dense [g][n][Hkv][d]; unweighted;
// n_tokens <= 64. a.layer, a.gamma and a.kv are 0.
loopvq_status launch_encode_evict(const EncodeArgs& a);

// Weighted centroid update of one k-means step: every codebook (h, j) of
// (layer, gamma, kv) becomes the per-element weighted mean of the
// sub-vectors assigned to each centroid (assignment [Hkv][J][n_tokens]);
// elements whose weight sum is zero keep their value.
loopvq_status launch_kmeans_update(const EncodeArgs& a, float* codebooks);

struct Bf16DecodeArgs {
  int batch, Hq, Hkv, d, max_seq_len;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* seq_lens;
  float sm_scale;
  int out_dtype;
  void* out;
  float* lse;
  void* workspace;
  int splits;
  void* stream;
};
loopvq_status launch_bf16_decode(const Bf16DecodeArgs& a);

// Split-K merge of float32 partials [pairs][splits][d+2] (m in log2 units,
// l, un-normalised o[d]) into out/lse.
loopvq_status launch_merge(const float* partials, int pairs, int splits, int d, int out_dtype,
                           void* out, float* lse, void* stream);

}  // namespace loopvq
