/*
 * loopvq.h - C ABI of the LoopVQ decode hot path on NVIDIA B200 (sm_100a).
 *
 * LoopVQ stores the KV cache of a looped transformer as vector-quantised
 * indices along the loop axis: one sub-vector joins c channels of g
 * consecutive loop steps of one token of one (layer, kv-head), and is
 * stored as a single 8-bit codebook index, i.e. 8/(c*g) bits per element
 * ("LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers",
 * abstract: "codes channels of multiple loop steps jointly", 0.5 bit per
 * element; airadar.tv "LoopVQ : Quantification du cache KV en 1 bit ...",
 * opening paragraph: one shared codebook index per sub-vector). The first
 * prefix_tokens and the latest recent_tokens tokens stay in bf16 (airadar.tv,
 * section "Utilisation": PREFIX_TOKENS=8 RECENT_TOKENS=64), and decoding
 * reads packed indices through fused kernels (airadar.tv, section
 * "Raisons": packed index storage and fused decode kernels).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Device pointers are raw CUDA device addresses owned by the caller. The
 *    library never allocates, frees or synchronises; it only enqueues
 *    kernels on `stream` (a cudaStream_t passed as void*, NULL = the legacy
 *    default stream) on the current device.
 *  - Every argument is checked on the host before anything is launched. A
 *    failed check returns an error status and launches nothing. A launch
 *    error reported by the CUDA runtime returns LOOPVQ_ERR_CUDA. Faults of
 *    the kernels themselves surface at the caller's next synchronisation.
 *  - Calls are reentrant: the library keeps no state between calls other
 *    than a per-device cache of the SM count.
 *  - Symbols: L layers, Hkv kv-heads, Hq query heads (Hq % Hkv == 0),
 *    d head_dim, T loop steps, g loop_group, G = T/g loop groups,
 *    c chan_group, J = d/c channel groups, D = c*g sub-vector length,
 *    E = 256 centroids, P prefix_tokens, R recent_tokens, Pg page_tokens.
 *    Loop step t belongs to loop group gamma = t / g at offset tau = t % g.
 */
#ifndef LOOPVQ_H
#define LOOPVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOOPVQ_OK = 0,
  LOOPVQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer, bad index */
  LOOPVQ_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement */
  LOOPVQ_ERR_WORKSPACE = 3,    /* workspace smaller than loopvq_decode_workspace_bytes */
  LOOPVQ_ERR_CUDA = 4          /* the CUDA runtime reported an error */
} loopvq_status;

enum { LOOPVQ_DTYPE_BF16 = 0, LOOPVQ_DTYPE_F32 = 1 };

/* Flag bits of the encoder's status word (per device, see
 * loopvq_encode_status). */
enum {
  /* a tensor-core encode gave up waiting for a tile's tensor-core result:
   * the tokens of that tile and of the CTA's later tiles were not written */
  LOOPVQ_ENCODE_STATUS_TIMEOUT = 1,
  /* ... and its last tensor-core operation did not finish within the
   * second, longer wait either */
  LOOPVQ_ENCODE_STATUS_UNDRAINED = 2,
  /* a slot_mapping entry at or past n_pages * page_tokens: that token was
   * not written */
  LOOPVQ_ENCODE_STATUS_BAD_SLOT = 4
};

/* Flag bits of a decode call's status word (the first int32 of its
 * workspace), set by the kernels, never cleared by them. */
enum {
  /* a block_table entry of a page the call reads lies outside [0, n_pages);
   * the page was skipped */
  LOOPVQ_DECODE_STATUS_BAD_PAGE = 1,
  /* the streaming kernel's shared-memory allocation did not start where its
   * address arithmetic needs it; its records are NaN (the host checks this
   * before launching and returns LOOPVQ_ERR_UNSUPPORTED, so this bit means a
   * device that changed under the library) */
  LOOPVQ_DECODE_STATUS_SHARED_BASE = 2,
  /* a range check of a build with LOOPVQ_RANGE_CHECK defined found an index
   * outside its buffer; the access was skipped (never set by the default
   * build, whose indices are in range by construction) */
  LOOPVQ_DECODE_STATUS_RANGE = 4,
  /* a bounded wait of the tensor-core prefill form (for the tensor cores or
   * a bulk copy) gave up; the affected records are NaN and the call's
   * outputs are not to be trusted */
  LOOPVQ_DECODE_STATUS_TIMEOUT = 8,
  /* with LOOPVQ_DECODE_STATUS_TIMEOUT: the work in flight could not be
   * waited for before the kernel exited */
  LOOPVQ_DECODE_STATUS_UNDRAINED = 16
};

/*
 * Static shape of one LoopVQ cache. Supported: head_dim % 8 == 0 and
 * head_dim <= 256; chan_group in {1,2,4,8,16} dividing head_dim; J = d/c a
 * multiple of 4 and at most 32; n_loops % loop_group == 0; D = c*g <= 32;
 * n_centroids == 256; page_tokens a multiple of 16, at most 256, and a
 * power-of-two multiple (1, 2, 4, ..) of the rotation block LB =
 * floor(32/J)*J; n_q_heads % n_kv_heads == 0.
 */
typedef struct {
  uint32_t struct_size;      /* sizeof(loopvq_config) */
  int32_t n_layers;          /* L */
  int32_t n_kv_heads;        /* Hkv */
  int32_t n_q_heads;         /* Hq */
  int32_t head_dim;          /* d */
  int32_t n_loops;           /* T */
  int32_t loop_group;        /* g: loop steps coded jointly */
  int32_t chan_group;        /* c: channels per sub-vector */
  int32_t n_centroids;       /* E, must be 256 (8-bit index) */
  int32_t prefix_tokens;     /* P, bf16 prefix window (8 on the pages) */
  int32_t recent_tokens;     /* R, bf16 recent window (64 on the pages) */
  int32_t page_tokens;       /* Pg, tokens per index page */
  int32_t n_pages;           /* physical pages per (layer, kv-head, loop group) */
  int32_t max_batch;         /* rows of block_table */
  int32_t max_pages_per_seq; /* columns of block_table */
} loopvq_config;

/*
 * Derived layout, the single source of truth for sizes and strides.
 *
 * Index pool (uint8), row-major
 *     [L][Hkv][G][n_pages][2 (K, V)][plane]
 * with one plane = Pg*J bytes holding the K (or V) indices of Pg token
 * slots.
 *
 * Both planes (K and V) share one layout. Slots come in blocks of
 * LB = floor(32/J)*J. Inside a block the bytes are stored in granules of GR
 * bytes (GR = 16 if J % 16 == 0, else 8 if J % 8 == 0, else 4) as
 *     [J/GR granules][LB slots][GR bytes],
 * and the J index bytes of slot i are rotated: the index of channel group
 * j sits at byte position (j - (i mod LB)) mod J of that slot's row. So
 * the byte offset of (slot i, group j) inside a plane is
 *     (i/LB)*LB*J + (pos/GR)*LB*GR + (i%LB)*GR + pos%GR,
 *     pos = (j - i%LB) mod J.
 * The rotation lets one warp lane per slot read its own row while the
 * lanes of a warp touch distinct columns of a [E][32] table (the key
 * lookup table, the value histogram), which keeps shared memory free of
 * bank conflicts, and the granules make a warp's row loads contiguous.
 *
 * Quantised token v of a sequence (v = position - P, for positions
 * P .. N-R-1) lives in page block_table[b][v / Pg], slot v % Pg.
 *
 * Codebooks (float32), row-major
 *     [L][Hkv][G][2 (K, V)][g][J][E][c]
 * so codeword e of channel group j for (layer, head, loop group, K/V) is
 * the D = g*c values cb[tau][j][e][ch], tau < g, ch < c (loop-major
 * sub-vector order: element tau*c + ch is channel j*c + ch of loop step
 * gamma*g + tau). Decoding loop step t reads only the contiguous slice
 * [J][E][c] at tau = t % g.
 *
 * bf16 windows, per (layer, loop step): [B][Hkv][P+R][d]. Slots 0..P-1 hold
 * the prefix, slots P..P+R-1 the recent tokens in any order (attention does
 * not depend on token order). The first min(N, P+R) slots are used.
 */
typedef struct {
  uint32_t struct_size;        /* sizeof(loopvq_layout) */
  int32_t J;                   /* channel groups d/c */
  int32_t D;                   /* sub-vector length c*g */
  int32_t n_loop_groups;       /* G */
  int32_t granule;             /* GR */
  int32_t rot_block;           /* LB */
  int32_t window_tokens;       /* P + R */
  size_t plane_bytes;          /* Pg*J */
  size_t page_bytes;           /* 2*Pg*J */
  size_t pool_bytes;           /* L*Hkv*G*n_pages*page_bytes */
  int64_t pool_stride_layer;   /* bytes */
  int64_t pool_stride_head;    /* bytes */
  int64_t pool_stride_group;   /* bytes */
  size_t codebook_bytes;       /* L*Hkv*G*2*g*J*E*c*4 */
  int64_t cb_stride_layer;     /* floats */
  int64_t cb_stride_head;      /* floats */
  int64_t cb_stride_group;     /* floats */
  int64_t cb_stride_kv;        /* floats */
  int64_t cb_stride_loop;      /* floats: one [J][E][c] slice */
  size_t window_bytes;         /* one of K or V for max_batch, one (layer, loop step) */
  double bits_per_element;     /* 8/(c*g) */
} loopvq_layout;

/*
 * Fill `out` with the layout of `cfg`. Host only, pure, no CUDA call.
 * Returns LOOPVQ_ERR_INVALID_ARG for null pointers, wrong struct_size or
 * non-positive sizes, LOOPVQ_ERR_UNSUPPORTED for shapes outside the list
 * above. bits_per_element follows the rate of the abstract: one 8-bit index
 * per c*g elements.
 */
loopvq_status loopvq_cache_layout(const loopvq_config* cfg, loopvq_layout* out);

/*
 * Nearest-centroid encoding of fresh bf16 keys or values into the pool
 * (the quantisation step of the abstract; the distance is the per-element
 * weighted squared distance, the plainest reading of the Fisher-weighted
 * k-means on airadar.tv's opening paragraph).
 *
 * For every token n < n_tokens, kv-head h and channel group j, forms the
 * sub-vector s[tau*c + ch] = x[tau][n][h][j*c + ch] over the g loop steps of
 * loop group `loop_group_idx`, and writes
 *     idx = argmin_e sum_i w_i (s_i - C[e]_i)^2     (exact ties: smallest e)
 * into the K (kv = 0) or V (kv = 1) plane of the pool slot
 * slot_mapping[n] = page*Pg + slot of (layer, h, loop_group_idx). Distances
 * are evaluated in float32 in the direct form above.
 *
 *  x             bf16, element (tau, n, h, ch) at
 *                x + tau*x_loop_stride + n*x_token_stride + h*d + ch
 *                (strides in elements, 16-byte aligned rows).
 *  w             float32 weights or NULL (all 1). Element (tau, n, h, ch) at
 *                w + tau*w_loop_stride + n*w_token_stride + h*d + ch;
 *                w_token_stride = 0 shares one weight vector over tokens.
 *                Weights must be finite and >= 0.
 *  codebooks     base of the whole codebook array (layout above).
 *  slot_mapping  int64 [n_tokens]; a negative entry skips that token.
 *                Entries must be < n_pages*Pg.
 *  pool          base of the whole pool (layout above).
 * n_tokens == 0 is a no-op that returns LOOPVQ_OK.
 */
loopvq_status loopvq_encode(const loopvq_config* cfg, int layer, int loop_group_idx, int kv,
                            int n_tokens, const void* x, int64_t x_loop_stride,
                            int64_t x_token_stride, const float* w, int64_t w_loop_stride,
                            int64_t w_token_stride, const float* codebooks,
                            const int64_t* slot_mapping, uint8_t* pool, void* stream);

/*
 * Reads the encoder status word of the current device into *flags
 * (LOOPVQ_ENCODE_STATUS_* bits that any loopvq_encode, loopvq_encode_evict or
 * loopvq_kmeans_step kernel set since the word was last cleared) and clears
 * it when `clear` is nonzero. This call synchronises with the device (it
 * copies a device word to the host). A word of zero means every encode so
 * far wrote all of its indices.
 */
loopvq_status loopvq_encode_status(int* flags, int clear);

/*
 * The window eviction of one decode step in one launch (airadar.tv, section
 * "Utilisation": the latest RECENT_TOKENS tokens stay in bf16, so each new
 * token pushes one token out of the recent window into the quantised cache).
 * Encodes n_tokens tokens, unweighted, exactly as loopvq_encode would for
 * every (layer, loop group, K/V) of the configuration: for combination
 * z = (layer*G + loop_group)*2 + kv the g loop slices are read at
 *     x + z*g*n_tokens*Hkv*d   as dense bf16 [g][n_tokens][Hkv][d],
 * i.e. x is [L][G][2][g][n_tokens][Hkv][d], and the indices go to the K
 * (kv = 0) or V plane of (layer, loop group) at slot_mapping[n] (the same
 * slot for every layer and group: the page tables are shared; a negative
 * entry skips the token).
 *  n_tokens   0 .. 64 (one evicted token per sequence of the batch);
 *             larger batches return LOOPVQ_ERR_UNSUPPORTED.
 *  x          16-byte aligned; codebooks and pool as for loopvq_encode.
 */
loopvq_status loopvq_encode_evict(const loopvq_config* cfg, int n_tokens, const void* x,
                                  const float* codebooks, const int64_t* slot_mapping,
                                  uint8_t* pool, void* stream);

/*
 * One weighted k-means (Lloyd) step on the codebooks of (layer,
 * loop_group_idx, K or V) for every kv-head and channel group: the offline
 * codebook fitting that the abstract's quantiser needs (Fisher-weighted
 * k-means, airadar.tv opening paragraph), run on the GPU.
 *
 * With the sub-vectors s and weights w of loopvq_encode (same x, w, strides
 * and rules):
 *   1. assignment: assign[(h*J + j)*n_tokens + n] = the index loopvq_encode
 *      would write for token n under the current codebooks (same float32
 *      arithmetic and tie rule);
 *   2. update, in place: every element i of centroid e becomes
 *          sum_{n: assign = e} w_ni s_ni / sum_{n: assign = e} w_ni,
 *      the minimiser of the cluster's weighted squared distance; an element
 *      whose weight sum is zero (an empty cluster, or zero weights) keeps its
 *      value. The sums are float32 and their order is not fixed, so repeated
 *      runs can differ in the last bits.
 *
 *  codebooks  base of the whole codebook array (layout above); read and
 *             written.
 *  assign     device buffer of at least loopvq_kmeans_assign_bytes(cfg,
 *             n_tokens) bytes; receives the step's assignment.
 * Returns LOOPVQ_ERR_WORKSPACE if assign_bytes is too small. n_tokens == 0
 * is a no-op that returns LOOPVQ_OK.
 */
size_t loopvq_kmeans_assign_bytes(const loopvq_config* cfg, int n_tokens);
loopvq_status loopvq_kmeans_step(const loopvq_config* cfg, int layer, int loop_group_idx, int kv,
                                 int n_tokens, const void* x, int64_t x_loop_stride,
                                 int64_t x_token_stride, const float* w, int64_t w_loop_stride,
                                 int64_t w_token_stride, float* codebooks, uint8_t* assign,
                                 size_t assign_bytes, void* stream);

/*
 * Bytes of scratch that loopvq_decode_attn needs for `batch` sequences of
 * at most `max_seq_len` tokens: a 256-byte status area (below), then
 * (batch*Hq + 256) segment records of 4 + head_dim float32 (a segment's
 * softmax maximum and sum and its unnormalised output), batch*Hq window
 * partials of the same size, batch*Hq key lookup tables of 256 x J float32
 * and batch*Hq 32-bit record counters. Host only, pure.
 */
size_t loopvq_decode_workspace_bytes(const loopvq_config* cfg, int batch, int max_seq_len);

/*
 * Fused decode attention of one query per (sequence, query head) at loop
 * step `loop_step` of layer `layer` over the LoopVQ cache (airadar.tv,
 * section "Raisons": fused decode kernels over packed index storage).
 *
 * For sequence b with N = seq_lens[b] tokens, the tokens are the
 * min(N, P+R) bf16 window slots of win_k/win_v plus the quantised tokens
 * v = 0 .. N-P-R-1 read from the pool and dequantised with the loop-tau
 * slice of the codebooks of (layer, kv-head, gamma). The call computes
 *     z_n = sm_scale * q . k_n,   out = sum_n softmax(z)_n v_n,
 *     lse = log(sum_n exp(z_n))   (natural log)
 * with float32 accumulation. Query head hq reads kv-head hq / (Hq/Hkv).
 *
 *  q            bf16 [batch][Hq][d], 16-byte aligned.
 *  pool         base of the pool; codebooks: base of the codebook array.
 *  block_table  int32 [batch][max_pages_per_seq] physical page per logical
 *               page; entries past a sequence's last page are not read.
 *  seq_lens     int32 [batch], each <= max_seq_len and with
 *               ceil((N-P-R)/Pg) <= max_pages_per_seq.
 *  win_k/win_v  bf16 [batch][Hkv][P+R][d] for (layer, loop_step).
 *  out          [batch][Hq][d], bf16 (out_dtype LOOPVQ_DTYPE_BF16, round to
 *               nearest even) or float32 (LOOPVQ_DTYPE_F32).
 *  lse          float32 [batch][Hq] or NULL. A sequence with N == 0 gives
 *               out = 0 and lse = -inf.
 *  workspace    device scratch of at least
 *               loopvq_decode_workspace_bytes(cfg, batch, max_seq_len),
 *               16-byte aligned. Its contents need no initialisation except
 *               the status word, the int32 at byte 0: the kernels OR
 *               LOOPVQ_DECODE_STATUS_* bits into it and never clear it. A
 *               caller that wants to know zeroes it before the call and
 *               reads it after synchronising; a nonzero word means the
 *               outputs of that call are not to be trusted.
 */
loopvq_status loopvq_decode_attn(const loopvq_config* cfg, int layer, int loop_step, int batch,
                                 int max_seq_len, const void* q, const uint8_t* pool,
                                 const float* codebooks, const int32_t* block_table,
                                 const int32_t* seq_lens, const void* win_k, const void* win_v,
                                 float sm_scale, int out_dtype, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Attention of a chunk of new queries over the cached context (the prefill
 * or chunked-prefill side of the same cache; airadar.tv, section
 * "Utilisation", names the prefill backend as a serving setting). For each
 * sequence b and each of its n_queries queries i, computes exactly what
 * loopvq_decode_attn computes for a single query: attention of
 * q[b][i][hq] over the min(N, P+R) window tokens and the N-P-R quantised
 * tokens of sequence b, N = seq_lens[b]. Attention among the chunk's own
 * tokens (causal, not yet cached) is the caller's; out and lse are returned
 * so that the caller merges the two with log-sum-exp weights.
 *
 *  q      bf16 [batch][n_queries][Hq][d], 16-byte aligned.
 *  out    [batch][n_queries][Hq][d] (bf16 or float32 as out_dtype).
 *  lse    float32 [batch][n_queries][Hq] or NULL.
 *  workspace  at least loopvq_prefill_workspace_bytes(cfg, batch, n_queries,
 *         max_seq_len) bytes; the status word as for loopvq_decode_attn.
 * Every other argument as for loopvq_decode_attn.
 *
 * Two forms, chosen per call:
 *  - bf16 output, n_queries >= 64, head_dim 128 and chan_group 4: the
 *    tensor-core form. Each tile of 64 tokens is dequantised once for a tile
 *    of 128 queries and both products run on the tensor cores; the key
 *    codewords enter in two bf16 parts (scores and lse keep float32-level
 *    precision), the value codewords and softmax weights in bf16 (about
 *    2^-9 relative in the output). A bounded wait that gives up sets
 *    LOOPVQ_DECODE_STATUS_TIMEOUT (and _UNDRAINED) in the status word.
 *  - otherwise: the decode kernels over batch*n_queries virtual sequences
 *    (neighbouring CTAs share each sequence's pages through L2), exact in
 *    float32 like loopvq_decode_attn.
 */
size_t loopvq_prefill_workspace_bytes(const loopvq_config* cfg, int batch, int n_queries,
                                      int max_seq_len);
loopvq_status loopvq_prefill_attn(const loopvq_config* cfg, int layer, int loop_step, int batch,
                                  int n_queries, int max_seq_len, const void* q,
                                  const uint8_t* pool, const float* codebooks,
                                  const int32_t* block_table, const int32_t* seq_lens,
                                  const void* win_k, const void* win_v, float sm_scale,
                                  int out_dtype, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * Decode attention that needs no workspace from the caller. The pages have
 * no counterpart for this call; it exists for callers that cannot allocate
 * device memory: code that receives only input and output pointers from a
 * host program that owns all device memory (a plugin or callback interface),
 * and code running under a fixed device-memory budget that forbids further
 * allocations. Such callers cannot provide the scratch that
 * loopvq_decode_attn takes.
 *
 * Computes exactly what loopvq_decode_attn computes, with the same
 * arguments except `workspace`/`workspace_bytes`. The split-K scratch is a
 * file-scope device array of LOOPVQ_STATIC_SCRATCH_BYTES bytes inside the
 * library: every GPU that loads the library holds it until the process
 * exits, and this call itself allocates and frees nothing. When
 * loopvq_decode_workspace_bytes(cfg, batch, max_seq_len) exceeds
 * LOOPVQ_STATIC_SCRATCH_BYTES the call returns LOOPVQ_ERR_WORKSPACE and
 * launches nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and the library remembers it for the
 * rest of the process; make that first call before any stream capture. The
 * remembered address belongs to the device's primary context: after
 * cudaDeviceReset, or anything else that destroys and recreates that
 * context, it is stale, and calling this entry point again in the same
 * process is not supported. All calls on a device share the one array and it keeps
 * the last call's contents (no initial contents are needed); calls whose
 * kernels overlap on the GPU, e.g. on two streams without ordering, race
 * on it and give undefined results.
 */
#define LOOPVQ_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
loopvq_status loopvq_decode_attn_noalloc(const loopvq_config* cfg, int layer, int loop_step,
                                         int batch, int max_seq_len, const void* q,
                                         const uint8_t* pool, const float* codebooks,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         const void* win_k, const void* win_v, float sm_scale,
                                         int out_dtype, void* out, float* lse, void* stream);

/*
 * Same-shape decode attention over a dense bf16 KV cache, the comparison
 * point for loopvq_decode_attn (the pages compare LoopVQ decode latency
 * with BF16 at 32K context: airadar.tv section "Raisons").
 *
 *  q        bf16 [batch][n_q_heads][head_dim]
 *  k, v     bf16 [batch][n_kv_heads][max_seq_len][head_dim] for one
 *           (layer, loop step), 16-byte aligned
 *  seq_lens int32 [batch], each <= max_seq_len
 * out/lse/workspace as for loopvq_decode_attn, with
 * loopvq_bf16_decode_workspace_bytes giving the scratch size.
 * head_dim % 8 == 0 and head_dim <= 256.
 */
size_t loopvq_bf16_decode_workspace_bytes(int batch, int n_q_heads, int head_dim,
                                          int max_seq_len);
loopvq_status loopvq_bf16_decode_attn(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                      int max_seq_len, const void* q, const void* k,
                                      const void* v, const int32_t* seq_lens, float sm_scale,
                                      int out_dtype, void* out, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* Static description of a status code. Never NULL. */
const char* loopvq_status_string(loopvq_status s);

#ifdef __cplusplus
}
#endif

#endif /* LOOPVQ_H */
