"""LoopVQ oracle: a plain, slow, float64 CPU statement of the decode hot path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The product (the CUDA
library and its Python binding) never calls it, and it shares no code, table
or helper with the CUDA side.

What it computes, and where the pages say so
---------------------------------------------
Sources are the five extracted web pages on LoopVQ; the authority is the
original English abstract on "LoopVQ: Sub 1-bit KV Cache Quantization for
Looped Transformers" (shd-paper.top, section "摘要（原文）", below called
*the abstract*).

* Loop-axis vector quantisation: the channels of several consecutive loop
  steps are coded jointly, one codebook index per sub-vector (the abstract;
  airadar.tv "LoopVQ : Quantification du cache KV en 1 bit ...", opening
  paragraph). A sub-vector joins ``c`` channels of ``g`` consecutive loop
  steps of one token of one (layer, kv-head), so ``D = c*g`` elements.
* Rate: 0.5 bit per element at the main operating point, 0.25 bit at the
  low one (the abstract; airadar.tv section "Raisons"). With an 8-bit index
  over ``c*g`` elements the rate is ``8/(c*g)``.
* Encoding is nearest-centroid under a per-element weighted squared
  distance. The pages only imply this step (codebooks are Fisher-weighted
  k-means, airadar.tv opening paragraph); the weighted distance is the
  plainest reading.
* The first 8 (prefix) and the latest 64 (recent) tokens stay in bf16
  (airadar.tv section "Utilisation": PREFIX_TOKENS=8 RECENT_TOKENS=64).
* Decode attention over the quantised cache (airadar.tv section "Raisons":
  packed index storage and fused decode kernels) is ordinary softmax
  attention of one query against the window tokens and the dequantised
  tokens.

Readings taken where the pages are silent (each one is listed, with its
reason, in the design notes of the repository):

* element order inside a sub-vector is loop-major: element ``tau*c + ch``
  is channel ``j*c + ch`` of loop ``gamma*g + tau``;
* one codebook of E=256 codewords per (layer, kv-head, loop group, K or V,
  channel group j); K and V are coded separately;
* exact ties in the distance go to the smallest centroid index;
* scores are ``sm_scale * q.k`` with ``sm_scale = 1/sqrt(d)``; the returned
  log-sum-exp is the natural log of the sum of ``exp`` of those scores;
* keys are quantised as cached (after any rotary embedding), so attention
  against a dequantised key is a plain dot product.

Pins (the tests under ``tests/test_oracle_*.py``) tie every function here to
something other than itself: the rate closed form, scipy's ``vq``,
``kmeans2`` and ``logsumexp``, torch's ``scaled_dot_product_attention``,
brute force over all assignments on tiny inputs, an exact codebook that must
reproduce the unquantised cache, token replication for integer weights,
split-and-merge identities and invariances.
"""

from __future__ import annotations

import math

import numpy as np

N_CENTROIDS = 256          # 8-bit index
PREFIX_TOKENS = 8          # airadar.tv, section "Utilisation"
RECENT_TOKENS = 64         # airadar.tv, section "Utilisation"


# ---------------------------------------------------------------------------
# Rate
# ---------------------------------------------------------------------------

def bits_per_element(c: int, g: int, index_bits: int = 8) -> float:
    """Bits stored per cached element: one ``index_bits`` index per ``c*g``
    elements (the abstract: "0.5 bits per element" with joint loop coding)."""
    return index_bits / (c * g)


def packed_bytes_per_plane(n_tokens: int, d: int, c: int) -> int:
    """Bytes of packed 8-bit indices for ``n_tokens`` tokens of one
    (layer, kv-head, loop group) and one of K or V. These bytes cover the
    ``g`` loop steps of the group: one byte per sub-vector, ``d/c``
    sub-vectors per token."""
    if d % c:
        raise ValueError("head_dim must be a multiple of c")
    return n_tokens * (d // c)


# ---------------------------------------------------------------------------
# Sub-vectors and codewords
# ---------------------------------------------------------------------------

def subvectors(X: np.ndarray, c: int) -> np.ndarray:
    """Join ``c`` channels of the ``g`` loop steps of one loop group.

    ``X`` holds the g loop slices of one group, shape ``[g][N][H][d]``.
    Returns ``S`` of shape ``[N][H][J][g*c]`` with
    ``S[n, h, j, tau*c + ch] = X[tau, n, h, j*c + ch]`` (loop-major order).
    """
    X = np.asarray(X, dtype=np.float64)
    g, N, H, d = X.shape
    if d % c:
        raise ValueError("head_dim must be a multiple of c")
    J = d // c
    S = np.empty((N, H, J, g * c), dtype=np.float64)
    for tau in range(g):
        for ch in range(c):
            # channels ch, c+ch, 2c+ch, ... are channel ch of groups 0..J-1
            S[:, :, :, tau * c + ch] = X[tau, :, :, ch::c]
    return S


def subvector_weights(w: np.ndarray | None, N: int, c: int) -> np.ndarray | None:
    """Arrange per-element weights like ``subvectors``.

    ``w`` is ``[g][N][H][d]`` (one weight per element) or ``[g][1][H][d]``
    (one weight per (loop, head, channel), shared by all tokens) or None
    (all weights 1)."""
    if w is None:
        return None
    w = np.asarray(w, dtype=np.float64)
    if w.shape[1] == 1 and N != 1:
        w = np.broadcast_to(w, (w.shape[0], N, w.shape[2], w.shape[3]))
    return subvectors(w, c)


def codewords(cb: np.ndarray) -> np.ndarray:
    """Codewords of one (layer, kv-head, loop group, K or V) codebook set.

    ``cb`` has shape ``[g][J][E][c]``: the loop-``tau`` slice
    ``cb[tau]`` is what decoding at loop step ``gamma*g + tau`` reads.
    Returns ``[J][E][g*c]`` in the same loop-major order as ``subvectors``.
    """
    cb = np.asarray(cb, dtype=np.float64)
    g, J, E, c = cb.shape
    W = np.empty((J, E, g * c), dtype=np.float64)
    for tau in range(g):
        W[:, :, tau * c:(tau + 1) * c] = cb[tau]
    return W


# ---------------------------------------------------------------------------
# Encoding
# ---------------------------------------------------------------------------

def weighted_sq_dist(S: np.ndarray, CW: np.ndarray,
                     Wt: np.ndarray | None = None) -> np.ndarray:
    """Direct-form weighted squared distance, float64.

    ``S`` is ``[N][J][D]`` (sub-vectors of one head), ``CW`` is
    ``[J][E][D]``, ``Wt`` is ``[N][J][D]`` or None (weight 1).
    Returns ``dist[n, j, e] = sum_i Wt[n,j,i] * (S[n,j,i] - CW[j,e,i])**2``.
    """
    S = np.asarray(S, dtype=np.float64)
    CW = np.asarray(CW, dtype=np.float64)
    N, J, D = S.shape
    E = CW.shape[1]
    dist = np.empty((N, J, E), dtype=np.float64)
    for j in range(J):
        diff = S[:, j, None, :] - CW[None, j, :, :]          # [N][E][D]
        sq = diff * diff
        if Wt is not None:
            sq = sq * np.asarray(Wt, dtype=np.float64)[:, j, None, :]
        dist[:, j, :] = sq.sum(axis=2)
    return dist


def encode_ref(S: np.ndarray, CW: np.ndarray,
               Wt: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Nearest centroid of every sub-vector: ``argmin_e dist[n, j, e]``.

    Exact ties go to the smallest index (``np.argmin`` returns the first
    minimum). Returns ``(idx [N][J] uint8, dist [N][J][E] float64)``.
    """
    dist = weighted_sq_dist(S, CW, Wt)
    idx = np.argmin(dist, axis=2)
    if CW.shape[1] > 256:
        raise ValueError("an 8-bit index holds at most 256 centroids")
    return idx.astype(np.uint8), dist


def encode_group_ref(X: np.ndarray, cb: np.ndarray,
                     w: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Encode the g loop slices ``X [g][N][H][d]`` of one loop group with the
    per-head codebooks ``cb [H][g][J][E][c]``.

    Returns ``idx [N][H][J]`` uint8 and ``dist [N][H][J][E]``.
    """
    X = np.asarray(X, dtype=np.float64)
    g, N, H, d = X.shape
    c = cb.shape[-1]
    S = subvectors(X, c)
    Wt = subvector_weights(w, N, c)
    J = d // c
    idx = np.empty((N, H, J), dtype=np.uint8)
    dist = np.empty((N, H, J, cb.shape[3]), dtype=np.float64)
    for h in range(H):
        i_h, d_h = encode_ref(S[:, h], codewords(cb[h]),
                              None if Wt is None else Wt[:, h])
        idx[:, h] = i_h
        dist[:, h] = d_h
    return idx, dist


# ---------------------------------------------------------------------------
# Codebook fitting: one weighted k-means (Lloyd) step
# ---------------------------------------------------------------------------
# The codebooks are fitted offline with Fisher-weighted k-means (airadar.tv,
# opening paragraph). A Lloyd step alternates the assignment (the encoder
# above, under the current codewords) and the update. Under the per-element
# weighted squared distance the update that minimises a cluster's distortion
# is, element by element, the weighted mean of its members; an element with
# no weight (an empty cluster) keeps its codeword value.

def centroid_update_ref(S: np.ndarray, CW: np.ndarray, idx: np.ndarray,
                        Wt: np.ndarray | None = None) -> np.ndarray:
    """Weighted centroid update for the codebooks of one head, float64.

    ``S`` is ``[N][J][D]``, ``CW`` the current codewords ``[J][E][D]``,
    ``idx`` the assignment ``[N][J]``, ``Wt`` ``[N][J][D]`` or None (weight
    1). Returns ``new[j, e, i] = sum_{n: idx[n,j]=e} Wt[n,j,i] S[n,j,i] /
    sum_{n: idx[n,j]=e} Wt[n,j,i]``, or ``CW[j, e, i]`` where that weight sum
    is zero.
    """
    S = np.asarray(S, dtype=np.float64)
    CW = np.asarray(CW, dtype=np.float64)
    idx = np.asarray(idx)
    N, J, D = S.shape
    W = np.ones_like(S) if Wt is None else np.asarray(Wt, dtype=np.float64)
    new = CW.copy()
    for j in range(J):
        for e in range(CW.shape[1]):
            members = idx[:, j] == e
            if not members.any():
                continue
            den = W[members, j, :].sum(axis=0)
            num = (W[members, j, :] * S[members, j, :]).sum(axis=0)
            keep = den == 0
            new[j, e] = np.where(keep, CW[j, e], num / np.where(keep, 1.0, den))
    return new


def codebook_from_codewords(CW: np.ndarray, g: int) -> np.ndarray:
    """Inverse of ``codewords``: ``[J][E][g*c]`` back to ``[g][J][E][c]``."""
    CW = np.asarray(CW, dtype=np.float64)
    J, E, D = CW.shape
    c = D // g
    cb = np.empty((g, J, E, c), dtype=np.float64)
    for tau in range(g):
        cb[tau] = CW[:, :, tau * c:(tau + 1) * c]
    return cb


def kmeans_step_group_ref(X: np.ndarray, cb: np.ndarray, w: np.ndarray | None = None,
                          assign: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """One weighted Lloyd step on the per-head codebooks ``cb [H][g][J][E][c]``
    of one loop group, with the g loop slices ``X [g][N][H][d]`` and weights
    ``w`` as for ``encode_group_ref``.

    The assignment is the encoder's under ``cb``, unless ``assign [N][H][J]``
    is given (then that one is used, e.g. to update from another
    implementation's choice among near-tied centroids). Returns
    ``(assignment [N][H][J] uint8, new codebooks [H][g][J][E][c])``.
    """
    X = np.asarray(X, dtype=np.float64)
    g, N, H, d = X.shape
    c = cb.shape[-1]
    if assign is None:
        assign, _ = encode_group_ref(X, cb, w)
    S = subvectors(X, c)
    Wt = subvector_weights(w, N, c)
    new = np.empty(cb.shape, dtype=np.float64)
    for h in range(H):
        CW_new = centroid_update_ref(S[:, h], codewords(cb[h]), assign[:, h],
                                     None if Wt is None else Wt[:, h])
        new[h] = codebook_from_codewords(CW_new, g)
    return np.asarray(assign, dtype=np.uint8), new


def weighted_distortion_ref(X: np.ndarray, cb: np.ndarray, assign: np.ndarray,
                            w: np.ndarray | None = None) -> float:
    """Total weighted squared distance of every sub-vector to the codeword
    it is assigned to (the objective a Lloyd step does not increase)."""
    X = np.asarray(X, dtype=np.float64)
    g, N, H, d = X.shape
    c = cb.shape[-1]
    S = subvectors(X, c)
    Wt = subvector_weights(w, N, c)
    total = 0.0
    for h in range(H):
        CW = codewords(cb[h])
        for j in range(d // c):
            diff = S[:, h, j, :] - CW[j][assign[:, h, j]]
            sq = diff * diff if Wt is None else Wt[:, h, j, :] * diff * diff
            total += float(sq.sum())
    return total


# ---------------------------------------------------------------------------
# Dequantisation and attention
# ---------------------------------------------------------------------------

def dequant_ref(idx: np.ndarray, cb: np.ndarray, tau: int) -> np.ndarray:
    """Reconstruct the loop-``tau`` slice of cached vectors.

    ``idx`` is ``[n][J]``, ``cb`` is ``[g][J][E][c]``. Returns ``[n][J*c]``
    with ``out[n, j*c + ch] = cb[tau, j, idx[n, j], ch]``.
    """
    cb = np.asarray(cb, dtype=np.float64)
    g, J, E, c = cb.shape
    idx = np.asarray(idx)
    n = idx.shape[0]
    out = np.empty((n, J * c), dtype=np.float64)
    for j in range(J):
        out[:, j * c:(j + 1) * c] = cb[tau, j][idx[:, j].astype(np.int64)]
    return out


def attn_partial_ref(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                     sm_scale: float) -> tuple[float, float, np.ndarray]:
    """Un-normalised softmax partial over a set of tokens.

    ``z_n = sm_scale * q . K_n``, ``m = max z``, ``l = sum exp(z - m)``,
    ``o = sum exp(z_n - m) V_n``. An empty set gives ``(-inf, 0, 0)``.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return -math.inf, 0.0, np.zeros(V.shape[1], dtype=np.float64)
    z = sm_scale * (K @ q)
    m = float(z.max())
    p = np.exp(z - m)
    return m, float(p.sum()), p @ V


def merge_partials_ref(parts) -> tuple[np.ndarray, float]:
    """Merge partials ``(m_s, l_s, o_s)`` of disjoint token sets.

    ``m* = max m_s``, ``l* = sum l_s exp(m_s - m*)``,
    ``out = sum o_s exp(m_s - m*) / l*``, ``lse = m* + ln l*``.
    """
    parts = [p for p in parts if p[1] > 0.0]
    if not parts:
        raise ValueError("no tokens")
    m_star = max(p[0] for p in parts)
    l_star = sum(p[1] * math.exp(p[0] - m_star) for p in parts)
    o = sum(p[2] * math.exp(p[0] - m_star) for p in parts)
    return o / l_star, m_star + math.log(l_star)


def attn_ref(q: np.ndarray, K: np.ndarray, V: np.ndarray,
             sm_scale: float) -> tuple[np.ndarray, float]:
    """Softmax attention of one query over all rows of K/V, float64.
    Returns ``(out [d], lse)``."""
    return merge_partials_ref([attn_partial_ref(q, K, V, sm_scale)])


def softmax_weights_ref(q: np.ndarray, K: np.ndarray, sm_scale: float) -> np.ndarray:
    """The attention probabilities ``p_n`` (used by the invariance pins)."""
    z = sm_scale * (np.asarray(K, np.float64) @ np.asarray(q, np.float64))
    e = np.exp(z - z.max())
    return e / e.sum()


def n_vq_tokens(seq_len: int, prefix: int = PREFIX_TOKENS,
                recent: int = RECENT_TOKENS) -> int:
    """Tokens held as indices: positions ``[prefix, seq_len - recent)``."""
    return max(0, seq_len - prefix - recent)


def n_window_tokens(seq_len: int, prefix: int = PREFIX_TOKENS,
                    recent: int = RECENT_TOKENS) -> int:
    """Tokens held in bf16: the first ``prefix`` and last ``recent``."""
    return min(seq_len, prefix + recent)


def decode_attn_ref(q: np.ndarray, win_K: np.ndarray, win_V: np.ndarray,
                    idx_K: np.ndarray, idx_V: np.ndarray,
                    cb_K: np.ndarray, cb_V: np.ndarray, tau: int,
                    sm_scale: float) -> tuple[np.ndarray, float]:
    """Decode attention of one query (one sequence, one query head) at loop
    offset ``tau`` inside its loop group.

    ``win_K/win_V [w][d]``: the bf16 window tokens (values already bf16).
    ``idx_K/idx_V [n_vq][J]``: indices of the quantised tokens.
    ``cb_K/cb_V [g][J][E][c]``: that head's codebooks for the loop group.
    Window tokens enter exactly; quantised tokens enter dequantised. The
    order of tokens does not matter to softmax attention.
    """
    K = np.concatenate([np.asarray(win_K, np.float64),
                        dequant_ref(idx_K, cb_K, tau)], axis=0)
    V = np.concatenate([np.asarray(win_V, np.float64),
                        dequant_ref(idx_V, cb_V, tau)], axis=0)
    return attn_ref(q, K, V, sm_scale)


# ---------------------------------------------------------------------------
# The packed, paged index pool (the library's documented storage format)
# ---------------------------------------------------------------------------
#
# Written from the layout text of include/loopvq.h, independently of the
# library's own code. The pool is
#     [n_layers][n_kv_heads][n_loop_groups][n_pages][2 (K, V)][plane]
# with a plane of page_tokens * J bytes.
# Both planes (K and V) share one layout: token slots come in blocks of
# LB = floor(32/J)*J. Inside a block, bytes are grouped in granules of GR
# bytes (GR = 16 if J % 16 == 0, else 8 if J % 8 == 0, else 4) laid out
#     [J / GR granules][LB slots][GR bytes],
# and the J index bytes of slot i are rotated: group j sits at byte position
# (j - (i mod LB)) mod J of that slot's row.

def pool_granule(J: int) -> int:
    if J % 16 == 0:
        return 16
    if J % 8 == 0:
        return 8
    if J % 4 == 0:
        return 4
    raise ValueError("J = head_dim / c must be a multiple of 4")


def rotation_block(J: int) -> int:
    """LB: slots per rotation block, the largest multiple of J not above 32."""
    if J > 32:
        raise ValueError("J above 32 is not part of the format")
    return (32 // J) * J


def plane_offset(slot: int, j: int, J: int, kv: int = 0, page_tokens: int = 0) -> int:
    """Byte offset of group ``j`` of token slot ``slot`` inside a plane. The
    K plane (``kv = 0``) and the V plane (``kv = 1``) share the layout;
    ``kv`` and ``page_tokens`` are accepted for the callers' convenience."""
    gr = pool_granule(J)
    lb = rotation_block(J)
    blk, rot = divmod(slot, lb)
    pos = (j - rot) % J
    gran, byte = divmod(pos, gr)
    return blk * lb * J + gran * lb * gr + rot * gr + byte


def pack_pages(idx_K: np.ndarray, idx_V: np.ndarray, pages: list[int],
               n_pages: int, page_tokens: int) -> np.ndarray:
    """Pack one sequence's indices of one (layer, head, loop group) into a
    page array ``[n_pages][2][page_tokens*J]``. Token ``v`` (0-based among the
    quantised tokens) goes to page ``pages[v // page_tokens]``, slot
    ``v % page_tokens``. Unused bytes are 0."""
    n, J = idx_K.shape
    out = np.zeros((n_pages, 2, page_tokens * J), dtype=np.uint8)
    for v in range(n):
        pg = pages[v // page_tokens]
        slot = v % page_tokens
        for j in range(J):
            out[pg, 0, plane_offset(slot, j, J, 0)] = idx_K[v, j]
            out[pg, 1, plane_offset(slot, j, J, 1, page_tokens)] = idx_V[v, j]
    return out


def plane_offsets(slots: np.ndarray, J: int, kv: int = 0, page_tokens: int = 0) -> np.ndarray:
    """Array form of ``plane_offset``: ``[n]`` slots -> ``[n][J]`` offsets."""
    slots = np.asarray(slots, dtype=np.int64)[:, None]
    j = np.arange(J, dtype=np.int64)[None, :]
    gr = pool_granule(J)
    lb = rotation_block(J)
    blk, rot = slots // lb, slots % lb
    pos = (j - rot) % J
    return blk * lb * J + (pos // gr) * lb * gr + rot * gr + pos % gr


def pack_sequence(pool: np.ndarray, idx: np.ndarray, block_row: np.ndarray,
                  page_tokens: int, kv: int) -> None:
    """Write one sequence's indices ``idx [n][J]`` of one (layer, head, loop
    group) into ``pool [n_pages][2][page_tokens*J]`` (in place) for K
    (``kv = 0``) or V (``kv = 1``), following ``block_row`` (its page table
    row)."""
    n, J = idx.shape
    v = np.arange(n, dtype=np.int64)
    phys = np.asarray(block_row, dtype=np.int64)[v // page_tokens]
    off = plane_offsets(v % page_tokens, J, kv, page_tokens)
    pool[phys[:, None], kv, off] = idx


def unpack_sequence(pool: np.ndarray, n: int, J: int, block_row: np.ndarray,
                    page_tokens: int, kv: int) -> np.ndarray:
    """Inverse of ``pack_sequence``."""
    v = np.arange(n, dtype=np.int64)
    phys = np.asarray(block_row, dtype=np.int64)[v // page_tokens]
    off = plane_offsets(v % page_tokens, J, kv, page_tokens)
    return pool[phys[:, None], kv, off]


def unpack_pages(page_array: np.ndarray, pages: list[int], n: int,
                 J: int, page_tokens: int) -> tuple[np.ndarray, np.ndarray]:
    """Inverse of ``pack_pages``: read back ``n`` tokens' K and V indices."""
    idx_K = np.empty((n, J), dtype=np.uint8)
    idx_V = np.empty((n, J), dtype=np.uint8)
    for v in range(n):
        pg = pages[v // page_tokens]
        slot = v % page_tokens
        for j in range(J):
            idx_K[v, j] = page_array[pg, 0, plane_offset(slot, j, J, 0)]
            idx_V[v, j] = page_array[pg, 1, plane_offset(slot, j, J, 1, page_tokens)]
    return idx_K, idx_V
