"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form from the pages, a
library routine (scipy, torch), brute force over all choices on a tiny
input, or an invariance of the mathematics. A plausible mistake in the
oracle (a dropped weight, a transposed sub-vector order, a wrong sign in the
log-sum-exp, an off-by-one window) fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import scipy.cluster.vq
import scipy.special
import torch

from oracle import loopvq_oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# Rate: "0.5 bits per element" and "0.25 bits" (LoopVQ: Sub 1-bit KV Cache
# Quantization for Looped Transformers, abstract; airadar.tv "Raisons").
# --------------------------------------------------------------------------

@pytest.mark.parametrize("c,g,bits", [(4, 4, 0.5), (8, 4, 0.25), (4, 2, 1.0), (2, 4, 1.0)])
def test_rate_closed_form(c, g, bits):
    assert O.bits_per_element(c, g) == bits


@pytest.mark.parametrize("d,c,g,n", [(64, 4, 4, 440), (128, 4, 4, 1000), (96, 8, 4, 77)])
def test_packed_bytes_give_rate(d, c, g, n):
    # one byte per sub-vector; the bytes of one plane cover g loop steps
    nbytes = O.packed_bytes_per_plane(n, d, c)
    assert nbytes * 8 / (n * d * g) == O.bits_per_element(c, g)


# --------------------------------------------------------------------------
# Encoder: nearest centroid under a weighted squared distance.
# --------------------------------------------------------------------------

def test_unweighted_encode_matches_scipy_vq():
    r = _rng(1)
    N, J, D, E = 300, 3, 16, 256
    S = r.normal(size=(N, J, D))
    CW = r.normal(size=(J, E, D))
    idx, dist = O.encode_ref(S, CW)
    for j in range(J):
        code, d_eu = scipy.cluster.vq.vq(S[:, j], CW[j], check_finite=True)
        np.testing.assert_array_equal(idx[:, j], code)
        np.testing.assert_allclose(np.sqrt(dist[np.arange(N), j, idx[:, j]]), d_eu,
                                   rtol=1e-9)


def test_weighted_encode_equals_vq_of_sqrtw_scaled_vectors():
    # sum_i w_i (s_i - C_i)^2 == || sqrt(w) s - sqrt(w) C ||^2
    r = _rng(2)
    N, J, D, E = 40, 2, 8, 64
    S = r.normal(size=(N, J, D))
    CW = r.normal(size=(J, E, D))
    Wt = np.exp(r.normal(size=(N, J, D)))
    idx, _ = O.encode_ref(S, CW, Wt)
    for n in range(N):
        for j in range(J):
            sw = np.sqrt(Wt[n, j])
            code, _ = scipy.cluster.vq.vq((S[n, j] * sw)[None], CW[j] * sw[None])
            assert idx[n, j] == code[0]


def test_single_nonzero_weight_is_1d_nearest():
    r = _rng(3)
    N, D, E = 50, 16, 32
    S = r.normal(size=(N, 1, D))
    CW = r.normal(size=(1, E, D))
    Wt = np.zeros((N, 1, D))
    Wt[:, 0, 5] = 2.5
    idx, _ = O.encode_ref(S, CW, Wt)
    expect = np.argmin(np.abs(S[:, 0, 5][:, None] - CW[0, :, 5][None, :]), axis=1)
    np.testing.assert_array_equal(idx[:, 0], expect)


def test_bruteforce_total_distortion_tiny():
    # E=4 centroids, 5 sub-vectors: enumerate all 4^5 assignments.
    r = _rng(4)
    n, D, E = 5, 3, 4
    S = r.normal(size=(n, 1, D))
    CW = r.normal(size=(1, E, D))
    Wt = np.exp(r.normal(size=(n, 1, D)))
    idx, _ = O.encode_ref(S, CW, Wt)
    best, best_a = math.inf, None
    for a in itertools.product(range(E), repeat=n):
        tot = 0.0
        for k in range(n):
            diff = S[k, 0] - CW[0, a[k]]
            tot += float(np.sum(Wt[k, 0] * diff * diff))
        if tot < best:
            best, best_a = tot, a
    assert tuple(int(x) for x in idx[:, 0]) == best_a


def test_weight_scale_invariance_and_centroid_permutation():
    r = _rng(5)
    N, J, D, E = 200, 2, 16, 256
    S = r.normal(size=(N, J, D))
    CW = r.normal(size=(J, E, D))
    Wt = np.exp(r.normal(size=(N, J, D)))
    idx, _ = O.encode_ref(S, CW, Wt)
    idx2, _ = O.encode_ref(S, CW, Wt * 7.25)
    np.testing.assert_array_equal(idx, idx2)
    perm = r.permutation(E)
    CWp = CW[:, perm, :]
    idx3, _ = O.encode_ref(S, CWp, Wt)
    np.testing.assert_array_equal(perm[idx3.astype(int)], idx.astype(int))


def test_expansion_form_agrees_with_direct_form():
    r = _rng(6)
    N, J, D, E = 64, 2, 16, 256
    S = r.normal(size=(N, J, D))
    CW = r.normal(size=(J, E, D))
    Wt = np.exp(r.normal(size=(N, J, D)))
    dist = O.weighted_sq_dist(S, CW, Wt)
    for j in range(J):
        w = Wt[:, j]
        expd = ((w * S[:, j] ** 2).sum(1)[:, None]
                - 2.0 * (w * S[:, j]) @ CW[j].T
                + w @ (CW[j] ** 2).T)
        np.testing.assert_allclose(dist[:, j], expd, rtol=1e-9, atol=1e-9)


def test_exact_ties_take_smallest_index():
    r = _rng(7)
    D, E = 16, 8
    CW = r.normal(size=(1, E, D))
    CW[0, 5] = CW[0, 2]          # duplicate codeword
    S = CW[0, 2][None, None, :] + 0.0
    idx, dist = O.encode_ref(S, CW)
    assert idx[0, 0] == 2 and dist[0, 0, 2] == 0.0 and dist[0, 0, 5] == 0.0


def test_group_weights_broadcast_over_tokens():
    r = _rng(8)
    g, N, H, d, c, E = 4, 30, 2, 16, 4, 16
    X = r.normal(size=(g, N, H, d))
    cb = r.normal(size=(H, g, d // c, E, c))
    w1 = np.exp(r.normal(size=(g, 1, H, d)))
    a, _ = O.encode_group_ref(X, cb, w1)
    b, _ = O.encode_group_ref(X, cb, np.broadcast_to(w1, (g, N, H, d)).copy())
    np.testing.assert_array_equal(a, b)


# --------------------------------------------------------------------------
# Exact codebook: if every sub-vector is a codeword, encoding returns the
# codeword's index with distance 0, dequantisation gives back the cache at
# every loop step, and attention equals torch's textbook SDPA.
# --------------------------------------------------------------------------

def _bf16_exact(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _exact_case(seed, g=4, c=4, d=64, n=120, E=256):
    r = _rng(seed)
    J = d // c
    cb = _bf16_exact(r.normal(size=(g, J, E, c))).astype(np.float64)
    # make codewords distinct: offset codeword e by e * 2^-4 on one element
    cb[0, :, :, 0] = _bf16_exact(np.round(cb[0, :, :, 0]) + np.arange(E)[None, :] / 16.0)
    idx = r.integers(0, E, size=(n, J))
    X = np.empty((g, n, 1, d))
    for tau in range(g):
        for v in range(n):
            for j in range(J):
                for ch in range(c):
                    X[tau, v, 0, j * c + ch] = cb[tau, j, idx[v, j], ch]
    return cb, idx, X


def test_exact_codebook_encode_returns_indices():
    cb, idx, X = _exact_case(9)
    got, dist = O.encode_group_ref(X, cb[None])
    np.testing.assert_array_equal(got[:, 0], idx)
    assert np.all(dist[:, 0][np.arange(idx.shape[0])[:, None], np.arange(idx.shape[1])[None, :],
                             idx] == 0.0)


def test_exact_codebook_dequant_reproduces_every_loop_step():
    cb, idx, X = _exact_case(10)
    for tau in range(cb.shape[0]):
        np.testing.assert_array_equal(O.dequant_ref(idx, cb, tau), X[tau, :, 0])


def test_exact_codebook_attention_equals_sdpa():
    r = _rng(11)
    cbK, idxK, XK = _exact_case(12)
    cbV, idxV, XV = _exact_case(13)
    d = XK.shape[-1]
    win_K = _bf16_exact(r.normal(size=(72, d)))
    win_V = _bf16_exact(r.normal(size=(72, d)))
    q = _bf16_exact(r.normal(size=d))
    scale = 1.0 / math.sqrt(d)
    for tau in range(4):
        out, lse = O.decode_attn_ref(q, win_K, win_V, idxK, idxV, cbK, cbV, tau, scale)
        K = torch.from_numpy(np.concatenate([win_K, XK[tau, :, 0]])).double()
        V = torch.from_numpy(np.concatenate([win_V, XV[tau, :, 0]])).double()
        qt = torch.from_numpy(q).double()
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt[None, None, None], K[None, None], V[None, None], scale=scale)[0, 0, 0]
        np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
        z = scale * (K.numpy() @ q)
        assert abs(lse - scipy.special.logsumexp(z)) < 1e-12


# --------------------------------------------------------------------------
# Attention invariants and the split/merge identity.
# --------------------------------------------------------------------------

def test_attention_matches_sdpa_and_logsumexp():
    r = _rng(14)
    n, d = 333, 128
    q, K, V = r.normal(size=d), r.normal(size=(n, d)) * 3, r.normal(size=(n, d))
    scale = 1 / math.sqrt(d)
    out, lse = O.attn_ref(q, K, V, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], scale=scale)[0, 0, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert abs(lse - scipy.special.logsumexp(scale * K @ q)) < 1e-12
    p = O.softmax_weights_ref(q, K, scale)
    assert abs(p.sum() - 1.0) < 1e-12
    np.testing.assert_allclose(p @ V, out, rtol=1e-12, atol=1e-12)


def test_attention_token_order_invariance():
    r = _rng(15)
    n, d = 200, 64
    q, K, V = r.normal(size=d), r.normal(size=(n, d)), r.normal(size=(n, d))
    perm = r.permutation(n)
    a, la = O.attn_ref(q, K, V, 0.125)
    b, lb = O.attn_ref(q, K[perm], V[perm], 0.125)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    assert abs(la - lb) < 1e-12


def test_all_equal_scores_give_mean_of_values():
    r = _rng(16)
    n, d = 97, 32
    K, V = r.normal(size=(n, d)), r.normal(size=(n, d))
    out, lse = O.attn_ref(np.zeros(d), K, V, 0.5)
    np.testing.assert_allclose(out, V.mean(axis=0), rtol=1e-12, atol=1e-13)
    assert abs(lse - math.log(n)) < 1e-12


@pytest.mark.parametrize("cuts", [[1], [50], [199], [7, 100, 150], list(range(10, 200, 10))])
def test_split_merge_equals_full(cuts):
    r = _rng(17)
    n, d = 200, 48
    q, K, V = r.normal(size=d) * 4, r.normal(size=(n, d)), r.normal(size=(n, d))
    full, lf = O.attn_ref(q, K, V, 0.3)
    bounds = [0] + cuts + [n]
    parts = [O.attn_partial_ref(q, K[a:b], V[a:b], 0.3) for a, b in zip(bounds[:-1], bounds[1:])]
    parts.append(O.attn_partial_ref(q, K[:0], V[:0], 0.3))   # an empty split
    out, lse = O.merge_partials_ref(parts)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)
    assert abs(lse - lf) < 1e-12


# --------------------------------------------------------------------------
# Windows: the first 8 and the latest 64 tokens stay bf16 (airadar.tv,
# section "Utilisation": PREFIX_TOKENS=8 RECENT_TOKENS=64).
# --------------------------------------------------------------------------

def test_window_counts_by_enumeration():
    for N in range(0, 300):
        win = [p for p in range(N) if p < 8 or p >= N - 64]
        vq = [p for p in range(N) if not (p < 8 or p >= N - 64)]
        assert O.n_window_tokens(N) == len(win)
        assert O.n_vq_tokens(N) == len(vq)
        if vq:
            assert vq[0] == 8 and vq[-1] == N - 65


def test_short_context_is_plain_attention():
    r = _rng(18)
    d, J = 64, 16
    for N in (1, 9, 72):
        K, V = _bf16_exact(r.normal(size=(N, d))), _bf16_exact(r.normal(size=(N, d)))
        q = _bf16_exact(r.normal(size=d))
        cb = r.normal(size=(4, J, 256, 4))
        empty = np.zeros((O.n_vq_tokens(N), J), dtype=np.uint8)
        out, lse = O.decode_attn_ref(q, K, V, empty, empty, cb, cb, 1, 0.125)
        ref, lref = O.attn_ref(q, K, V, 0.125)
        np.testing.assert_array_equal(out, ref)
        assert lse == lref


# --------------------------------------------------------------------------
# The packed pool format (the library's own storage layout, as the header
# states it): a hand-worked table of offsets plus a bijection check.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("J", [12, 16, 24, 32, 8, 4, 20, 28])
@pytest.mark.parametrize("kv", [0, 1])
def test_plane_offsets_form_a_bijection(J, kv):
    n = 3 * O.rotation_block(J)
    seen = set()
    for slot in range(n):
        for j in range(J):
            seen.add(O.plane_offset(slot, j, J, kv, n))
    assert seen == set(range(n * J))


@pytest.mark.parametrize("J", [12, 16, 24, 32, 8])
def test_rotation_spreads_lanes_over_distinct_columns(J):
    # at every step s, the slots of one block read distinct (replica, group)
    # pairs, each group appearing floor(32/J) times: the property the format
    # exists for.
    lb = O.rotation_block(J)
    for s in range(J):
        cols = []
        for rot in range(lb):
            pos_of = {(j - rot) % J: j for j in range(J)}
            cols.append((rot // J, pos_of[s]))
        assert len(set(cols)) == lb


def test_plane_offsets_hand_worked():
    # J=32, granule 16. slot 0, group 0 -> pos 0 -> byte 0.
    assert O.plane_offset(0, 0, 32) == 0
    # slot 1 (lane 1), group 1 -> pos 0 -> granule 0, lane 1 -> 16.
    assert O.plane_offset(1, 1, 32) == 16
    # slot 1, group 0 -> pos 31 -> granule 1 (512 B in), lane 1 (16), byte 15.
    assert O.plane_offset(1, 0, 32) == 512 + 16 + 15
    # slot 33 is lane 1 of block 1 (1024 B in): group 1 -> 1024 + 16.
    assert O.plane_offset(33, 1, 32) == 1024 + 16
    # J=12: LB=24, granule 4. slot 2, group 0 -> pos 10 -> granule 2
    # (2*24*4 = 192), row 2 (8), byte 2.
    assert O.plane_offset(2, 0, 12) == 192 + 8 + 2
    # J=12, slot 31 is row 7 of block 1 (24*12 = 288 B in): group 7 -> pos 0.
    assert O.plane_offset(31, 7, 12) == 288 + 28
    # J=24, granule 8. slot 5, group 6 -> pos 1 -> 5*8 + 1.
    assert O.plane_offset(5, 6, 24) == 41
    # The V plane has the same layout. J=32: slot 5, group 3 -> pos 30 ->
    # granule 1 (512), row 5 (80), byte 14.
    assert O.plane_offset(5, 3, 32, 1, 64) == 512 + 80 + 14
    # J=12: slot 95 is row 23 of block 3 (3*288 = 864): group 11 -> pos 0 ->
    # granule 0, row 23 (92), byte 0.
    assert O.plane_offset(95, 11, 12, 1, 96) == 864 + 92


def test_pack_unpack_round_trip():
    r = _rng(19)
    J, Pg, n = 12, 96, 250
    iK = r.integers(0, 256, size=(n, J)).astype(np.uint8)
    iV = r.integers(0, 256, size=(n, J)).astype(np.uint8)
    pages = [4, 0, 2]
    arr = O.pack_pages(iK, iV, pages, 5, Pg)
    assert arr.shape == (5, 2, Pg * J)
    k2, v2 = O.unpack_pages(arr, pages, n, J, Pg)
    np.testing.assert_array_equal(k2, iK)
    np.testing.assert_array_equal(v2, iV)
    assert not arr[1].any() and not arr[3].any()


@pytest.mark.parametrize("J", [12, 16, 32, 24])
def test_vector_packer_matches_scalar_packer(J):
    r = _rng(20)
    Pg = 2 * O.rotation_block(J) if O.rotation_block(J) != 32 else 64
    n = 3 * Pg - 5
    iK = r.integers(0, 256, size=(n, J)).astype(np.uint8)
    iV = r.integers(0, 256, size=(n, J)).astype(np.uint8)
    pages = [3, 1, 0]
    ref = O.pack_pages(iK, iV, pages, 4, Pg)
    pool = np.zeros((4, 2, Pg * J), dtype=np.uint8)
    O.pack_sequence(pool, iK, np.array(pages), Pg, 0)
    O.pack_sequence(pool, iV, np.array(pages), Pg, 1)
    np.testing.assert_array_equal(pool, ref)
    np.testing.assert_array_equal(O.unpack_sequence(pool, n, J, np.array(pages), Pg, 1), iV)
    for s in range(0, Pg, 7):
        for kv in (0, 1):
            np.testing.assert_array_equal(O.plane_offsets(np.array([s]), J, kv, Pg)[0],
                                          [O.plane_offset(s, j, J, kv, Pg) for j in range(J)])


# ---------------------------------------------------------------------------
# Weighted k-means (Lloyd) step: scipy's kmeans2, token replication,
# optimality of the update, descent of the objective
# ---------------------------------------------------------------------------

def _lloyd_case(seed, N=600, H=1, d=16, g=2, c=4, E=256, per_element=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((g, N, H, d))
    cb = rng.standard_normal((H, g, d // c, E, c)) * 0.8
    w = rng.lognormal(0.0, 1.0, (g, N, H, d)) if per_element else None
    return X, cb, w


def test_unweighted_lloyd_step_matches_scipy_kmeans2():
    # one iteration of scipy's kmeans2 from a given code book is the same
    # step: assignment by vq, then means, empty clusters kept in place
    X, cb, _ = _lloyd_case(11, N=700, E=64)
    idx, new = O.kmeans_step_group_ref(X, cb)
    S = O.subvectors(X, 4)
    CW = O.codewords(cb[0])
    empty = 0
    for j in range(S.shape[2]):
        import warnings
        with warnings.catch_warnings():
            warnings.simplefilter("ignore")
            ref_cb, ref_lab = scipy.cluster.vq.kmeans2(S[:, 0, j, :], CW[j].copy(), iter=1,
                                                       minit="matrix")
        np.testing.assert_array_equal(idx[:, 0, j], ref_lab)
        np.testing.assert_allclose(O.codewords(new[0])[j], ref_cb, rtol=1e-12, atol=1e-12)
        empty += int(np.sum(np.bincount(ref_lab, minlength=64) == 0))
    assert empty > 0                       # the kept-in-place rule was exercised


def test_integer_token_weights_equal_token_replication():
    # a weight k on every element of a token is the token counted k times
    X, cb, _ = _lloyd_case(12, N=300, E=32)
    rng = np.random.default_rng(13)
    k = rng.integers(1, 5, size=X.shape[1])
    w = np.broadcast_to(k[None, :, None, None].astype(np.float64), X.shape).copy()
    idx_w, new_w = O.kmeans_step_group_ref(X, cb, w)
    Xr = np.repeat(X, k, axis=1)
    idx_r, new_r = O.kmeans_step_group_ref(Xr, cb)
    np.testing.assert_array_equal(np.repeat(idx_w, k, axis=0), idx_r)
    np.testing.assert_allclose(new_w, new_r, rtol=1e-12, atol=1e-12)
    S = O.subvectors(Xr, 4)
    for j in range(S.shape[2]):
        ref_cb, _ = scipy.cluster.vq.kmeans2(S[:, 0, j, :], O.codewords(cb[0])[j].copy(), iter=1,
                                             minit="matrix", missing="warn")
        np.testing.assert_allclose(O.codewords(new_w[0])[j], ref_cb, rtol=1e-12, atol=1e-12)


def test_weighted_update_is_the_clusters_minimiser():
    # for the given assignment, each updated element zeroes the gradient of
    # the cluster's weighted distortion, and moving it only costs more
    X, cb, w = _lloyd_case(14, N=500, E=16)
    idx, new = O.kmeans_step_group_ref(X, cb, w)
    S, Wt = O.subvectors(X, 4)[:, 0], O.subvector_weights(w, X.shape[1], 4)[:, 0]
    CW = O.codewords(new[0])
    rng = np.random.default_rng(15)
    for j in range(S.shape[1]):
        for e in np.unique(idx[:, 0, j]):
            m = idx[:, 0, j] == e
            grad = (Wt[m, j] * (CW[j, e] - S[m, j])).sum(axis=0)
            assert np.max(np.abs(grad)) < 1e-9 * max(1.0, Wt[m, j].sum())
            base = (Wt[m, j] * (S[m, j] - CW[j, e]) ** 2).sum()
            for _ in range(3):
                moved = CW[j, e] + rng.normal(0, 1e-3, CW.shape[2])
                assert (Wt[m, j] * (S[m, j] - moved) ** 2).sum() > base


def test_weight_scale_leaves_the_step_unchanged():
    X, cb, w = _lloyd_case(16, N=400, E=32)
    i1, n1 = O.kmeans_step_group_ref(X, cb, w)
    i2, n2 = O.kmeans_step_group_ref(X, cb, w * 7.5)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(n1, n2, rtol=1e-12, atol=1e-13)


def test_lloyd_steps_never_increase_the_weighted_distortion():
    X, cb, w = _lloyd_case(17, N=800, H=2, E=32)
    idx, _ = O.encode_group_ref(X, cb, w)
    prev = O.weighted_distortion_ref(X, cb, idx, w)
    for _ in range(4):
        idx, cb = O.kmeans_step_group_ref(X, cb, w)
        after_update = O.weighted_distortion_ref(X, cb, idx, w)
        assert after_update <= prev * (1 + 1e-12)
        idx, _ = O.encode_group_ref(X, cb, w)
        prev2 = O.weighted_distortion_ref(X, cb, idx, w)
        assert prev2 <= after_update * (1 + 1e-12)
        prev = prev2


def test_empty_clusters_and_zero_weights_keep_their_codewords():
    X, cb, w = _lloyd_case(18, N=50, E=256)
    w[:, :, :, 0] = 0.0                    # element 0 of group 0 (channel 0, every loop) has no weight
    idx, new = O.kmeans_step_group_ref(X, cb, w)
    used = np.zeros((cb.shape[2], cb.shape[3]), dtype=bool)
    for j in range(cb.shape[2]):
        used[j, np.unique(idx[:, 0, j])] = True
    assert (~used).sum() > 0
    for j in range(cb.shape[2]):
        np.testing.assert_array_equal(new[0, :, j][:, ~used[j]], cb[0, :, j][:, ~used[j]])
    # channel 0 is element tau*c + 0 of group 0 for every tau: kept where weight-free
    np.testing.assert_array_equal(new[0, :, 0, :, 0], cb[0, :, 0, :, 0])


def test_update_with_a_given_assignment_uses_it():
    X, cb, w = _lloyd_case(19, N=200, E=16)
    rng = np.random.default_rng(20)
    forced = rng.integers(0, 16, size=(X.shape[1], 1, 4)).astype(np.uint8)
    idx, new = O.kmeans_step_group_ref(X, cb, w, assign=forced)
    np.testing.assert_array_equal(idx, forced)
    S, Wt = O.subvectors(X, 4)[:, 0], O.subvector_weights(w, X.shape[1], 4)[:, 0]
    m = forced[:, 0, 2] == 5
    want = (Wt[m, 2] * S[m, 2]).sum(0) / Wt[m, 2].sum(0)
    np.testing.assert_allclose(O.codewords(new[0])[2, 5], want, rtol=1e-12)


def test_lloyd_step_shared_weights_equal_repeated_per_token_weights():
    # a weight vector shared over tokens ([g][1][H][d]) is the same vector given to every token
    X, cb, w = _lloyd_case(21, N=300, H=2, E=32)
    shared = w[:, :1]
    i1, n1 = O.kmeans_step_group_ref(X, cb, shared)
    i2, n2 = O.kmeans_step_group_ref(X, cb, np.repeat(shared, X.shape[1], axis=1))
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(n1, n2, rtol=0, atol=0)


def test_weighted_distortion_hand_worked():
    # g = 2 loop steps, c = 2 channels, one head, d = 2 (J = 1), D = 4; two
    # tokens, two centroids, unequal weights. Loop-major sub-vectors:
    #   s0 = (1, 2, 3, 4), s1 = (0, -1, 2, 0); codewords c0 = (1, 1, 1, 1),
    #   c1 = (0, 0, 2, 2); weights w0 = (2, 1, 0.5, 3), w1 = (1, 4, 2, 0).
    # Assignment (0, 1):
    #   token 0: w0 . (0, 1, 2, 3)^2 = 0 + 1 + 2 + 27 = 30
    #   token 1: w1 . (0, -1, 0, -2)^2 = 0 + 4 + 0 + 0 = 4           -> 34
    # Unweighted: 14 + 5 = 19. Assignment (1, 0):
    #   w0 . (1, 2, 1, 2)^2 = 18.5;  w1 . (-1, -2, 1, -1)^2 = 19     -> 37.5
    # Weights shared over tokens (token 0's vector for both):
    #   30 + (2, 1, 0.5, 3) . (0, 1, 0, 4) = 30 + 13                   -> 43
    X = np.zeros((2, 2, 1, 2))
    X[0, 0, 0], X[1, 0, 0] = (1, 2), (3, 4)
    X[0, 1, 0], X[1, 1, 0] = (0, -1), (2, 0)
    cb = np.zeros((1, 2, 1, 2, 2))                      # [H][g][J][E][c]
    cb[0, 0, 0, 0], cb[0, 1, 0, 0] = (1, 1), (1, 1)
    cb[0, 0, 0, 1], cb[0, 1, 0, 1] = (0, 0), (2, 2)
    w = np.zeros((2, 2, 1, 2))
    w[0, 0, 0], w[1, 0, 0] = (2, 1), (0.5, 3)
    w[0, 1, 0], w[1, 1, 0] = (1, 4), (2, 0)
    a01 = np.array([[[0]], [[1]]], dtype=np.uint8)        # [N][H][J]
    a10 = np.array([[[1]], [[0]]], dtype=np.uint8)
    assert O.weighted_distortion_ref(X, cb, a01, w) == 34.0
    assert O.weighted_distortion_ref(X, cb, a01, None) == 19.0
    assert O.weighted_distortion_ref(X, cb, a10, w) == 37.5
    assert O.weighted_distortion_ref(X, cb, a01, w[:, :1]) == 43.0
    # the encoder agrees: under these weights token 0 prefers c1 (18.5 < 30)
    idx, dist = O.encode_group_ref(X, cb, w)
    assert dist[0, 0, 0].tolist() == [30.0, 18.5] and dist[1, 0, 0].tolist() == [19.0, 4.0]
    assert idx[:, 0, 0].tolist() == [1, 1]
