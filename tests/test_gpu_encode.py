"""GPU parity of loopvq_encode (through the C ABI) against the oracle's
brute-force float64 argmin. Indices are bit-exact except in near ties (the
oracle's best two distances within 1e-5 relative), where the GPU's choice
must be within that margin of the best."""

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from synthetic import SHAPES, Shape, codebooks_for_layer, loop_group_kv, weights

from _cases import check_indices, random_codebooks

from _guard import Guarded

pytestmark = pytest.mark.gpu

W128 = Shape("w128", n_layers=2, n_kv_heads=2, n_q_heads=2, head_dim=128, n_loops=8,
             loop_group=4, chan_group=4, batch=1, context=0, head_scale=(0.5, 2.0), seed=201)
J12 = Shape("j12e", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=96, n_loops=4, loop_group=4,
            chan_group=8, batch=1, context=0, page_tokens=96, kind="ar1", seed=202)


def _cfg(s: Shape, n_layers: int, n_pages: int) -> L.LoopVQConfig:
    return L.LoopVQConfig(n_layers=n_layers, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                          head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                          chan_group=s.chan_group, n_pages=n_pages, max_batch=1,
                          max_pages_per_seq=n_pages, prefix_tokens=s.prefix,
                          recent_tokens=s.recent, page_tokens=s.page_tokens)


def _run(s, n_layers, layer, gamma, kv, x, w, cb, slots, n_pages):
    cfg = _cfg(s, n_layers, n_pages)
    pool = Guarded((n_layers, s.n_kv_heads, s.G, n_pages, 2, s.page_tokens * s.J), torch.uint8,
                   fill=0)
    L.loopvq_encode(cfg, layer, gamma, kv, x.cuda() if x.device.type == "cpu" else x,
                    None if w is None else w.cuda(), cb.cuda(),
                    torch.as_tensor(slots, dtype=torch.int64).cuda(), pool.t)
    pool.check("pool")
    return pool.t.cpu().numpy()


def _gpu_indices(pool, s, layer, gamma, kv, slots):
    out = np.zeros((len(slots), s.n_kv_heads, s.J), dtype=np.uint8)
    for n, sl in enumerate(slots):
        if sl < 0:
            continue
        page, slot = divmod(int(sl), s.page_tokens)
        off = O.plane_offsets(np.array([slot]), s.J, kv, s.page_tokens)[0]
        for h in range(s.n_kv_heads):
            out[n, h] = pool[layer, h, gamma, page, kv, off]
    return out


def _slots(n, n_pages, Pg, seed, skip_every=0):
    r = np.random.default_rng(seed)
    slots = r.permutation(n_pages * Pg)[:n].astype(np.int64)
    if skip_every:
        slots[::skip_every] = -1
    return slots


@pytest.mark.parametrize("kv", [0, 1])
def test_tiny_config_fitted_codebooks(kv):
    s = SHAPES["tiny"]
    n = s.n_vq
    x = loop_group_kv(s, 0, 0, kv, n)
    cb = codebooks_for_layer(s, 0, n_samples=1024)[None]          # [1][H][G][2][g][J][E][c]
    n_pages = 8
    slots = np.arange(n, dtype=np.int64)                           # contiguous, page order
    pool = _run(s, 1, 0, 0, kv, x, None, cb, slots, n_pages)
    idx_ref, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, kv].double().numpy())
    got = _gpu_indices(pool, s, 0, 0, kv, slots)
    check_indices(got, dist)
    # and the pool bytes are exactly the oracle's packing of those indices
    ref_pool = np.zeros_like(pool[0, 0, 0])
    O.pack_sequence(ref_pool, idx_ref[:, 0], np.arange(n_pages), s.page_tokens, kv)
    if (got == idx_ref).all():
        np.testing.assert_array_equal(pool[0, 0, 0], ref_pool)


@pytest.mark.parametrize("per_token", [True, False])
def test_weighted_encode_with_skips_and_paging(per_token):
    s = W128
    n, n_pages, layer, gamma, kv = 300, 7, 1, 1, 0
    x = loop_group_kv(s, layer, gamma, kv, n)
    w = weights(s, n, per_token, layer, gamma, kv)
    cb = random_codebooks(s, 2, 5)
    slots = _slots(n, n_pages, s.page_tokens, 9, skip_every=7)
    pool = _run(s, 2, layer, gamma, kv, x, w, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[layer, :, gamma, kv].double().numpy(),
                                 w.double().numpy())
    got = _gpu_indices(pool, s, layer, gamma, kv, slots)
    keep = slots >= 0
    check_indices(got[keep], dist[keep])
    # skipped tokens, other layers, other groups and the V planes stay untouched
    assert not pool[0].any() and not pool[layer, :, 0].any() and not pool[:, :, :, :, 1].any()
    written = set()
    for sl in slots[keep]:
        page, slot = divmod(int(sl), s.page_tokens)
        for o in O.plane_offsets(np.array([slot]), s.J, kv, s.page_tokens)[0]:
            written.add((page, int(o)))
    mask = np.zeros((n_pages, s.page_tokens * s.J), dtype=bool)
    for page, o in written:
        mask[page, o] = True
    assert not pool[layer, :, gamma, :, kv][:, ~mask].any()


def test_j12_quarter_bit_encode():
    s = J12
    n, n_pages = 500, 6
    x = loop_group_kv(s, 0, 0, 1, n)
    cb = random_codebooks(s, 1, 6)
    slots = _slots(n, n_pages, s.page_tokens, 10)
    pool = _run(s, 1, 0, 0, 1, x, None, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 1].double().numpy())
    check_indices(_gpu_indices(pool, s, 0, 0, 1, slots), dist)


def test_exact_codewords_and_duplicate_ties():
    # sub-vectors equal to bf16-representable codewords: distance 0, exact
    # index; duplicated codewords resolve to the smaller index.
    s = W128.with_(n_kv_heads=1, n_q_heads=1)
    g, J, c, E = s.loop_group, s.J, s.chan_group, 256
    gen = torch.Generator().manual_seed(3)
    cb = torch.randn(1, 1, s.G, 2, g, J, E, c, generator=gen).to(torch.bfloat16).float()
    cb[0, 0, 0, 0, :, :, 200] = cb[0, 0, 0, 0, :, :, 17]        # codeword 200 == 17
    n = 256
    idx = torch.randint(0, E, (n, J), generator=gen)
    idx[:5] = 200
    x = torch.empty(g, n, 1, s.head_dim)
    for tau in range(g):
        for j in range(J):
            x[tau, :, 0, j * c:(j + 1) * c] = cb[0, 0, 0, 0, tau, j][idx[:, j]]
    x = x.to(torch.bfloat16)
    slots = np.arange(n, dtype=np.int64)
    pool = _run(s, 1, 0, 0, 0, x, None, cb, slots, 4)
    got = _gpu_indices(pool, s, 0, 0, 0, slots)[:, 0].astype(np.int64)
    expect = idx.numpy().copy()
    expect[expect == 200] = 17
    np.testing.assert_array_equal(got, expect)


def test_strided_input_views():
    s = W128.with_(n_kv_heads=2)
    n = 200
    big = loop_group_kv(s, 0, 0, 0, 2 * n)
    x = big[:, ::2]                                               # token stride 2*H*d
    assert x.stride(1) == 2 * s.n_kv_heads * s.head_dim
    cb = random_codebooks(s, 1, 8)
    slots = _slots(n, 5, s.page_tokens, 11)
    pool = _run(s, 1, 0, 0, 0, big.cuda()[:, ::2], None, cb, slots, 5)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 0].double().numpy())
    check_indices(_gpu_indices(pool, s, 0, 0, 0, slots), dist)


def test_zero_tokens_is_a_noop():
    s = W128
    cfg = _cfg(s, 2, 3)
    pool = torch.zeros(10, dtype=torch.uint8, device="cuda")
    x = torch.zeros(s.loop_group, 0, s.n_kv_heads, s.head_dim, dtype=torch.bfloat16, device="cuda")
    L.loopvq_encode(cfg, 0, 0, 0, x, None, torch.zeros(16, device="cuda"),
                    torch.zeros(1, dtype=torch.int64, device="cuda"), pool)
    torch.cuda.synchronize()
    assert not pool.any()


@pytest.mark.parametrize("n", [1, 8, 37, 64])
def test_small_batches_weighted_with_skips(n):
    # batches of at most 64 tokens (the window eviction at each decode step)
    # take the warp-per-token kernel
    s = W128
    layer, gamma, kv, n_pages = 1, 0, 1, 3
    x = loop_group_kv(s, layer, gamma, kv, n)
    w = weights(s, n, True, layer, gamma, kv)
    cb = random_codebooks(s, 2, 12)
    slots = _slots(n, n_pages, s.page_tokens, 13, skip_every=5 if n > 5 else 0)
    pool = _run(s, 2, layer, gamma, kv, x, w, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[layer, :, gamma, kv].double().numpy(),
                                 w.double().numpy())
    keep = slots >= 0
    check_indices(_gpu_indices(pool, s, layer, gamma, kv, slots)[keep], dist[keep])


def test_small_batch_j12_and_ties():
    s = J12
    n, n_pages = 24, 2
    x = loop_group_kv(s, 0, 0, 0, n)
    cb = random_codebooks(s, 1, 14)
    slots = _slots(n, n_pages, s.page_tokens, 15)
    pool = _run(s, 1, 0, 0, 0, x, None, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 0].double().numpy())
    check_indices(_gpu_indices(pool, s, 0, 0, 0, slots), dist)
    # exact codewords with a duplicated codeword: the smaller index wins
    t = W128.with_(n_kv_heads=1, n_q_heads=1)
    g, J, c, E = t.loop_group, t.J, t.chan_group, 256
    gen = torch.Generator().manual_seed(16)
    cbt = torch.randn(1, 1, t.G, 2, g, J, E, c, generator=gen).to(torch.bfloat16).float()
    cbt[0, 0, 0, 1, :, :, 250] = cbt[0, 0, 0, 1, :, :, 3]        # codeword 250 == 3
    m = 40
    idx = torch.randint(0, E, (m, J), generator=gen)
    idx[::3] = 250
    xt = torch.empty(g, m, 1, t.head_dim)
    for tau in range(g):
        for jj in range(J):
            xt[tau, :, 0, jj * c:(jj + 1) * c] = cbt[0, 0, 0, 1, tau, jj][idx[:, jj]]
    pool = _run(t, 1, 0, 0, 1, xt.to(torch.bfloat16), None, cbt, np.arange(m, dtype=np.int64), 2)
    got = _gpu_indices(pool, t, 0, 0, 1, np.arange(m))[:, 0].astype(np.int64)
    expect = idx.numpy().copy()
    expect[expect == 250] = 3
    np.testing.assert_array_equal(got, expect)


@pytest.mark.parametrize("per_token", [True, False])
def test_prefill_batches_take_the_tensor_core_form(per_token):
    # batches of 2048 tokens and more: tcgen05 contraction plus exact rescore
    s = W128
    n, n_pages, layer, gamma, kv = 2100, 40, 0, 1, 0
    x = loop_group_kv(s, layer, gamma, kv, n)
    w = weights(s, n, per_token, layer, gamma, kv)
    cb = random_codebooks(s, 2, 21)
    slots = _slots(n, n_pages, s.page_tokens, 22, skip_every=11)
    pool = _run(s, 2, layer, gamma, kv, x, w, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[layer, :, gamma, kv].double().numpy(),
                                 w.double().numpy())
    keep = slots >= 0
    check_indices(_gpu_indices(pool, s, layer, gamma, kv, slots)[keep], dist[keep])


def test_prefill_tensor_core_j12_fitted_and_ties():
    s = J12
    n, n_pages = 2304, 26
    x = loop_group_kv(s, 0, 0, 1, n)
    cb = codebooks_for_layer(s, 0, n_samples=2048, iters=8)[None]
    slots = _slots(n, n_pages, s.page_tokens, 23)
    pool = _run(s, 1, 0, 0, 1, x, None, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 1].double().numpy())
    check_indices(_gpu_indices(pool, s, 0, 0, 1, slots), dist)
    # exact codewords with a duplicated codeword through the tensor-core form
    t = W128.with_(n_kv_heads=1, n_q_heads=1)
    g, J, c, E = t.loop_group, t.J, t.chan_group, 256
    gen = torch.Generator().manual_seed(24)
    cbt = torch.randn(1, 1, t.G, 2, g, J, E, c, generator=gen).to(torch.bfloat16).float()
    cbt[0, 0, 0, 0, :, :, 99] = cbt[0, 0, 0, 0, :, :, 5]          # codeword 99 == 5
    m = 2048
    idx = torch.randint(0, E, (m, J), generator=gen)
    idx[::7] = 99
    xt = torch.empty(g, m, 1, t.head_dim)
    for tau in range(g):
        for jj in range(J):
            xt[tau, :, 0, jj * c:(jj + 1) * c] = cbt[0, 0, 0, 0, tau, jj][idx[:, jj]]
    pool = _run(t, 1, 0, 0, 0, xt.to(torch.bfloat16), None, cbt, np.arange(m, dtype=np.int64), 33)
    got = _gpu_indices(pool, t, 0, 0, 0, np.arange(m))[:, 0].astype(np.int64)
    expect = idx.numpy().copy()
    expect[expect == 99] = 5
    np.testing.assert_array_equal(got, expect)


def test_prefill_tensor_core_d8():
    # c = 2, g = 4: 8-element sub-vectors, K' = 48
    s = Shape("c2enc", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=64, n_loops=4, loop_group=4,
              chan_group=2, batch=1, context=0, seed=203)
    n, n_pages = 2200, 36
    x = loop_group_kv(s, 0, 0, 0, n)
    w = weights(s, n, True, 0, 0, 0)
    cb = random_codebooks(s, 1, 25)
    slots = _slots(n, n_pages, s.page_tokens, 26)
    pool = _run(s, 1, 0, 0, 0, x, w, cb, slots, n_pages)
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 0].double().numpy(),
                                 w.double().numpy())
    check_indices(_gpu_indices(pool, s, 0, 0, 0, slots), dist)


def test_eviction_encode_of_every_layer_group_and_plane_in_one_launch():
    # The one-launch eviction encode writes, for every (layer, loop group,
    # K/V), exactly the bytes that loopvq_encode writes for that combination
    # (the same float32 arithmetic), and those indices are the oracle's
    # nearest centroids; skipped slots and every other byte stay untouched.
    s = Shape("evict", n_layers=2, n_kv_heads=2, n_q_heads=2, head_dim=64, n_loops=8,
              loop_group=4, chan_group=4, batch=1, context=0, seed=210)
    L_, G, n, n_pages = 2, s.G, 12, 4
    cfg = _cfg(s, L_, n_pages)
    cb = random_codebooks(s, L_, 211)
    xs = torch.stack([torch.stack([torch.stack([loop_group_kv(s, l, gm, kv, n, stream=3)
                                                for kv in range(2)]) for gm in range(G)])
                      for l in range(L_)])                         # [L][G][2][g][n][H][d]
    slots = _slots(n, n_pages, s.page_tokens, 212, skip_every=5)
    pool = Guarded((L_, s.n_kv_heads, G, n_pages, 2, s.page_tokens * s.J), torch.uint8, fill=0)
    L.loopvq_encode_evict(cfg, xs.cuda(), cb.cuda(), torch.as_tensor(slots).cuda(), pool.t)
    pool.check("pool")
    got = pool.t.cpu().numpy()
    ref = torch.zeros_like(pool.t)
    for l in range(L_):
        for gm in range(G):
            for kv in range(2):
                L.loopvq_encode(cfg, l, gm, kv, xs[l, gm, kv].cuda(), None, cb.cuda(),
                                torch.as_tensor(slots).cuda(), ref)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got, ref.cpu().numpy())
    keep = slots >= 0
    for l in range(L_):
        for gm in range(G):
            for kv in range(2):
                _, dist = O.encode_group_ref(xs[l, gm, kv].double().numpy(),
                                             cb[l, :, gm, kv].double().numpy())
                idx = _gpu_indices(got, s, l, gm, kv, slots)
                check_indices(idx[keep], dist[keep])


def test_slots_past_the_pool_are_skipped_and_flagged():
    # A slot_mapping entry at or past n_pages * page_tokens is not written and
    # sets LOOPVQ_ENCODE_STATUS_BAD_SLOT; a negative one is a plain skip.
    s = SHAPES["tiny"]
    n, n_pages = 40, 2
    cfg = _cfg(s, 1, n_pages)
    cb = random_codebooks(s, 1, 213)
    x = loop_group_kv(s, 0, 0, 0, n, stream=5)
    slots = _slots(n, n_pages, s.page_tokens, 214)
    slots[3] = n_pages * s.page_tokens          # one past the pool
    slots[7] = -1
    L.loopvq_encode_status(clear=True)
    pool = _run(s, 1, 0, 0, 0, x, None, cb, slots, n_pages)
    assert L.loopvq_encode_status(clear=True) & L.LOOPVQ_ENCODE_STATUS_BAD_SLOT
    ok = np.ones(n, dtype=bool)
    ok[[3, 7]] = False
    _, dist = O.encode_group_ref(x.double().numpy(), cb[0, :, 0, 0].double().numpy())
    idx = _gpu_indices(pool, s, 0, 0, 0, np.where(ok, slots, -1))
    check_indices(idx[ok], dist[ok])
    assert L.loopvq_encode_status() == 0        # cleared
