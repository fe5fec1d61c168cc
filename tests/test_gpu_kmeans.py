"""GPU parity of loopvq_kmeans_step (one weighted Lloyd step, through the C
ABI) against the oracle. The assignment follows the encoder's rule (bit-exact
except in near ties); the updated codewords are compared with the oracle's
weighted means computed from the GPU's own assignment, within the float32
summation bound of the member count; elements without weight must keep their
exact value, and codebooks outside the step's (layer, loop group, K/V) must
not change."""

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from synthetic import Shape, loop_group_kv, weights

from _cases import check_indices, random_codebooks
from _guard import Guarded

pytestmark = pytest.mark.gpu

W128 = Shape("km128", n_layers=2, n_kv_heads=2, n_q_heads=2, head_dim=128, n_loops=8,
             loop_group=4, chan_group=4, batch=1, context=0, head_scale=(0.5, 2.0), seed=301)
C8 = Shape("km96", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=96, n_loops=4, loop_group=4,
           chan_group=8, batch=1, context=0, page_tokens=96, kind="ar1", seed=302)
C2 = Shape("km64", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=64, n_loops=4, loop_group=4,
           chan_group=2, batch=1, context=0, seed=303)
EPS32 = 2.0 ** -24


def _cfg(s: Shape, n_layers: int) -> L.LoopVQConfig:
    return L.LoopVQConfig(n_layers=n_layers, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                          head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                          chan_group=s.chan_group, n_pages=1, max_batch=1, max_pages_per_seq=1,
                          page_tokens=s.page_tokens)


def _step(s, n_layers, layer, gamma, kv, x, w, cb_gpu):
    cfg = _cfg(s, n_layers)
    n = x.shape[1]
    assign = Guarded((L.loopvq_kmeans_assign_bytes(cfg, n),), torch.uint8, fill=255)
    L.loopvq_kmeans_step(cfg, layer, gamma, kv, x.cuda(), None if w is None else w.cuda(),
                         cb_gpu, assign.t)
    assign.check("assignment")
    return assign.t.cpu().numpy().reshape(s.n_kv_heads, s.J, n).transpose(2, 0, 1)   # [n][H][J]


def _check_step(s, x, w, cb_old, a_gpu, cb_new_gpu):
    """cb_old, cb_new_gpu: [H][g][J][E][c] of the step's slice."""
    X = x.double().numpy()
    W = None if w is None else w.double().numpy()
    _, dist = O.encode_group_ref(X, cb_old, W)
    check_indices(a_gpu, dist)
    _, ref = O.kmeans_step_group_ref(X, cb_old, W, assign=a_gpu)
    # float32 sums of the members: bound (count + 2) * 2^-24 on num and den,
    # relative to the mean magnitude sum w|s| / sum w
    _, scale = O.kmeans_step_group_ref(np.abs(X), np.abs(cb_old), W, assign=a_gpu)
    counts = np.zeros((s.n_kv_heads, s.J, 256))
    for h in range(s.n_kv_heads):
        for j in range(s.J):
            counts[h, j] = np.bincount(a_gpu[:, h, j], minlength=256)
    cnt = counts[:, None, :, :, None]                                  # [H][1][J][E][1]
    tol = 4.0 * (cnt + 2.0) * EPS32 * scale
    err = np.abs(cb_new_gpu - ref)
    assert np.all(err <= tol), float(np.max(err / np.maximum(tol, 1e-300)))
    # clusters without members keep their exact codewords
    empty = np.broadcast_to(cnt == 0, cb_old.shape)
    assert empty.any()
    np.testing.assert_array_equal(cb_new_gpu[empty], cb_old[empty])


@pytest.mark.parametrize("per_token", [True, False])
def test_kmeans_step_tensor_core_assignment(per_token):
    # 2304 tokens: the tensor-core encoder assigns, then the weighted update
    s = W128
    n, layer, gamma, kv = 2304, 1, 1, 0
    x = loop_group_kv(s, layer, gamma, kv, n)
    w = weights(s, n, per_token, layer, gamma, kv)
    cb = random_codebooks(s, 2, 31)
    cb_gpu = cb.cuda()
    a = _step(s, 2, layer, gamma, kv, x, w, cb_gpu)
    new = cb_gpu.cpu()
    _check_step(s, x, w, cb[layer, :, gamma, kv].double().numpy(), a,
                new[layer, :, gamma, kv].double().numpy())
    # nothing outside (layer, gamma, kv) moved
    mask = torch.ones(cb.shape[:4], dtype=torch.bool)
    mask[layer, :, gamma, kv] = False
    assert torch.equal(new[mask], cb[mask])


def test_kmeans_step_direct_assignment_unweighted():
    s = W128
    n, layer, gamma, kv = 700, 0, 0, 1
    x = loop_group_kv(s, layer, gamma, kv, n)
    cb = random_codebooks(s, 2, 32)
    cb_gpu = cb.cuda()
    a = _step(s, 2, layer, gamma, kv, x, None, cb_gpu)
    _check_step(s, x, None, cb[layer, :, gamma, kv].double().numpy(), a,
                cb_gpu.cpu()[layer, :, gamma, kv].double().numpy())


@pytest.mark.parametrize("shape,n", [(C8, 2100), (C8, 300), (C2, 2048), (C2, 50)])
def test_kmeans_step_other_groupings(shape, n):
    # c = 8 (D = 32: 64 KB of accumulators) and c = 2 (D = 8)
    s = shape
    x = loop_group_kv(s, 0, 0, 1, n)
    w = weights(s, n, True, 0, 0, 1)
    cb = random_codebooks(s, 1, 33)
    cb_gpu = cb.cuda()
    a = _step(s, 1, 0, 0, 1, x, w, cb_gpu)
    _check_step(s, x, w, cb[0, :, 0, 1].double().numpy(), a,
                cb_gpu.cpu()[0, :, 0, 1].double().numpy())


def test_zero_weight_elements_keep_their_codewords():
    s = W128
    n = 900
    x = loop_group_kv(s, 0, 0, 0, n)
    w = weights(s, n, True, 0, 0, 0)
    w[:, :, :, 5] = 0.0                    # channel 5: element 4*tau + 1 of group 1, no weight anywhere
    cb = random_codebooks(s, 2, 34)
    cb_gpu = cb.cuda()
    _step(s, 2, 0, 0, 0, x, w, cb_gpu)
    new = cb_gpu.cpu()
    assert torch.equal(new[0, :, 0, 0, :, 1, :, 1], cb[0, :, 0, 0, :, 1, :, 1])


def test_repeated_steps_do_not_increase_the_weighted_distortion():
    s = W128
    n, layer, gamma, kv = 2304, 0, 1, 1
    x = loop_group_kv(s, layer, gamma, kv, n)
    w = weights(s, n, True, layer, gamma, kv)
    X, W = x.double().numpy(), w.double().numpy()
    cb_gpu = random_codebooks(s, 2, 35).cuda()
    prev = None
    for _ in range(4):
        old = cb_gpu.cpu()[layer, :, gamma, kv].double().numpy()
        a = _step(s, 2, layer, gamma, kv, x, w, cb_gpu)
        before = O.weighted_distortion_ref(X, old, a, W)
        new = cb_gpu.cpu()[layer, :, gamma, kv].double().numpy()
        after = O.weighted_distortion_ref(X, new, a, W)
        assert after <= before * (1 + 1e-6)
        if prev is not None:                     # reassignment: near ties move within 1e-5 of the best
            assert before <= prev * (1 + 2e-5)
        prev = after
