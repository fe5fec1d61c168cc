"""GPU parity of loopvq_decode_attn (through the C ABI) against the oracle.

Tolerances: float32 output, per (sequence, head), max|o - ref| / max|ref|
<= 1e-4; bf16 output, max abs error <= 2e-2 (floored at one bf16 ulp of the
reference); log-sum-exp within 1e-4.
"""

import numpy as np
import pytest
import torch

from synthetic import SHAPES, Shape

from _cases import DecodeCase, check_decode

pytestmark = pytest.mark.gpu

RAG128 = Shape("rag128", n_layers=2, n_kv_heads=2, n_q_heads=2, head_dim=128, n_loops=4,
               loop_group=4, chan_group=4, batch=7, context=0, head_scale=(0.5, 2.0), seed=11)
J12 = Shape("j12", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=96, n_loops=8, loop_group=4,
            chan_group=8, batch=4, context=0, page_tokens=96, kind="ar1", seed=12)
GQA = Shape("gqa", n_layers=1, n_kv_heads=2, n_q_heads=4, head_dim=64, n_loops=4, loop_group=2,
            chan_group=4, batch=2, context=0, seed=13)
D256 = Shape("d256", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=256, n_loops=4,
             loop_group=4, chan_group=8, batch=2, context=0, seed=14)


@pytest.mark.parametrize("t", [0, 1, 2, 3])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_tiny_config_every_loop_step(t, dt):
    s = SHAPES["tiny"]
    case = DecodeCase(s, [s.context], loop_step=t, fitted_codebooks=True, seed=t)
    out, lse = case.run_gpu(dt)
    check_decode(case, out, lse, dt)


@pytest.mark.parametrize("t", [0, 3])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_ragged_batch_window_edges(t, dt):
    # N <= 72 (window only), N = 73 (one quantised token), partial pages,
    # several splits, layer 1 of 2.
    case = DecodeCase(RAG128, [1, 9, 72, 73, 200, 777, 2100], layer=1, n_layers=2, loop_step=t,
                      seed=100 + t)
    out, lse = case.run_gpu(dt)
    check_decode(case, out, lse, dt)


def test_empty_sequence_gives_zero_and_neg_inf():
    case = DecodeCase(RAG128, [0, 150], seed=3)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_j12_quarter_bit(dt):
    # d=96, c=8, g=4: 32-element sub-vectors, 0.25 bit, J=12 (24-slot rotation)
    case = DecodeCase(J12, [50, 73, 300, 1500], loop_step=5, seed=21)
    out, lse = case.run_gpu(dt)
    check_decode(case, out, lse, dt)


def test_gqa_ratio_two():
    case = DecodeCase(GQA, [100, 1000], loop_step=3, seed=31)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


def test_head_dim_256():
    case = DecodeCase(D256, [80, 700], loop_step=2, seed=41)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


def test_large_magnitude_scores():
    # q scaled by 30: softmax close to one-hot, running maximum moves a lot
    case = DecodeCase(RAG128, [500, 3000], q_scale=30.0, seed=51)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


def test_zero_query_is_mean_of_values():
    # all scores equal: out = mean of every token's (dequantised) value
    case = DecodeCase(RAG128, [72, 1000], q_scale=0.0, seed=61)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)
    assert abs(lse[1, 0] - np.log(1000)) < 1e-4


def test_long_single_sequence_many_splits():
    s = RAG128.with_(n_kv_heads=1, n_q_heads=1)
    case = DecodeCase(s, [20000], loop_step=2, seed=71)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


def test_full_long_context_config_sampled():
    # the 32K configuration at full size (one layer: batch 8, 16 heads,
    # context 32768), checked on sampled (sequence, head) pairs
    s = SHAPES["long32k"]
    case = DecodeCase(s.with_(n_layers=1), [s.context] * s.batch, loop_step=3, seed=81,
                      spare_pages=0)
    out, lse = case.run_gpu(torch.bfloat16)
    pairs = [(0, 0), (3, 7), (7, 15), (5, 2)]
    check_decode(case, out, lse, torch.bfloat16, pairs=pairs)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32, pairs=pairs)


# Every (J, c) instantiation the library dispatches, beyond the shapes above:
# J = 8 (four replicas per group in a 32-slot block), J = 24 (24-slot blocks,
# lanes 24..31 idle) and the c = 2 forms.
OTHER_SHAPES = [
    Shape("j8c4", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=32, n_loops=4, loop_group=4,
          chan_group=4, batch=3, context=0, seed=31),
    Shape("j8c8", n_layers=1, n_kv_heads=1, n_q_heads=2, head_dim=64, n_loops=4, loop_group=4,
          chan_group=8, batch=3, context=0, seed=32),
    Shape("j24c4", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=96, n_loops=4, loop_group=4,
          chan_group=4, batch=3, context=0, page_tokens=96, seed=33),
    Shape("j16c8", n_layers=1, n_kv_heads=1, n_q_heads=2, head_dim=128, n_loops=4, loop_group=4,
          chan_group=8, batch=3, context=0, seed=38),
    Shape("j32c2", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=64, n_loops=4, loop_group=4,
          chan_group=2, batch=3, context=0, seed=34),
    Shape("j24c2", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=48, n_loops=4, loop_group=4,
          chan_group=2, batch=3, context=0, page_tokens=96, seed=35),
    Shape("j12c2", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=24, n_loops=4, loop_group=4,
          chan_group=2, batch=3, context=0, page_tokens=48, seed=36),
    Shape("j16c2", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=32, n_loops=4, loop_group=4,
          chan_group=2, batch=3, context=0, seed=37),
]


@pytest.mark.parametrize("shape", OTHER_SHAPES, ids=lambda s: s.name)
def test_every_dispatched_group_shape(shape):
    case = DecodeCase(shape, [73, 640, 2500], loop_step=2, seed=40)
    out, lse = case.run_gpu(torch.float32)
    check_decode(case, out, lse, torch.float32)


def test_out_of_range_page_entries_are_skipped_and_flagged():
    # Block-table entries outside [0, n_pages) are not read: the kernel skips
    # those pages, sets LOOPVQ_DECODE_STATUS_BAD_PAGE in the workspace's status
    # word, and the result is attention over the remaining tokens.
    import math as _m

    import sub_bit_vq_b200 as L
    from oracle import loopvq_oracle as O

    from _guard import Guarded, status_word, workspace

    s = RAG128
    case = DecodeCase(s, [400, 1000], seed=6)
    good = case.bt.clone()
    bad = good.clone()
    bad[1, 2] = case.n_pages + 7                     # past the pool
    bad[1, 5] = -3                                   # negative
    dev = "cuda"
    cfg = case.config()
    out = Guarded((case.B, s.n_q_heads, s.head_dim), torch.float32, fill=float("nan"))
    lse = Guarded((case.B, s.n_q_heads), torch.float32, fill=float("nan"))
    ws = workspace(L.loopvq_decode_workspace_bytes(cfg, case.B, case.max_seq_len))
    L.loopvq_decode_attn(cfg, 0, case.t, case.q.to(dev), torch.from_numpy(case.pool).to(dev),
                         case.cb.to(dev), bad.to(dev),
                         torch.tensor(case.seq_lens, dtype=torch.int32, device=dev),
                         case.win_k.to(dev), case.win_v.to(dev), out.t, ws.t, case.max_seq_len,
                         lse=lse.t, sm_scale=case.sm_scale)
    for g_, what in ((out, "output"), (lse, "lse"), (ws, "workspace")):
        g_.check(what)
    assert status_word(ws) & L.LOOPVQ_DECODE_STATUS_BAD_PAGE
    o, ls = out.t.cpu().numpy(), lse.t.cpu().numpy()
    # sequence 0 is untouched; sequence 1 lost the tokens of its logical pages 2 and 5
    for h in range(s.n_q_heads):
        ref, lref = case.oracle(0, h)
        assert np.max(np.abs(o[0, h] - ref)) / np.max(np.abs(ref)) <= 1e-4
        iK, iV = case.indices(1, h)
        keep = np.ones(iK.shape[0], dtype=bool)
        for pg in (2, 5):
            keep[pg * s.page_tokens:(pg + 1) * s.page_tokens] = False
        nw = O.n_window_tokens(case.seq_lens[1], s.prefix, s.recent)
        ref, lref = O.decode_attn_ref(case.q[1, h].double().numpy(),
                                      case.win_k[1, h, :nw].double().numpy(),
                                      case.win_v[1, h, :nw].double().numpy(), iK[keep], iV[keep],
                                      case.cb[0, h, 0, 0].double().numpy(),
                                      case.cb[0, h, 0, 1].double().numpy(), case.tau,
                                      1.0 / _m.sqrt(s.head_dim))
        assert np.max(np.abs(o[1, h] - ref)) / np.max(np.abs(ref)) <= 1e-4
        assert abs(ls[1, h] - lref) <= 1e-4
