"""The decode entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin that only receives
input and output pointers from a host program that owns the device memory,
or code held to a fixed memory budget), so they cannot pass the workspace
loopvq_decode_attn takes. loopvq_decode_attn_noalloc keeps the split
scratch in the library's own static device array instead. This test calls
it through the C ABI twice in a row and checks both results against the
workspace entry point within the float32 tolerance of the other decode
tests. It sits in its own file, collected last, and needs no state from
other tests.
"""

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from sub_bit_vq_b200 import binding as B
from synthetic import Shape

from _cases import TOL_F32_REL, TOL_LSE, DecodeCase
from _guard import Guarded, status_word, workspace

pytestmark = pytest.mark.gpu

SHAPE = Shape("noalloc", n_layers=2, n_kv_heads=2, n_q_heads=4, head_dim=128, n_loops=4,
              loop_group=4, chan_group=4, batch=4, context=0, head_scale=(0.5, 2.0), seed=91)


def _inputs(case, dev="cuda"):
    s = case.shape
    return dict(
        cfg=case.config(), q=case.q.to(dev), pool=torch.from_numpy(case.pool).to(dev),
        cb=case.cb.to(dev), bt=case.bt.to(dev),
        sl=torch.tensor(case.seq_lens, dtype=torch.int32, device=dev),
        wk=case.win_k.to(dev), wv=case.win_v.to(dev),
        out=torch.full((case.B, s.n_q_heads, s.head_dim), float("nan"), device=dev),
        lse=torch.full((case.B, s.n_q_heads), float("nan"), device=dev))


def _workspace_reference(case, a):
    """out/lse of the workspace entry point, its scratch filled with NaN."""
    need = L.loopvq_decode_workspace_bytes(a["cfg"], case.B, case.max_seq_len)
    assert 0 < need <= B.LOOPVQ_STATIC_SCRATCH_BYTES
    ws = workspace(need)
    L.loopvq_decode_attn(a["cfg"], case.layer, case.t, a["q"], a["pool"], a["cb"], a["bt"], a["sl"],
                         a["wk"], a["wv"], a["out"], ws.t, case.max_seq_len, lse=a["lse"],
                         sm_scale=case.sm_scale)
    ws.check("workspace")
    assert status_word(ws) == 0
    return a["out"].cpu().numpy(), a["lse"].cpu().numpy()


def _noalloc(case, a):
    out = Guarded(a["out"].shape, a["out"].dtype, fill=float("nan"))
    lse = Guarded(a["lse"].shape, a["lse"].dtype, fill=float("nan"))
    B.loopvq_decode_attn_noalloc(a["cfg"], case.layer, case.t, a["q"], a["pool"], a["cb"],
                                 a["bt"], a["sl"], a["wk"], a["wv"], out.t, case.max_seq_len,
                                 lse=lse.t, sm_scale=case.sm_scale)
    out.check("output")
    lse.check("lse")
    return out.t.cpu().numpy(), lse.t.cpu().numpy()


def _compare(case, got, ref):
    (o, ls), (ro, rl) = got, ref
    for b in range(case.B):
        for h in range(case.shape.n_q_heads):
            if case.seq_lens[b] == 0:
                assert np.all(o[b, h] == 0) and ls[b, h] == -np.inf
                continue
            rel = np.max(np.abs(o[b, h] - ro[b, h])) / np.max(np.abs(ro[b, h]))
            assert rel <= TOL_F32_REL, (b, h, rel)
            assert abs(ls[b, h] - rl[b, h]) <= TOL_LSE


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # Two different calls in a row: a batch with one long sequence, then a
    # smaller batch of short sequences. The second call writes fewer split
    # records than the first left in the shared static array, so a record it
    # did not write would surface as a mismatch.
    first = DecodeCase(SHAPE, [60, 73, 900, 20000], layer=1, n_layers=2, loop_step=2, seed=5)
    second = DecodeCase(SHAPE.with_(batch=3), [75, 0, 640], layer=0, n_layers=2, loop_step=1,
                        seed=6)
    for case in (first, second):
        a = _inputs(case)
        ref = _workspace_reference(case, a)
        _compare(case, _noalloc(case, a), ref)


def test_noalloc_repeated_call_gives_the_same_result():
    case = DecodeCase(SHAPE, [200, 1500, 73, 4000], layer=0, n_layers=2, loop_step=3, seed=7)
    a = _inputs(case)
    ref = _workspace_reference(case, a)
    for _ in range(2):
        _compare(case, _noalloc(case, a), ref)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    # a batch whose split records exceed the static array: clear error, no launch
    cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=32, n_q_heads=32, head_dim=256, n_loops=4,
                         loop_group=4, chan_group=8, n_pages=4096, max_batch=512,
                         max_pages_per_seq=4096)
    assert L.loopvq_decode_workspace_bytes(cfg, 512, 4096 * 64) > B.LOOPVQ_STATIC_SCRATCH_BYTES
    st = B.library().loopvq_decode_attn_noalloc(cfg.c_ref(), 0, 0, 512, 4096 * 64, 0x1000, 0x2000,
                                                0x3000, 0x4000, 0x5000, 0x6000, 0x7000, 0.1, 0,
                                                0x8000, None, None)
    assert st == B.LOOPVQ_ERR_WORKSPACE
