"""GPU parity of loopvq_prefill_attn: a chunk of Q new queries per sequence
attending over the sequence's cached context (bf16 windows + quantised
tokens), checked query by query against the oracle's decode attention.

Tolerances: those of the decode tests (float32 output per (query, head)
max|o - ref| / max|ref| <= 1e-4; bf16 max abs <= 2e-2 floored at one bf16
ulp; lse within 1e-4).
"""

import math

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from synthetic import Shape

from _cases import TOL_BF16_ABS, TOL_F32_REL, TOL_LSE, DecodeCase, bf16_ulp
from _guard import Guarded, status_word, workspace

pytestmark = pytest.mark.gpu

S128 = Shape("pf128", n_layers=1, n_kv_heads=2, n_q_heads=4, head_dim=128, n_loops=4, loop_group=4,
             chan_group=4, batch=4, context=0, head_scale=(0.5, 2.0), seed=71)


def _run(case, q, out_dtype):
    dev = "cuda"
    s = case.shape
    B, Q = q.shape[0], q.shape[1]
    cfg = case.config()
    out = Guarded((B, Q, s.n_q_heads, s.head_dim), out_dtype, fill=float("nan"))
    lse = Guarded((B, Q, s.n_q_heads), torch.float32, fill=float("nan"))
    ws = workspace(L.loopvq_prefill_workspace_bytes(cfg, B, Q, case.max_seq_len))
    L.loopvq_prefill_attn(cfg, 0, case.t, q.to(dev), torch.from_numpy(case.pool).to(dev),
                          case.cb.to(dev), case.bt.to(dev),
                          torch.tensor(case.seq_lens, dtype=torch.int32, device=dev),
                          case.win_k.to(dev), case.win_v.to(dev), out.t, ws.t, case.max_seq_len,
                          lse=lse.t, sm_scale=case.sm_scale)
    for g_, what in ((out, "output"), (lse, "lse"), (ws, "workspace")):
        g_.check(what)
    assert status_word(ws) == 0
    return out.t.float().cpu().numpy(), lse.t.cpu().numpy()


@pytest.mark.parametrize("Q", [16, 128])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_prefill_chunk_over_the_cache(Q, dt):
    case = DecodeCase(S128, [0, 73, 1500, 4000], loop_step=1, seed=80 + Q)
    s = S128
    g = torch.Generator().manual_seed(Q)
    q = torch.randn(case.B, Q, s.n_q_heads, s.head_dim, generator=g).to(torch.bfloat16)
    out, lse = _run(case, q, dt)
    r = np.random.default_rng(Q)
    picks = [(b, int(i), int(h)) for b in range(case.B)
             for i, h in zip(r.integers(0, Q, 6), r.integers(0, s.n_q_heads, 6))]
    picks += [(3, Q - 1, h) for h in range(s.n_q_heads)]
    ratio = s.n_q_heads // s.n_kv_heads
    for b, i, h in picks:
        N = case.seq_lens[b]
        o = out[b, i, h].astype(np.float64)
        if N == 0:
            assert np.all(o == 0) and lse[b, i, h] == -np.inf
            continue
        hkv = h // ratio
        iK, iV = case.indices(b, hkv)
        nw = O.n_window_tokens(N, s.prefix, s.recent)
        ref, lref = O.decode_attn_ref(q[b, i, h].double().numpy(),
                                      case.win_k[b, hkv, :nw].double().numpy(),
                                      case.win_v[b, hkv, :nw].double().numpy(), iK, iV,
                                      case.cb[0, hkv, 0, 0].double().numpy(),
                                      case.cb[0, hkv, 0, 1].double().numpy(), case.tau,
                                      1.0 / math.sqrt(s.head_dim))
        if dt == torch.float32:
            assert np.max(np.abs(o - ref)) / np.max(np.abs(ref)) <= TOL_F32_REL, (b, i, h)
        else:
            assert np.all(np.abs(o - ref) <= np.maximum(TOL_BF16_ABS, bf16_ulp(ref))), (b, i, h)
        assert abs(float(lse[b, i, h]) - lref) <= TOL_LSE, (b, i, h)


def test_one_query_chunk_equals_decode():
    # Q = 1 is the decode call: identical results, bit for bit
    case = DecodeCase(S128, [73, 900, 2000], loop_step=2, seed=90)
    out_d, lse_d = case.run_gpu(torch.float32)
    out_p, lse_p = _run(case, case.q[:, None].contiguous(), torch.float32)
    np.testing.assert_array_equal(out_p[:, 0], out_d)
    np.testing.assert_array_equal(lse_p[:, 0], lse_d)
