"""GPU parity of the dense bf16-KV comparison kernel against the oracle's
float64 attention (same tolerances as the LoopVQ kernel)."""

import math

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O

from _cases import TOL_F32_REL, TOL_LSE, TOL_BF16_ABS, bf16_ulp
from _guard import Guarded

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_bf16_kv_decode(d, dt):
    g = torch.Generator().manual_seed(d)
    B, Hq, Hkv, S = 4, 4, 2, 3000
    seq = [0, 1, 777, S]
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, S, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, S, d, generator=g).to(torch.bfloat16)
    out = Guarded((B, Hq, d), dt, fill=float("nan"))
    lse = Guarded((B, Hq), torch.float32, fill=float("nan"))
    ws = Guarded((L.loopvq_bf16_decode_workspace_bytes(B, Hq, d, S) // 4,), torch.float32)
    L.loopvq_bf16_decode_attn(q.cuda(), k.cuda(), v.cuda(),
                              torch.tensor(seq, dtype=torch.int32, device="cuda"), out.t, ws.t, lse=lse.t)
    for g_, what in ((out, "output"), (lse, "lse"), (ws, "workspace")):
        g_.check(what)
    o, ls = out.t.float().cpu().numpy(), lse.t.cpu().numpy()
    scale = 1 / math.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            if seq[b] == 0:
                assert np.all(o[b, h] == 0) and ls[b, h] == -np.inf
                continue
            hk = h // (Hq // Hkv)
            ref, lref = O.attn_ref(q[b, h].double().numpy(), k[b, hk, :seq[b]].double().numpy(),
                                   v[b, hk, :seq[b]].double().numpy(), scale)
            if dt == torch.float32:
                assert np.max(np.abs(o[b, h] - ref)) / np.max(np.abs(ref)) <= TOL_F32_REL
            else:
                assert np.all(np.abs(o[b, h] - ref) <= np.maximum(TOL_BF16_ABS, bf16_ulp(ref)))
            assert abs(ls[b, h] - lref) <= TOL_LSE
