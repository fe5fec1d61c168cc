"""Status words and checked builds, on the GPU, without faulting it.

* The short-wait build (libloopvq_shortwait.so) gives the tensor-core
  encoder's per-tile wait no tries: every CTA gives up on its first tile,
  then waits (bounded) for the tensor cores to finish before it frees their
  memory, and reports LOOPVQ_ENCODE_STATUS_TIMEOUT. The test checks that the
  flag is set, that nothing was written, and that the context still runs the
  normal library correctly afterwards.
* The range-check build (libloopvq_rangecheck.so) checks the decode
  kernel's indices against their buffers; on the parity cases it must find
  nothing and give the same results as the default build.
"""

import ctypes
import os

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from sub_bit_vq_b200 import binding as B
from synthetic import SHAPES, Shape, loop_group_kv

from _cases import DecodeCase, check_decode, check_indices, random_codebooks
from _guard import Guarded

pytestmark = pytest.mark.gpu

PKG = os.path.dirname(B.__file__)


def _variant(name):
    path = os.path.join(PKG, f"libloopvq_{name}.so")
    if not os.path.exists(path):
        pytest.fail(f"{path} not built (python sub_bit_vq_b200/build.py builds the test variants)")
    return B.load_library(path)


def test_encoder_timeout_is_reported_and_the_context_stays_usable():
    lib = _variant("shortwait")
    s = SHAPES["sweep"].with_(n_kv_heads=2, n_q_heads=2)
    n, n_pages = 2304, 36                       # a prefill-sized batch: the tensor-core form
    cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                         head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                         chan_group=s.chan_group, n_pages=n_pages, max_batch=1,
                         max_pages_per_seq=n_pages)
    cb = random_codebooks(s, 1, 215).cuda()
    x = loop_group_kv(s, 0, 0, 0, n, stream=6).cuda()
    slots = torch.arange(n, dtype=torch.int64, device="cuda")
    pool = Guarded((L.loopvq_cache_layout(cfg)["pool_bytes"],), torch.uint8, fill=0)
    flags = ctypes.c_int(0)
    assert lib.loopvq_encode_status(ctypes.byref(flags), 1) == 0
    st = lib.loopvq_encode(cfg.c_ref(), 0, 0, 0, n, x.data_ptr(), x.stride(0), x.stride(1), None, 0, 0,
                           cb.data_ptr(), slots.data_ptr(), pool.t.data_ptr(), None)
    assert st == B.LOOPVQ_OK
    torch.cuda.synchronize()
    assert lib.loopvq_encode_status(ctypes.byref(flags), 1) == 0
    assert flags.value & B.LOOPVQ_ENCODE_STATUS_TIMEOUT
    assert not flags.value & B.LOOPVQ_ENCODE_STATUS_UNDRAINED
    pool.check("pool")
    assert not bool(pool.t.any()), "a tile that timed out wrote indices"
    # the context is fine: the default build encodes the same batch correctly
    L.loopvq_encode(cfg, 0, 0, 0, x, None, cb, slots, pool.t)
    torch.cuda.synchronize()
    assert L.loopvq_encode_status(clear=True) == 0
    plane = pool.t.cpu().numpy().reshape(s.n_kv_heads, 1, n_pages, 2, -1)
    _, dist = O.encode_group_ref(x.double().cpu().numpy(), cb[0, :, 0, 0].double().cpu().numpy())
    got = np.empty((n, s.n_kv_heads, s.J), dtype=np.uint8)
    v = np.arange(n)
    for h in range(s.n_kv_heads):
        got[:, h] = O.unpack_sequence(plane[h, 0], n, s.J, np.arange(n_pages), s.page_tokens, 0)
    check_indices(got, dist)


@pytest.mark.parametrize("t", [0, 3])
def test_range_check_build_agrees_with_the_default_build(t):
    lib = _variant("rangecheck")
    rag = Shape("rc", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=128, n_loops=4, loop_group=4,
                chan_group=4, batch=5, context=0, seed=17)
    case = DecodeCase(rag, [0, 73, 640, 3000, 9000], loop_step=t, seed=300 + t)
    ref_out, ref_lse = case.run_gpu(torch.float32)
    old = B._lib
    B._lib = lib
    try:
        out, lse = case.run_gpu(torch.float32)  # the guard and status checks of run_gpu apply
    finally:
        B._lib = old
    check_decode(case, out, lse, torch.float32)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=0)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=0)
