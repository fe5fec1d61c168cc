"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, computes the documented layout, and rejects bad arguments
with the documented status before launching anything (no GPU needed)."""

import ctypes
import os
import re

import pytest

import sub_bit_vq_b200 as L
from sub_bit_vq_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(loopvq_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"loopvq_cache_layout", "loopvq_encode", "loopvq_decode_attn"} <= names
    lib = B.library()
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(B.EXPORTED) <= names


def _cfg(**kw):
    base = dict(n_layers=2, n_kv_heads=3, n_q_heads=6, head_dim=128, n_loops=8, loop_group=4,
                chan_group=4, n_pages=10, max_batch=4, max_pages_per_seq=5)
    base.update(kw)
    return L.LoopVQConfig(**base)


@pytest.mark.parametrize("c,g,bits", [(4, 4, 0.5), (8, 4, 0.25), (4, 2, 1.0), (8, 1, 1.0)])
def test_layout_rate_and_sizes(c, g, bits):
    d = 128 if c != 8 else 96
    cfg = _cfg(head_dim=d, chan_group=c, loop_group=g, n_loops=2 * g,
               page_tokens=96 if d // c == 12 else 64)
    lay = L.loopvq_cache_layout(cfg)
    assert lay["bits_per_element"] == bits == 8 / (c * g)
    J = d // c
    assert lay["J"] == J and lay["D"] == c * g and lay["n_loop_groups"] == 2
    Pg = cfg.page_tokens
    assert lay["plane_bytes"] == Pg * J and lay["page_bytes"] == 2 * Pg * J
    assert lay["pool_bytes"] == cfg.n_layers * cfg.n_kv_heads * 2 * cfg.n_pages * 2 * Pg * J
    assert lay["pool_stride_group"] == cfg.n_pages * 2 * Pg * J
    assert lay["pool_stride_head"] == 2 * lay["pool_stride_group"]
    assert lay["pool_stride_layer"] == cfg.n_kv_heads * lay["pool_stride_head"]
    assert lay["cb_stride_loop"] == J * 256 * c
    assert lay["cb_stride_kv"] == g * lay["cb_stride_loop"]
    assert lay["codebook_bytes"] == 4 * cfg.n_layers * cfg.n_kv_heads * 2 * 2 * g * J * 256 * c
    assert lay["rot_block"] == (32 // J) * J
    assert lay["granule"] == (16 if J % 16 == 0 else 8 if J % 8 == 0 else 4)
    # packed bytes of one plane cover g loop steps: 8/(c*g) bits per element
    assert lay["plane_bytes"] * 8 / (Pg * d * g) == bits


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=130), B.LOOPVQ_ERR_INVALID_ARG),        # d % c
    (dict(n_loops=6), B.LOOPVQ_ERR_INVALID_ARG),           # T % g
    (dict(n_q_heads=4), B.LOOPVQ_ERR_INVALID_ARG),         # Hq % Hkv
    (dict(n_layers=0), B.LOOPVQ_ERR_INVALID_ARG),
    (dict(n_centroids=128), B.LOOPVQ_ERR_UNSUPPORTED),
    (dict(chan_group=2), B.LOOPVQ_ERR_UNSUPPORTED),         # J = 64 > 32
    (dict(loop_group=8, n_loops=8, chan_group=8), B.LOOPVQ_ERR_UNSUPPORTED),  # D = 64
    (dict(page_tokens=48), B.LOOPVQ_ERR_UNSUPPORTED),       # not a multiple of LB = 32
    (dict(page_tokens=96), B.LOOPVQ_ERR_UNSUPPORTED),       # 3 blocks of LB = 32: not a power of two
    (dict(prefix_tokens=200, recent_tokens=100), B.LOOPVQ_ERR_UNSUPPORTED),
])
def test_layout_rejects(kw, status):
    with pytest.raises(L.LoopVQError) as ei:
        L.loopvq_cache_layout(_cfg(**kw))
    assert ei.value.status == status


def test_layout_rejects_wrong_struct_size():
    c = _cfg().c_struct()
    c.struct_size = 12
    out = B._Layout()
    assert B.library().loopvq_cache_layout(ctypes.byref(c), ctypes.byref(out)) == \
        B.LOOPVQ_ERR_INVALID_ARG


def _decode_raw(cfg, **over):
    # fake, aligned, never dereferenced addresses: every check below fails
    # before the library touches the device
    a = dict(layer=0, loop_step=0, batch=1, max_seq_len=100, q=0x1000, pool=0x2000,
             cb=0x3000, bt=0x4000, sl=0x5000, wk=0x6000, wv=0x7000, scale=0.1, odt=0,
             out=0x8000, lse=None, ws=0x9000, ws_bytes=0)
    a.update(over)
    return B.library().loopvq_decode_attn(
        ctypes.byref(cfg.c_struct()), a["layer"], a["loop_step"], a["batch"],
        a["max_seq_len"], a["q"], a["pool"], a["cb"], a["bt"], a["sl"], a["wk"], a["wv"],
        a["scale"], a["odt"], a["out"], a["lse"], a["ws"], a["ws_bytes"], None)


def test_decode_rejects_before_launch():
    cfg = _cfg()
    E = B.LOOPVQ_ERR_INVALID_ARG
    assert _decode_raw(cfg, q=None) == E
    assert _decode_raw(cfg, out=None) == E
    assert _decode_raw(cfg, layer=2) == E
    assert _decode_raw(cfg, loop_step=8) == E
    assert _decode_raw(cfg, batch=5) == E
    assert _decode_raw(cfg, odt=7) == E
    assert _decode_raw(cfg, scale=-1.0) == E
    assert _decode_raw(cfg, q=0x1002) == E                       # misaligned
    assert _decode_raw(cfg, max_seq_len=72 + 5 * 64 + 1) == E   # > max_pages_per_seq
    need = L.loopvq_decode_workspace_bytes(cfg, 1, 100)
    assert need > 0
    assert _decode_raw(cfg, ws_bytes=need - 4) == B.LOOPVQ_ERR_WORKSPACE


def test_encode_rejects_before_launch():
    cfg = _cfg()
    lib = B.library()

    def enc(layer=0, grp=0, kv=0, n=4, x=0x1000, xl=512, xt=1024, w=None, cb=0x3000,
            sm=0x4000, pool=0x5000):
        return lib.loopvq_encode(ctypes.byref(cfg.c_struct()), layer, grp, kv, n, x, xl, xt, w,
                                 0, 0, cb, sm, pool, None)
    E = B.LOOPVQ_ERR_INVALID_ARG
    assert enc(n=0, x=None, cb=None, sm=None, pool=None) == B.LOOPVQ_OK   # no-op
    assert enc(layer=2) == E
    assert enc(grp=2) == E
    assert enc(kv=2) == E
    assert enc(n=-1) == E
    assert enc(x=None) == E
    assert enc(x=0x1001) == E
    assert enc(xt=3) == E
    assert enc(sm=0x4004) == E


def test_kmeans_step_rejects_before_launch():
    cfg = _cfg()
    lib = B.library()
    n = 10
    need = L.loopvq_kmeans_assign_bytes(cfg, n)
    assert need == 3 * (128 // 4) * n                 # Hkv * J * n_tokens
    assert L.loopvq_kmeans_assign_bytes(cfg, -1) == 0

    def km(layer=0, grp=0, kv=0, n=n, x=0x1000, xl=512, xt=1024, w=None, wl=0, wt=0, cb=0x3000,
           assign=0x4000, nbytes=need):
        return lib.loopvq_kmeans_step(ctypes.byref(cfg.c_struct()), layer, grp, kv, n, x, xl, xt, w,
                                      wl, wt, cb, assign, nbytes, None)
    E = B.LOOPVQ_ERR_INVALID_ARG
    assert km(n=0, x=None, cb=None, assign=None, nbytes=0) == B.LOOPVQ_OK   # no-op
    assert km(layer=2) == E
    assert km(grp=2) == E
    assert km(kv=2) == E
    assert km(n=-1) == E
    assert km(x=None) == E
    assert km(cb=None) == E
    assert km(assign=None) == E
    assert km(x=0x1001) == E
    assert km(xt=3) == E
    assert km(w=0x2004) == E
    assert km(w=0x2000, wt=3) == E
    assert km(cb=0x3004) == E
    assert km(nbytes=need - 1) == B.LOOPVQ_ERR_WORKSPACE


def test_workspace_bytes_formula():
    cfg = _cfg()
    # a 256-byte status area, then one record (m, l, 2 spare, o[d]) of float32
    # per (pair, streaming CTA) slot: pairs + 256 slots, one window partial of
    # the same size per pair, one key lookup table of 256 x J float32 per
    # pair and one 32-bit record counter per pair (rounded up to 16 bytes)
    n = L.loopvq_decode_workspace_bytes(cfg, 2, 72 + 5 * 64)
    rec = 4 * (4 + cfg.head_dim)
    pairs, J = 2 * cfg.n_q_heads, cfg.head_dim // cfg.chan_group
    counters = -(-pairs * 4 // 16) * 16
    assert n == 256 + rec * (pairs + 256) + rec * pairs + pairs * 256 * J * 4 + counters
    # more sequences need more records
    assert L.loopvq_decode_workspace_bytes(cfg, 4, 72 + 5 * 64) > n
    assert L.loopvq_decode_workspace_bytes(cfg, 0, 10) == 0


def test_status_strings():
    for s in range(5):
        assert L.loopvq_status_string(s)
    assert "unknown" in L.loopvq_status_string(99)


def test_python_api_exports_the_documented_calls():
    for name in ("LoopVQConfig", "loopvq_cache_layout", "loopvq_encode", "loopvq_encode_evict",
                 "loopvq_kmeans_assign_bytes",
                 "loopvq_kmeans_step", "loopvq_decode_workspace_bytes", "loopvq_decode_attn",
                 "loopvq_bf16_decode_workspace_bytes", "loopvq_bf16_decode_attn",
                 "loopvq_decode_attn_noalloc", "loopvq_status_string"):
        assert callable(getattr(L, name)), name
    cfg = _cfg()
    lay = L.loopvq_cache_layout(cfg)
    assert lay["bits_per_element"] == 0.5
    assert L.loopvq_kmeans_assign_bytes(cfg, 7) == 3 * 32 * 7


def test_static_scratch_size_matches_the_header():
    # the binding's copy of LOOPVQ_STATIC_SCRATCH_BYTES is the header's value
    text = open(os.path.join(ROOT, "include", "loopvq.h")).read()
    m = re.search(r"#define\s+LOOPVQ_STATIC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "LOOPVQ_STATIC_SCRATCH_BYTES not found in include/loopvq.h"
    assert int(m.group(1)) << int(m.group(2)) == B.LOOPVQ_STATIC_SCRATCH_BYTES
    assert L.LOOPVQ_STATIC_SCRATCH_BYTES == B.LOOPVQ_STATIC_SCRATCH_BYTES


def test_status_bits_match_the_header():
    text = open(os.path.join(ROOT, "include", "loopvq.h")).read()
    for name in ("LOOPVQ_DECODE_STATUS_BAD_PAGE", "LOOPVQ_DECODE_STATUS_SHARED_BASE",
                 "LOOPVQ_ENCODE_STATUS_TIMEOUT", "LOOPVQ_ENCODE_STATUS_UNDRAINED",
                 "LOOPVQ_ENCODE_STATUS_BAD_SLOT", "LOOPVQ_DECODE_STATUS_RANGE",
                 "LOOPVQ_DECODE_STATUS_TIMEOUT", "LOOPVQ_DECODE_STATUS_UNDRAINED"):
        m = re.search(name + r"\s*=\s*(\d+)", text)
        assert m, name
        assert getattr(B, name) == int(m.group(1)) == getattr(L, name)


def test_encode_evict_rejects_before_launch():
    cfg = _cfg()
    lib = B.library()
    E = B.LOOPVQ_ERR_INVALID_ARG
    ev = lambda n=4, x=0x1000, cb=0x2000, sl=0x3000, pool=0x4000: lib.loopvq_encode_evict(
        cfg.c_ref(), n, x, cb, sl, pool, None)
    assert ev(n=0) == B.LOOPVQ_OK                     # nothing to do, nothing launched
    assert ev(n=-1) == E
    assert ev(n=65) == B.LOOPVQ_ERR_UNSUPPORTED
    assert ev(x=0) == E and ev(cb=0) == E and ev(sl=0) == E and ev(pool=0) == E
    assert ev(x=0x1008) == E and ev(cb=0x2004) == E and ev(sl=0x3004) == E


def test_encode_status_rejects_a_null_pointer():
    assert B.library().loopvq_encode_status(None, 0) == B.LOOPVQ_ERR_INVALID_ARG


def test_prefill_rejects_before_launch_and_sizes_its_workspace():
    cfg = _cfg()
    lib = B.library()
    need = L.loopvq_prefill_workspace_bytes(cfg, 2, 5, 72 + 5 * 64)
    assert need == L.loopvq_decode_workspace_bytes(cfg, 2, 72 + 5 * 64) + \
        (need - L.loopvq_decode_workspace_bytes(cfg, 2, 72 + 5 * 64))
    assert need > L.loopvq_decode_workspace_bytes(cfg, 2, 72 + 5 * 64)
    assert L.loopvq_prefill_workspace_bytes(cfg, 2, 0, 100) == 0

    def call(nq=5, ws=0x5000, nbytes=need):
        return lib.loopvq_prefill_attn(cfg.c_ref(), 0, 0, 2, nq, 72 + 5 * 64, 0x1000, 0x2000, 0x3000,
                                       0x4000, 0x4100, 0x6000, 0x7000, 0.1, 0, 0x8000, None, ws,
                                       nbytes, None)
    assert call(nq=0) == B.LOOPVQ_ERR_INVALID_ARG
    assert call(ws=0) == B.LOOPVQ_ERR_INVALID_ARG
    assert call(nbytes=need - 1) == B.LOOPVQ_ERR_WORKSPACE
