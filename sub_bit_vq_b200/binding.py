"""Python binding of libloopvq (ctypes). Argument marshalling only.

Every function has the name of the C entry point it wraps (see
``include/loopvq.h``). Tensors are passed as raw device pointers; the stream
is the caller's current torch stream unless one is given. A non-OK status
raises ``LoopVQError``. There is no fallback: if ``libloopvq.so`` is missing
the import fails.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LOOPVQ_LIB names another in-tree build of the same sources (a test build
# such as libloopvq_rangecheck.so); the default is libloopvq.so.
LIB_PATH = os.path.join(_HERE, os.environ.get("LOOPVQ_LIB", "libloopvq.so"))

LOOPVQ_OK = 0
LOOPVQ_ERR_INVALID_ARG = 1
LOOPVQ_ERR_UNSUPPORTED = 2
LOOPVQ_ERR_WORKSPACE = 3
LOOPVQ_ERR_CUDA = 4
LOOPVQ_DTYPE_BF16 = 0
LOOPVQ_DTYPE_F32 = 1
LOOPVQ_ENCODE_STATUS_TIMEOUT = 1
LOOPVQ_ENCODE_STATUS_UNDRAINED = 2
LOOPVQ_ENCODE_STATUS_BAD_SLOT = 4
LOOPVQ_DECODE_STATUS_BAD_PAGE = 1
LOOPVQ_DECODE_STATUS_SHARED_BASE = 2
LOOPVQ_DECODE_STATUS_RANGE = 4
LOOPVQ_DECODE_STATUS_TIMEOUT = 8
LOOPVQ_DECODE_STATUS_UNDRAINED = 16


class LoopVQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {loopvq_status_string(status)} (status {status})")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32)] + [
        (n, ctypes.c_int32) for n in (
            "n_layers", "n_kv_heads", "n_q_heads", "head_dim", "n_loops", "loop_group",
            "chan_group", "n_centroids", "prefix_tokens", "recent_tokens", "page_tokens",
            "n_pages", "max_batch", "max_pages_per_seq")]


class _Layout(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32),
        ("J", ctypes.c_int32), ("D", ctypes.c_int32), ("n_loop_groups", ctypes.c_int32),
        ("granule", ctypes.c_int32), ("rot_block", ctypes.c_int32),
        ("window_tokens", ctypes.c_int32),
        ("plane_bytes", ctypes.c_size_t), ("page_bytes", ctypes.c_size_t),
        ("pool_bytes", ctypes.c_size_t),
        ("pool_stride_layer", ctypes.c_int64), ("pool_stride_head", ctypes.c_int64),
        ("pool_stride_group", ctypes.c_int64),
        ("codebook_bytes", ctypes.c_size_t),
        ("cb_stride_layer", ctypes.c_int64), ("cb_stride_head", ctypes.c_int64),
        ("cb_stride_group", ctypes.c_int64), ("cb_stride_kv", ctypes.c_int64),
        ("cb_stride_loop", ctypes.c_int64),
        ("window_bytes", ctypes.c_size_t),
        ("bits_per_element", ctypes.c_double),
    ]


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built ({path}); run python sub_bit_vq_b200/build.py")
    lib = ctypes.CDLL(path)
    P, I, I64, F, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                        ctypes.c_size_t)
    cfgp = ctypes.POINTER(_Config)
    lib.loopvq_status_string.restype = ctypes.c_char_p
    lib.loopvq_status_string.argtypes = [I]
    lib.loopvq_cache_layout.restype = I
    lib.loopvq_cache_layout.argtypes = [cfgp, ctypes.POINTER(_Layout)]
    lib.loopvq_encode.restype = I
    lib.loopvq_encode.argtypes = [cfgp, I, I, I, I, P, I64, I64, P, I64, I64, P, P, P, P]
    lib.loopvq_encode_status.restype = I
    lib.loopvq_encode_status.argtypes = [ctypes.POINTER(ctypes.c_int), I]
    lib.loopvq_encode_evict.restype = I
    lib.loopvq_encode_evict.argtypes = [cfgp, I, P, P, P, P, P]
    lib.loopvq_prefill_workspace_bytes.restype = SZ
    lib.loopvq_prefill_workspace_bytes.argtypes = [cfgp, I, I, I]
    lib.loopvq_prefill_attn.restype = I
    lib.loopvq_prefill_attn.argtypes = [cfgp, I, I, I, I, I, P, P, P, P, P, P, P, F, I, P, P, P, SZ,
                                        P]
    lib.loopvq_decode_workspace_bytes.restype = SZ
    lib.loopvq_decode_workspace_bytes.argtypes = [cfgp, I, I]
    lib.loopvq_decode_attn.restype = I
    lib.loopvq_decode_attn.argtypes = [cfgp, I, I, I, I, P, P, P, P, P, P, P, F, I, P, P, P, SZ,
                                       P]
    lib.loopvq_decode_attn_noalloc.restype = I
    lib.loopvq_decode_attn_noalloc.argtypes = [cfgp, I, I, I, I, P, P, P, P, P, P, P, F, I, P, P, P]
    lib.loopvq_bf16_decode_workspace_bytes.restype = SZ
    lib.loopvq_bf16_decode_workspace_bytes.argtypes = [I, I, I, I]
    lib.loopvq_bf16_decode_attn.restype = I
    lib.loopvq_bf16_decode_attn.argtypes = [I, I, I, I, I, P, P, P, P, F, I, P, P, P, SZ, P]
    lib.loopvq_kmeans_assign_bytes.restype = SZ
    lib.loopvq_kmeans_assign_bytes.argtypes = [cfgp, I]
    lib.loopvq_kmeans_step.restype = I
    lib.loopvq_kmeans_step.argtypes = [cfgp, I, I, I, I, P, I64, I64, P, I64, I64, P, P, SZ, P]
    return lib


_lib = _load()

EXPORTED = ("loopvq_status_string", "loopvq_cache_layout", "loopvq_encode", "loopvq_encode_evict",
            "loopvq_encode_status", "loopvq_prefill_workspace_bytes", "loopvq_prefill_attn",
            "loopvq_decode_workspace_bytes", "loopvq_decode_attn", "loopvq_decode_attn_noalloc",
            "loopvq_bf16_decode_workspace_bytes", "loopvq_bf16_decode_attn",
            "loopvq_kmeans_assign_bytes", "loopvq_kmeans_step")


def library() -> ctypes.CDLL:
    return _lib


def load_library(path: str) -> ctypes.CDLL:
    """Another build of the library (e.g. a test build), with the same
    argument types declared."""
    return _load(path)


@dataclass(frozen=True)
class LoopVQConfig:
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    n_loops: int
    loop_group: int
    chan_group: int
    n_pages: int
    max_batch: int
    max_pages_per_seq: int
    n_centroids: int = 256
    prefix_tokens: int = 8
    recent_tokens: int = 64
    page_tokens: int = 64

    def c_struct(self) -> _Config:
        c = _Config()
        c.struct_size = ctypes.sizeof(_Config)
        for name, _ in _Config._fields_[1:]:
            setattr(c, name, int(getattr(self, name)))
        return c

    def c_ref(self):
        """A cached ``ctypes.byref`` of the C struct (the config is frozen)."""
        ref = self.__dict__.get("_ref")
        if ref is None:
            s = self.c_struct()
            ref = (s, ctypes.byref(s))
            object.__setattr__(self, "_ref", ref)
        return ref[1]


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != LOOPVQ_OK:
        raise LoopVQError(fn, status)


def loopvq_status_string(status: int) -> str:
    return _lib.loopvq_status_string(int(status)).decode()


def loopvq_cache_layout(cfg: LoopVQConfig) -> dict:
    out = _Layout()
    _check("loopvq_cache_layout", _lib.loopvq_cache_layout(cfg.c_ref(), ctypes.byref(out)))
    return {name: getattr(out, name) for name, _ in _Layout._fields_}


def loopvq_encode(cfg: LoopVQConfig, layer: int, loop_group_idx: int, kv: int, x: torch.Tensor,
                  w: torch.Tensor | None, codebooks: torch.Tensor, slot_mapping: torch.Tensor,
                  pool: torch.Tensor, stream=None) -> None:
    """x: bf16 ``[g][n][Hkv][d]`` with the last two dims dense; w: float32
    ``[g][n][Hkv][d]``, ``[g][1][Hkv][d]`` (shared over tokens) or None."""
    g, n = x.shape[0], x.shape[1]
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if x.stride(3) != 1 or x.stride(2) != x.shape[3]:
        raise ValueError("x rows [Hkv][d] must be dense")
    wl = wt = 0
    if w is not None:
        if w.dtype != torch.float32 or w.stride(3) != 1 or w.stride(2) != w.shape[3]:
            raise ValueError("w must be float32 with dense [Hkv][d] rows")
        wl = w.stride(0)
        wt = w.stride(1) if w.shape[1] != 1 else 0
    st = _lib.loopvq_encode(cfg.c_ref(), layer, loop_group_idx, kv, n, _ptr(x),
                            x.stride(0), x.stride(1) if n > 1 else 0, _ptr(w), wl, wt,
                            _ptr(codebooks), _ptr(slot_mapping), _ptr(pool), _stream(stream))
    _check("loopvq_encode", st)


def loopvq_encode_status(clear: bool = False) -> int:
    """The encoder status word of the current device (LOOPVQ_ENCODE_STATUS_*
    bits); synchronises with the device."""
    v = ctypes.c_int(0)
    _check("loopvq_encode_status", _lib.loopvq_encode_status(ctypes.byref(v), int(clear)))
    return v.value


def loopvq_encode_evict(cfg: LoopVQConfig, x: torch.Tensor, codebooks: torch.Tensor,
                        slot_mapping: torch.Tensor, pool: torch.Tensor, stream=None) -> None:
    """x: dense bf16 ``[L][G][2][g][n][Hkv][d]``, the evicted tokens of every
    (layer, loop group, K/V); slot_mapping: int64 ``[n]``."""
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be dense bfloat16 [L][G][2][g][n][Hkv][d]")
    n = x.shape[4]
    st = _lib.loopvq_encode_evict(cfg.c_ref(), n, _ptr(x), _ptr(codebooks), _ptr(slot_mapping),
                                  _ptr(pool), _stream(stream))
    _check("loopvq_encode_evict", st)


def _xw_strides(x: torch.Tensor, w: torch.Tensor | None) -> tuple[int, int, int, int]:
    n = x.shape[1]
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if x.stride(3) != 1 or x.stride(2) != x.shape[3]:
        raise ValueError("x rows [Hkv][d] must be dense")
    wl = wt = 0
    if w is not None:
        if w.dtype != torch.float32 or w.stride(3) != 1 or w.stride(2) != w.shape[3]:
            raise ValueError("w must be float32 with dense [Hkv][d] rows")
        wl = w.stride(0)
        wt = w.stride(1) if w.shape[1] != 1 else 0
    return x.stride(0), (x.stride(1) if n > 1 else 0), wl, wt


def loopvq_kmeans_assign_bytes(cfg: LoopVQConfig, n_tokens: int) -> int:
    return int(_lib.loopvq_kmeans_assign_bytes(cfg.c_ref(), n_tokens))


def loopvq_kmeans_step(cfg: LoopVQConfig, layer: int, loop_group_idx: int, kv: int, x: torch.Tensor,
                       w: torch.Tensor | None, codebooks: torch.Tensor, assign: torch.Tensor,
                       stream=None) -> None:
    """One weighted Lloyd step on the codebooks of (layer, loop_group_idx,
    kv), in place. x and w as for loopvq_encode; assign: uint8 with at least
    loopvq_kmeans_assign_bytes(cfg, n) bytes, receives [Hkv][J][n]."""
    n = x.shape[1]
    xl, xt, wl, wt = _xw_strides(x, w)
    if assign.dtype != torch.uint8:
        raise TypeError("assign must be uint8")
    st = _lib.loopvq_kmeans_step(cfg.c_ref(), layer, loop_group_idx, kv, n, _ptr(x), xl, xt,
                                 _ptr(w), wl, wt, _ptr(codebooks), _ptr(assign),
                                 assign.numel(), _stream(stream))
    _check("loopvq_kmeans_step", st)


def loopvq_decode_workspace_bytes(cfg: LoopVQConfig, batch: int, max_seq_len: int) -> int:
    return int(_lib.loopvq_decode_workspace_bytes(cfg.c_ref(), batch,
                                                  max_seq_len))


def loopvq_decode_attn(cfg: LoopVQConfig, layer: int, loop_step: int, q: torch.Tensor,
                       pool: torch.Tensor, codebooks: torch.Tensor, block_table: torch.Tensor,
                       seq_lens: torch.Tensor, win_k: torch.Tensor, win_v: torch.Tensor,
                       out: torch.Tensor, workspace: torch.Tensor, max_seq_len: int,
                       lse: torch.Tensor | None = None, sm_scale: float | None = None,
                       stream=None) -> None:
    batch = q.shape[0]
    if sm_scale is None:
        sm_scale = cfg.head_dim ** -0.5
    odt = LOOPVQ_DTYPE_F32 if out.dtype == torch.float32 else LOOPVQ_DTYPE_BF16
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    st = _lib.loopvq_decode_attn(
        cfg.c_ref(), layer, loop_step, batch, max_seq_len, _ptr(q), _ptr(pool),
        _ptr(codebooks), _ptr(block_table), _ptr(seq_lens), _ptr(win_k), _ptr(win_v),
        float(sm_scale), odt, _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("loopvq_decode_attn", st)


def loopvq_prefill_workspace_bytes(cfg: LoopVQConfig, batch: int, n_queries: int,
                                   max_seq_len: int) -> int:
    return int(_lib.loopvq_prefill_workspace_bytes(cfg.c_ref(), batch, n_queries, max_seq_len))


def loopvq_prefill_attn(cfg: LoopVQConfig, layer: int, loop_step: int, q: torch.Tensor,
                        pool: torch.Tensor, codebooks: torch.Tensor, block_table: torch.Tensor,
                        seq_lens: torch.Tensor, win_k: torch.Tensor, win_v: torch.Tensor,
                        out: torch.Tensor, workspace: torch.Tensor, max_seq_len: int,
                        lse: torch.Tensor | None = None, sm_scale: float | None = None,
                        stream=None) -> None:
    """q: bf16 ``[B][Q][Hq][d]``; out ``[B][Q][Hq][d]``; lse ``[B][Q][Hq]``."""
    batch, nq = q.shape[0], q.shape[1]
    if sm_scale is None:
        sm_scale = cfg.head_dim ** -0.5
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    odt = LOOPVQ_DTYPE_F32 if out.dtype == torch.float32 else LOOPVQ_DTYPE_BF16
    st = _lib.loopvq_prefill_attn(
        cfg.c_ref(), layer, loop_step, batch, nq, max_seq_len, _ptr(q), _ptr(pool), _ptr(codebooks),
        _ptr(block_table), _ptr(seq_lens), _ptr(win_k), _ptr(win_v), float(sm_scale), odt, _ptr(out),
        _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("loopvq_prefill_attn", st)


LOOPVQ_STATIC_SCRATCH_BYTES = 32 << 20


def loopvq_decode_attn_noalloc(cfg: LoopVQConfig, layer: int, loop_step: int, q: torch.Tensor,
                               pool: torch.Tensor, codebooks: torch.Tensor,
                               block_table: torch.Tensor, seq_lens: torch.Tensor,
                               win_k: torch.Tensor, win_v: torch.Tensor, out: torch.Tensor,
                               max_seq_len: int, lse: torch.Tensor | None = None,
                               sm_scale: float | None = None, stream=None) -> None:
    """loopvq_decode_attn without a workspace argument: the split scratch is
    the library's own static device array (for callers that cannot
    allocate device memory). Calls that overlap on the GPU race on it."""
    batch = q.shape[0]
    if sm_scale is None:
        sm_scale = cfg.head_dim ** -0.5
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    odt = LOOPVQ_DTYPE_F32 if out.dtype == torch.float32 else LOOPVQ_DTYPE_BF16
    st = _lib.loopvq_decode_attn_noalloc(
        cfg.c_ref(), layer, loop_step, batch, max_seq_len, _ptr(q), _ptr(pool), _ptr(codebooks),
        _ptr(block_table), _ptr(seq_lens), _ptr(win_k), _ptr(win_v), float(sm_scale), odt,
        _ptr(out), _ptr(lse), _stream(stream))
    _check("loopvq_decode_attn_noalloc", st)


def loopvq_bf16_decode_workspace_bytes(batch: int, n_q_heads: int, head_dim: int,
                                       max_seq_len: int) -> int:
    return int(_lib.loopvq_bf16_decode_workspace_bytes(batch, n_q_heads, head_dim, max_seq_len))


def loopvq_bf16_decode_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            seq_lens: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                            lse: torch.Tensor | None = None, sm_scale: float | None = None,
                            stream=None) -> None:
    """q: bf16 ``[B][Hq][d]``; k, v: bf16 ``[B][Hkv][max_seq][d]``."""
    batch, hq, d = q.shape
    hkv, max_seq = k.shape[1], k.shape[2]
    if sm_scale is None:
        sm_scale = d ** -0.5
    odt = LOOPVQ_DTYPE_F32 if out.dtype == torch.float32 else LOOPVQ_DTYPE_BF16
    st = _lib.loopvq_bf16_decode_attn(batch, hq, hkv, d, max_seq, _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(seq_lens), float(sm_scale), odt, _ptr(out), _ptr(lse),
                                      _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream))
    _check("loopvq_bf16_decode_attn", st)
