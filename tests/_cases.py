"""Builders of seeded parity cases shared by the GPU tests.

A case holds host (numpy/torch CPU) copies of every input, runs the oracle
on them, and can upload them to the GPU for the library. Inputs come from
``synthetic`` only; expected values come from ``oracle`` only.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from synthetic import Shape, block_tables, codebooks_for_layer, queries, window_kv

from _guard import Guarded, status_word, workspace

TOL_F32_REL = 1e-4      # fp32 output: per-row max|o - ref| / max|ref|
TOL_BF16_ABS = 2e-2     # bf16 output: max abs, floored at one bf16 ulp of ref
TOL_LSE = 1e-4


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 1e-30)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def random_codebooks(shape: Shape, n_layers: int, seed: int) -> torch.Tensor:
    """``[L][Hkv][G][2][g][J][E][c]`` N(0,1) float32 codebooks (decode parity
    does not need fitted codebooks)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(n_layers, shape.n_kv_heads, shape.G, 2, shape.loop_group, shape.J, 256,
                       shape.chan_group, generator=g)


class DecodeCase:
    """Decode-attention inputs for one (layer, loop step) and every sequence
    of a ragged batch, with random indices packed by the oracle's packer."""

    def __init__(self, shape: Shape, seq_lens, *, layer=0, n_layers=1, loop_step=0, seed=0,
                 q_scale=1.0, fitted_codebooks=False, spare_pages=3, max_pages=None):
        self.shape = shape
        self.seq_lens = list(seq_lens)
        self.B = len(self.seq_lens)
        self.layer, self.n_layers, self.t = layer, n_layers, loop_step
        self.gamma, self.tau = loop_step // shape.loop_group, loop_step % shape.loop_group
        H, Hq, d, J, Pg = shape.n_kv_heads, shape.n_q_heads, shape.head_dim, shape.J, shape.page_tokens
        self.bt, self.n_pages = block_tables(shape, self.B, self.seq_lens, spare_pages=spare_pages,
                                             max_pages=max_pages)
        self.max_pages = self.bt.shape[1]
        if fitted_codebooks:
            cb_l = codebooks_for_layer(shape, layer, n_samples=1024)
            cb = random_codebooks(shape, n_layers, seed + 7)
            cb[layer] = cb_l
        else:
            cb = random_codebooks(shape, n_layers, seed + 7)
        self.cb = cb
        # Every byte of the pool is random: the slots a sequence owns carry
        # its indices (read back per sequence with the oracle's unpacker),
        # everything else is garbage the kernel must not read.
        r = np.random.default_rng(seed)
        self.pool = r.integers(0, 256, size=(n_layers, H, shape.G, self.n_pages, 2, Pg * J),
                               dtype=np.uint8)
        q = queries(shape, layer, loop_step, batch=self.B).float() * q_scale
        self.q = q.to(torch.bfloat16)
        self.win_k = window_kv(shape, layer, loop_step, 0, batch=self.B)
        self.win_v = window_kv(shape, layer, loop_step, 1, batch=self.B)
        self.max_seq_len = max(self.seq_lens + [0])
        self.sm_scale = 1.0 / math.sqrt(d)

    def config(self) -> L.LoopVQConfig:
        s = self.shape
        return L.LoopVQConfig(n_layers=self.n_layers, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                              head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                              chan_group=s.chan_group, n_pages=self.n_pages, max_batch=self.B,
                              max_pages_per_seq=self.max_pages, prefix_tokens=s.prefix,
                              recent_tokens=s.recent, page_tokens=s.page_tokens)

    def oracle(self, b: int, hq: int):
        s = self.shape
        hkv = hq // (s.n_q_heads // s.n_kv_heads)
        N = self.seq_lens[b]
        nw = O.n_window_tokens(N, s.prefix, s.recent)
        iK, iV = self.indices(b, hkv)
        cbK = self.cb[self.layer, hkv, self.gamma, 0].double().numpy()
        cbV = self.cb[self.layer, hkv, self.gamma, 1].double().numpy()
        if N == 0:
            return np.zeros(s.head_dim), -math.inf
        return O.decode_attn_ref(self.q[b, hq].double().numpy(),
                                 self.win_k[b, hkv, :nw].double().numpy(),
                                 self.win_v[b, hkv, :nw].double().numpy(),
                                 iK, iV, cbK, cbV, self.tau, self.sm_scale)

    def indices(self, b: int, hkv: int):
        """Logical (idx_K, idx_V) ``[n_vq][J]`` of sequence b, kv-head hkv."""
        s = self.shape
        n = O.n_vq_tokens(self.seq_lens[b], s.prefix, s.recent)
        plane = self.pool[self.layer, hkv, self.gamma]
        row = self.bt[b].numpy()
        return (O.unpack_sequence(plane, n, s.J, row, s.page_tokens, 0),
                O.unpack_sequence(plane, n, s.J, row, s.page_tokens, 1))

    def run_gpu(self, out_dtype=torch.float32, dev="cuda"):
        cfg = self.config()
        pool = torch.from_numpy(self.pool).to(dev)
        cb = self.cb.to(dev)
        bt = self.bt.to(dev)
        sl = torch.tensor(self.seq_lens, dtype=torch.int32, device=dev)
        q = self.q.to(dev)
        wk, wv = self.win_k.to(dev), self.win_v.to(dev)
        s = self.shape
        out = Guarded((self.B, s.n_q_heads, s.head_dim), out_dtype, fill=float("nan"), device=dev)
        lse = Guarded((self.B, s.n_q_heads), torch.float32, fill=float("nan"), device=dev)
        ws = workspace(L.loopvq_decode_workspace_bytes(cfg, self.B, self.max_seq_len), device=dev)
        L.loopvq_decode_attn(cfg, self.layer, self.t, q, pool, cb, bt, sl, wk, wv, out.t, ws.t,
                             self.max_seq_len, lse=lse.t, sm_scale=self.sm_scale)
        torch.cuda.synchronize()
        out.check("output")
        lse.check("lse")
        ws.check("workspace")
        assert status_word(ws) == 0, f"decode status {status_word(ws)}"
        return out.t.float().cpu().numpy(), lse.t.cpu().numpy()


def check_decode(case: DecodeCase, out: np.ndarray, lse: np.ndarray, out_dtype, pairs=None):
    """Compare GPU out/lse with the oracle on every (b, hq) (or `pairs`)."""
    s = case.shape
    if pairs is None:
        pairs = [(b, h) for b in range(case.B) for h in range(s.n_q_heads)]
    worst = 0.0
    for b, h in pairs:
        ref, lref = case.oracle(b, h)
        o = out[b, h].astype(np.float64)
        assert np.all(np.isfinite(o)), (b, h)
        if case.seq_lens[b] == 0:
            assert np.all(o == 0) and lse[b, h] == -np.inf
            continue
        if out_dtype == torch.float32:
            rel = np.max(np.abs(o - ref)) / max(np.max(np.abs(ref)), 1e-30)
            assert rel <= TOL_F32_REL, (b, h, rel)
            worst = max(worst, rel)
        else:
            err = np.abs(o - ref)
            lim = np.maximum(TOL_BF16_ABS, bf16_ulp(ref))
            assert np.all(err <= lim), (b, h, float(np.max(err - lim)))
            worst = max(worst, float(np.max(err)))
        assert abs(float(lse[b, h]) - lref) <= TOL_LSE, (b, h, float(lse[b, h]), lref)
    return worst


def check_indices(gpu_idx: np.ndarray, dist: np.ndarray, rel: float = 1e-5) -> int:
    """Indices must equal the oracle's argmin except in near ties: when the
    oracle's best two distances d1 <= d2 differ by less than rel*d1, the GPU
    choice must lie within rel*d1 of d1. Returns the number of near-tie
    cases that took a different index."""
    flat_d = dist.reshape(-1, dist.shape[-1])
    flat_i = gpu_idx.reshape(-1).astype(np.int64)
    srt = np.sort(flat_d, axis=1)
    d1, d2 = srt[:, 0], srt[:, 1]
    ref = np.argmin(flat_d, axis=1)
    tie = (d2 - d1) < rel * d1
    bad_exact = (~tie) & (flat_i != ref)
    assert not bad_exact.any(), f"{int(bad_exact.sum())} indices differ outside near ties"
    chosen = flat_d[np.arange(flat_d.shape[0]), flat_i]
    assert np.all(chosen - d1 <= rel * d1 + 0.0), "near-tie choice outside the margin"
    return int(((flat_i != ref) & tie).sum())


class DeviceDecodeCase:
    """Decode inputs at full configuration size for one (layer, loop step).

    The pool lives on the GPU only: either random bytes drawn there (seeded),
    or a pool the caller filled (e.g. with the GPU encoder). The oracle of a
    pair reads back just that pair's pages. Codebooks, queries and windows
    are host tensors copied to the GPU once."""

    def __init__(self, shape: Shape, seq_lens, *, loop_step=0, seed=0, q_scale=1.0, cb=None,
                 pool=None, bt=None, dev="cuda"):
        self.shape = shape
        self.seq_lens = list(seq_lens)
        self.B = len(self.seq_lens)
        self.layer, self.n_layers, self.t = 0, 1, loop_step
        self.gamma, self.tau = loop_step // shape.loop_group, loop_step % shape.loop_group
        H, J, Pg = shape.n_kv_heads, shape.J, shape.page_tokens
        if bt is None:
            bt = block_tables(shape, self.B, self.seq_lens, spare_pages=1)
        self.bt, self.n_pages = bt[0].cpu(), bt[1]
        self.max_pages = self.bt.shape[1]
        self.cb = random_codebooks(shape, 1, seed + 7) if cb is None else cb.cpu()
        if pool is None:
            g = torch.Generator(device=dev)
            g.manual_seed(seed)
            pool = torch.randint(0, 256, (1, H, shape.G, self.n_pages, 2, Pg * J), generator=g,
                                 dtype=torch.uint8, device=dev)
        self.pool = pool
        self.q = (queries(shape, 0, loop_step, batch=self.B).float() * q_scale).to(torch.bfloat16)
        self.win_k = window_kv(shape, 0, loop_step, 0, batch=self.B)
        self.win_v = window_kv(shape, 0, loop_step, 1, batch=self.B)
        self.max_seq_len = max(self.seq_lens + [0])
        self.sm_scale = 1.0 / math.sqrt(shape.head_dim)
        self.dev = dev

    config = DecodeCase.config
    oracle = DecodeCase.oracle

    def indices(self, b: int, hkv: int):
        s = self.shape
        n = O.n_vq_tokens(self.seq_lens[b], s.prefix, s.recent)
        pages = -(-n // s.page_tokens)
        phys = self.bt[b, :pages].long().to(self.dev)
        plane = self.pool.view(1, s.n_kv_heads, s.G, self.n_pages, 2, -1)[0, hkv, self.gamma][phys]
        plane = plane.cpu().numpy()                    # this pair's pages, in table order
        row = np.arange(pages)
        return (O.unpack_sequence(plane, n, s.J, row, s.page_tokens, 0),
                O.unpack_sequence(plane, n, s.J, row, s.page_tokens, 1))

    def run_gpu(self, out_dtype=torch.float32):
        dev = self.dev
        cfg = self.config()
        s = self.shape
        cb, bt = self.cb.to(dev), self.bt.to(dev)
        sl = torch.tensor(self.seq_lens, dtype=torch.int32, device=dev)
        q, wk, wv = self.q.to(dev), self.win_k.to(dev), self.win_v.to(dev)
        out = Guarded((self.B, s.n_q_heads, s.head_dim), out_dtype, fill=float("nan"), device=dev)
        lse = Guarded((self.B, s.n_q_heads), torch.float32, fill=float("nan"), device=dev)
        ws = workspace(L.loopvq_decode_workspace_bytes(cfg, self.B, self.max_seq_len), device=dev)
        L.loopvq_decode_attn(cfg, self.layer, self.t, q, self.pool, cb, bt, sl, wk, wv, out.t, ws.t,
                             self.max_seq_len, lse=lse.t, sm_scale=self.sm_scale)
        torch.cuda.synchronize()
        out.check("output")
        lse.check("lse")
        ws.check("workspace")
        assert status_word(ws) == 0, f"decode status {status_word(ws)}"
        return out.t.float().cpu().numpy(), lse.t.cpu().numpy()


def sample_pairs(B: int, Hq: int, n: int, seed: int, whole=()):
    """``n`` random (sequence, head) pairs plus every head of the sequences in
    ``whole``."""
    r = np.random.default_rng(seed)
    pairs = {(int(b), int(h)) for b, h in zip(r.integers(0, B, n), r.integers(0, Hq, n))}
    pairs |= {(b, h) for b in whole for h in range(Hq)}
    return sorted(pairs)
