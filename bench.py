#!/usr/bin/env python
"""Benchmark of the LoopVQ decode hot path on B200.

One step = one decode token of the whole stack on the 32K-context workload
(48 layers, 16 kv-heads, head_dim 128, 4 loop steps coded in one group of
g=4 with c=4 channels, 0.5 bit per element, batch 8, context 32768 with 8
prefix + 64 recent bf16 tokens): for every loop step t and layer l one fused
decode-attention call, then the eviction encode of the token that leaves the
recent window (batch tokens, every layer, loop group and K/V). The reported
metric is microseconds per loop step (48 decode calls) of the whole job;
`roofline` gives the decode kernel's effective cache-read bandwidth against
the measured HBM copy bandwidth.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun (N > 1) every rank runs the same per-GPU workload (weak
scaling, no collective on the data path); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "VQ-KV decode attn µs/loop-step @32K; effective cache GB/s vs HBM roofline"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="loopvq", choices=["loopvq", "reference"])
    ap.add_argument("--config", default="long32k")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the bf16-KV comparison and the prefill encode leg")
    ap.add_argument("--layers", type=int, default=None,
                    help="fewer layers with the same per-call shape (small profiling case)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    return ap.parse_args()


# --------------------------------------------------------------------------
# process group
# --------------------------------------------------------------------------

def dist_init(n_gpus: int):
    """One process per GPU (torchrun env). NCCL between GPUs; gloo when no
    GPU is visible (the host-side logic is exercised that way on CPU)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=300)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(elapsed_ms: float, steps: int, n_loops: int, world: int):
    """µs per loop step of the whole job and ms per bench step. Every rank
    runs `steps` steps of `n_loops` loop steps on its own replica (weak
    scaling); elapsed_ms is the max over ranks."""
    loop_steps = steps * n_loops * world
    return elapsed_ms * 1e3 / loop_steps, elapsed_ms / steps


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def call_percentiles(times: list[float]) -> list[float]:
    """p10, median and p90 of per-call times (nearest rank on the sorted list)."""
    t = sorted(times)
    if not t:
        return [float("nan")] * 3
    pick = lambda q: t[min(len(t) - 1, max(0, int(round(q * (len(t) - 1)))))]
    return [pick(0.1), pick(0.5), pick(0.9)]


def recorded_traffic(kernel_src: str, key: str):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh).get(key)
    if not d:
        return None
    with open(os.path.join(ROOT, kernel_src), "rb") as fh:
        h = hashlib.sha256(fh.read()).hexdigest()[:16]
    return d["dram_bytes_per_launch"] if d.get("source_sha256_16") == h else None


# --------------------------------------------------------------------------
# workload
# --------------------------------------------------------------------------

class Workload:
    """Device-resident inputs of the decode step for one GPU."""

    def __init__(self, shape, device, quick_codebooks=False):
        import torch

        import sub_bit_vq_b200 as L
        from synthetic import block_tables, codebooks_for_layer, loop_group_kv, queries, window_kv

        s = self.shape = shape
        self.dev = device
        B, H, Hq, d, T, g, G = (s.batch, s.n_kv_heads, s.n_q_heads, s.head_dim, s.n_loops,
                                s.loop_group, s.G)
        self.seq_lens = [s.context] * B
        bt, n_used = block_tables(s, B, self.seq_lens)
        self.n_pages = n_used + 1                  # one spare page takes the eviction writes
        self.cfg = L.LoopVQConfig(
            n_layers=s.n_layers, n_kv_heads=H, n_q_heads=Hq, head_dim=d, n_loops=T,
            loop_group=g, chan_group=s.chan_group, n_pages=self.n_pages, max_batch=B,
            max_pages_per_seq=bt.shape[1], prefix_tokens=s.prefix, recent_tokens=s.recent,
            page_tokens=s.page_tokens)
        lay = L.loopvq_cache_layout(self.cfg)
        self.layout = lay
        self.bt = bt.to(device)
        self.sl = torch.tensor(self.seq_lens, dtype=torch.int32, device=device)
        self.max_seq_len = s.context
        # codebooks: Lloyd k-means per (layer, head, group, K/V, channel group)
        self.cb = torch.empty(s.n_layers, H, G, 2, g, s.J, 256, s.chan_group, device=device)
        for l in range(s.n_layers):
            self.cb[l] = codebooks_for_layer(s, l, device=device,
                                             n_samples=1024 if quick_codebooks else 2048,
                                             iters=20)
        # packed index pool, filled by the GPU encoder from synthetic K/V
        self.pool = torch.zeros(lay["pool_bytes"], dtype=torch.uint8, device=device)
        n_vq = s.n_vq
        v = torch.arange(n_vq, device=device)
        slots = torch.cat([self.bt[b][v // s.page_tokens].long() * s.page_tokens + v % s.page_tokens
                           for b in range(B)])
        chunk = 1 << 16
        for l in range(s.n_layers):
            for gamma in range(G):
                for kv in range(2):
                    x = loop_group_kv(s, l, gamma, kv, B * n_vq, device=device)
                    for c0 in range(0, B * n_vq, chunk):
                        L.loopvq_encode(self.cfg, l, gamma, kv, x[:, c0:c0 + chunk], None, self.cb,
                                        slots[c0:c0 + chunk], self.pool)
                    del x
        # bf16 windows, queries and outputs for every (layer, loop step)
        W = s.window
        self.win_k = torch.empty(s.n_layers, T, B, H, W, d, dtype=torch.bfloat16, device=device)
        self.win_v = torch.empty_like(self.win_k)
        self.q = torch.empty(s.n_layers, T, B, Hq, d, dtype=torch.bfloat16, device=device)
        for l in range(s.n_layers):
            for t in range(T):
                self.win_k[l, t] = window_kv(s, l, t, 0, device=device)
                self.win_v[l, t] = window_kv(s, l, t, 1, device=device)
                self.q[l, t] = queries(s, l, t, device=device)
        self.out = torch.empty(s.n_layers, T, B, Hq, d, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(s.n_layers, T, B, Hq, dtype=torch.float32, device=device)
        ws = L.loopvq_decode_workspace_bytes(self.cfg, B, self.max_seq_len)
        self.ws = torch.zeros(ws // 4 + 4, dtype=torch.float32, device=device)   # zero counters
        # eviction encode inputs: the token leaving the recent window, g loops
        self.evict = torch.empty(s.n_layers, G, 2, g, B, H, d, dtype=torch.bfloat16, device=device)
        for l in range(s.n_layers):
            for gamma in range(G):
                for kv in range(2):
                    self.evict[l, gamma, kv] = loop_group_kv(s, l, gamma, kv, B, device=device,
                                                             stream=7)
        spare = self.n_pages - 1
        self.evict_slots = torch.arange(B, device=device, dtype=torch.int64) + spare * s.page_tokens
        torch.cuda.synchronize()

    def decode_call(self, l, t, stream):
        import sub_bit_vq_b200 as L
        L.loopvq_decode_attn(self.cfg, l, t, self.q[l, t], self.pool, self.cb, self.bt, self.sl,
                             self.win_k[l, t], self.win_v[l, t], self.out[l, t], self.ws,
                             self.max_seq_len, lse=self.lse[l, t], stream=stream)

    def evict_encode(self, stream):
        """The tokens leaving the recent window, every layer, loop group and
        K/V, in one launch."""
        import sub_bit_vq_b200 as L
        L.loopvq_encode_evict(self.cfg, self.evict, self.cb, self.evict_slots, self.pool, stream=stream)

    def launches_per_step(self):
        """Kernels per step: two per decode call (the pair kernel, the
        streaming kernel) and one for the eviction encode."""
        s = self.shape
        return s.n_loops * s.n_layers * 2 + 1

    def step(self, stream, events=None):
        s = self.shape
        for t in range(s.n_loops):
            for l in range(s.n_layers):
                if events is not None:
                    e0, e1 = events.pop()
                    e0.record(stream)
                    self.decode_call(l, t, stream.cuda_stream)
                    e1.record(stream)
                else:
                    self.decode_call(l, t, stream.cuda_stream)
        self.evict_encode(stream.cuda_stream)

    def algorithmic_bytes_per_call(self):
        s = self.shape
        n_vq = s.n_vq
        idx = 2 * s.J * n_vq * s.batch * s.n_q_heads
        win = 2 * min(s.context, s.window) * s.head_dim * 2 * s.batch * s.n_kv_heads
        cb = 2 * 256 * s.head_dim * 4 * s.n_kv_heads
        io = s.batch * s.n_q_heads * (s.head_dim * 2 * 2 + 4)
        return idx + win + cb + io


# --------------------------------------------------------------------------
# CPU baseline: the oracle on the host cores
# --------------------------------------------------------------------------

def cpu_baseline(shape, budget_s=10.0):
    """Time the float64 oracle on (sequence, head) slices of one decode call
    of the workload and scale to one loop step (all layers); returns the
    cpu_baseline record. Inputs are random indices and codebooks of the
    workload's shape (timing does not depend on their values)."""
    import numpy as np
    import torch

    from oracle import loopvq_oracle as O

    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    torch.set_num_threads(threads)
    s = shape
    r = np.random.default_rng(0)
    n_vq = s.n_vq
    nw = min(s.context, s.window)
    cb = r.normal(size=(s.loop_group, s.J, 256, s.chan_group))
    q = r.normal(size=s.head_dim)
    wk, wv = r.normal(size=(nw, s.head_dim)), r.normal(size=(nw, s.head_dim))
    iK = r.integers(0, 256, size=(n_vq, s.J), dtype=np.uint8)
    iV = r.integers(0, 256, size=(n_vq, s.J), dtype=np.uint8)
    done, t0 = 0, time.perf_counter()
    while True:
        O.decode_attn_ref(q, wk, wv, iK, iV, cb, cb, 1, 1.0 / math.sqrt(s.head_dim))
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= 64:
            break
    per_pair = el / done
    pairs_per_loop_step = s.batch * s.n_q_heads * s.n_layers
    us = per_pair * pairs_per_loop_step * 1e6
    return {"value": us, "unit": "µs/loop-step", "cores": threads, "kind": "oracle",
            "sample": f"{done} (sequence, head) slices of one call at full context "
                      f"({n_vq} quantised + {nw} window tokens) in {el:.1f} s, "
                      f"scaled x{pairs_per_loop_step} to one loop step (extrapolated)"}


# --------------------------------------------------------------------------
# extras: bf16-KV comparison and prefill encode throughput
# --------------------------------------------------------------------------

def bf16_comparison(shape, device, reps=20):
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import queries

    s = shape
    B, H, d, N = s.batch, s.n_kv_heads, s.head_dim, s.context
    nbuf = 3
    ks = [torch.randn(B, H, N, d, device=device, dtype=torch.bfloat16) for _ in range(nbuf)]
    vs = [torch.randn(B, H, N, d, device=device, dtype=torch.bfloat16) for _ in range(nbuf)]
    q = queries(s, 0, 0, device=device)
    sl = torch.full((B,), N, dtype=torch.int32, device=device)
    out = torch.empty(B, s.n_q_heads, d, dtype=torch.bfloat16, device=device)
    ws = torch.empty(L.loopvq_bf16_decode_workspace_bytes(B, s.n_q_heads, d, N) // 4 + 4,
                     device=device)
    st = torch.cuda.current_stream()
    for i in range(3):
        L.loopvq_bf16_decode_attn(q, ks[i % nbuf], vs[i % nbuf], sl, out, ws, stream=st.cuda_stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    torch.cuda.synchronize()
    for i in range(reps):
        ev[i][0].record(st)
        L.loopvq_bf16_decode_attn(q, ks[i % nbuf], vs[i % nbuf], sl, out, ws, stream=st.cuda_stream)
        ev[i][1].record(st)
    torch.cuda.synchronize()
    us = statistics.median(a.elapsed_time(b) * 1e3 for a, b in ev)
    nbytes = 2 * B * H * N * d * 2 + B * s.n_q_heads * d * 4
    del ks, vs
    torch.cuda.empty_cache()
    return {"us_per_call": us, "gbps": nbytes / us / 1e3, "bytes_per_call": nbytes,
            "shape": f"B={B} Hkv={H} d={d} N={N} bf16 K/V"}


def alg_bytes_per_call(shape, seq_lens) -> int:
    """Bytes one decode call must move: the packed K and V indices of every
    quantised token of every (sequence, query head), the bf16 window tokens,
    the loop-step slice of the K and V codebooks of every kv-head, and q,
    out (bf16) and lse."""
    s = shape
    n_vq = sum(max(0, n - s.window) for n in seq_lens)
    n_win = sum(min(n, s.window) for n in seq_lens)
    idx = 2 * s.J * n_vq * s.n_q_heads
    win = 2 * n_win * s.head_dim * 2 * s.n_kv_heads
    cb = 2 * 256 * s.head_dim * 4 * s.n_kv_heads
    io = len(seq_lens) * s.n_q_heads * (s.head_dim * 2 * 2 + 4)
    return idx + win + cb + io


def encoded_layers(shape, n_layers, seq_lens, gammas, device, chunk=1 << 18):
    """A pool of `n_layers` layers whose indices the GPU encoder wrote from the
    synthetic loop-group K/V of the shape (codebooks fitted by Lloyd on
    samples of the same distribution), for the loop groups `gammas`. Returns
    (config, pool, codebooks, block table)."""
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import block_tables, codebooks_for_layer, loop_group_kv

    s = shape
    B = len(seq_lens)
    bt, n_pages = block_tables(s, B, seq_lens)
    cfg = L.LoopVQConfig(n_layers=n_layers, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                         head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                         chan_group=s.chan_group, n_pages=n_pages, max_batch=B,
                         max_pages_per_seq=bt.shape[1], prefix_tokens=s.prefix,
                         recent_tokens=s.recent, page_tokens=s.page_tokens)
    pool = torch.zeros(L.loopvq_cache_layout(cfg)["pool_bytes"], dtype=torch.uint8, device=device)
    cb = torch.empty(n_layers, s.n_kv_heads, s.G, 2, s.loop_group, s.J, 256, s.chan_group,
                     device=device)
    btd = bt.to(device)
    slots = []
    for b, n in enumerate(seq_lens):
        v = torch.arange(max(0, n - s.window), device=device)
        slots.append(btd[b][v // s.page_tokens].long() * s.page_tokens + v % s.page_tokens)
    slots = torch.cat(slots)
    total = int(slots.numel())
    for l in range(n_layers):
        cb[l] = codebooks_for_layer(s, l, device=device, n_samples=1024, iters=10)
        for gamma in gammas:
            for kv in range(2):
                for k, c0 in enumerate(range(0, total, chunk)):
                    n = min(chunk, total - c0)
                    x = loop_group_kv(s, l, gamma, kv, n, device=device, stream=k)
                    L.loopvq_encode(cfg, l, gamma, kv, x, None, cb, slots[c0:c0 + n], pool)
                    del x
    torch.cuda.synchronize()
    return cfg, pool, cb, btd


def time_calls(calls, reps, warm=3):
    """Per-call device times (CUDA events around each call, queue kept full)
    and the back-to-back average of `reps` calls without events, in µs.
    `calls` is a list of callables taking a stream handle; they rotate."""
    import torch
    st = torch.cuda.current_stream()
    for i in range(warm):
        calls[i % len(calls)](st.cuda_stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    torch.cuda.synchronize()
    for i in range(reps):
        ev[i][0].record(st)
        calls[i % len(calls)](st.cuda_stream)
        ev[i][1].record(st)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) * 1e3 for a, b in ev]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(reps):
        calls[i % len(calls)](st.cuda_stream)
    e1.record(st)
    torch.cuda.synchronize()
    return per, e0.elapsed_time(e1) * 1e3 / reps


def decode_row(shape, seq_lens, n_layers, loop_steps, device, peak, l2_bytes, rotate_seqs=None):
    """One measured decode configuration: the LoopVQ call (layers, or
    sequence subsets, rotate so that the calls of a round move at least 4x
    the L2 size) and the same-shape bf16-KV kernel beside it."""
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import queries, window_kv

    s = shape
    B = len(seq_lens)
    gammas = sorted({t // s.loop_group for t in loop_steps})
    all_lens = seq_lens if rotate_seqs is None else seq_lens * rotate_seqs
    cfg, pool, cb, bt = encoded_layers(s, n_layers, all_lens, gammas, device)
    nb = len(all_lens)
    sl_all = torch.tensor(all_lens, dtype=torch.int32, device=device)
    max_len = max(seq_lens)
    wsb = L.loopvq_decode_workspace_bytes(cfg, B, max_len)
    alg = alg_bytes_per_call(s, seq_lens)
    n_rot = max(1, -(-4 * l2_bytes // alg))
    calls = []
    keep = []
    for k in range(n_rot):
        l = k % n_layers
        r = (k // n_layers) % (nb // B)
        t = loop_steps[k % len(loop_steps)]
        q = queries(s, l, t, batch=nb, device=device)[r * B:(r + 1) * B].contiguous()
        wk = window_kv(s, l, t, 0, batch=nb, device=device)[r * B:(r + 1) * B].contiguous()
        wv = window_kv(s, l, t, 1, batch=nb, device=device)[r * B:(r + 1) * B].contiguous()
        out = torch.empty(B, s.n_q_heads, s.head_dim, dtype=torch.bfloat16, device=device)
        lse = torch.empty(B, s.n_q_heads, device=device)
        ws = torch.zeros(wsb // 4 + 4, device=device)
        btr, slr = bt[r * B:(r + 1) * B], sl_all[r * B:(r + 1) * B]
        keep.append((q, wk, wv, out, lse, ws, btr, slr))

        def call(stream, l=l, t=t, a=keep[-1]):
            L.loopvq_decode_attn(cfg, l, t, a[0], pool, cb, a[6], a[7], a[1], a[2], a[3], a[5],
                                 max_len, lse=a[4], stream=stream)
        calls.append(call)
    per, avg = time_calls(calls, reps=max(30, n_rot))
    p10, med, p90 = call_percentiles(per)
    row = {"batch": B, "context": max_len, "us_per_call": med, "us_p10_median_p90": [p10, med, p90],
           "us_back_to_back": avg, "alg_bytes_per_call": alg, "gbps": alg / med / 1e3,
           "frac_of_measured_hbm": alg / med / 1e3 / peak, "rotation": n_rot}
    del keep, calls, pool
    torch.cuda.empty_cache()
    # the same-shape bf16-KV kernel: distinct K/V per rotation
    n_rot_b = max(1, -(-4 * l2_bytes // (2 * B * s.n_kv_heads * max_len * s.head_dim * 2)))
    ks = [torch.randn(B, s.n_kv_heads, max_len, s.head_dim, device=device, dtype=torch.bfloat16)
          for _ in range(n_rot_b)]
    vs = [torch.randn_like(k) for k in ks]
    qb = queries(s, 0, 0, batch=B, device=device)
    slb = torch.tensor(seq_lens, dtype=torch.int32, device=device)
    outb = torch.empty(B, s.n_q_heads, s.head_dim, dtype=torch.bfloat16, device=device)
    wsb2 = torch.empty(L.loopvq_bf16_decode_workspace_bytes(B, s.n_q_heads, s.head_dim, max_len) // 4 + 4,
                       device=device)
    bcalls = [lambda st, k=k, v=v: L.loopvq_bf16_decode_attn(qb, k, v, slb, outb, wsb2, stream=st)
              for k, v in zip(ks, vs)]
    per_b, _ = time_calls(bcalls, reps=20)
    row["bf16_us_per_call"] = statistics.median(per_b)
    row["vq_speedup_vs_bf16"] = row["bf16_us_per_call"] / med
    del ks, vs
    torch.cuda.empty_cache()
    return row


def decode_rows(device, peak):
    """The decode batch sweep (batch 1..256 at context 16384, 16 heads,
    d = 128, 0.5 bit) and the per-call rows of the other configurations,
    each beside the same-shape bf16-KV kernel."""
    import torch
    from synthetic import SHAPES

    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    sw = SHAPES["sweep"]
    sweep = []
    for B in (1, 2, 4, 8, 16, 32, 64, 128, 256):
        rot = max(1, min(256 // B, -(-4 * l2 // alg_bytes_per_call(sw, [sw.context] * B))))
        sweep.append(decode_row(sw.with_(batch=B), [sw.context] * B, 1, [0, sw.n_loops - 1], device,
                                peak, l2, rotate_seqs=rot))
    rows = {"sweep": sweep}
    o = SHAPES["ouro14"]
    rows["ouro14"] = decode_row(o, [o.context] * o.batch, 4, [0, o.n_loops - 1], device, peak, l2)
    dp = SHAPES["deep025"]
    rows["deep025"] = decode_row(dp.with_(n_layers=1), [dp.context] * dp.batch, 1,
                                 [0, dp.n_loops - 1], device, peak, l2)
    rows["prefill"] = prefill_row(device, peak)
    return rows


def prefill_row(device, peak, Q=128, B=2):
    """A chunk of Q = 128 new queries per sequence over a 16384-token cached
    context (16 heads, d = 128, 0.5 bit), against Q single-query decode
    calls on the same cache."""
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import SHAPES, queries, window_kv

    s = SHAPES["sweep"].with_(batch=B)
    cfg, pool, cb, bt = encoded_layers(s, 1, [s.context] * B, [0], device)
    sl = torch.full((B,), s.context, dtype=torch.int32, device=device)
    g = torch.Generator(device=device).manual_seed(5)
    q = torch.randn(B, Q, s.n_q_heads, s.head_dim, generator=g, device=device).to(torch.bfloat16)
    wk, wv = window_kv(s, 0, 0, 0, batch=B, device=device), window_kv(s, 0, 0, 1, batch=B, device=device)
    out = torch.empty(B, Q, s.n_q_heads, s.head_dim, dtype=torch.bfloat16, device=device)
    lse = torch.empty(B, Q, s.n_q_heads, device=device)
    ws = torch.zeros(L.loopvq_prefill_workspace_bytes(cfg, B, Q, s.context) // 4 + 4, device=device)
    call = lambda st: L.loopvq_prefill_attn(cfg, 0, 0, q, pool, cb, bt, sl, wk, wv, out, ws, s.context,
                                            lse=lse, stream=st)
    per, _ = time_calls([call], reps=10)
    us = statistics.median(per)
    alg = alg_bytes_per_call(s, [s.context] * B)     # the cache once, plus Q-fold q/out
    alg += B * (Q - 1) * s.n_q_heads * (s.head_dim * 2 * 2 + 4)
    # the same queries one decode call at a time
    qd = q[:, 0].contiguous()
    outd = torch.empty(B, s.n_q_heads, s.head_dim, dtype=torch.bfloat16, device=device)
    wsd = torch.zeros(L.loopvq_decode_workspace_bytes(cfg, B, s.context) // 4 + 4, device=device)
    dcall = lambda st: L.loopvq_decode_attn(cfg, 0, 0, qd, pool, cb, bt, sl, wk, wv, outd, wsd, s.context,
                                            stream=st)
    perd, _ = time_calls([dcall], reps=20)
    return {"batch": B, "queries_per_seq": Q, "context": s.context, "us_per_call": us,
            "queries_per_s": B * Q * s.n_q_heads / (us * 1e-6), "alg_bytes_per_call": alg,
            "gbps": alg / us / 1e3, "frac_of_measured_hbm": alg / us / 1e3 / peak,
            "decode_us_per_query_chunk_of_1": statistics.median(perd),
            "speedup_vs_q_decode_calls": Q * statistics.median(perd) / us}


def encode_prefill(device, reps=3):
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import SHAPES, codebooks_for_layer, loop_group_kv, weights

    s = SHAPES["sweep"]
    n = 32768
    cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                         head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                         chan_group=s.chan_group, n_pages=n // s.page_tokens, max_batch=1,
                         max_pages_per_seq=n // s.page_tokens)
    cb = codebooks_for_layer(s, 0, device=device, n_samples=1024, iters=10)[None].contiguous()
    pool = torch.zeros(L.loopvq_cache_layout(cfg)["pool_bytes"], dtype=torch.uint8, device=device)
    x = loop_group_kv(s, 0, 0, 0, n, device=device)
    w = weights(s, n, True, device=device)
    slots = torch.arange(n, device=device, dtype=torch.int64)
    st = torch.cuda.current_stream()
    L.loopvq_encode(cfg, 0, 0, 0, x, w, cb, slots, pool, stream=st.cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(reps):
        L.loopvq_encode(cfg, 0, 0, 0, x, w, cb, slots, pool, stream=st.cuda_stream)
    e1.record(st)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3 / reps
    nsub = n * s.n_kv_heads * s.J
    return {"subvectors_per_s": nsub / sec, "ms_per_call": sec * 1e3,
            "shape": f"{n} tokens x {s.n_kv_heads} heads x {s.J} groups, D={s.D}, "
                     f"per-token LogNormal weights, one of K/V",
            "kernel": "tcgen05 scaled-fp16 contraction + exact float32 rescore (tensor cores)",
            "bounds": encode_bounds(nsub, s.D, sec)}


def encode_bounds(nsub: int, D: int, sec: float) -> dict:
    """The encoder's three candidate bounds for nsub sub-vectors of D
    elements with per-token weights, as fractions achieved in `sec`:
    - hbm: bf16 x and float32 w read, one index byte written;
    - tensor: the cross and weight terms of the distance, 2 * (2 D) * 256
      flops per sub-vector (the algorithmic count, issued as one fp16
      product per term), against the measured bf16 GEMM rate (fp16 runs
      at the same rate);
    - alu: 256 candidates x 3 operations (bias add, compare, select) per
      sub-vector, against 148 SMs x 128 float32 lanes x the maximum SM clock."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = json.load(open(p)) if os.path.exists(p) else {}
    hbm = float(d.get("hbm_gbs", FALLBACK_HBM_GBS)) * 1e9
    tflops = float(d.get("bf16_tflops", 1590.0)) * 1e12
    mhz = float(d.get("sm_max_mhz", 1965.0)) * 1e6
    byt = nsub * (D * 2 + D * 4 + 1)
    flop = nsub * 2 * (2 * D) * 256
    alu = nsub * 256 * 3
    alu_peak = 148 * 128 * mhz
    return {"hbm_frac": byt / sec / hbm, "tensor_frac": flop / sec / tflops,
            "alu_frac": alu / sec / alu_peak, "bytes": byt, "flops": flop, "alu_ops": alu,
            "peaks": "MEASURED_PEAKS.json hbm_gbs and bf16_tflops; alu from 148 x 128 lanes x sm_max_mhz"}


def kmeans_step(device, reps=3):
    """One weighted Lloyd step of the codebooks of one (layer, loop group,
    K/V) on the 32768-token prefill sample: the assignment (the encoder,
    writing indices to an array) plus the weighted centroid update. The
    update kernel is timed alone too, against the HBM bytes it must move."""
    import torch

    import sub_bit_vq_b200 as L
    from synthetic import SHAPES, codebooks_for_layer, loop_group_kv, weights

    s = SHAPES["sweep"]
    n = 32768
    cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=s.n_kv_heads, n_q_heads=s.n_q_heads,
                         head_dim=s.head_dim, n_loops=s.n_loops, loop_group=s.loop_group,
                         chan_group=s.chan_group, n_pages=n // s.page_tokens, max_batch=1,
                         max_pages_per_seq=n // s.page_tokens)
    cb = codebooks_for_layer(s, 0, device=device, n_samples=1024, iters=10)[None].contiguous()
    x = loop_group_kv(s, 0, 0, 0, n, device=device)
    w = weights(s, n, True, device=device)
    assign = torch.empty(L.loopvq_kmeans_assign_bytes(cfg, n), dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    L.loopvq_kmeans_step(cfg, 0, 0, 0, x, w, cb, assign, stream=st.cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(reps):
        L.loopvq_kmeans_step(cfg, 0, 0, 0, x, w, cb, assign, stream=st.cuda_stream)
    e1.record(st)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / reps
    # the encoder alone on the same inputs: the step minus it is the update
    pool = torch.zeros(L.loopvq_cache_layout(cfg)["pool_bytes"], dtype=torch.uint8, device=device)
    cfg_e = cfg
    slots = torch.arange(n, device=device, dtype=torch.int64)
    L.loopvq_encode(cfg_e, 0, 0, 0, x, w, cb, slots, pool, stream=st.cuda_stream)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(reps):
        L.loopvq_encode(cfg_e, 0, 0, 0, x, w, cb, slots, pool, stream=st.cuda_stream)
    e1.record(st)
    torch.cuda.synchronize()
    enc_ms = e0.elapsed_time(e1) / reps
    nsub = n * s.n_kv_heads * s.J
    upd_ms = max(step_ms - enc_ms, 1e-6)
    # update: x (bf16) and w (fp32) once, the assignment once, codebooks read and written
    upd_bytes = n * s.n_kv_heads * s.head_dim * s.loop_group * (2 + 4) + nsub + \
        2 * s.n_kv_heads * s.J * 256 * s.D * 4
    return {"ms_per_step": step_ms, "subvectors_per_s": nsub / (step_ms / 1e3),
            "assign_ms": enc_ms, "update_ms": upd_ms,
            "update_gbps": upd_bytes / (upd_ms / 1e3) / 1e9, "update_bytes": upd_bytes,
            "shape": f"{n} tokens x {s.n_kv_heads} heads x {s.J} groups, D={s.D}, "
                     f"per-token LogNormal weights, one of K/V"}


# --------------------------------------------------------------------------
# main
# --------------------------------------------------------------------------

def workload_config(shape, world):
    """The `config` dict of a line: the same for both arms."""
    return {"workload": shape.name, "layers": shape.n_layers, "kv_heads": shape.n_kv_heads,
            "head_dim": shape.head_dim, "loops": shape.n_loops, "g": shape.loop_group,
            "c": shape.chan_group, "bits_per_element": 8 / shape.D, "batch": shape.batch,
            "context": shape.context, "prefix": shape.prefix, "recent": shape.recent,
            "global_batch": shape.batch * world, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2: 277 MB per call, layers rotate"}


def main():
    args = parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from synthetic import SHAPES
    shape = SHAPES[args.config]
    if args.layers is not None:
        shape = shape.with_(n_layers=args.layers)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:                                  # rank 0 alone times the oracle
            return 0
        for _ in range(args.warmup):
            cpu_baseline(shape, budget_s=0.5)
        vals = [cpu_baseline(shape, budget_s=max(1.0, 60.0 / max(args.steps, 1)))
                for _ in range(args.steps)]
        v = statistics.median(x["value"] for x in vals)
        rec = dict(vals[-1])
        rec["value"] = v
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "µs/loop-step",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": v * shape.n_loops / 1e3, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_config(shape, world),
                "cpu_baseline": rec,
                "e2e": {"value": v, "unit": "µs/loop-step", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    rank, world, local = dist_init(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    wl = Workload(shape, dev)
    st = torch.cuda.current_stream()

    for _ in range(args.warmup):
        wl.step(st)
    torch.cuda.synchronize()
    barrier(world)

    # timed region: K whole steps, one pair of events, nothing else on the stream
    K = args.steps
    ev_start, ev_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local if world > 1 else 0)
    clk.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev_start.record(st)
    for _ in range(K):
        wl.step(st)
    ev_end.record(st)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clk.stop()
    elapsed_ms = ev_start.elapsed_time(ev_end)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    loop_steps = K * shape.n_loops * world
    value, ms_per_step = whole_job_value(elapsed_ms, K, shape.n_loops, world)

    # per-call device times of the decode call (a separate pass, events around
    # every call): the roofline's launch duration
    n_calls = max(1, min(K, 3)) * shape.n_loops * shape.n_layers
    call_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(n_calls)]
    pending = list(reversed(call_events))
    torch.cuda.synchronize()
    for _ in range(max(1, min(K, 3))):
        wl.step(st, events=pending)
    torch.cuda.synchronize()
    call_us = [a.elapsed_time(b) * 1e3 for a, b in call_events]
    avg_call_us = sum(call_us) / len(call_us)

    # end to end through the public API with host buffers: per step the
    # queries, the new token's K/V rows and the evicted token come from
    # pinned host memory, and every output goes back to the host.
    s = shape
    h_q = torch.empty_like(wl.q, device="cpu").pin_memory()
    h_q.copy_(wl.q.cpu())
    h_newk = torch.empty(s.n_layers, s.n_loops, s.batch, s.n_kv_heads, s.head_dim,
                         dtype=torch.bfloat16).pin_memory()
    h_newk.copy_(wl.win_k[:, :, :, :, -1].cpu())
    h_newv = torch.empty_like(h_newk).pin_memory()
    h_newv.copy_(wl.win_v[:, :, :, :, -1].cpu())
    h_ev = torch.empty_like(wl.evict, device="cpu").pin_memory()
    h_ev.copy_(wl.evict.cpu())
    h_out = torch.empty_like(wl.out, device="cpu").pin_memory()
    h_lse = torch.empty_like(wl.lse, device="cpu").pin_memory()
    h2d = h_q.numel() * 2 + h_newk.numel() * 2 * 2 + h_ev.numel() * 2
    d2h = h_out.numel() * 2 + h_lse.numel() * 4

    def e2e_step():
        wl.q.copy_(h_q, non_blocking=True)
        wl.win_k[:, :, :, :, -1].copy_(h_newk, non_blocking=True)
        wl.win_v[:, :, :, :, -1].copy_(h_newv, non_blocking=True)
        wl.evict.copy_(h_ev, non_blocking=True)
        wl.step(st)
        h_out.copy_(wl.out, non_blocking=True)
        h_lse.copy_(wl.lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(K):
        e2e_step()
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_val = e2e_ms * 1e3 / loop_steps

    alg = wl.algorithmic_bytes_per_call()
    peak, peak_src = measured_peaks()
    achieved = alg / avg_call_us / 1e3           # GB/s
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": recorded_traffic(
                    "sub_bit_vq_b200/csrc/decode.cu", "vq_decode_long32k"),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, copy)" if
                peak_src == "measured" else "fallback 6650 GB/s",
                "kernel": "vq_pair_kernel + vq_stream_kernel (one decode call, per-call events)",
                "algorithmic_bytes_per_launch": alg, "avg_launch_us": avg_call_us,
                "launch_us_p10_median_p90": call_percentiles(call_us),
                "calls_timed": len(call_us),
                "frac_of_8tbs": achieved / 8000.0}

    line = {"metric": METRIC, "value": value, "unit": "µs/loop-step", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
            "data": "synthetic", "config": workload_config(shape, world),
            "e2e": {"value": e2e_val, "unit": "µs/loop-step", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": wl.launches_per_step() * K,
            "clocks": clocks, "roofline": roofline}

    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(shape)
    if rank == 0 and not args.no_extras:
        del wl
        torch.cuda.empty_cache()
        line["bf16_kv"] = bf16_comparison(shape, dev)
        line["bf16_kv"]["vq_speedup_per_call"] = line["bf16_kv"]["us_per_call"] / avg_call_us
        line["decode_rows"] = decode_rows(dev, peak)
        line["encode_prefill"] = encode_prefill(dev)
        line["kmeans_step"] = kmeans_step(dev)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
