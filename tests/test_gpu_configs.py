"""GPU parity of loopvq_decode_attn at the full size of every workload.

Each case runs one decode call through the C ABI at a configuration's real
shape (one layer) and compares sampled (sequence, head) pairs, plus every
head of a few whole sequences, with the oracle on the same inputs:

* ouro14 (24 layers of 16 heads, d = 128, batch 16, context 8192);
* deep025 (40 heads, d = 96, c = 8 so J = 12 and 0.25 bit, 16 loop steps in
  groups of 4, batch 32, context 16384) at the first and last loop step;
* the batch sweep's decode shapes (16 heads, d = 128, context 16384) at
  batch 1, 64 and 256, and a ragged batch of 256 in which every streaming
  CTA holds many (sequence, head) segments;
* long32k (batch 8, context 32768) with the configuration's own generator
  (1% of key channels scaled by 8), fitted codebooks and indices written by
  the GPU encoder, whose choices are checked against the oracle's nearest
  centroid on sampled tokens first.

Tolerances are those of the other decode tests: float32 output per pair
max|o - ref| / max|ref| <= 1e-4, bf16 output max abs <= 2e-2 (floored at one
bf16 ulp of the reference), log-sum-exp within 1e-4.
"""

import numpy as np
import pytest
import torch

import sub_bit_vq_b200 as L
from oracle import loopvq_oracle as O
from synthetic import SHAPES, block_tables, codebooks_for_layer, loop_group_kv

from _cases import DeviceDecodeCase, check_decode, check_indices, sample_pairs
from test_partition_host import segments

pytestmark = pytest.mark.gpu


def _both_dtypes(case, pairs):
    for dt in (torch.float32, torch.bfloat16):
        out, lse = case.run_gpu(dt)
        check_decode(case, out, lse, dt, pairs=pairs)


@pytest.mark.parametrize("t", [0, 3])
def test_ouro14_full_batch(t):
    s = SHAPES["ouro14"]
    case = DeviceDecodeCase(s, [s.context] * s.batch, loop_step=t, seed=200 + t)
    _both_dtypes(case, sample_pairs(s.batch, s.n_q_heads, 40, seed=t, whole=(0, s.batch - 1)))


@pytest.mark.parametrize("t", [0, 15])
def test_deep025_full_batch(t):
    s = SHAPES["deep025"]
    assert s.J == 12 and s.D == 32 and s.G == 4
    case = DeviceDecodeCase(s, [s.context] * s.batch, loop_step=t, seed=300 + t)
    _both_dtypes(case, sample_pairs(s.batch, s.n_q_heads, 50, seed=t, whole=(0, 17)))


@pytest.mark.parametrize("batch", [1, 64, 256])
def test_sweep_decode_shapes(batch):
    s = SHAPES["sweep"].with_(batch=batch)
    case = DeviceDecodeCase(s, [s.context] * batch, loop_step=2, seed=400 + batch)
    whole = (0,) if batch == 1 else (0, batch - 1)
    _both_dtypes(case, sample_pairs(batch, s.n_q_heads, 40, seed=batch, whole=whole))


def test_ragged_batch_of_256_many_segments_per_cta():
    s = SHAPES["sweep"].with_(batch=256)
    r = np.random.default_rng(7)
    lens = [int(x) for x in r.integers(0, s.context + 1, size=256)]
    lens[:6] = [0, 1, 72, 73, 137, s.context]         # empty, window only, edges, full
    case = DeviceDecodeCase(s, lens, loop_step=1, seed=500)
    # the streaming partition: CTAs x segments (one per pair a CTA touches)
    pages = [max(0, -(-(n - s.window) // s.page_tokens)) for n in lens]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n_cta = min(sms, 256, sum(pages) * s.n_q_heads)
    segs, _ = segments(pages, s.n_q_heads, n_cta)
    per_cta = np.bincount([c for _, c, _, _ in segs], minlength=n_cta)
    assert per_cta.min() >= 5, per_cta.min()
    pairs = sample_pairs(256, s.n_q_heads, 40, seed=8, whole=(0, 1, 2, 3, 4, 5, 200))
    _both_dtypes(case, pairs)


def test_long32k_generator_with_gpu_encoded_indices():
    s = SHAPES["long32k"].with_(n_layers=1)
    dev = "cuda"
    B, n_vq, Pg, J, H = s.batch, s.n_vq, s.page_tokens, s.J, s.n_kv_heads
    cb = codebooks_for_layer(s, 0, device=dev, n_samples=2048)[None].contiguous()
    bt = block_tables(s, B, [s.context] * B, spare_pages=1)
    n_pages = bt[1]
    cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=H, n_q_heads=s.n_q_heads, head_dim=s.head_dim,
                         n_loops=s.n_loops, loop_group=s.loop_group, chan_group=s.chan_group,
                         n_pages=n_pages, max_batch=B, max_pages_per_seq=bt[0].shape[1])
    pool = torch.zeros(L.loopvq_cache_layout(cfg)["pool_bytes"], dtype=torch.uint8, device=dev)
    btd = bt[0].to(dev)
    v = torch.arange(n_vq, device=dev)
    slots = torch.cat([btd[b][v // Pg].long() * Pg + v % Pg for b in range(B)])
    pv = pool.view(1, H, 1, n_pages, 2, Pg * J)
    r = np.random.default_rng(9)
    toks = np.sort(r.choice(B * n_vq, size=384, replace=False))
    for kv in range(2):
        x = loop_group_kv(s, 0, 0, kv, B * n_vq, device=dev)
        for c0 in range(0, B * n_vq, 1 << 16):
            L.loopvq_encode(cfg, 0, 0, kv, x[:, c0:c0 + (1 << 16)], None, cb, slots[c0:c0 + (1 << 16)],
                            pool)
        torch.cuda.synchronize()
        # the encoder against the oracle's nearest centroid on sampled tokens
        xs = x[:, torch.from_numpy(toks).to(dev)].cpu()
        del x
        ref_idx, dist = O.encode_group_ref(xs.double().numpy(), cb[0, :, 0, kv].double().cpu().numpy())
        got = np.empty_like(ref_idx)
        sl = slots[torch.from_numpy(toks).to(dev)].cpu().numpy()
        for i, slot in enumerate(sl):
            page, k = divmod(int(slot), Pg)
            row = pv[0, :, 0, page, kv].cpu().numpy()                    # [H][Pg*J]
            got[i] = row[:, O.plane_offsets(np.array([k]), J, kv, Pg)[0]]
        check_indices(got, dist)
    for t in (0, 3):
        case = DeviceDecodeCase(s, [s.context] * B, loop_step=t, seed=600 + t, cb=cb, pool=pool,
                                bt=bt)
        _both_dtypes(case, sample_pairs(B, s.n_q_heads, 24, seed=t, whole=(3,)))
