"""Workload shapes of the decode hot path.

Each shape is one decode configuration: a looped transformer with
``n_loops`` loop steps coded in groups of ``loop_group`` (g) consecutive
steps, ``chan_group`` (c) channels per sub-vector and an 8-bit index, i.e.
``8/(c*g)`` bits per cached element.
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Shape:
    name: str
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    n_loops: int
    loop_group: int
    chan_group: int
    batch: int
    context: int
    prefix: int = 8
    recent: int = 64
    page_tokens: int = 64
    n_centroids: int = 256
    # value model of the looped cache: "base_noise" draws one base vector per
    # token and adds 0.3*N(0,1) per loop step; "ar1" is an AR(1) chain over
    # loop steps with correlation ``loop_corr`` and unit variance.
    kind: str = "base_noise"
    loop_corr: float = 0.8
    head_scale: tuple[float, float] | None = None   # U(lo, hi) per (layer, head, K/V)
    key_outlier_frac: float = 0.0                    # Bernoulli mask over key channels
    key_outlier_scale: float = 8.0
    seed: int = 1000

    @property
    def J(self) -> int:
        return self.head_dim // self.chan_group

    @property
    def G(self) -> int:
        return self.n_loops // self.loop_group

    @property
    def D(self) -> int:
        return self.chan_group * self.loop_group

    @property
    def window(self) -> int:
        return self.prefix + self.recent

    @property
    def n_vq(self) -> int:
        return max(0, self.context - self.window)

    @property
    def pages_per_seq(self) -> int:
        return -(-self.n_vq // self.page_tokens)

    def with_(self, **kw) -> "Shape":
        return replace(self, **kw)


SHAPES: dict[str, Shape] = {
    # 1 layer, 1 kv-head, d=64, 4 loops in one group of 4, c=4 -> 0.5 bit,
    # context 512 (8 prefix + 64 recent bf16), batch 1.
    "tiny": Shape("tiny", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=64,
                  n_loops=4, loop_group=4, chan_group=4, batch=1, context=512,
                  seed=1001),
    # Ouro-1.4B-like decode step: 24 layers, 16 kv-heads (MHA), d=128,
    # 4 loops, g=4, c=4 (0.5 bit), batch 16, context 8192, per-head scales.
    "ouro14": Shape("ouro14", n_layers=24, n_kv_heads=16, n_q_heads=16,
                    head_dim=128, n_loops=4, loop_group=4, chan_group=4,
                    batch=16, context=8192, head_scale=(0.5, 2.0), seed=1002),
    # Long context at 0.5 bit: 48 layers, batch 8, context 32768, with 1% of
    # key channels scaled by 8.
    "long32k": Shape("long32k", n_layers=48, n_kv_heads=16, n_q_heads=16,
                     head_dim=128, n_loops=4, loop_group=4, chan_group=4,
                     batch=8, context=32768, head_scale=(0.5, 2.0),
                     key_outlier_frac=0.01, seed=1003),
    # 0.25 bit, deep recurrence: d=96, 40 kv-heads, 16 loops in groups of 4,
    # c=8 (32-element sub-vectors), batch 32, context 16384, AR(1) loops.
    # The layer count is not given; 4 layers are enough to rotate buffers
    # past the L2 cache. Pages hold 96 tokens: a multiple of the 24-slot
    # rotation block of J = 12 groups (and of 16).
    "deep025": Shape("deep025", n_layers=4, n_kv_heads=40, n_q_heads=40,
                     head_dim=96, n_loops=16, loop_group=4, chan_group=8,
                     batch=32, context=16384, kind="ar1", loop_corr=0.8,
                     page_tokens=96, seed=1004),
    # Encoder + batch sweep: 16 heads, d=128, 4 loops, g=4, c=4; the encode
    # leg is a 32768-token prefill, the sweep is batch 1..256 at 16384.
    "sweep": Shape("sweep", n_layers=1, n_kv_heads=16, n_q_heads=16,
                   head_dim=128, n_loops=4, loop_group=4, chan_group=4,
                   batch=16, context=16384, seed=1005),
}
