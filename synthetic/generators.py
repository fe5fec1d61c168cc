"""Seeded random draws for the synthetic workloads (torch, CPU or CUDA).

Everything here is input generation: values of a looped K/V cache, queries,
weights, k-means codebooks (the offline codebook step, out of the hot path,
stood in for by plain Lloyd iterations on samples of the same distribution)
and page tables. Draws are reproducible for a given (shape, seed, device).
"""

from __future__ import annotations

import math

import torch

from .configs import Shape

_MASK62 = (1 << 62) - 1


def _seed(*parts: int) -> int:
    s = 0x9E3779B97F4A7C15 & _MASK62
    for p in parts:
        s = (s * 1000003 + (int(p) & _MASK62) + 0x632BE5AB) & _MASK62
    return s


def _gen(device, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


_TAG_SCALE, _TAG_OUTLIER, _TAG_KV, _TAG_WIN, _TAG_Q, _TAG_W, _TAG_CB, _TAG_PAGES = range(8)


def head_scales(shape: Shape, device="cpu") -> torch.Tensor:
    """``[L][Hkv][2]`` scale per (layer, kv-head, K or V), U(lo, hi) or 1."""
    L, H = shape.n_layers, shape.n_kv_heads
    if shape.head_scale is None:
        return torch.ones(L, H, 2, device=device)
    lo, hi = shape.head_scale
    g = _gen(device, shape.seed, _TAG_SCALE)
    return lo + (hi - lo) * torch.rand(L, H, 2, generator=g, device=device)


def key_outlier_mask(shape: Shape, device="cpu") -> torch.Tensor:
    """``[L][Hkv][d]`` per-key-channel scale: ``key_outlier_scale`` on a
    Bernoulli(``key_outlier_frac``) subset of (layer, head, channel), else 1."""
    L, H, d = shape.n_layers, shape.n_kv_heads, shape.head_dim
    if shape.key_outlier_frac <= 0.0:
        return torch.ones(L, H, d, device=device)
    g = _gen(device, shape.seed, _TAG_OUTLIER)
    hit = torch.rand(L, H, d, generator=g, device=device) < shape.key_outlier_frac
    return torch.where(hit, torch.full_like(hit, shape.key_outlier_scale, dtype=torch.float32),
                       torch.ones_like(hit, dtype=torch.float32))


def _loop_series(shape: Shape, n_steps: int, tail: tuple, g: torch.Generator,
                 device) -> torch.Tensor:
    """``[n_steps, *tail]`` float32 values over consecutive loop steps.

    ``base_noise``: one N(0,1) base per element plus 0.3*N(0,1) per step
    (redundancy along the loop axis). ``ar1``: x0 ~ N(0,1),
    x_t = r*x_{t-1} + sqrt(1-r^2)*N(0,1), unit variance, correlation r.
    """
    if shape.kind == "base_noise":
        base = torch.randn(tail, generator=g, device=device)
        eps = torch.randn((n_steps,) + tuple(tail), generator=g, device=device)
        return base.unsqueeze(0) + 0.3 * eps
    if shape.kind == "ar1":
        r = shape.loop_corr
        s = math.sqrt(1.0 - r * r)
        x = torch.randn(tail, generator=g, device=device)
        out = [x]
        for _ in range(1, n_steps):
            x = r * x + s * torch.randn(tail, generator=g, device=device)
            out.append(x)
        return torch.stack(out)
    raise ValueError(shape.kind)


def _channel_scale(shape: Shape, layer: int, kv: int, device) -> torch.Tensor:
    """``[Hkv][d]`` multiplicative scale of (layer, K or V)."""
    sc = head_scales(shape, device)[layer, :, kv]                 # [H]
    out = sc[:, None].expand(shape.n_kv_heads, shape.head_dim).clone()
    if kv == 0:
        out = out * key_outlier_mask(shape, device)[layer]
    return out


def loop_group_kv(shape: Shape, layer: int, gamma: int, kv: int, n_tokens: int,
                  device="cpu", stream: int = 0) -> torch.Tensor:
    """The ``g`` loop slices of loop group ``gamma`` for ``n_tokens`` tokens:
    ``[g][n_tokens][Hkv][d]`` bf16. ``stream`` picks independent token sets."""
    g = _gen(device, shape.seed, _TAG_KV, layer, gamma, kv, stream)
    x = _loop_series(shape, shape.loop_group,
                     (n_tokens, shape.n_kv_heads, shape.head_dim), g, device)
    x = x * _channel_scale(shape, layer, kv, device)[None, None]
    return x.to(torch.bfloat16)


def window_kv(shape: Shape, layer: int, loop_step: int, kv: int, batch: int | None = None,
              device="cpu") -> torch.Tensor:
    """bf16 window tokens (prefix + recent) at one loop step:
    ``[B][Hkv][prefix+recent][d]``."""
    B = shape.batch if batch is None else batch
    g = _gen(device, shape.seed, _TAG_WIN, layer, loop_step, kv)
    x = _loop_series(shape, 1, (B, shape.n_kv_heads, shape.window, shape.head_dim),
                     g, device)[0]
    x = x * _channel_scale(shape, layer, kv, device)[None, :, None, :]
    return x.to(torch.bfloat16)


def queries(shape: Shape, layer: int, loop_step: int, batch: int | None = None,
            device="cpu") -> torch.Tensor:
    """``[B][Hq][d]`` bf16 queries, N(0,1)."""
    B = shape.batch if batch is None else batch
    g = _gen(device, shape.seed, _TAG_Q, layer, loop_step)
    return torch.randn(B, shape.n_q_heads, shape.head_dim, generator=g,
                       device=device).to(torch.bfloat16)


def weights(shape: Shape, n_tokens: int, per_token: bool, layer: int = 0,
            gamma: int = 0, kv: int = 0, device="cpu") -> torch.Tensor:
    """Per-element Fisher-style weights ~ LogNormal(0, 1), float32:
    ``[g][n_tokens][Hkv][d]`` if ``per_token`` else ``[g][1][Hkv][d]``."""
    g = _gen(device, shape.seed, _TAG_W, layer, gamma, kv, int(per_token))
    n = n_tokens if per_token else 1
    return torch.exp(torch.randn(shape.loop_group, n, shape.n_kv_heads, shape.head_dim,
                                 generator=g, device=device))


def lloyd_kmeans(X: torch.Tensor, n_centroids: int, iters: int,
                 g: torch.Generator, chunk: int = 256) -> torch.Tensor:
    """Batched plain Lloyd k-means. ``X [NC][M][D]`` float32 ->
    ``[NC][E][D]``. Initial centroids are E distinct samples per set; a
    centroid with no members keeps its previous value."""
    NC, M, D = X.shape
    E = n_centroids
    if M < E:
        raise ValueError("need at least as many samples as centroids")
    pick = torch.rand(NC, M, generator=g, device=X.device).argsort(dim=1)[:, :E]
    C = torch.gather(X, 1, pick[:, :, None].expand(NC, E, D)).clone()
    for _ in range(iters):
        for s in range(0, NC, chunk):
            x = X[s:s + chunk]
            c = C[s:s + chunk]
            d2 = (x * x).sum(-1, keepdim=True) - 2.0 * torch.bmm(x, c.transpose(1, 2)) \
                + (c * c).sum(-1)[:, None, :]
            a = d2.argmin(dim=2)                                         # [n][M]
            sums = torch.zeros_like(c).scatter_add_(1, a[:, :, None].expand(-1, -1, D), x)
            cnt = torch.zeros(c.shape[0], E, device=X.device).scatter_add_(
                1, a, torch.ones_like(a, dtype=torch.float32))
            C[s:s + chunk] = torch.where(cnt[:, :, None] > 0,
                                         sums / cnt.clamp_min(1.0)[:, :, None], c)
    return C


def codebooks_for_layer(shape: Shape, layer: int, device="cpu", n_samples: int = 4096,
                        iters: int = 20) -> torch.Tensor:
    """k-means codebooks of one layer in the library's layout:
    ``[Hkv][G][2 (K, V)][g][J][E][c]`` float32.

    Training samples for each (head, loop group, K/V, channel group) are
    drawn from the same distribution as the cache (same value model, head
    scale and key outlier channels), as ``[g][c]`` blocks."""
    H, G, g_, J, c, E = (shape.n_kv_heads, shape.G, shape.loop_group, shape.J,
                        shape.chan_group, shape.n_centroids)
    gen = _gen(device, shape.seed, _TAG_CB, layer)
    out = torch.empty(H, G, 2, g_, J, E, c, device=device)
    for kv in range(2):
        scale = _channel_scale(shape, layer, kv, device).view(H, J, c)   # [H][J][c]
        for gamma in range(G):
            x = _loop_series(shape, g_, (H, J, n_samples, c), gen, device)  # [g][H][J][M][c]
            x = x * scale[None, :, :, None, :]
            X = x.permute(1, 2, 3, 0, 4).reshape(H * J, n_samples, g_ * c)
            C = lloyd_kmeans(X.contiguous(), E, iters, gen)                 # [H*J][E][g*c]
            out[:, gamma, kv] = C.view(H, J, E, g_, c).permute(0, 3, 1, 2, 4)
    return out


def block_tables(shape: Shape, batch: int, seq_lens: list[int], device="cpu",
                 max_pages: int | None = None, spare_pages: int = 0):
    """Random page tables. Each sequence gets ``ceil(n_vq / page_tokens)``
    distinct physical pages drawn from one shuffled pool.

    Returns ``(block_table [B][max_pages] int32, n_pages)`` where unused
    entries are -1 and ``n_pages`` is the physical page count."""
    need = [max(0, -(-max(0, n - shape.window) // shape.page_tokens)) for n in seq_lens]
    total = sum(need) + spare_pages
    mp = max(need + [1]) if max_pages is None else max_pages
    g = _gen("cpu", shape.seed, _TAG_PAGES, batch, total)
    perm = torch.randperm(max(total, 1), generator=g)
    bt = torch.full((batch, mp), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[k:k + n].to(torch.int32)
        k += n
    return bt.to(device), max(total, 1)
