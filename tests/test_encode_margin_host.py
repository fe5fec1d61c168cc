"""Host check of the rescore margin of the tensor-core encoder.

The kernel scores a token against the 256 centroids as S_e = a . b_e with
a = [w*s, w] and b_e = [-2 C_e, C_e*C_e], from operands split into bf16
high and low parts (a.b ~= a_hi.b_hi + a_hi.b_lo + a_lo.b_hi, accumulated in
float32), and rescores exactly every centroid within
    margin = 2^-12 * (sum_i |a_i| max_e |b_ei| + sum_i w_i s_i^2)
of the smallest approximate score. That is correct when the exact nearest
centroid always lies within the margin. This test models the split
products (exact: bf16 x bf16 fits float32) and a float32 accumulation in
operand order, and checks on wide and nearly tied data that
  * each approximate score is within 2^-14.3 * sum_i |a_i b_ei| of the exact one;
  * the exact argmin is among the rescored candidates."""

import numpy as np
import pytest


def bf16_rn(x):
    """Round float32 values to bfloat16 (nearest, ties to even), as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def split(x):
    hi = bf16_rn(x)
    lo = bf16_rn((x - hi).astype(np.float32))
    return hi, lo


def approx_scores(a, B):
    """a [K2] float32, B [E][K2] float32 -> S [E] float32 from the split operands."""
    ah, al = split(a)
    Bh, Bl = split(B)
    terms = np.concatenate([ah[None] * Bh, ah[None] * Bl, al[None] * Bh], axis=1)   # exact in float32
    acc = np.zeros(B.shape[0], dtype=np.float32)
    for k in range(terms.shape[1]):
        acc = (acc + terms[:, k]).astype(np.float32)
    return acc


def make(seed, n, D, s_scale, w_sigma, ties):
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((256, D)).astype(np.float32)
    if ties:                                   # centroids that differ in one element's last bits
        C[1::2] = C[0::2] + np.float32(1e-6) * rng.standard_normal((128, D)).astype(np.float32)
    s = (rng.standard_normal((n, D)) * s_scale).astype(np.float32)
    s = bf16_rn(s)                             # the kernel's inputs are bf16
    w = np.exp(rng.standard_normal((n, D)) * w_sigma).astype(np.float32)
    return s, w, C


@pytest.mark.parametrize("D,s_scale,w_sigma,ties", [(16, 1.0, 1.0, False), (16, 30.0, 2.0, False),
                                                    (8, 1.0, 1.0, True), (32, 0.01, 1.0, True)])
def test_split_scores_stay_inside_the_margin(D, s_scale, w_sigma, ties):
    s, w, C = make(1000 + D, 300, D, s_scale, w_sigma, ties)
    B = np.concatenate([-2.0 * C, C * C], axis=1).astype(np.float32)               # [E][2D]
    bmax = np.abs(B).max(axis=0)
    for n in range(s.shape[0]):
        a = np.concatenate([w[n] * s[n], w[n]]).astype(np.float32)
        exact = B.astype(np.float64) @ a.astype(np.float64)
        approx = approx_scores(a, B).astype(np.float64)
        scale = np.abs(B.astype(np.float64)) @ np.abs(a.astype(np.float64))
        assert np.all(np.abs(approx - exact) <= 2.0 ** -14.3 * scale)
        margin = 2.0 ** -12 * (np.abs(a).astype(np.float64) @ bmax + float(np.sum(w[n] * s[n] * s[n], dtype=np.float64)))
        # the exact distances, and the centroid the direct form would pick
        d = (w[n].astype(np.float64) * (s[n].astype(np.float64) - C.astype(np.float64)) ** 2).sum(axis=1)
        best = int(np.argmin(d))
        assert approx[best] <= approx.min() + margin
