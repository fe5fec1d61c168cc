"""Host check of the rescore margin of the tensor-core encoder.

The kernel scores a token against the 256 centroids as S_e = a . b_e with
a = [w*s, w] and b_e = [-2 C_e, C_e*C_e], from fp16 operands scaled by
powers of two: the -2C half of B by 2^beta1 and the C*C half by 2^beta2 (the
largest |b| of each half lands in [2^13, 2^14)), a row of A by
2^(rho - beta) per half, with rho chosen so that the row's largest scaled
|a| lands in [2^13, 2^14). Products of fp16 values are exact in float32 and
summed in float32, so the scores are S'_e ~= 2^rho S_e. The kernel rescores
exactly every centroid within
    margin = 2^-8.5 2^rho sum_k |a_k| max_e |b_ek| + 2^-17 2^rho sum_i w_i s_i^2
             + 2^-23 (sum_k |alpha_k| + sum_k max_e |beta'_ek|)
of the smallest S'. This test models the scaling, fp16 rounding (nearest,
ties to even, subnormals included) and a float32 accumulation in operand
order, and checks on ordinary, wide, tiny, nearly tied and mixed-magnitude
data that
  * every approximate score is within the stated error bound of 2^rho S_e;
  * the exact argmin, and the argmin of the float32 direct form the kernel
    rescores with, are among the rescored candidates."""

import numpy as np
import pytest

TOP = 13


def exp_of(m):
    """floor(log2 m) of a positive float32 (-127 for zero or subnormal)."""
    return int((np.float32(m).view(np.uint32) >> 23) & 0xFF) - 127


def col_scales(B, D):
    m_lo, m_hi = float(np.abs(B[:, :D]).max()), float(np.abs(B[:, D:]).max())
    beta1 = TOP - exp_of(m_lo) if m_lo > 0 else 0
    beta2 = TOP - exp_of(m_hi) if m_hi > 0 else 0
    return beta1, beta2


def scores(a, B, D, beta1, beta2):
    """The kernel's scores S' [E] (float32), rho and the scaled operands."""
    m1 = float(np.abs(a[:D]).max())
    m2 = float(np.abs(a[D:]).max())
    e1 = exp_of(m1) - beta1 if m1 > 0 else -100000
    e2 = exp_of(m2) - beta2 if m2 > 0 else -100000
    er = max(e1, e2)
    lo = max(-126, -126 + beta1, -126 + beta2)
    hi = min(127, 127 + beta1, 127 + beta2)
    rho = max(lo, min(hi, 0 if er == -100000 else TOP - er))
    fa = np.array([2.0 ** (rho - beta1)] * D + [2.0 ** (rho - beta2)] * D, dtype=np.float32)
    fb = np.array([2.0 ** beta1] * D + [2.0 ** beta2] * D, dtype=np.float32)
    alpha = (a * fa).astype(np.float32)
    betap = (B * fb[None]).astype(np.float32)
    A16 = alpha.astype(np.float16).astype(np.float32)
    B16 = betap.astype(np.float16).astype(np.float32)
    terms = (A16[None] * B16).astype(np.float32)          # exact: fp16 x fp16 fits float32
    acc = np.zeros(B.shape[0], dtype=np.float32)
    for k in range(terms.shape[1]):
        acc = (acc + terms[:, k]).astype(np.float32)
    return acc, rho, alpha, betap


def direct_f32(s, w, C):
    """encode_kernel's float32 direct form, in its term order."""
    d = np.zeros(C.shape[0], dtype=np.float32)
    for i in range(C.shape[1]):
        df = (s[i] - C[:, i]).astype(np.float32)
        d = (np.float32(w[i]) * df * df + d).astype(np.float32)   # fma rounds once; bound covers both
    return d


def bf16_rn(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def make(seed, n, D, s_scale, w_sigma, c_scale, ties, mixed):
    rng = np.random.default_rng(seed)
    C = (rng.standard_normal((256, D)) * c_scale).astype(np.float32)
    if ties:                                   # centroids that differ in one element's last bits
        C[1::2] = C[0::2] + np.float32(1e-6 * c_scale) * rng.standard_normal((128, D)).astype(np.float32)
    s = bf16_rn((rng.standard_normal((n, D)) * s_scale).astype(np.float32))   # the kernel's inputs are bf16
    w = np.exp(rng.standard_normal((n, D)) * w_sigma).astype(np.float32)
    if mixed:                                  # weights spanning many binades within a row
        w *= np.float32(2.0) ** rng.integers(-30, 30, size=(n, D)).astype(np.float32)
    return s, w, C


CASES = [  # D, s_scale, w_sigma, c_scale, ties, mixed
    (16, 1.0, 1.0, 1.0, False, False),
    (16, 30.0, 2.0, 30.0, False, False),
    (8, 1.0, 1.0, 1.0, True, False),
    (32, 0.01, 1.0, 0.01, True, False),
    (16, 1e-3, 1.0, 1e-3, False, False),
    (16, 1.0, 1.0, 1.0, False, True),
    (16, 500.0, 3.0, 500.0, False, False),
]


@pytest.mark.parametrize("D,s_scale,w_sigma,c_scale,ties,mixed", CASES)
def test_scaled_fp16_scores_stay_inside_the_margin(D, s_scale, w_sigma, c_scale, ties, mixed):
    s, w, C = make(1000 + D, 200, D, s_scale, w_sigma, c_scale, ties, mixed)
    B = np.concatenate([-2.0 * C, C * C], axis=1).astype(np.float32)               # [E][2D]
    bmax = np.abs(B).max(axis=0).astype(np.float64)
    beta1, beta2 = col_scales(B, D)
    fb = np.array([2.0 ** beta1] * D + [2.0 ** beta2] * D)
    q_abs = float((bmax * fb).sum())
    for n in range(s.shape[0]):
        a = np.concatenate([w[n] * s[n], w[n]]).astype(np.float32)
        approx, rho, alpha, betap = scores(a, B, D, beta1, beta2)
        approx = approx.astype(np.float64)
        # exact scores from the exact reals a = w*s (not its float32 rounding) and b
        a_exact = np.concatenate([w[n].astype(np.float64) * s[n].astype(np.float64), w[n].astype(np.float64)])
        C64 = C.astype(np.float64)
        b_exact = np.concatenate([-2.0 * C64, C64 * C64], axis=1)
        exact = (2.0 ** rho) * (b_exact @ a_exact)
        al = np.abs(alpha.astype(np.float64))
        bound = 2.0 ** -9.98 * (np.abs(betap.astype(np.float64)) @ al) + \
            2.0 ** -24.9 * (al.sum() + np.abs(betap.astype(np.float64)).sum(axis=1))
        assert np.all(np.abs(approx - exact) <= bound), n
        wss = float(np.sum(w[n].astype(np.float64) * s[n].astype(np.float64) ** 2))
        pu = float(np.abs(a).astype(np.float64) @ bmax)
        margin = 2.0 ** rho * (2.0 ** -8.5 * pu + 2.0 ** -17 * wss) + 2.0 ** -23 * (al.sum() + q_abs)
        thr = approx.min() + margin
        d64 = (w[n].astype(np.float64) * (s[n].astype(np.float64) - C64) ** 2).sum(axis=1)
        assert approx[int(np.argmin(d64))] <= thr, n
        assert approx[int(np.argmin(direct_f32(s[n], w[n], C)))] <= thr, n


def test_scaled_operands_fit_fp16():
    # the largest scaled |a| and |b| lie in [2^13, 2^14): no fp16 overflow
    s, w, C = make(7, 50, 16, 100.0, 3.0, 100.0, False, True)
    B = np.concatenate([-2.0 * C, C * C], axis=1).astype(np.float32)
    beta1, beta2 = col_scales(B, 16)
    for n in range(s.shape[0]):
        a = np.concatenate([w[n] * s[n], w[n]]).astype(np.float32)
        _, _, alpha, betap = scores(a, B, 16, beta1, beta2)
        assert 2.0 ** 13 <= np.abs(alpha).max() < 2.0 ** 14
        assert np.abs(betap).max() < 2.0 ** 14
        assert np.all(np.isfinite(alpha.astype(np.float16)))
