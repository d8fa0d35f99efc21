"""The support extraction's cut, checked on the CPU in the kernel's fp32 arithmetic.

Given tau_i, the backward lists row i's support {j : scale * S_ij > tau_i} in one score pass
(support extraction, fwd.cu).  The pass compares raw fp32 scores with one threshold per row,
t = fl(tau / scale) lowered by 2^-20 of itself, and applies the exact test (one fused
multiply-add, scale * S - tau > 0) to the scores it lists.  That is only right if the raw cut never
drops a score whose scaled value exceeds tau.  Here, with numpy's IEEE fp32 (the kernel is built
without flush-to-zero), every fp32 score within 64 ulps of tau / scale on either side is tested
against the exact rule, over taus and scales of both signs of tau and many magnitudes.
"""
import numpy as np
import pytest

F = np.float32


def kernel_cut(tau: float, scale: float) -> np.float32:
    t = F(tau) / F(scale)
    if np.isfinite(t):
        t = F(t - F(abs(t) * F(2.0**-20)))
    return t


def exact_hit(c: np.ndarray, tau: float, scale: float) -> np.ndarray:
    # scale * c is exact in fp64 (24-bit by 24-bit mantissas); the fp64 subtraction keeps the sign
    return np.float64(F(scale)) * c.astype(np.float64) - np.float64(F(tau)) > 0


def neighbours(x: np.float32, n: int = 64) -> np.ndarray:
    up, down = [x], [x]
    for _ in range(n):
        up.append(np.nextafter(up[-1], F(np.inf)))
        down.append(np.nextafter(down[-1], F(-np.inf)))
    return np.array(down[::-1] + up[1:], dtype=F)


SCALES = [0.125, 0.25, 1 / np.sqrt(3.0), 0.3, 1e-3, 7.5, 2.0**-7 * 3]


@pytest.mark.parametrize("scale", SCALES)
def test_cut_keeps_every_support_score(scale):
    rng = np.random.default_rng(12)
    taus = np.concatenate([rng.normal(0, 3, 300), rng.normal(0, 1e-3, 50), 10.0 ** rng.uniform(-30, 4, 100),
                           -(10.0 ** rng.uniform(-30, 4, 100)), [0.0, 1.0, -1.0, 2.0, 1.5]])
    for tau in taus.astype(F):
        t = kernel_cut(float(tau), scale)
        c = neighbours(F(tau) / F(scale))
        hit = exact_hit(c, float(tau), scale)
        listed = c > t
        assert not np.any(hit & ~listed), (float(tau), scale)
        # the cut is tight: what it lets through beyond the support lies within 2^-19 of the threshold
        extra = c[listed & ~hit]
        if extra.size and np.isfinite(t):
            ref = abs(float(F(tau) / F(scale)))
            assert np.all(np.abs(extra.astype(np.float64) - float(F(tau) / F(scale))) <= ref * 2.0**-19 + 1e-38)


def test_infinite_tau_cuts_everything():
    # a row with no allowed key has tau = +inf: no score passes the cut
    t = kernel_cut(np.inf, 0.125)
    assert t == np.inf
    c = np.array([np.finfo(F).max, 1e30, 0.0, -1.0], dtype=F)
    assert not np.any(c > t)


def test_random_rows_support_matches_the_definition():
    # whole rows of random scores: the listed-then-tested entries are exactly {j : scale * S_j > tau}
    rng = np.random.default_rng(3)
    for _ in range(200):
        scale = float(rng.choice(SCALES))
        s = rng.normal(0, 8, 4096).astype(F)
        tau = F(np.sort(s * F(scale))[-rng.integers(1, 40)])  # a tau that equals some scaled score
        t = kernel_cut(float(tau), scale)
        listed = np.flatnonzero(s > t)
        kept = listed[exact_hit(s[listed], float(tau), scale)]
        np.testing.assert_array_equal(kept, np.flatnonzero(exact_hit(s, float(tau), scale)))
