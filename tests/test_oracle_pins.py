"""Pins for the fp64 oracle against facts the pages and mathematics fix.

None of these re-types the oracle's own formula: each checks it against a
different route -- hand-derived closed forms (tests/golden), the argmax
definition solved by a generic optimiser, brute force over supports with the
KKT conditions, a library root finder, textbook averages, and finite
differences.  Chosen so that a dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle fails at least one of them.

Passages: page "svd-sst2-roberta-adasplash" sections 2.1 (argmax definition),
2.2 (Theorem 1, closed form and KKT), 2.3 (Theorem 2, bracket and bisection
bound), 2.4 (Jacobian); model cards "roberta-base-adasplash" and
"distilbert-sst2-adasplash" (bracket [max-2, max-2/sqrt(L)]).
"""
import itertools
import math
from pathlib import Path

import numpy as np
import pytest
import torch
from scipy import optimize

from oracle import oracle as orc

GOLDEN = Path(__file__).parent / "golden" / "entmax15_closed_forms.txt"


def _rows(seed, count, nmin=1, nmax=40, spread=(0.2, 6.0)):
    rng = np.random.default_rng(seed)
    for _ in range(count):
        n = int(rng.integers(nmin, nmax + 1))
        sd = float(rng.uniform(*spread))
        yield rng.normal(0.0, sd, size=n)


# ---------------------------------------------------------------- bf16 input
def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3, size=20000).astype(np.float32)
    # exact ties and carries into the exponent
    extra = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -(1.0 + 2 ** -8),
                      np.float32(1.9999999), 65504.0, 1e-30, -0.0, 0.0, 3.0e38], dtype=np.float32)
    x = np.concatenate([x, extra])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_bf16(x), ref)


# ---------------------------------------------------------- golden fixtures
def _golden():
    out = []
    for line in GOLDEN.read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        name, s, tau, p = (f.strip() for f in line.split("|"))
        out.append((name, np.array(s.split(), float), float(tau), np.array(p.split(), float)))
    return out


@pytest.mark.parametrize("name,s,tau,p", _golden(), ids=[g[0] for g in _golden()])
def test_golden_closed_forms(name, s, tau, p):
    t, _ = orc.tau_sort(s)
    assert t == pytest.approx(tau, abs=1e-14)
    np.testing.assert_allclose(orc.entmax15(s), p, atol=1e-14)
    # the pages' bisection reaches the same root within its stated bound
    tb = orc.tau_bisect(s)
    width = 2.0 - 2.0 / math.sqrt(s.size)
    assert abs(tb - tau) <= width / 2 ** 26 + 1e-15


# ------------------------------------------------------ closed-form cases
def test_two_element_closed_form():
    rng = np.random.default_rng(1)
    for _ in range(500):
        a, b = rng.normal(0, 2, size=2)
        hi, lo = max(a, b), min(a, b)
        d = hi - lo
        expect = hi - 2.0 if d >= 2.0 else 0.5 * (hi + lo) - math.sqrt(2.0 - (d / 2.0) ** 2)
        assert orc.tau_sort([a, b])[0] == pytest.approx(expect, abs=1e-12)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 64, 1000])
def test_equal_scores_uniform(n):
    c = 0.37
    s = np.full(n, c)
    t, k = orc.tau_sort(s)
    assert k == n
    assert t == pytest.approx(c - 2.0 / math.sqrt(n), abs=1e-12)
    np.testing.assert_allclose(orc.entmax15(s), np.full(n, 1.0 / n), rtol=1e-10)


def test_gap_of_two_gives_one_hot():
    rng = np.random.default_rng(2)
    for _ in range(200):
        n = int(rng.integers(2, 50))
        s = rng.uniform(-5, 0, size=n)
        j = int(rng.integers(n))
        s[j] = s.max() + 2.0 + rng.uniform(0, 3)
        p = orc.entmax15(s)
        assert p[j] == pytest.approx(1.0, abs=1e-15)
        assert np.count_nonzero(p) == 1
        assert orc.tau_sort(s)[0] == pytest.approx(s[j] - 2.0, abs=1e-12)


# -------------------------------------------------------------- invariants
def test_shift_invariance_and_permutation_equivariance():
    rng = np.random.default_rng(3)
    for s in _rows(4, 300):
        c = float(rng.normal(0, 10))
        t, _ = orc.tau_sort(s)
        t2, _ = orc.tau_sort(s + c)
        assert t2 == pytest.approx(t + c, abs=1e-9)
        np.testing.assert_allclose(orc.entmax15(s + c), orc.entmax15(s), atol=1e-10)
        perm = rng.permutation(s.size)
        np.testing.assert_allclose(orc.entmax15(s[perm]), orc.entmax15(s)[perm], atol=1e-12)


def test_simplex_membership():
    for s in _rows(5, 500, nmax=300):
        p = orc.entmax15(s)
        assert (p >= 0).all()
        assert p.sum() == pytest.approx(1.0, abs=1e-12)
        t, k = orc.tau_sort(s)
        # exact zeros below tau, positive weights above (KKT, Theorem 1)
        assert np.all((p > 0) == (s > t))
        assert k == np.count_nonzero(p)


def test_g_at_root_and_brackets():
    """Theorem 2: g is decreasing, g(lo) >= 1 >= g(hi) on both brackets, g(tau*) = 1."""
    for s in _rows(6, 300):
        n = s.size
        t, _ = orc.tau_sort(s)
        assert orc.g(s, t) == pytest.approx(1.0, abs=1e-12)
        m = s.max()
        assert orc.g(s, m - 2.0) >= 1.0 - 1e-15
        assert orc.g(s, m - 2.0 / math.sqrt(n)) <= 1.0 + 1e-12
        assert orc.g(s, s.min() - 2.0) >= 1.0 - 1e-15
        assert orc.g(s, m) == 0.0
        grid = np.linspace(s.min() - 3, m, 50)
        vals = [orc.g(s, x) for x in grid]
        assert all(a >= b for a, b in zip(vals, vals[1:]))


# ------------------------------------------------ bisection vs exact root
def test_bisection_matches_exact_within_bound():
    for s in _rows(7, 400, nmax=500):
        n = s.size
        t, _ = orc.tau_sort(s)
        tb = orc.tau_bisect(s, 25)
        width = 2.0 - 2.0 / math.sqrt(n)
        assert abs(tb - t) <= width / 2 ** 26 + 1e-12
        tw = orc.tau_bisect_wide(s, 25)
        assert abs(tw - t) <= (s.max() - s.min() + 2.0) / 2 ** 25 + 1e-12


# ---------------------------------------- brute force over supports (KKT)
def _kkt_bruteforce(s):
    """Enumerate every non-empty support; keep the roots that satisfy KKT."""
    found = []
    n = s.size
    for k in range(1, n + 1):
        for sup in itertools.combinations(range(n), k):
            z = s[list(sup)]
            # sum (z - t)^2 = 4  ->  k t^2 - 2 t sum z + sum z^2 - 4 = 0
            a, b, c = k, -2.0 * z.sum(), float((z * z).sum() - 4.0)
            disc = b * b - 4 * a * c
            if disc < 0:
                continue
            for t in ((-b - math.sqrt(disc)) / (2 * a), (-b + math.sqrt(disc)) / (2 * a)):
                inside = all(s[i] > t for i in sup)
                outside = all(s[i] <= t for i in range(n) if i not in sup)
                if inside and outside:
                    found.append(t)
    return found


def test_kkt_bruteforce_small_rows():
    for s in _rows(8, 300, nmin=1, nmax=4, spread=(0.1, 3.0)):
        roots = _kkt_bruteforce(s)
        assert len(roots) >= 1
        assert max(roots) - min(roots) < 1e-9  # unique multiplier
        assert orc.tau_sort(s)[0] == pytest.approx(roots[0], abs=1e-10)


# ---------------------------------------------------- argmax definition
def test_argmax_definition_by_optimiser():
    """Section 2.1: entmax_1.5(s) = argmax_{p in simplex} p.s + (4/3) sum (p - p^1.5)."""
    for s in _rows(9, 40, nmin=2, nmax=6, spread=(0.3, 2.5)):
        n = s.size

        def neg(p):
            p = np.clip(p, 0.0, None)
            return -(p @ s + (4.0 / 3.0) * np.sum(p - p ** 1.5))

        best = None
        for x0 in (np.full(n, 1.0 / n), np.eye(n)[int(np.argmax(s))] * 0.9 + 0.1 / n):
            r = optimize.minimize(neg, x0, method="SLSQP", bounds=[(0, 1)] * n,
                                  constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1.0}],
                                  options={"ftol": 1e-14, "maxiter": 500})
            if best is None or r.fun < best.fun:
                best = r
        np.testing.assert_allclose(orc.entmax15(s), np.clip(best.x, 0, None), atol=2e-4)


# -------------------------------------------------- Jacobian (section 2.4)
def _fd_jacobian(s, h=1e-6):
    n = s.size
    J = np.empty((n, n))
    for j in range(n):
        e = np.zeros(n)
        e[j] = h
        J[:, j] = (orc.entmax15(s + e) - orc.entmax15(s - e)) / (2 * h)
    return J


def test_jvp_matches_finite_differences():
    rng = np.random.default_rng(10)
    checked = 0
    for s in _rows(11, 200, nmin=2, nmax=12, spread=(0.5, 3.0)):
        t, _ = orc.tau_sort(s)
        if np.min(np.abs(s - t)) < 1e-3:
            continue  # kink of the piecewise-smooth map
        J = _fd_jacobian(s)
        gv = rng.normal(size=s.size)
        ds = orc.entmax15_jvp(orc.entmax15(s), gv)
        np.testing.assert_allclose(ds, J.T @ gv, atol=1e-6)
        checked += 1
    assert checked > 100


def test_jacobian_structure():
    """J symmetric, J 1 = 0 (shift invariance), zero rows/cols off the support."""
    for s in _rows(12, 100, nmin=2, nmax=15, spread=(0.5, 3.0)):
        p = orc.entmax15(s)
        n = s.size
        J = np.stack([orc.entmax15_jvp(p, np.eye(n)[k]) for k in range(n)])  # row k = e_k^T J
        np.testing.assert_allclose(J, J.T, atol=1e-12)
        np.testing.assert_allclose(J.sum(axis=1), 0.0, atol=1e-12)
        off = p == 0
        assert np.all(J[off] == 0) and np.all(J[:, off] == 0)


# -------------------------------------------------------------- attention
def _rand_qkv(seed, B, H, L, D, sd=1.0):
    rng = np.random.default_rng(seed)
    f = lambda: orc.round_bf16(rng.normal(0, sd, size=(B, H, L, D)).astype(np.float32))
    return f(), f(), f(), f()


def _allowed(L, causal, window, mask_row):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    a = np.ones((L, L), bool)
    if causal:
        a &= j <= i
    if window:
        a &= j >= i - window + 1
    if mask_row is not None:
        a &= mask_row[None, :].astype(bool)
    return a


def test_attention_forward_by_root_finder():
    """Scores by matmul, tau by Brent's method on g(tau) = 1, then p and p @ V."""
    B, H, L, D = 2, 2, 24, 8
    Q, K, V, _ = _rand_qkv(13, B, H, L, D, sd=1.3)
    mask = np.ones((B, L), np.uint8)
    mask[1, 17:] = 0
    for causal, window in ((False, 0), (True, 0), (True, 5)):
        O, tau = orc.attn_fwd(Q, K, V, mask, causal, window, scale=0.3)
        for b in range(B):
            a = _allowed(L, causal, window, mask[b])
            for h in range(H):
                S = 0.3 * Q[b, h] @ K[b, h].T
                for i in range(L):
                    s = S[i, a[i]]
                    if s.size == 0:  # window entirely inside the padding
                        assert np.isinf(tau[b, h, i]) and np.all(O[b, h, i] == 0)
                        continue
                    f = lambda t: np.sum(np.clip((s - t) / 2, 0, None) ** 2) - 1.0
                    t = optimize.brentq(f, s.min() - 2.5, s.max(), xtol=1e-15, rtol=1e-15)
                    p = np.clip((s - t) / 2, 0, None) ** 2
                    assert tau[b, h, i] == pytest.approx(t, abs=1e-11)
                    np.testing.assert_allclose(O[b, h, i], p @ V[b, h][a[i]], atol=1e-11)


def test_uniform_attention_is_masked_average():
    """Q = 0 -> all allowed scores equal -> O_i is the plain mean of the allowed V rows."""
    B, H, L, D = 2, 3, 40, 8
    _, K, V, _ = _rand_qkv(14, B, H, L, D)
    Q = np.zeros_like(K)
    lens = [40, 23]
    mask = np.zeros((B, L), np.uint8)
    for b, n in enumerate(lens):
        mask[b, :n] = 1
    O, tau = orc.attn_fwd(Q, K, V, mask, scale=0.125)
    for b, n in enumerate(lens):
        np.testing.assert_allclose(O[b], np.broadcast_to(V[b, :, :n].mean(axis=1, keepdims=True), O[b].shape),
                                   atol=1e-13)
        np.testing.assert_allclose(tau[b], -2.0 / math.sqrt(n), atol=1e-13)
    W = 7
    O, tau = orc.attn_fwd(Q, K, V, None, causal=True, window=W, scale=0.125)
    for i in range(L):
        lo = max(0, i - W + 1)
        np.testing.assert_allclose(O[:, :, i], V[:, :, lo:i + 1].mean(axis=2), atol=1e-13)
        np.testing.assert_allclose(tau[:, :, i], -2.0 / math.sqrt(i + 1 - lo), atol=1e-13)


def test_causal_first_row_and_large_gap():
    B, H, L, D = 1, 2, 16, 8
    Q, K, V, _ = _rand_qkv(15, B, H, L, D)
    O, tau = orc.attn_fwd(Q, K, V, None, causal=True, scale=0.2)
    np.testing.assert_allclose(O[:, :, 0], V[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(tau[:, :, 0], 0.2 * np.sum(Q[:, :, 0] * K[:, :, 0], axis=-1) - 2.0, atol=1e-13)
    # a key aligned with the query and far above the rest takes all the weight
    Q2 = np.zeros((1, 1, 8, 4))
    K2 = np.zeros((1, 1, 8, 4))
    V2 = np.arange(32, dtype=float).reshape(1, 1, 8, 4)
    Q2[0, 0, :, 0] = 1.0
    K2[0, 0, 5, 0] = 10.0
    O2, _ = orc.attn_fwd(Q2, K2, V2, None, scale=1.0)
    np.testing.assert_allclose(O2[0, 0], np.broadcast_to(V2[0, 0, 5], (8, 4)), atol=1e-15)


def test_rows_subset_matches_full():
    B, H, L, D = 2, 2, 33, 16
    Q, K, V, _ = _rand_qkv(16, B, H, L, D)
    mask = np.ones((B, L), np.uint8)
    mask[0, 30:] = 0
    O, tau = orc.attn_fwd(Q, K, V, mask, True, 9, 0.25)
    ids = np.array([0, 5, 32, 33, 70, 131])
    Or, tr = orc.attn_fwd_rows(Q, K, V, ids, mask, True, 9, 0.25)
    np.testing.assert_array_equal(Or, O.reshape(-1, D)[ids])
    np.testing.assert_array_equal(tr, tau.reshape(-1)[ids])
    Ob, tb = orc.attn_fwd_rows(Q, K, V, ids, mask, True, 9, 0.25, tau_method="bisect")
    assert np.max(np.abs(tb - tr)) < 2.0 / 2 ** 26
    assert np.max(np.abs(Ob - Or)) < 1e-6


def test_empty_row_convention():
    B, H, L, D = 1, 1, 8, 4
    Q, K, V, dO = _rand_qkv(17, B, H, L, D)
    mask = np.zeros((B, L), np.uint8)
    O, tau = orc.attn_fwd(Q, K, V, mask)
    assert np.all(O == 0) and np.all(np.isinf(tau))
    dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, mask)
    assert np.all(dQ == 0) and np.all(dK == 0) and np.all(dV == 0)


@pytest.mark.parametrize("causal,window,masked", [(False, 0, False), (False, 0, True), (True, 0, False), (True, 3, True)])
def test_backward_matches_finite_differences(causal, window, masked):
    """Central differences of L = <dO, O> through the oracle forward (fp64)."""
    B, H, L, D = 1, 1, 7, 5
    scale = 0.6
    mask = None
    if masked:
        mask = np.ones((B, L), np.uint8)
        mask[0, 5:] = 0
    done = 0
    for seed in range(40):
        Q, K, V, dO = _rand_qkv(100 + seed, B, H, L, D)
        O, tau = orc.attn_fwd(Q, K, V, mask, causal, window, scale)
        a = _allowed(L, causal, window, None if mask is None else mask[0])
        S = scale * Q[0, 0] @ K[0, 0].T
        gaps = np.abs(S - tau[0, 0][:, None])[a]
        if gaps.min() < 1e-3:
            continue
        dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, mask, causal, window, scale)
        h = 1e-6
        for X, dX in ((Q, dQ), (K, dK), (V, dV)):
            num = np.zeros_like(X)
            for idx in np.ndindex(X.shape):
                old = X[idx]
                X[idx] = old + h
                Lp = np.sum(dO * orc.attn_fwd(Q, K, V, mask, causal, window, scale)[0])
                X[idx] = old - h
                Lm = np.sum(dO * orc.attn_fwd(Q, K, V, mask, causal, window, scale)[0])
                X[idx] = old
                num[idx] = (Lp - Lm) / (2 * h)
            np.testing.assert_allclose(dX, num, atol=2e-6)
        done += 1
        if done == 3:
            break
    assert done >= 1


# ------------------------------------------------------- grouped-query attention
def test_gqa_head_mapping_by_constant_values():
    """V constant per key/value head g -> every output row of a query head reading g equals that
    constant (the weights sum to one), which fixes the head map h -> h // (H/H_kv) without the oracle."""
    B, H, Hkv, L, D = 2, 6, 2, 12, 4
    rng = np.random.default_rng(21)
    Q = orc.round_bf16(rng.normal(0, 1, (B, H, L, D)).astype(np.float32))
    K = orc.round_bf16(rng.normal(0, 1, (B, Hkv, L, D)).astype(np.float32))
    c = np.arange(B * Hkv, dtype=float).reshape(B, Hkv) + 1.0
    V = np.broadcast_to(c[:, :, None, None], (B, Hkv, L, D)).copy()
    O, _ = orc.attn_fwd_gqa(Q, K, V, causal=True, scale=0.5)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(O[b, h], c[b, h // (H // Hkv)], atol=1e-13)


def test_gqa_single_kv_head_equals_shared_keys():
    """H_kv = 1: every query head sees the same K and V, as plain attention with K, V broadcast."""
    B, H, L, D = 1, 3, 10, 8
    Q, K, V, _ = _rand_qkv(22, B, H, L, D)
    K1, V1 = K[:, :1], V[:, :1]
    O, tau = orc.attn_fwd_gqa(Q, K1, V1, scale=0.4)
    for h in range(H):
        Oh, th = orc.attn_fwd(Q[:, h:h + 1], K1, V1, scale=0.4)
        np.testing.assert_array_equal(O[:, h], Oh[:, 0])
        np.testing.assert_array_equal(tau[:, h], th[:, 0])


def test_gqa_backward_matches_finite_differences():
    """Central differences of <dO, O> w.r.t. the SHARED key/value heads: pins the sum over the group."""
    B, H, Hkv, L, D = 1, 4, 2, 6, 3
    scale = 0.7
    done = 0
    for seed in range(40):
        rng = np.random.default_rng(300 + seed)
        Q = rng.normal(0, 1, (B, H, L, D))
        K = rng.normal(0, 1, (B, Hkv, L, D))
        V = rng.normal(0, 1, (B, Hkv, L, D))
        dO = rng.normal(0, 1, (B, H, L, D))
        O, tau = orc.attn_fwd_gqa(Q, K, V, None, True, 0, scale)
        ok = True
        for h in range(H):
            S = scale * Q[0, h] @ K[0, h // (H // Hkv)].T
            a = _allowed(L, True, 0, None)
            if np.abs(S - tau[0, h][:, None])[a].min() < 1e-3:
                ok = False
        if not ok:
            continue
        dQ, dK, dV = orc.attn_bwd_gqa(Q, K, V, dO, None, True, 0, scale)
        assert dK.shape == K.shape and dV.shape == V.shape and dQ.shape == Q.shape
        eps = 1e-6
        for X, dX in ((Q, dQ), (K, dK), (V, dV)):
            num = np.zeros_like(X)
            for idx in np.ndindex(X.shape):
                old = X[idx]
                X[idx] = old + eps
                Lp = np.sum(dO * orc.attn_fwd_gqa(Q, K, V, None, True, 0, scale)[0])
                X[idx] = old - eps
                Lm = np.sum(dO * orc.attn_fwd_gqa(Q, K, V, None, True, 0, scale)[0])
                X[idx] = old
                num[idx] = (Lp - Lm) / (2 * eps)
            np.testing.assert_allclose(dX, num, atol=2e-6)
        done += 1
        if done == 2:
            break
    assert done >= 1


# ------------------------------------------------------------ general alpha
# alpha-entmax (page "svd-sst2-roberta-adasplash", section 4, the entmax_bisect routine):
# p = max(0, (alpha-1)(s - tau))^(1/(alpha-1)), sum p = 1, for alpha in (1, 2].
ALPHAS = (1.1, 1.25, 1.5, 1.75, 2.0)


def _sparsemax_textbook(z):
    """Sparsemax by sorting (Martins & Astudillo 2016, Algorithm 1): k(z) = max{k : 1 + k z_(k) >
    sum_{j<=k} z_(j)}, tau = (sum_{j<=k} z_(j) - 1) / k, p = max(0, z - tau)."""
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    ks = np.arange(1, z.size + 1)
    k = ks[1 + ks * zs > cs][-1]
    tau = (cs[k - 1] - 1.0) / k
    return np.clip(z - tau, 0.0, None), tau


def test_alpha_two_is_textbook_sparsemax():
    for s in _rows(31, 200, nmin=1, nmax=40, spread=(0.2, 4.0)):
        p_ref, t_ref = _sparsemax_textbook(s)
        assert orc.tau_alpha(s, 2.0) == pytest.approx(t_ref, abs=1e-12)
        np.testing.assert_allclose(orc.entmax_alpha(s, 2.0), p_ref, atol=1e-12)


def test_alpha_one_point_five_matches_closed_form():
    """The generic solver at alpha = 1.5 against the sorted closed form of Theorem 1."""
    for s in _rows(32, 200, nmin=1, nmax=60):
        assert orc.tau_alpha(s, 1.5) == pytest.approx(orc.tau_sort(s)[0], abs=1e-12)
        np.testing.assert_allclose(orc.entmax_alpha(s, 1.5), orc.entmax15(s), atol=1e-12)


def test_alpha_near_one_tends_to_softmax():
    """alpha -> 1+: alpha-entmax tends to softmax (the pages fall back to softmax at alpha = 1)."""
    rng = np.random.default_rng(33)
    for _ in range(20):
        s = rng.normal(0, 1.0, size=12)
        sm = np.exp(s - s.max())
        sm /= sm.sum()
        np.testing.assert_allclose(orc.entmax_alpha(s, 1.0 + 1e-4), sm, atol=2e-3)


@pytest.mark.parametrize("alpha", [1.25, 1.75, 2.0])
def test_alpha_argmax_definition_by_optimiser(alpha):
    """alpha-entmax(s) = argmax_{p in simplex} p.s + sum (p - p^alpha) / (alpha (alpha - 1))
    (the Tsallis-entropy definition of which section 2.1 is the alpha = 1.5 case)."""
    c = 1.0 / (alpha * (alpha - 1.0))
    for s in _rows(34, 25, nmin=2, nmax=6, spread=(0.3, 2.5)):
        n = s.size

        def neg(p):
            p = np.clip(p, 0.0, None)
            return -(p @ s + c * np.sum(p - p ** alpha))

        best = None
        for x0 in (np.full(n, 1.0 / n), np.eye(n)[int(np.argmax(s))] * 0.9 + 0.1 / n):
            r = optimize.minimize(neg, x0, method="SLSQP", bounds=[(0, 1)] * n,
                                  constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1.0}],
                                  options={"ftol": 1e-14, "maxiter": 500})
            if best is None or r.fun < best.fun:
                best = r
        np.testing.assert_allclose(orc.entmax_alpha(s, alpha), np.clip(best.x, 0, None), atol=3e-4)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_alpha_invariants_and_bisection_bound(alpha):
    """Simplex, shift invariance, max-gap one-hot (gap >= 1/(alpha-1)), and the pages' 25 halvings
    within half the final bracket of the converged root."""
    a = alpha - 1.0
    for s in _rows(35, 100, nmin=1, nmax=30):
        p = orc.entmax_alpha(s, alpha)
        assert np.all(p >= 0) and abs(p.sum() - 1.0) < 1e-10
        np.testing.assert_allclose(orc.entmax_alpha(s + 3.7, alpha), p, atol=1e-11)
        t = orc.tau_alpha(s, alpha)
        width = (1.0 - s.size ** (-a)) / a
        assert abs(orc.tau_alpha_bisect(s, alpha, 25) - t) <= width / 2 ** 26 + 1e-12
    s = np.array([0.0, -1.0 / a, -1.0 / a - 0.5, -3.0 / a])
    np.testing.assert_allclose(orc.entmax_alpha(s, alpha), [1.0, 0.0, 0.0, 0.0], atol=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.75, 2.0])
def test_alpha_jvp_matches_finite_differences(alpha):
    rng = np.random.default_rng(36)
    checked = 0
    for s in _rows(37, 120, nmin=2, nmax=10, spread=(0.5, 3.0)):
        t = orc.tau_alpha(s, alpha)
        if np.min(np.abs(s - t)) < 1e-3:
            continue
        h = 1e-6
        J = np.empty((s.size, s.size))
        for j in range(s.size):
            e = np.zeros(s.size)
            e[j] = h
            J[:, j] = (orc.entmax_alpha(s + e, alpha) - orc.entmax_alpha(s - e, alpha)) / (2 * h)
        gv = rng.normal(size=s.size)
        ds = orc.entmax_alpha_jvp(orc.entmax_alpha(s, alpha), gv, alpha)
        np.testing.assert_allclose(ds, J.T @ gv, atol=2e-6)
        checked += 1
    assert checked > 50


@pytest.mark.parametrize("alpha", [1.25, 2.0])
def test_alpha_attention_backward_matches_finite_differences(alpha):
    B, H, L, D = 1, 1, 6, 4
    scale = 0.6
    done = 0
    for seed in range(60):
        Q, K, V, dO = _rand_qkv(400 + seed, B, H, L, D)
        O, tau = orc.attn_fwd(Q, K, V, None, True, 0, scale, alpha=alpha)
        S = scale * Q[0, 0] @ K[0, 0].T
        a = _allowed(L, True, 0, None)
        if np.abs(S - tau[0, 0][:, None])[a].min() < 1e-3:
            continue
        # forward against the scalar root finder, row by row
        for i in range(L):
            s = S[i, a[i]]
            f = lambda t: np.sum(np.clip((alpha - 1) * (s - t), 0, None) ** (1 / (alpha - 1))) - 1.0
            assert tau[0, 0, i] == pytest.approx(optimize.brentq(f, s.max() - 1 / (alpha - 1) - 1, s.max(),
                                                                 xtol=1e-15), abs=1e-10)
        dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, None, True, 0, scale, alpha=alpha)
        eps = 1e-6
        for X, dX in ((Q, dQ), (K, dK), (V, dV)):
            num = np.zeros_like(X)
            for idx in np.ndindex(X.shape):
                old = X[idx]
                X[idx] = old + eps
                Lp = np.sum(dO * orc.attn_fwd(Q, K, V, None, True, 0, scale, alpha=alpha)[0])
                X[idx] = old - eps
                Lm = np.sum(dO * orc.attn_fwd(Q, K, V, None, True, 0, scale, alpha=alpha)[0])
                X[idx] = old
                num[idx] = (Lp - Lm) / (2 * eps)
            np.testing.assert_allclose(dX, num, atol=3e-6)
        done += 1
        if done == 2:
            break
    assert done >= 1


# ------------------------------------------------------------ alpha = 1 (softmax)
# The pages' alpha-entmax routine returns softmax when |alpha - 1| < 1e-4 (page
# "svd-sst2-roberta-adasplash", section 4, entmax_bisect): p = exp(s - tau), tau = log sum exp(s).
def test_softmax_closed_forms():
    # n equal scores c: p = 1/n, tau = c + log n
    for n, c in ((1, 0.3), (5, -2.0), (64, 7.5)):
        s = np.full(n, c)
        assert orc.tau_softmax(s) == pytest.approx(c + math.log(n), abs=1e-13)
        np.testing.assert_allclose(orc.softmax(s), np.full(n, 1.0 / n), atol=1e-14)
    # two scores: the logistic function of their gap
    for a, b in ((0.0, 1.0), (3.0, -2.5), (1000.0, 999.0)):
        s = np.array([a, b])
        assert orc.softmax(s)[0] == pytest.approx(1.0 / (1.0 + math.exp(b - a)), abs=1e-13)
        assert orc.tau_softmax(s) == pytest.approx(max(a, b) + math.log1p(math.exp(-abs(a - b))), abs=1e-12)
    # a shift moves tau by the same amount and leaves p alone
    for s in _rows(51, 40, nmin=1, nmax=30):
        assert orc.tau_softmax(s + 4.25) == pytest.approx(orc.tau_softmax(s) + 4.25, abs=1e-12)
        np.testing.assert_allclose(orc.softmax(s + 4.25), orc.softmax(s), atol=1e-14)
    assert orc.tau_softmax(np.array([])) == math.inf


def test_softmax_is_the_gibbs_argmax():
    """softmax(s) = argmax over the simplex of p.s - sum p log p, and the maximum is log sum exp(s)
    (the alpha -> 1 member of the entropy family whose alpha = 1.5 case is section 2.1)."""
    rng = np.random.default_rng(52)
    for _ in range(12):
        n = int(rng.integers(2, 8))
        s = rng.normal(0, 1.5, size=n)

        def neg(p):
            q = np.clip(p, 1e-300, None)
            return -(p @ s - np.sum(q * np.log(q)))

        cons = ({"type": "eq", "fun": lambda p: np.sum(p) - 1.0},)
        res = optimize.minimize(neg, np.full(n, 1.0 / n), method="SLSQP", bounds=[(0.0, 1.0)] * n,
                                constraints=cons, options={"ftol": 1e-14, "maxiter": 500})
        np.testing.assert_allclose(orc.softmax(s), res.x, atol=2e-4)
        assert -res.fun == pytest.approx(orc.tau_softmax(s), abs=1e-8)


def test_softmax_is_the_alpha_one_limit():
    """alpha-entmax (pinned on its own above) tends to softmax as alpha -> 1+, the gap shrinking with
    alpha - 1."""
    for s in _rows(53, 10, nmin=2, nmax=12, spread=(0.3, 1.5)):
        sm = orc.softmax(s)
        errs = [np.max(np.abs(orc.entmax_alpha(s, 1.0 + e) - sm)) for e in (1e-1, 1e-2, 1e-3)]
        assert errs[0] > errs[1] > errs[2] and errs[2] < 2e-3


def test_softmax_jvp_matches_finite_differences():
    """The Jacobian-vector product at alpha = 1 (w = p) against central differences of softmax."""
    rng = np.random.default_rng(54)
    for _ in range(20):
        n = int(rng.integers(1, 10))
        s = rng.normal(0, 2.0, size=n)
        gv = rng.normal(size=n)
        h = 1e-6
        J = np.empty((n, n))
        for j in range(n):
            e = np.zeros(n)
            e[j] = h
            J[:, j] = (orc.softmax(s + e) - orc.softmax(s - e)) / (2 * h)
        ds = orc.entmax_alpha_jvp(orc.softmax(s), gv, 1.0)
        np.testing.assert_allclose(ds, J.T @ gv, atol=2e-8)


def test_softmax_attention_special_cases():
    """alpha = 1 attention: Q = 0 gives every allowed key weight 1/n (O = mean of the allowed V rows,
    tau = log n); causal row 0 sees key 0 alone (O = V_0, tau = S_00); a fully padded batch gives
    O = 0, tau = +inf; one key far above the rest takes all the weight."""
    B, H, L, D = 2, 2, 20, 8
    _, K, V, _ = _rand_qkv(55, B, H, L, D)
    Q = np.zeros_like(K)
    mask = np.ones((B, L), np.uint8)
    mask[1, 13:] = 0
    mask[1, 2] = 0
    O, tau = orc.attn_fwd(Q, K, V, mask, False, 0, 0.125, alpha=1.0)
    for b in range(B):
        keep = mask[b].astype(bool)
        for h in range(H):
            np.testing.assert_allclose(O[b, h], np.broadcast_to(V[b, h][keep].mean(0), (L, D)), atol=1e-13)
            np.testing.assert_allclose(tau[b, h], math.log(keep.sum()), atol=1e-13)
    Q, K, V, _ = _rand_qkv(56, B, H, L, D)
    O, tau = orc.attn_fwd(Q, K, V, None, True, 0, 0.3, alpha=1.0)
    np.testing.assert_allclose(O[:, :, 0], V[:, :, 0], atol=1e-13)
    np.testing.assert_allclose(tau[:, :, 0], 0.3 * np.einsum("bhd,bhd->bh", Q[:, :, 0], K[:, :, 0]), atol=1e-12)
    mask = np.ones((B, L), np.uint8)
    mask[0] = 0
    O, tau = orc.attn_fwd(Q, K, V, mask, False, 0, 0.3, alpha=1.0)
    assert np.all(O[0] == 0) and np.all(np.isinf(tau[0]))
    # key 5 aligned with every query and far longer than the others
    K2 = K.copy()
    K2[:, :, 5] = 60.0 * Q.mean(axis=2)
    O, _ = orc.attn_fwd(Q, K2, V, None, False, 0, 1.0, alpha=1.0)
    S = np.einsum("bhid,bhjd->bhij", Q, K2)
    gap = S[:, :, :, 5] - np.delete(S, 5, axis=3).max(axis=3)
    rows = gap > 40.0
    assert rows.sum() > 10
    err = np.abs(O - V[:, :, 5:6, :])[rows]
    assert err.max() < 1e-12


def test_softmax_attention_backward_matches_finite_differences():
    """dQ, dK, dV at alpha = 1 against central differences of <dO, O>, with a causal window and a
    padded key."""
    B, H, L, D = 1, 2, 7, 4
    scale = 0.7
    Q, K, V, dO = _rand_qkv(57, B, H, L, D)
    mask = np.ones((B, L), np.uint8)
    mask[0, 3] = 0
    args = (mask, True, 4, scale)
    dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, *args, alpha=1.0)
    eps = 1e-6
    for X, dX in ((Q, dQ), (K, dK), (V, dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + eps
            Lp = np.sum(dO * orc.attn_fwd(Q, K, V, *args, alpha=1.0)[0])
            X[idx] = old - eps
            Lm = np.sum(dO * orc.attn_fwd(Q, K, V, *args, alpha=1.0)[0])
            X[idx] = old
            num[idx] = (Lp - Lm) / (2 * eps)
        np.testing.assert_allclose(dX, num, atol=3e-7)
    assert np.all(dK[0, :, 3] == 0) and np.all(dV[0, :, 3] == 0)


# ------------------------------------------------------- auxiliary rows
def test_aux_rows_uniform_and_one_hot():
    """Otil_i = sum_j sqrt(p_ij) V_j, r_i = sum_j sqrt(p_ij).  Q = 0: p = 1/n on the allowed keys, so
    r = sqrt(n) and Otil = (sum of the allowed V rows) / sqrt(n).  A key far above the rest: p is
    one-hot, r = 1 and Otil = that key's V row."""
    B, H, L, D = 2, 2, 24, 8
    _, K, V, _ = _rand_qkv(31, B, H, L, D)
    Q = np.zeros_like(K)
    mask = np.zeros((B, L), np.uint8)
    mask[0, :24] = 1
    mask[1, :9] = 1
    ids = np.arange(B * H * L)
    Ot, r = orc.attn_aux_rows(Q, K, V, ids, mask, scale=0.125)
    for rid in ids:
        b, h, i = rid // (H * L), (rid // L) % H, rid % L
        n = int(mask[b].sum())
        assert r[rid] == pytest.approx(math.sqrt(n), abs=1e-12)
        np.testing.assert_allclose(Ot[rid], V[b, h, :n].sum(axis=0) / math.sqrt(n), atol=1e-12)
    Q2 = np.zeros((1, 1, 8, 4))
    K2 = np.zeros((1, 1, 8, 4))
    V2 = np.arange(32, dtype=float).reshape(1, 1, 8, 4)
    Q2[0, 0, :, 0] = 1.0
    K2[0, 0, 3, 0] = 10.0
    Ot2, r2 = orc.attn_aux_rows(Q2, K2, V2, np.arange(8), None, scale=1.0)
    np.testing.assert_allclose(r2, 1.0, atol=1e-15)
    np.testing.assert_allclose(Ot2, np.broadcast_to(V2[0, 0, 3], (8, 4)), atol=1e-15)
    # a row with no allowed key
    m0 = np.zeros((1, 8), np.uint8)
    Ot3, r3 = orc.attn_aux_rows(Q2, K2, V2, [0, 5], m0, scale=1.0)
    assert np.all(Ot3 == 0) and np.all(r3 == 0)


def test_aux_rows_by_kkt_bruteforce():
    """Tiny heads: tau of every row by enumerating supports (KKT), then sqrt(p) = (s - tau)/2 on the
    support and the two sums written out."""
    rng = np.random.default_rng(32)
    for trial in range(20):
        L, D = int(rng.integers(1, 5)), int(rng.integers(1, 5))
        Q = rng.normal(0, 1.5, (1, 1, L, D))
        K = rng.normal(0, 1.5, (1, 1, L, D))
        V = rng.normal(0, 1.0, (1, 1, L, D))
        Ot, r = orc.attn_aux_rows(Q, K, V, np.arange(L), None, scale=0.7)
        for i in range(L):
            s = 0.7 * (K[0, 0] @ Q[0, 0, i])
            tau = _kkt_bruteforce(s)[0]
            w = np.where(s > tau, (s - tau) / 2.0, 0.0)
            assert r[i] == pytest.approx(w.sum(), abs=1e-10)
            np.testing.assert_allclose(Ot[i], w @ V[0, 0], atol=1e-10)


def test_aux_rows_give_the_score_gradient():
    """The backward's row scalar from the auxiliary rows, u_i = dO_i . Otil_i / r_i, against central
    finite differences of <dO_i, O_i> in the scores: on the support, d<dO_i, O_i>/ds_j =
    sqrt(p_j) (dO_i . V_j - u_i) (section 2.4), so u_i = dO_i . V_j - (FD_j / sqrt(p_j))."""
    rng = np.random.default_rng(33)
    L, D = 12, 6
    Q = rng.normal(0, 1.0, (1, 1, L, D))
    K = rng.normal(0, 1.0, (1, 1, L, D))
    V = rng.normal(0, 1.0, (1, 1, L, D))
    dO = rng.normal(0, 1.0, (L, D))
    scale = 1.3
    Ot, r = orc.attn_aux_rows(Q, K, V, np.arange(L), None, scale=scale)
    checked = 0
    for i in range(L):
        s = scale * (K[0, 0] @ Q[0, 0, i])
        p = orc.entmax15(s)
        u = dO[i] @ Ot[i] / r[i]
        tau = orc.tau_sort(s)[0]
        if np.min(np.abs(s - tau)) < 1e-3:
            continue  # a kink: skip
        h = 1e-6
        for j in np.nonzero(p > 0)[0]:
            e = np.zeros(L)
            e[j] = h
            fd = (dO[i] @ (orc.entmax15(s + e) @ V[0, 0]) - dO[i] @ (orc.entmax15(s - e) @ V[0, 0])) / (2 * h)
            assert dO[i] @ V[0, 0, j] - fd / math.sqrt(p[j]) == pytest.approx(u, abs=1e-5)
            checked += 1
    assert checked > 10
