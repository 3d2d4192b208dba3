"""Pins for the fp64 oracle against facts fixed by the pages and by mathematics.

The oracle is checked here against things other than itself: closed forms of special cases
(the second-order Taylor kernel, a constant kernel whose output is a running mean, kernels
that select a single group), a different evaluation route of eq. (3) (the norm of L^T sbar
instead of the quadratic form), invariances, and brute force on tiny inputs.  Each one is
chosen so that a plausible slip (a dropped term or eps, a wrong scale or sign, a transposed
L, exclusive instead of inclusive causality, a wrong GQA head map, a wrong group index)
fails at least one test.

Citations: "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of arXiv 2610.13674),
section 核心公式, equations numbered in order of appearance (2) grouped score, (3) kernel,
(4) prefix states, (5) readout; the abstract of arXiv 2610.13674 ("Starting from a
second-order Taylor approximation").
"""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _one_head_problem(rng, T, d, dv, G, gid=None):
    q = _rand(rng, 1, 1, T, d)
    k = _rand(rng, 1, 1, T, d)
    v = _rand(rng, 1, 1, T, dv)
    if gid is None:
        gid = rng.integers(1, G + 1, size=(1, d)).astype(np.int32)
        gid[0, :G] = np.arange(1, G + 1)  # every group non-empty
    return q, k, v, gid


def _slot(Lsmall, gmax=I.GMAX):
    L = np.zeros((1, gmax + 1, gmax + 1))
    n = Lsmall.shape[0]
    L[0, :n, :n] = Lsmall
    return L


def _causal_weighted_mean(W, v):
    """yhat_i = sum_{j<=i} W_ij v_j / sum_{j<=i} W_ij for one head (numpy)."""
    Wm = np.tril(W)
    return (Wm @ v) / Wm.sum(axis=1, keepdims=True)


def _both(q, k, v, gid, L, G, eps):
    yd = oracle.dense(q, k, v, gid, L, np.array(G, np.int32).reshape(-1), eps)
    yr = oracle.recurrent(q, k, v, gid, L, np.array(G, np.int32).reshape(-1), eps)
    return yd, yr


# --- closed forms --------------------------------------------------------------------------

def test_taylor_special_case():
    """G=1, L=[[1,0],[1/2,1/2]] gives M=[[1,1/2],[1/2,1/2]] and kappa = eps + 1 + s + s^2/2,
    the second-order Taylor expansion of exp(s) (abstract), with s = q.k/sqrt(d)."""
    rng = np.random.default_rng(11)
    T, d, dv, eps = 40, 16, 8, 0.25
    q, k, v, _ = _one_head_problem(rng, T, d, dv, 1)
    gid = np.ones((1, d), np.int32)
    L = _slot(np.array([[1.0, 0.0], [0.5, 0.5]]))
    s = (q[0, 0] @ k[0, 0].T) / np.sqrt(d)
    W = eps + 1.0 + s + 0.5 * s * s
    np.testing.assert_allclose(oracle.kappa(q[0, 0], k[0, 0], gid[0], L[0], 1, eps), W,
                               rtol=1e-13, atol=1e-13)
    ref = _causal_weighted_mean(W, v[0, 0])
    yd, yr = _both(q, k, v, gid, L, 1, eps)
    np.testing.assert_allclose(yd[0, 0], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(yr[0, 0], ref, rtol=1e-10, atol=1e-11)


def test_constant_kernel_is_inclusive_running_mean():
    """L = e0 e0^T makes kappa = eps + 1 for every pair, so yhat_i is the mean of v_0..v_i
    (inclusive causality, eq. (4) j <= i)."""
    rng = np.random.default_rng(12)
    T, d, dv = 33, 8, 5
    q, k, v, gid = _one_head_problem(rng, T, d, dv, 3)
    Ls = np.zeros((4, 4))
    Ls[0, 0] = 1.0
    ref = np.cumsum(v[0, 0], axis=0) / np.arange(1, T + 1)[:, None]
    yd, yr = _both(q, k, v, gid, _slot(Ls), 3, 1e-6)
    np.testing.assert_allclose(yd[0, 0], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(yr[0, 0], ref, rtol=1e-10, atol=1e-11)


def test_single_group_selector():
    """M = diag(1, 0, 1): kappa = eps + 1 + s_2^2 with s_2 summed over the dims whose group
    id is 2 only (eq. (2)); the dims of group 1 must not contribute."""
    rng = np.random.default_rng(13)
    T, d, dv, eps = 30, 12, 4, 0.5
    q, k, v, gid = _one_head_problem(rng, T, d, dv, 2)
    Ls = np.diag([1.0, 0.0, 1.0])
    m2 = gid[0] == 2
    s2 = (q[0, 0][:, m2] @ k[0, 0][:, m2].T) / np.sqrt(d)
    W = eps + 1.0 + s2 * s2
    np.testing.assert_allclose(oracle.kappa(q[0, 0], k[0, 0], gid[0], _slot(Ls)[0], 2, eps), W,
                               rtol=1e-13, atol=1e-13)
    yd, yr = _both(q, k, v, gid, _slot(Ls), 2, eps)
    ref = _causal_weighted_mean(W, v[0, 0])
    np.testing.assert_allclose(yd[0, 0], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(yr[0, 0], ref, rtol=1e-10, atol=1e-11)


def test_cross_term_selector():
    """L = [[1,0,0],[1,0,0],[0,0,0]] gives M with M_00 = M_01 = M_11 = 1, so
    kappa = eps + (1 + s_1)^2: checks the factor 2 on the linear term and the 1/sqrt(d)."""
    rng = np.random.default_rng(14)
    T, d, dv, eps = 25, 10, 3, 0.125
    q, k, v, gid = _one_head_problem(rng, T, d, dv, 2)
    Ls = np.array([[1.0, 0, 0], [1.0, 0, 0], [0, 0, 0]])
    m1 = gid[0] == 1
    s1 = (q[0, 0][:, m1] @ k[0, 0][:, m1].T) / np.sqrt(d)
    W = eps + (1.0 + s1) ** 2
    yd, yr = _both(q, k, v, gid, _slot(Ls), 2, eps)
    ref = _causal_weighted_mean(W, v[0, 0])
    np.testing.assert_allclose(yd[0, 0], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(yr[0, 0], ref, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("G", [1, 3, 6, 8])
def test_norm_form_of_kappa(G):
    """eq. (3) through a different route: sbar^T L L^T sbar = ||L^T sbar||^2.  A full (not
    triangular) random L makes L L^T differ from L^T L, so a transposed factor fails."""
    rng = np.random.default_rng(20 + G)
    T, d = 17, 24
    q, k, _, gid = _one_head_problem(rng, T, d, 2, G)
    Ls = rng.standard_normal((G + 1, G + 1))
    eps = 0.3
    sbar = np.ones((T, T, G + 1))
    for g in range(1, G + 1):
        m = gid[0] == g
        sbar[:, :, g] = (q[0, 0][:, m] @ k[0, 0][:, m].T) / np.sqrt(d)
    W = eps + np.sum(np.einsum("ijg,gm->ijm", sbar, Ls) ** 2, axis=-1)
    got = oracle.kappa(q[0, 0], k[0, 0], gid[0], _slot(Ls)[0], G, eps)
    np.testing.assert_allclose(got, W, rtol=1e-12, atol=1e-12)


def test_gqa_head_map():
    """Query head h reads key/value head floor(h*Hkv/Hq): with a constant kernel each head's
    output is the running mean of its own key/value head's v."""
    rng = np.random.default_rng(15)
    B, Hq, Hkv, T, d, dv = 2, 6, 2, 9, 8, 3
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, dv)) + np.arange(Hkv)[None, :, None, None] * 10
    gid = np.ones((Hq, d), np.int32)
    L = np.zeros((Hq, 9, 9))
    L[:, 0, 0] = 1.0
    G = np.ones(Hq, np.int32)
    yd = oracle.dense(q, k, v, gid, L, G, 1e-6)
    yr = oracle.recurrent(q, k, v, gid, L, G, 1e-6)
    for h in range(Hq):
        ref = np.cumsum(v[:, h * Hkv // Hq], axis=1) / np.arange(1, T + 1)[None, :, None]
        np.testing.assert_allclose(yd[:, h], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(yr[:, h], ref, rtol=1e-10, atol=1e-11)


def test_prefix_state_definition():
    """The recurrence's final state equals the eq. (4) sums written as whole-sequence
    contractions: H0 = sum_j [v;1], H1 = sum_j k_j [v;1]^T, H2 = sum_j k_j k_j^T [v;1]."""
    rng = np.random.default_rng(16)
    p = I.small_layer(3, B=2, T=21, Hq=4, Hkv=2, dtype="f32", d=8, dv=6)
    _, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    vv = np.concatenate([p.v, np.ones(p.v.shape[:-1] + (1,), np.float32)], axis=-1).astype(np.float64)
    k64 = p.k.astype(np.float64)
    np.testing.assert_allclose(st.H0, vv.sum(axis=2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st.H1, np.einsum("bhjr,bhjn->bhrn", k64, vv), rtol=1e-12,
                               atol=1e-11)
    np.testing.assert_allclose(st.H2, np.einsum("bhjr,bhjt,bhjn->bhrtn", k64, k64, vv),
                               rtol=1e-12, atol=1e-10)
    del rng


# --- invariants ----------------------------------------------------------------------------

def test_positivity():
    """M = L L^T is PSD, so kappa >= eps on every pair and the normaliser of row i is at
    least (i+1) eps (eq. (3), 'PSD parameterisation guarantees a positive denominator')."""
    p = I.config0()
    kap = oracle.kappa(p.q[0, 0], p.k[0, 0], p.group_id[0], p.L[0], int(p.G[0]), p.eps)
    assert kap.min() >= p.eps * (1 - 1e-9)
    q = p.slice_tokens(0, 64)
    _, den = oracle.dense(q.q, q.k, q.v, q.group_id, q.L, q.G, q.eps, return_den=True)
    assert np.all(den[0, 0] >= (np.arange(64) + 1) * q.eps)
    p1 = I.small_layer(4, B=1, T=48, Hq=4, Hkv=2, dtype="bf16")
    for h in range(4):
        kap = oracle.kappa(p1.q[0, h], p1.k[0, h // 2], p1.group_id[h], p1.L[h], int(p1.G[h]),
                           p1.eps)
        assert kap.min() >= p1.eps * (1 - 1e-9)


def test_permutation_invariance():
    """Relabelling head dimensions consistently in q, k and group_id changes nothing."""
    p = I.small_layer(5, B=1, T=37, Hq=4, Hkv=2, dtype="f32")
    perm = np.random.default_rng(5).permutation(p.q.shape[-1])
    y0 = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    y1 = oracle.recurrent(p.q[..., perm], p.k[..., perm], p.v, p.group_id[:, perm], p.L, p.G,
                          p.eps)
    np.testing.assert_allclose(y1, y0, rtol=1e-10, atol=1e-12)


def test_scale_invariance():
    """kappa scales by c^2 under L -> cL, eps -> c^2 eps; the normalised output does not."""
    p = I.small_layer(6, B=1, T=29, Hq=2, Hkv=1, dtype="f32")
    y0 = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, 0.01)
    y1 = oracle.dense(p.q, p.k, p.v, p.group_id, 3.0 * p.L.astype(np.float64), p.G, 0.09)
    np.testing.assert_allclose(y1, y0, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("case", ["config0", "gqa_bf16", "g8_dv32", "tiny_T1"])
def test_dense_equals_recurrent(case):
    """eqs. (4)-(5) reproduce eqs. (2)-(3) summed over j <= i: the two independent oracle
    routes agree to 1e-10 relative (the pages report 1.18e-6..1.28e-6 for their own,
    lower-precision, dense/HD check)."""
    if case == "config0":
        p = I.config0()
    elif case == "gqa_bf16":
        p = I.small_layer(7, B=2, T=150, Hq=14, Hkv=2, dtype="bf16")
    elif case == "g8_dv32":
        rng = np.random.default_rng(8)
        p = I.small_layer(8, B=1, T=70, Hq=2, Hkv=1, dtype="f32", d=16, dv=32)
        p.G[:] = 8
        p.group_id[:] = rng.integers(1, 9, size=p.group_id.shape)
        p.group_id[:, :8] = np.arange(1, 9)
        p.L[:] = np.stack([I.random_L(rng, 8) for _ in range(2)])
    else:
        p = I.small_layer(9, B=3, T=1, Hq=2, Hkv=2, dtype="f32")
    yd = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    yr = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    scale = np.abs(yd).max(axis=-1, keepdims=True)
    assert np.max(np.abs(yr - yd) / np.maximum(scale, 1e-300)) < 1e-10


def test_decode_continuation():
    """Prefill of T tokens then n single-token steps from the saved state equals a prefill of
    T + n tokens (eq. (4) is a prefix sum), in outputs and in the final state."""
    p = I.small_layer(10, B=2, T=40, Hq=4, Hkv=2, dtype="bf16")
    y_all, st_all = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps,
                                     return_state=True)
    pre = p.slice_tokens(0, 33)
    _, st = oracle.recurrent(pre.q, pre.k, pre.v, pre.group_id, pre.L, pre.G, pre.eps,
                             return_state=True)
    for t in range(33, 40):
        s = p.slice_tokens(t, t + 1)
        y, st = oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps, state=st,
                                 return_state=True)
        np.testing.assert_allclose(y[:, :, 0], y_all[:, :, t], rtol=1e-11, atol=1e-12)
    for a, b in ((st.H0, st_all.H0), (st.H1, st_all.H1), (st.H2, st_all.H2)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-9)


def test_brute_force_tiny():
    """T <= 8: the definition evaluated with scalar Python loops only (explicit L L^T, s_g
    summed per group, weighted causal mean), against both oracle routes."""
    rng = np.random.default_rng(17)
    T, d, dv, G, eps = 6, 5, 3, 3, 0.2
    q, k, v, gid = _one_head_problem(rng, T, d, dv, G)
    Ls = np.tril(rng.standard_normal((G + 1, G + 1)))
    M = [[sum(Ls[a][m] * Ls[b][m] for m in range(G + 1)) for b in range(G + 1)]
         for a in range(G + 1)]
    ref = np.zeros((T, dv))
    for i in range(T):
        num = [0.0] * dv
        den = 0.0
        for j in range(i + 1):
            sb = [1.0] + [0.0] * G
            for r in range(d):
                sb[gid[0][r]] += q[0, 0, i, r] * k[0, 0, j, r] / d ** 0.5
            kap = eps + sum(sb[a] * M[a][b] * sb[b] for a in range(G + 1) for b in range(G + 1))
            den += kap
            for n in range(dv):
                num[n] += kap * v[0, 0, j, n]
        ref[i] = [x / den for x in num]
    yd, yr = _both(q, k, v, gid, _slot(Ls), G, eps)
    np.testing.assert_allclose(yd[0, 0], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(yr[0, 0], ref, rtol=1e-11, atol=1e-12)


def test_argument_validation():
    p = I.small_layer(11, B=1, T=4, Hq=2, Hkv=1, dtype="f32")
    bad = p.group_id.copy()
    bad[0, 0] = 0
    with pytest.raises(ValueError):
        oracle.dense(p.q, p.k, p.v, bad, p.L, p.G, p.eps)
    badG = p.G.copy()
    badG[1] = 9
    with pytest.raises(ValueError):
        oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, badG, p.eps)


def test_golden_regression_record():
    """The oracle still reproduces the stored record of its own config-0 outputs (written by
    tests/golden/make_golden.py; the pages print no worked example to pin instead)."""
    import json
    import os
    rec = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "config0_rows.json")))
    p = I.config0()
    y, den = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_den=True)
    for n, i in enumerate(rec["rows"]):
        np.testing.assert_allclose(y[0, 0, i, :8], rec["yhat_first8"][n], rtol=1e-12)
        np.testing.assert_allclose(den[0, 0, i], rec["normaliser"][n], rtol=1e-12)


def test_dense_rows_match_dense():
    """Sampled-row evaluation returns exactly the rows of the full dense form."""
    p = I.small_layer(12, B=2, T=50, Hq=4, Hkv=2, dtype="bf16")
    y = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    rows = [(0, 0, 0), (1, 3, 49), (0, 2, 17), (1, 1, 33)]
    yr = oracle.dense_rows(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(yr[n], y[b, h, i])


# --- contribution statistic, eq. (1) ------------------------------------------------------------

def test_chi_constant_inputs_closed_form():
    """q = a and k = c everywhere: every causal pair contributes |a c| / sqrt(d), and the
    pair count cancels |Omega| = T (T + 1) / 2, so chi = |a c| / 8 for d = 64."""
    T, d = 37, 64
    q = np.full((1, 1, T, d), -1.5)
    k = np.full((1, 1, T, d), 0.75)
    np.testing.assert_allclose(oracle.chi(q, k), abs(-1.5 * 0.75) / 8.0, rtol=1e-13)


def test_chi_linear_keys_closed_form():
    """q = 1, k_j = j + 1: sum_i sum_{j<=i} (j + 1) = T (T + 1)(T + 2) / 6, so chi =
    (T + 2) / (3 sqrt(d)) after dividing by T (T + 1) / 2.  Summing over every j instead of
    j <= i, or dividing by T^2, gives a different value."""
    T, d = 50, 64
    q = np.ones((1, 1, T, d))
    k = np.broadcast_to((np.arange(T) + 1.0)[None, None, :, None], (1, 1, T, d)).copy()
    np.testing.assert_allclose(oracle.chi(q, k), (T + 2) / (3.0 * 8.0), rtol=1e-12)


def test_chi_is_causal_not_full():
    """Only the last query sees the last key: a key spike at j = T - 1 contributes once."""
    T, d = 16, 64
    q = np.ones((1, 1, T, d))
    k = np.zeros((1, 1, T, d))
    k[0, 0, T - 1, 5] = 8.0
    chi = oracle.chi(q, k)
    pairs = T * (T + 1) / 2
    assert chi[0, 0, 5] == pytest.approx(8.0 / 8.0 / pairs, rel=1e-13)
    assert np.count_nonzero(chi) == 1


def test_chi_invariances_and_gqa():
    """Sign flips of q or k leave chi unchanged, scales multiply it, a permutation of the
    dimensions permutes it, and query head h reads key head floor(h * Hkv / Hq)."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, T, d = 2, 4, 2, 23, 64
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    base = oracle.chi(q, k)
    np.testing.assert_allclose(oracle.chi(-q, k), base, rtol=1e-13)
    np.testing.assert_allclose(oracle.chi(q, -2.0 * k), 2.0 * base, rtol=1e-13)
    perm = rng.permutation(d)
    np.testing.assert_allclose(oracle.chi(q[..., perm], k[..., perm]), base[..., perm],
                               rtol=1e-13)
    # GQA: heads 0, 1 read k head 0, heads 2, 3 read k head 1
    k2 = np.concatenate([k[:, :1], k[:, :1], k[:, 1:], k[:, 1:]], axis=1)
    np.testing.assert_allclose(oracle.chi(q, k2), base, rtol=1e-13)


def test_chi_equals_prefix_sum_form():
    """sum_i |q_i| (sum_{j<=i} |k_j|): a different evaluation route (cumulative sums)."""
    rng = np.random.default_rng(12)
    T, d = 40, 64
    q = rng.standard_normal((1, 1, T, d))
    k = rng.standard_normal((1, 1, T, d))
    ref = (np.abs(q[0, 0]) * np.cumsum(np.abs(k[0, 0]), axis=0)).sum(0) / 8.0 / (T * (T + 1) / 2)
    np.testing.assert_allclose(oracle.chi(q, k)[0, 0], ref, rtol=1e-12)
