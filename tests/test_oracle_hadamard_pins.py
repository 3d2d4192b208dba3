"""Pins for the oracle's ungrouped Hadamard form: eq. (5) with free a, b_r, C_rt.

The abstract of arXiv 2610.13674 describes this form: the second-order Taylor kernel with its
shared coefficients relaxed into per-dimension linear terms and cross-dimensional quadratic
terms. Eq. (5) ("OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式) is its readout.
The oracle evaluates it two ways, as pairwise kernels and through the H0/H1/H2 states. They
are checked here against:
- each other, on the unnormalised readout u;
- the grouped oracle, after expanding its coefficients;
- the Taylor kernel's closed form;
- a worked example done by hand;
- the facts that an antisymmetric C contributes nothing and that a kernel scaled by -1 gives
  the same output;
- IEEE behaviour when the normaliser is zero.
"""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I


def _problem(rng, B, Hq, Hkv, T, dh, dv):
    return (rng.standard_normal((B, Hq, T, dh)), rng.standard_normal((B, Hkv, T, dh)),
            rng.standard_normal((B, Hkv, T, dv)))


def _coef(rng, Hq, dh, a0=3.0):
    a = a0 + rng.random(Hq)
    b = rng.standard_normal((Hq, dh))
    C = 0.3 * rng.standard_normal((Hq, dh, dh))  # neither symmetric nor definite
    return a, b, C


def test_dense_and_recurrent_agree_on_u():
    """Eq. (5) over the states of eq. (4) equals the pairwise kernel summed over j <= i, for
    coefficients with no structure at all (GQA 4/2, ragged sizes)."""
    rng = np.random.default_rng(11)
    q, k, v = _problem(rng, 2, 4, 2, 37, 8, 5)
    a, b, C = _coef(rng, 4, 8)
    yd, ud = oracle.hadamard_dense(q, k, v, a, b, C, return_u=True)
    yr, ur = oracle.hadamard_recurrent(q, k, v, a, b, C, return_u=True)
    scale = np.abs(ud).max(axis=-1, keepdims=True)
    assert np.max(np.abs(ud - ur) / scale) < 1e-11
    np.testing.assert_allclose(yd, yr, rtol=1e-9, atol=1e-9)


def test_grouped_expansion_reproduces_grouped_kernel():
    """The grouped kernel of eq. (3) expanded into (a, b, C) gives the grouped oracle's
    output through the Hadamard dense form, which never sees L or the group ids."""
    p = I.small_layer(21, B=2, T=50, Hq=4, Hkv=2, dtype="f32")
    a, b, C = oracle.grouped_coefficients(p.group_id, p.L, p.G, p.eps)
    yh = oracle.hadamard_dense(p.q, p.k, p.v, a, b, C)
    yg = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    assert np.max(np.abs(yh - yg)) <= 1e-10 * np.abs(yg).max()


def test_taylor_coefficients():
    """a = 1, b_r = 1, C_rt = 1/2 give kappa = 1 + s + s^2/2 with s = q.k/sqrt(dh): the
    second-order Taylor expansion of exp(s) that the abstract starts from."""
    rng = np.random.default_rng(3)
    T, dh, dv = 20, 16, 3
    q, k, v = _problem(rng, 1, 1, 1, T, dh, dv)
    y = oracle.hadamard_recurrent(q, k, v, np.ones(1), np.ones((1, dh)),
                                  np.full((1, dh, dh), 0.5))
    s = q[0, 0] @ k[0, 0].T / np.sqrt(dh)
    W = np.tril(1.0 + s + 0.5 * s * s)
    ref = (W @ v[0, 0]) / W.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(y[0, 0], ref, rtol=1e-11, atol=1e-12)


def test_hand_worked_example():
    """dh = 4 (so x_r = q_r k_r / 2), dv = 1, T = 2; a = 1, b = e_0, C = E_01.
    Token 0: q = (2,2,0,0), k = (1,1,0,0), v = 1. Token 1: q = (2,0,0,0), k = (2,2,0,0), v = 4.
      kappa_00: x = (1,1,0,0) -> 1 + 1 + 1*1 = 3;  yhat_0 = 1
      kappa_10: x = (1,0,0,0) -> 1 + 1 + 0 = 2
      kappa_11: x = (2,0,0,0) -> 1 + 2 + 0 = 3;    yhat_1 = (2*1 + 3*4) / 5 = 14/5."""
    q = np.array([[2, 2, 0, 0], [2, 0, 0, 0]], float).reshape(1, 1, 2, 4)
    k = np.array([[1, 1, 0, 0], [2, 2, 0, 0]], float).reshape(1, 1, 2, 4)
    v = np.array([[1.0], [4.0]]).reshape(1, 1, 2, 1)
    a = np.ones(1)
    b = np.zeros((1, 4))
    b[0, 0] = 1.0
    C = np.zeros((1, 4, 4))
    C[0, 0, 1] = 1.0
    for f in (oracle.hadamard_dense, oracle.hadamard_recurrent):
        y, u = f(q, k, v, a, b, C, return_u=True)
        np.testing.assert_allclose(y[0, 0, :, 0], [1.0, 2.8], rtol=1e-15)
        np.testing.assert_allclose(u[0, 0, :, 1], [3.0, 5.0], rtol=1e-15)


def test_only_the_symmetric_part_of_C_counts():
    """x^T C x vanishes for antisymmetric C, so C, C^T and (C + C^T)/2 give one output, and
    C + (any antisymmetric matrix) changes nothing."""
    rng = np.random.default_rng(5)
    q, k, v = _problem(rng, 1, 2, 1, 25, 6, 4)
    a, b, C = _coef(rng, 2, 6)
    A = rng.standard_normal((2, 6, 6))
    A = A - A.transpose(0, 2, 1)
    ref = oracle.hadamard_recurrent(q, k, v, a, b, C)
    for C2 in (C.transpose(0, 2, 1), 0.5 * (C + C.transpose(0, 2, 1)), C + A):
        np.testing.assert_allclose(oracle.hadamard_recurrent(q, k, v, a, b, C2), ref,
                                   rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(oracle.hadamard_dense(q, k, v, a, b, C + A), ref, rtol=1e-9,
                               atol=1e-10)


def test_single_linear_and_cross_terms():
    """b = beta e_r and C = gamma E_rt select one linear and one cross term: kappa =
    a + beta x_r + gamma x_r x_t with x_r = q_r k_r / sqrt(dh). This catches a swapped q/k,
    a transposed index, or a wrong scale on either term."""
    rng = np.random.default_rng(8)
    T, dh, dv, r, t = 15, 9, 2, 2, 7
    q, k, v = _problem(rng, 1, 1, 1, T, dh, dv)
    a, beta, gamma = 4.0, 0.7, -0.4
    b = np.zeros((1, dh))
    b[0, r] = beta
    C = np.zeros((1, dh, dh))
    C[0, r, t] = gamma
    xr = np.outer(q[0, 0, :, r], k[0, 0, :, r]) / np.sqrt(dh)
    xt = np.outer(q[0, 0, :, t], k[0, 0, :, t]) / np.sqrt(dh)
    W = np.tril(a + beta * xr + gamma * xr * xt)
    ref = (W @ v[0, 0]) / W.sum(axis=1, keepdims=True)
    for f in (oracle.hadamard_dense, oracle.hadamard_recurrent):
        np.testing.assert_allclose(f(q, k, v, np.array([a]), b, C)[0, 0], ref, rtol=1e-11,
                                   atol=1e-12)


def test_non_positive_normalisers():
    """Free coefficients can make the kernel non-positive. A kernel scaled by -1 gives the
    same yhat, because numerator and normaliser flip together. A zero kernel gives 0/0 = NaN
    in every row. The pages define no other behaviour; the oracle reads the division plainly."""
    rng = np.random.default_rng(9)
    q, k, v = _problem(rng, 1, 1, 1, 12, 4, 3)
    a, b, C = _coef(rng, 1, 4)
    for f in (oracle.hadamard_dense, oracle.hadamard_recurrent):
        y_pos, u_pos = f(q, k, v, a, b, C, return_u=True)
        y_neg, u_neg = f(q, k, v, -a, -b, -C, return_u=True)
        np.testing.assert_allclose(y_neg, y_pos, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(u_neg, -u_pos, rtol=1e-12, atol=1e-12)
        # constant kernel -1: the running mean of v, normaliser -(i + 1)
        y_m, u_m = f(q, k, v, -np.ones(1), np.zeros((1, 4)), np.zeros((1, 4, 4)), return_u=True)
        mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, 13)[:, None]
        np.testing.assert_allclose(y_m[0, 0], mean, rtol=1e-13)
        np.testing.assert_allclose(u_m[0, 0, :, -1], -np.arange(1, 13), rtol=0)
        with np.errstate(invalid="ignore"):
            y0 = f(q, k, v, np.zeros(1), np.zeros((1, 4)), np.zeros((1, 4, 4)))
        assert np.isnan(y0).all()


def test_state_carries_across_calls():
    """Two recurrent calls joined by the state of eq. (4) give the one-call result."""
    rng = np.random.default_rng(10)
    q, k, v = _problem(rng, 2, 4, 2, 30, 6, 3)
    a, b, C = _coef(rng, 4, 6)
    y, st = oracle.hadamard_recurrent(q, k, v, a, b, C, return_state=True)
    y1, st1 = oracle.hadamard_recurrent(q[:, :, :11], k[:, :, :11], v[:, :, :11], a, b, C,
                                        return_state=True)
    y2, st2 = oracle.hadamard_recurrent(q[:, :, 11:], k[:, :, 11:], v[:, :, 11:], a, b, C,
                                        state=st1, return_state=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=2), y)
    np.testing.assert_array_equal(st2.H2, st.H2)


def test_bad_shapes_are_rejected():
    rng = np.random.default_rng(1)
    q, k, v = _problem(rng, 1, 3, 2, 4, 4, 2)  # Hq not a multiple of Hkv
    with pytest.raises(ValueError):
        oracle.hadamard_dense(q, k, v, np.ones(3), np.zeros((3, 4)), np.zeros((3, 4, 4)))
    q, k, v = _problem(rng, 1, 2, 1, 4, 4, 2)
    with pytest.raises(ValueError):
        oracle.hadamard_recurrent(q, k, v, np.ones(2), np.zeros((2, 3)), np.zeros((2, 4, 4)))
