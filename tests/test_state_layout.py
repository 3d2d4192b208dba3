"""The state layout that include/oal.h documents, checked against the oracle on the CPU.

A saved state is meant to be read by other programs, so its documented contents must be
right on their own: the packed rows (the pairs r <= t of [k; 1] in the stated order) filled
from the oracle's H0/H1/H2, weighted by the stated coefficients and contracted with the
query's packed products, give eq. (5)'s u of the last token, whose ratio is the oracle's
output of that token."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._packed import F, coef_from_header, pack_oracle_state, packed_pairs


@pytest.mark.parametrize("seed,B,T,Hq,Hkv", [(21, 2, 37, 4, 2), (22, 1, 9, 14, 2),
                                             (23, 1, 64, 8, 1)])
def test_documented_state_reads_out_the_last_token(seed, B, T, Hq, Hkv):
    p = I.small_layer(seed, B=B, T=T, Hq=Hq, Hkv=Hkv, dtype="f32")
    y, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    S = pack_oracle_state(st)                       # [B, Hkv, F, 65]
    coef = coef_from_header(p.group_id, p.L, p.G, p.eps)
    pairs = packed_pairs()
    r, t = pairs[:, 0], pairs[:, 1]
    grp = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            qhat = np.concatenate([p.q[b, h, T - 1].astype(np.float64), [1.0]])
            phi = coef[h, :F] * qhat[r] * qhat[t]
            u = phi @ S[b, h // grp]                 # eq. (5), inclusive of the last token
            np.testing.assert_allclose(u[:64] / u[64], y[b, h, T - 1], rtol=1e-9, atol=1e-12)


def test_coefficient_rows_by_hand():
    """Three rows of the documented table written out by hand for one head: a cross term
    inside the bulk group, a linear row of an outlier dimension and the constant row."""
    p = I.small_layer(24, B=1, T=4, Hq=2, Hkv=1, dtype="f32")
    coef = coef_from_header(p.group_id, p.L, p.G, p.eps)
    pairs = [tuple(x) for x in packed_pairs().tolist()]
    h = 0
    Gh = int(p.G[h])
    M = p.L[h, :Gh + 1, :Gh + 1].astype(np.float64) @ p.L[h, :Gh + 1, :Gh + 1].T
    bulk = [r for r in range(64) if p.group_id[h, r] == 1]
    out = [r for r in range(64) if p.group_id[h, r] != 1][0]
    a, c = bulk[0], bulk[1]
    assert coef[h, pairs.index((a, c))] == pytest.approx(2 * M[1, 1] / 64)
    g = int(p.group_id[h, out])
    assert coef[h, pairs.index((out, 64))] == pytest.approx(2 * M[g, 0] / 8)
    assert coef[h, pairs.index((64, 64))] == pytest.approx(M[0, 0] + p.eps)


def test_hadamard_state_reads_out_with_its_coefficients():
    """The state of the Hadamard form has the same packed rows; its readout weights follow
    from kappa = a + b.x + x^T C x with x_r = q_r k_r / 8: a on the constant row, b_r / 8 on
    the linear row of r, (C_rt + C_tr) / 64 on a cross row r < t and C_rr / 64 on a square."""
    rng = np.random.default_rng(25)
    p = I.small_layer(25, B=1, T=21, Hq=4, Hkv=2, dtype="f32")
    Hq = 4
    a = rng.uniform(1.0, 2.0, Hq)
    b = rng.normal(0.0, 0.5, (Hq, 64))
    C = rng.normal(0.0, 0.2, (Hq, 64, 64))
    y, st = oracle.hadamard_recurrent(p.q, p.k, p.v, a, b, C, return_state=True)
    S = pack_oracle_state(st)
    pairs = packed_pairs()
    r, t = pairs[:, 0], pairs[:, 1]
    T = p.q.shape[2]
    for h in range(Hq):
        cr = np.where(t == 64, 0, np.minimum(r, 63))
        ct = np.minimum(t, 63)
        coef = np.where(r == t, C[h, cr, ct], C[h, cr, ct] + C[h, ct, cr]) / 64.0
        coef = np.where(t == 64, b[h, np.minimum(r, 63)] / 8.0, coef)
        coef = np.where((r == 64) & (t == 64), a[h], coef)
        qhat = np.concatenate([p.q[0, h, T - 1].astype(np.float64), [1.0]])
        u = (coef * qhat[r] * qhat[t]) @ S[0, h // 2]
        np.testing.assert_allclose(u[:64] / u[64], y[0, h, T - 1], rtol=1e-9, atol=1e-12)
