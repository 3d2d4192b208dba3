"""Pins for the oracle's gradients of the dense grouped form (eqs. (2)-(3), summed over j <= i
and normalised): the backward pass that joint training of the kernel coefficients needs
("OAL: 按 QK 离群贡献分组的正二次注意力核", the pipeline figure: LoRA and kernel parameters
trained together).

The forward oracle is pinned elsewhere. The gradients are pinned against it here:
- central finite differences of the scalar loss sum(dy * yhat), for q, k, v, L and eps, with
  GQA and several groups;
- exact identities:
  * with kappa scaled as L -> cL, <dL, L> = -2 eps deps;
  * shifting every v by a constant c shifts every yhat by c, so sum_j dv_j = sum_i dy_i;
  * a constant kernel (L = 0) has dq = dk = dL = 0, deps = 0, and dv_j = sum_{i>=j} dy_i / (i+1).
"""
import numpy as np
import pytest

import oracle


def _problem(seed, B=2, Hq=4, Hkv=2, T=9, dh=6, dv=3, Gmax=3, eps=0.3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, T, dh))
    k = rng.standard_normal((B, Hkv, T, dh))
    v = rng.standard_normal((B, Hkv, T, dv))
    G = rng.integers(1, Gmax + 1, size=Hq).astype(np.int32)
    G[0] = Gmax
    gid = np.ones((Hq, dh), np.int32)
    L = np.zeros((Hq, Gmax + 1, Gmax + 1))
    for h in range(Hq):
        gid[h] = rng.integers(1, G[h] + 1, size=dh)
        gid[h, :G[h]] = np.arange(1, G[h] + 1)
        n = G[h] + 1
        L[h, :n, :n] = rng.standard_normal((n, n)) * 0.6 + np.eye(n)
    dy = rng.standard_normal((B, Hq, T, dv))
    return dict(q=q, k=k, v=v, group_id=gid, L=L, G=G, eps=eps), dy


def _loss(args, dy):
    return float(np.sum(dy * oracle.dense(**args)))


def _fd(args, dy, name, idx, h=1e-6):
    plus, minus = dict(args), dict(args)
    if name == "eps":
        plus["eps"], minus["eps"] = args["eps"] + h, args["eps"] - h
    else:
        a_p, a_m = args[name].copy(), args[name].copy()
        a_p[idx] += h
        a_m[idx] -= h
        plus[name], minus[name] = a_p, a_m
    return (_loss(plus, dy) - _loss(minus, dy)) / (2 * h)


@pytest.mark.parametrize("seed", [0, 1])
def test_finite_differences(seed):
    args, dy = _problem(seed)
    g = oracle.dense_backward(dy=dy, **args)
    rng = np.random.default_rng(100 + seed)
    checks = []
    for name, grad in (("q", g["dq"]), ("k", g["dk"]), ("v", g["dv"])):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in args[name].shape)
            checks.append((name, idx, grad[idx]))
    for h in range(args["L"].shape[0]):  # every live entry of L for every head
        n = int(args["G"][h]) + 1
        for a in range(n):
            for m in range(n):
                checks.append(("L", (h, a, m), g["dL"][h, a, m]))
    checks.append(("eps", None, g["deps"]))
    for name, idx, analytic in checks:
        numeric = _fd(args, dy, name, idx)
        assert abs(analytic - numeric) <= 1e-6 * max(1.0, abs(numeric)), (name, idx, analytic,
                                                                          numeric)


def test_entries_outside_each_heads_block_are_zero():
    args, dy = _problem(2)
    dL = oracle.dense_backward(dy=dy, **args)["dL"]
    for h in range(dL.shape[0]):
        n = int(args["G"][h]) + 1
        mask = np.ones(dL.shape[1:], bool)
        mask[:n, :n] = False
        assert np.all(dL[h][mask] == 0.0)


def test_scaling_identity():
    """kappa(cL) = eps + c^2 (kappa - eps) and sum_j dkappa_ij kappa_ij = 0 for every row
    (yhat is a kappa-weighted mean), so d/dc of the loss at c = 1 is -2 eps deps."""
    for eps in (0.0, 0.3, 2.0):
        args, dy = _problem(3, eps=eps)
        g = oracle.dense_backward(dy=dy, **args)
        lhs = float(np.sum(g["dL"] * args["L"]))
        assert abs(lhs + 2 * eps * g["deps"]) <= 1e-10 * max(1.0, np.abs(g["dL"]).max())


def test_value_shift_identity():
    """yhat_i(v + c) = yhat_i(v) + c, so the v-gradient summed over tokens equals the sum of
    dy over tokens and over the query heads of the group."""
    args, dy = _problem(4)
    g = oracle.dense_backward(dy=dy, **args)
    B, Hq, T, dv = dy.shape
    Hkv = args["k"].shape[1]
    per_kv = dy.reshape(B, Hkv, Hq // Hkv, T, dv).sum(axis=(2, 3))
    np.testing.assert_allclose(g["dv"].sum(axis=2), per_kv, rtol=1e-10, atol=1e-12)


def test_constant_kernel():
    """L = 0 leaves kappa = eps: yhat is the running mean of v, and only v has a gradient."""
    args, dy = _problem(5)
    args["L"][:] = 0.0
    g = oracle.dense_backward(dy=dy, **args)
    assert np.all(g["dq"] == 0) and np.all(g["dk"] == 0) and np.all(g["dL"] == 0)
    assert abs(g["deps"]) < 1e-12
    B, Hq, T, dv = dy.shape
    Hkv = args["k"].shape[1]
    w = dy / np.arange(1, T + 1)[None, None, :, None]
    tail = np.flip(np.cumsum(np.flip(w, axis=2), axis=2), axis=2)  # sum_{i>=j} dy_i / (i+1)
    ref = tail.reshape(B, Hkv, Hq // Hkv, T, dv).sum(axis=2)
    np.testing.assert_allclose(g["dv"], ref, rtol=1e-12, atol=1e-14)
