"""Property-based checks of the oracle over random small problems (hypothesis): the two
evaluation routes of each form agree, chunking a recurrence through its state changes nothing,
and the gradients agree with finite differences in a random direction.  Sizes stay tiny so the
whole file runs in seconds."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

GMAX = 8


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    Hkv = draw(st.integers(1, 2))
    grp = draw(st.integers(1, 3))
    Hq = Hkv * grp
    T = draw(st.integers(1, 12))
    d = draw(st.sampled_from([4, 8, 16]))
    dv = draw(st.integers(1, 5))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    G = rng.integers(1, min(GMAX, d) + 1, size=Hq).astype(np.int32)
    gid = np.zeros((Hq, d), np.int32)
    L = np.zeros((Hq, GMAX + 1, GMAX + 1))
    for h in range(Hq):
        gid[h] = rng.integers(1, G[h] + 1, size=d)
        gid[h, :G[h]] = np.arange(1, G[h] + 1)
        n = G[h] + 1
        L[h, :n, :n] = rng.standard_normal((n, n)) * 0.5
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, dv))
    eps = float(rng.uniform(0.05, 1.0))
    return dict(q=q, k=k, v=v, group_id=gid, L=L, G=G, eps=eps), rng


@settings(max_examples=40, deadline=None)
@given(problems())
def test_grouped_dense_equals_recurrent(pr):
    args, _ = pr
    yd = oracle.dense(**args)
    yr = oracle.recurrent(**args)
    assert np.max(np.abs(yd - yr)) <= 1e-9 * max(1.0, np.abs(yd).max())


@settings(max_examples=40, deadline=None)
@given(problems(), st.integers(0, 11))
def test_recurrence_split_anywhere(pr, cut):
    args, _ = pr
    T = args["q"].shape[2]
    cut = min(cut, T)
    y, st_all = oracle.recurrent(**args, return_state=True)
    a = {**args, "q": args["q"][:, :, :cut], "k": args["k"][:, :, :cut],
         "v": args["v"][:, :, :cut]}
    b = {**args, "q": args["q"][:, :, cut:], "k": args["k"][:, :, cut:],
         "v": args["v"][:, :, cut:]}
    ya, sa = oracle.recurrent(**a, return_state=True)
    yb, sb = oracle.recurrent(**b, state=sa, return_state=True)
    np.testing.assert_array_equal(np.concatenate([ya, yb], axis=2), y)
    np.testing.assert_array_equal(sb.H2, st_all.H2)


@settings(max_examples=30, deadline=None)
@given(problems())
def test_hadamard_routes_agree(pr):
    args, rng = pr
    Hq, d = args["q"].shape[1], args["q"].shape[3]
    a = 2.0 + rng.random(Hq)
    b = 0.2 * rng.standard_normal((Hq, d))
    C = rng.standard_normal((Hq, d, d)) * 0.3
    _, ud = oracle.hadamard_dense(args["q"], args["k"], args["v"], a, b, C, return_u=True)
    _, ur = oracle.hadamard_recurrent(args["q"], args["k"], args["v"], a, b, C, return_u=True)
    assert np.max(np.abs(ud - ur)) <= 1e-9 * max(1.0, np.abs(ud).max())


@settings(max_examples=25, deadline=None)
@given(problems())
def test_backward_directional_derivative(pr):
    """<grad, direction> equals the central difference of the loss along that direction."""
    args, rng = pr
    dy = rng.standard_normal(args["q"].shape[:3] + (args["v"].shape[3],))
    g = oracle.dense_backward(dy=dy, **args)
    dirs = {n: rng.standard_normal(args[n].shape) for n in ("q", "k", "v")}
    dirL = np.zeros_like(args["L"])
    for h, Gh in enumerate(args["G"]):
        dirL[h, :Gh + 1, :Gh + 1] = rng.standard_normal((Gh + 1, Gh + 1))
    de = float(rng.standard_normal())
    analytic = (sum(float(np.sum(g["d" + n] * dirs[n])) for n in ("q", "k", "v"))
                + float(np.sum(g["dL"] * dirL)) + g["deps"] * de)
    h = 1e-6

    def loss(s):
        moved = {**args, "q": args["q"] + s * dirs["q"], "k": args["k"] + s * dirs["k"],
                 "v": args["v"] + s * dirs["v"], "L": args["L"] + s * dirL,
                 "eps": args["eps"] + s * de}
        return float(np.sum(dy * oracle.dense(**moved)))

    numeric = (loss(h) - loss(-h)) / (2 * h)
    assert abs(analytic - numeric) <= 1e-5 * max(1.0, abs(numeric))
