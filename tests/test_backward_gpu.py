"""GPU parity of the dense backward pass (oal_dense_backward_gpu) against the oracle's
gradients (oracle.dense_backward, pinned by finite differences and exact identities in
tests/test_oracle_backward_pins.py).  fp32 arithmetic on both input dtypes: each gradient
within 1e-4 of the oracle, relative to its largest entry, or to 1e-3 of the gradient's
natural scale when that is larger.

The floor matters only where a gradient vanishes in exact arithmetic.  At T = 1 the single
row attends to itself alone, so yhat_0 = v_0 and every dkappa = dy . (v_0 - yhat_0) / D is
zero: dq, dk and dL are exactly 0 (the oracle returns fp64 rounding, ~1e-18) and the fp32
kernel returns fp32 rounding of the same cancellation (~1e-9).  A relative error against
~1e-18 is meaningless there.  The natural scale of a gradient is the product of the
magnitudes its chain-rule terms multiply: max|dy| max|v| max|q|,|k| for dq and dk (dkappa
carries dy (v - yhat), dkappa/dq carries k), max|dy| for dv, max|dy| max|v| max|L| for dL."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests.test_gpu_parity import dev_inputs, oal  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _rel(a, b, scale=0.0):
    """max |a - b| over max(max |b|, 1e-3 * scale)."""
    den = max(float(np.abs(b).max()), 1e-3 * scale, 1e-30)
    return float(np.abs(np.asarray(a, np.float64) - b).max() / den)


def _natural_scales(p, dy):
    a = lambda x: float(np.abs(np.asarray(x, np.float64)).max()) if np.size(x) else 0.0  # noqa: E731
    qk = max(a(p.q), a(p.k))
    return {"dq": a(dy) * a(p.v) * qk, "dk": a(dy) * a(p.v) * qk, "dv": a(dy),
            "dL": a(dy) * a(p.v) * a(p.L)}


@pytest.mark.parametrize("dtype,B,T,Hq,Hkv", [("f32", 2, 70, 4, 2), ("bf16", 1, 131, 8, 1),
                                              ("f32", 1, 1, 2, 2)])
def test_dense_backward_matches_oracle(oal, cuda, dtype, B, T, Hq, Hkv):
    p = I.small_layer(700 + T, B=B, T=T, Hq=Hq, Hkv=Hkv, dtype=dtype)
    rng = np.random.default_rng(T)
    dy = rng.standard_normal((B, Hq, T, 64))
    ref = oracle.dense_backward(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, dy)
    q, k, v, g, L, G = dev_inputs(p, cuda)
    got = oal.dense_backward(q, k, v, g, L, G, p.eps, torch.from_numpy(dy).float())
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    scale = _natural_scales(p, dy)
    for name in ("dq", "dk", "dv", "dL"):
        assert _rel(got[name].cpu().numpy(), ref[name], scale[name]) <= 1e-4, name
    dL = got["dL"].cpu().numpy()
    for h in range(Hq):  # zero outside each head's live block
        n = int(p.G[h]) + 1
        mask = np.ones(dL.shape[1:], bool)
        mask[:n, :n] = False
        assert np.all(dL[h][mask] == 0.0)
    assert abs(float(got["deps"]) - ref["deps"]) <= 1e-4 * max(1.0, abs(ref["deps"]))


def test_dense_backward_is_reproducible(oal, cuda):
    """Every output is summed in a fixed order: two calls agree bit for bit."""
    p = I.small_layer(790, B=1, T=90, Hq=4, Hkv=2, dtype="bf16")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    dy = torch.randn(1, 4, 90, 64, generator=torch.Generator().manual_seed(3))
    a = oal.dense_backward(q, k, v, g, L, G, p.eps, dy)
    b = oal.dense_backward(q, k, v, g, L, G, p.eps, dy)
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dL", "deps"):
        assert torch.equal(a[name], b[name]), name


# ---- the training-scale (chunked) backward: oal_backward ---------------------------------

@pytest.mark.parametrize("dtype,B,T,Hq,Hkv", [("f32", 2, 70, 4, 2), ("bf16", 1, 131, 8, 1),
                                              ("f32", 1, 1, 2, 2), ("f32", 1, 64, 2, 1),
                                              ("f32", 1, 65, 2, 1), ("bf16", 1, 300, 7, 1)])
def test_chunked_backward_matches_oracle(oal, cuda, dtype, B, T, Hq, Hkv):
    """Chunk boundaries at 64 tokens: one partial chunk, exactly one chunk, a one-token
    second chunk, several chunks; GQA up to 8 query heads per kv head."""
    p = I.small_layer(800 + T, B=B, T=T, Hq=Hq, Hkv=Hkv, dtype=dtype)
    rng = np.random.default_rng(T + 1)
    dy = rng.standard_normal((B, Hq, T, 64))
    ref = oracle.dense_backward(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, dy)
    q, k, v, g, L, G = dev_inputs(p, cuda)
    got = oal.backward(q, k, v, g, L, G, p.eps, torch.from_numpy(dy).float())
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    scale = _natural_scales(p, dy)
    for name in ("dq", "dk", "dv", "dL"):
        assert _rel(got[name].cpu().numpy(), ref[name], scale[name]) <= 1e-4, name
    assert abs(float(got["deps"]) - ref["deps"]) <= 1e-4 * max(1.0, abs(ref["deps"]))


def test_chunked_backward_matches_dense_gpu(oal, cuda):
    """Against the dense GPU gradient (independent pair sums) on a longer sequence."""
    p = I.small_layer(820, B=1, T=700, Hq=14, Hkv=2, dtype="bf16")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    dy = torch.randn(1, 14, 700, 64, generator=torch.Generator().manual_seed(5))
    a = oal.backward(q, k, v, g, L, G, p.eps, dy)
    b = oal.dense_backward(q, k, v, g, L, G, p.eps, dy)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    for name in ("dq", "dk", "dv", "dL"):
        x, y = a[name].double(), b[name].double()
        assert float((x - y).abs().max() / y.abs().max()) <= 1e-4, name
    assert abs(float(a["deps"]) - float(b["deps"])) <= 1e-4 * max(1.0, abs(float(b["deps"])))


def test_chunked_backward_full_layer_identities(oal, cuda):
    """A Qwen2.5-0.5B-shaped layer (B=1, T=4096, 14/2 heads, bf16) at training scale: the
    gradients are reproducible bit for bit and satisfy identities that hold at any size --
    <dL, L> = -2 eps deps (kappa(cL) = eps + c^2 (kappa - eps), and yhat is a kappa-weighted
    mean) and sum_j dv_j = sum over tokens and group heads of dy (yhat(v + c) = yhat(v) + c)."""
    p = I.config1()
    q, k, v, g, L, G = dev_inputs(p, cuda)
    dy = torch.randn(1, 14, 4096, 64, generator=torch.Generator().manual_seed(6))
    ws = oal.backward_workspace(q, k, v)
    a = oal.backward(q, k, v, g, L, G, p.eps, dy, workspace=ws)
    b = oal.backward(q, k, v, g, L, G, p.eps, dy, workspace=ws)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    for name in ("dq", "dk", "dv", "dL", "deps"):
        assert torch.equal(a[name], b[name]), name
        assert bool(torch.isfinite(a[name]).all()), name
    lhs = float((a["dL"].double() * L.double()).sum())
    assert abs(lhs + 2 * p.eps * float(a["deps"])) <= 1e-3 * float(a["dL"].abs().max())
    per_kv = dy.double().reshape(1, 2, 7, 4096, 64).sum(dim=(2, 3))
    got = a["dv"].double().cpu().sum(dim=2)
    assert float((got - per_kv).abs().max()) <= 1e-3 * float(per_kv.abs().max())
