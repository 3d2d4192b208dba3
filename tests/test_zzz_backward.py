"""GPU parity of the dense backward pass (oal_dense_backward_gpu) against the oracle's
gradients (oracle.dense_backward, pinned by finite differences and exact identities in
tests/test_oracle_backward_pins.py).  fp32 arithmetic on both input dtypes: each gradient
within 1e-4 of the oracle, relative to its largest entry."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests.test_gpu_parity import dev_inputs, oal  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _rel(a, b):
    return float(np.abs(np.asarray(a, np.float64) - b).max() / max(np.abs(b).max(), 1e-30))


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
    for name in ("dq", "dk", "dv", "dL"):
        assert _rel(got[name].cpu().numpy(), ref[name]) <= 1e-4, name
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
