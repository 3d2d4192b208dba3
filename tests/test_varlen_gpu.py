"""GPU parity of the variable-length batch (oal_prefill_varlen): every sequence of a packed
batch equals an oal_prefill of that sequence alone, bit for bit (the same kernels run on the
same block), outputs and state; and matches the oracle.  Several streams, an empty sequence,
ragged lengths."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, TOL_F32, row_rel_err
from tests.test_gpu_parity import oal  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("dtype,chunk,lens,nstreams", [("bf16", 128, [300, 0, 129, 1000], 2),
                                                       ("f32", 64, [64, 77, 5], 1),
                                                       ("bf16", 256, [200, 31], 3)])
def test_varlen_equals_separate_prefills(oal, cuda, dtype, chunk, lens, nstreams):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    base = I.small_layer(600 + sum(lens), B=1, T=1, Hq=4, Hkv=2, dtype=dtype)
    g, L, G = (torch.from_numpy(x).to(cuda) for x in (base.group_id, base.L, base.G))
    probs = [I.small_layer(610 + i, B=1, T=t, Hq=4, Hkv=2, dtype=dtype) for i, t in
             enumerate(lens)]
    for pr in probs:  # one layer: the same groups and L for every sequence
        pr.group_id, pr.L, pr.G = base.group_id, base.L, base.G
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda, dt)  # noqa: E731
    qs = [t(pr.q[0]) for pr in probs]
    ks = [t(pr.k[0]) for pr in probs]
    vs = [t(pr.v[0]) for pr in probs]
    streams = [torch.cuda.Stream(device=cuda) for _ in range(nstreams)]
    outs, states = oal.prefill_varlen(qs, ks, vs, g, L, G, base.eps, chunk, streams=streams)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    for i, pr in enumerate(probs):
        y1, st1 = oal.prefill(qs[i][None], ks[i][None], vs[i][None], g, L, G, base.eps, chunk)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], y1[0])
        assert torch.equal(states[i, :44], st1[:44])
        assert torch.equal(states[i, 256:st1.numel()], st1[256:])
        if lens[i]:
            ref = oracle.recurrent(pr.q, pr.k, pr.v, pr.group_id, pr.L, pr.G, pr.eps)
            tol = TOL_BF16 if dtype == "bf16" else TOL_F32
            assert row_rel_err(outs[i].cpu().numpy()[None], ref) <= tol
