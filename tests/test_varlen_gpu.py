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


def _layer_batch(cuda, lens, Hq, Hkv, seed):
    base = I.small_layer(seed, B=1, T=1, Hq=Hq, Hkv=Hkv, dtype="bf16")
    g, L, G = (torch.from_numpy(x).to(cuda) for x in (base.group_id, base.L, base.G))
    probs = [I.small_layer(seed + 1 + i, B=1, T=t, Hq=Hq, Hkv=Hkv, dtype="bf16")
             for i, t in enumerate(lens)]
    for pr in probs:  # one layer: the same groups and L for every sequence
        pr.group_id, pr.L, pr.G = base.group_id, base.L, base.G
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda, torch.bfloat16)  # noqa: E731
    qs = [t(pr.q[0]) for pr in probs]
    ks = [t(pr.k[0]) for pr in probs]
    vs = [t(pr.v[0]) for pr in probs]
    return base, g, L, G, probs, qs, ks, vs


def _short64():
    """64 lengths of 64..320 tokens (the bench's short-sequence batch)."""
    rng = np.random.default_rng(902)
    rng.integers(64, 2049, size=16)
    return [int(x) for x in rng.integers(64, 321, size=64)]


_SHORT64 = _short64()


@pytest.mark.parametrize("lens,Hq,Hkv", [([300, 0, 129, 1000, 1, 128, 127, 640], 14, 2),
                                         ([5] * 40 + [700, 0, 0, 33], 4, 2),
                                         ([2048, 64, 1500], 8, 1),
                                         (_SHORT64, 14, 2)])
def test_packed_equals_separate_prefills(oal, cuda, lens, Hq, Hkv):
    """One launch per kernel for the whole batch gives each sequence exactly what an
    oal_prefill of it alone gives (same per-chunk arithmetic and summation order), outputs
    and state, and matches the oracle."""
    base, g, L, G, probs, qs, ks, vs = _layer_batch(cuda, lens, Hq, Hkv, 640 + len(lens))
    q, k, v, _ = oal.pack_sequences(qs, ks, vs)
    launches = oal.launch_count()
    out, states = oal.prefill_packed(q, k, v, lens, Hq, Hkv, g, L, G, base.eps)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert oal.launch_count() - launches <= 4  # deltas, intra-chunk, scan, readout
    off = 0
    for i, pr in enumerate(probs):
        T = lens[i]
        yi = out[off * Hq * 64:(off + T) * Hq * 64].view(Hq, T, 64)
        off += T
        y1, st1 = oal.prefill(qs[i][None], ks[i][None], vs[i][None], g, L, G, base.eps, 128)
        torch.cuda.synchronize()
        assert torch.equal(yi, y1[0]), i
        assert torch.equal(states[i, :44], st1[:44]), i
        assert torch.equal(states[i, 256:st1.numel()], st1[256:]), i
        if T and i % 3 == 0:
            ref = oracle.recurrent(pr.q, pr.k, pr.v, pr.group_id, pr.L, pr.G, pr.eps)
            assert row_rel_err(yi.cpu().numpy()[None], ref) <= TOL_BF16


def test_packed_empty_sequences(oal, cuda):
    """A batch of empty sequences: no kernel but the scan runs; every state is a valid empty
    state (header, coefficients, zero sums) that decode can continue."""
    lens = [0, 0, 0]
    base, g, L, G, probs, qs, ks, vs = _layer_batch(cuda, lens, 4, 2, 660)
    q, k, v, _ = oal.pack_sequences(qs, ks, vs)
    out, states = oal.prefill_packed(q, k, v, lens, 4, 2, g, L, G, base.eps)
    torch.cuda.synchronize()
    assert oal.device_error() == 0 and out.numel() == 0
    _, st1 = oal.prefill(qs[0][None], ks[0][None], vs[0][None], g, L, G, base.eps, 128)
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(states[i, :44], st1[:44])
        assert torch.equal(states[i, 256:st1.numel()], st1[256:])
