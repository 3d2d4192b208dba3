"""GPU parity on further shapes and degenerate cases, against the fp64 oracle: group counts
G = 1 and 8 on both bf16 prefill paths, a constant kernel (L = e0 e0^T, whose output is the
running mean of v) through prefill and decode, and decode for every query-heads-per-kv-head
count the decode kernel is specialised on.  Same tolerances as tests/test_gpu_parity.py."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, TOL_F32, row_rel_err
from tests._packed import F, pack_oracle_state, read_state
from tests.test_gpu_parity import dev_inputs, gpu_prefill, oal, tol  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("chunk", [128, 64])
def test_group_count_extremes_bf16(oal, cuda, chunk):
    """G = 1 and G = 8 (two and nine score tiles) on the bf16 paths: tensor cores at chunk
    128, CUDA cores at chunk 64; GQA 8/2."""
    rng = np.random.default_rng(6)
    p = I.small_layer(305, B=2, T=333, Hq=8, Hkv=2, dtype="bf16")
    for h in range(8):
        Gh = 1 if h % 2 == 0 else 8
        p.G[h] = Gh
        p.group_id[h] = rng.integers(1, Gh + 1, size=64)
        p.group_id[h, :Gh] = np.arange(1, Gh + 1)
        p.L[h] = I.random_L(rng, Gh)
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    y, _ = gpu_prefill(oal, p, cuda, chunk)
    assert row_rel_err(y, ref) <= TOL_BF16


@pytest.mark.parametrize("dtype,chunk", [("bf16", 128), ("f32", 64)])
def test_constant_kernel_is_running_mean(oal, cuda, dtype, chunk):
    """L = e0 e0^T leaves kappa = eps + 1 for every pair, so yhat is the inclusive running
    mean of v (eqs. (3) and (5)); then one decode step extends the mean."""
    p = I.small_layer(306, B=1, T=261, Hq=4, Hkv=2, dtype=dtype)
    p.L[:] = 0.0
    p.L[:, 0, 0] = 1.0
    T = 260
    q, k, v, g, L, G = dev_inputs(p, cuda)
    y, state = oal.prefill(q[:, :, :T].contiguous(), k[:, :, :T].contiguous(),
                           v[:, :, :T].contiguous(), g, L, G, p.eps, chunk)
    ws = oal.decode_workspace(1, 4, 2, cuda)
    y1 = oal.decode_step(q[:, :, T:].contiguous(), k[:, :, T:].contiguous(),
                         v[:, :, T:].contiguous(), state, ws)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    vv = np.repeat(p.v.astype(np.float64), 2, axis=1)  # query head h reads kv head h // 2
    mean = np.cumsum(vv, axis=2) / np.arange(1, T + 2)[None, None, :, None]
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    assert row_rel_err(y.cpu().numpy(), mean[:, :, :T]) <= tol
    assert row_rel_err(y1.cpu().numpy()[:, :, 0], mean[:, :, T]) <= tol


@pytest.mark.parametrize("Hq,Hkv,dtype", [(2, 2, "bf16"), (6, 2, "bf16"), (5, 1, "bf16"),
                                           (8, 1, "bf16"), (8, 1, "f32")])
def test_decode_group_sizes(oal, cuda, Hq, Hkv, dtype):
    """Decode for every query-heads-per-kv-head count the kernel is specialised on that the
    Qwen shape does not reach (1, 3, 5, 8): three steps after a ragged prefill."""
    B, T0, n = 2, 150, 3
    p = I.small_layer(320 + 10 * Hq + Hkv, B=B, T=T0 + n, Hq=Hq, Hkv=Hkv, dtype=dtype)
    y_all, st_all = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps,
                                     return_state=True)
    _, state = gpu_prefill(oal, p.slice_tokens(0, T0), cuda, 128)
    ws = oal.decode_workspace(B, Hq, Hkv, cuda)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    for t in range(T0, T0 + n):
        sl = lambda x: x[:, :, t:t + 1].contiguous()  # noqa: E731
        y = oal.decode_step(sl(q), sl(k), sl(v), state, ws)
        torch.cuda.synchronize()
        assert row_rel_err(y.cpu().numpy()[:, :, 0], y_all[:, :, t]) <= tol(p)
    assert oal.device_error() == 0
    hdr, _, S = read_state(state.cpu().numpy(), B, Hq, Hkv)
    assert hdr["tokens"] == T0 + n
    ref = pack_oracle_state(st_all)
    assert np.max(np.abs(S[:, :, :F] - ref) / np.abs(ref).max(axis=2, keepdims=True)) < 1e-5


def test_decode_step_in_a_cuda_graph(oal, cuda):
    """A decode step captured once in a CUDA graph and replayed token after token (new
    inputs copied into the captured buffers) continues the sequence like eager calls."""
    B, Hq, Hkv, T0, n = 2, 14, 2, 140, 4
    p = I.small_layer(330, B=B, T=T0 + n, Hq=Hq, Hkv=Hkv, dtype="bf16")
    y_all = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    _, state = gpu_prefill(oal, p.slice_tokens(0, T0), cuda, 128)
    ws = oal.decode_workspace(B, Hq, Hkv, cuda)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    sq = q[:, :, T0:T0 + 1].clone()
    sk = k[:, :, T0:T0 + 1].clone()
    sv = v[:, :, T0:T0 + 1].clone()
    out = torch.empty(B, Hq, 1, 64, dtype=torch.float32, device=cuda)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        oal.decode_step(sq, sk, sv, state, ws, out=out)
    # capturing does not run the step: the state still holds T0 tokens
    for t in range(T0, T0 + n):
        sq.copy_(q[:, :, t:t + 1])
        sk.copy_(k[:, :, t:t + 1])
        sv.copy_(v[:, :, t:t + 1])
        graph.replay()
        torch.cuda.synchronize()
        assert row_rel_err(out.cpu().numpy()[:, :, 0], y_all[:, :, t]) <= TOL_BF16
    assert oal.device_error() == 0
    hdr, _, _ = read_state(state.cpu().numpy(), B, Hq, Hkv)
    assert hdr["tokens"] == T0 + n
