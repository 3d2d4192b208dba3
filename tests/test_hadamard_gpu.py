"""GPU parity of the ungrouped Hadamard form (oal_prefill_hadamard, oal_dense_hadamard_gpu):
eq. (5) of "OAL: 按 QK 离群贡献分组的正二次注意力核" (section 核心公式) with free a, b_r, C_rt,
the relaxation the abstract of arXiv 2610.13674 describes.  The oracle is
oracle.hadamard_recurrent / hadamard_dense (pinned in tests/test_oracle_hadamard_pins.py).
bf16 inputs with chunk 128 run on tensor cores (bf16 operands, fp32 accumulation: the bf16
tolerance); every other case computes in fp32 on CUDA cores (the fp32 tolerance)."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, TOL_F32, row_rel_err
from tests.test_gpu_parity import dev_inputs, oal  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _coefs(seed, Hq, d=64):
    """a in [2, 3), |b| small, C = W W^T / d + I/2 plus an antisymmetric part: the kernel
    is bounded below by a - |b|^2 / 2 > 0, so the normalisers stay well away from zero."""
    rng = np.random.default_rng(seed)
    a = 2.0 + rng.random(Hq)
    b = 0.1 * rng.standard_normal((Hq, d))
    W = rng.standard_normal((Hq, d, d))
    A = 0.2 * rng.standard_normal((Hq, d, d))
    C = W @ W.transpose(0, 2, 1) / d + 0.5 * np.eye(d) + (A - A.transpose(0, 2, 1))
    return a.astype(np.float32), b.astype(np.float32), C.astype(np.float32)


def _t(x, dev):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev)


def _tol(oal, p, chunk):
    shape = oal.make_shape(p.q.shape[0], p.q.shape[2], p.q.shape[1], p.k.shape[1], chunk,
                           oal.OAL_BF16 if p.dtype == "bf16" else oal.OAL_F32)
    return TOL_BF16 if oal.prefill_path(shape) == oal.OAL_PATH_TENSOR else TOL_F32


@pytest.mark.parametrize("dtype,chunk", [("f32", 64), ("f32", 128), ("bf16", 64),
                                         ("bf16", 128), ("bf16", 256)])
def test_prefill_hadamard_matches_oracle(oal, cuda, dtype, chunk):
    p = I.small_layer(500 + chunk, B=2, T=301, Hq=4, Hkv=2, dtype=dtype)
    a, b, C = _coefs(7, 4)
    ref = oracle.hadamard_recurrent(p.q, p.k, p.v, a, b, C)
    q, k, v, *_ = dev_inputs(p, cuda)
    y, _ = oal.prefill_hadamard(q, k, v, _t(a, cuda), _t(b, cuda), _t(C, cuda), chunk)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert row_rel_err(y.cpu().numpy(), ref) <= _tol(oal, p, chunk)


@pytest.mark.parametrize("T", [1, 127, 128, 129, 640])
def test_tensor_hadamard_edges(oal, cuda, T):
    """Tensor-core path at a single token, one partial and one full chunk, a one-token second
    chunk and five chunks; GQA 7 query heads per kv head."""
    p = I.small_layer(520 + T, B=1, T=T, Hq=7, Hkv=1, dtype="bf16")
    a, b, C = _coefs(11, 7)
    ref = oracle.hadamard_recurrent(p.q, p.k, p.v, a, b, C)
    q, k, v, *_ = dev_inputs(p, cuda)
    y, _ = oal.prefill_hadamard(q, k, v, _t(a, cuda), _t(b, cuda), _t(C, cuda), 128)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert row_rel_err(y.cpu().numpy(), ref) <= TOL_BF16


def test_tensor_hadamard_full_layer(oal, cuda):
    """A Qwen2.5-0.5B-shaped layer (B=1, T=4096, 14 query / 2 kv heads), every row against
    the oracle's recurrence."""
    p = I.small_layer(530, B=1, T=4096, Hq=14, Hkv=2, dtype="bf16")
    a, b, C = _coefs(12, 14)
    ref = oracle.hadamard_recurrent(p.q, p.k, p.v, a, b, C)
    q, k, v, *_ = dev_inputs(p, cuda)
    y, _ = oal.prefill_hadamard(q, k, v, _t(a, cuda), _t(b, cuda), _t(C, cuda), 128)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert row_rel_err(y.cpu().numpy(), ref) <= TOL_BF16


def test_tensor_hadamard_state_matches_cuda_core_state(oal, cuda):
    """Both paths leave the same coefficient table (bit for bit: one prep kernel) and the same
    fp32 prefix state (the chunk deltas are exact on both; only the summation order differs)."""
    p = I.small_layer(531, B=2, T=700, Hq=4, Hkv=2, dtype="bf16")
    a, b, C = _coefs(13, 4)
    q, k, v, *_ = dev_inputs(p, cuda)
    ta, tb, tC = _t(a, cuda), _t(b, cuda), _t(C, cuda)
    _, s_tc = oal.prefill_hadamard(q, k, v, ta, tb, tC, 128)
    _, s_cc = oal.prefill_hadamard(q, k, v, ta, tb, tC, 64)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    head = 256 + ((4 * 2176 * 4 + 255) // 256) * 256
    assert torch.equal(s_tc[:head], s_cc[:head])
    x = s_tc[head:].view(torch.float32).double()
    y = s_cc[head:].view(torch.float32).double()
    assert float((x - y).abs().max() / y.abs().max()) <= 1e-5


def test_dense_hadamard_matches_oracle(oal, cuda):
    p = I.small_layer(510, B=1, T=150, Hq=4, Hkv=1, dtype="f32")
    a, b, C = _coefs(8, 4)
    ref = oracle.hadamard_dense(p.q, p.k, p.v, a, b, C)
    q, k, v, *_ = dev_inputs(p, cuda)
    y = oal.dense_hadamard(q, k, v, _t(a, cuda), _t(b, cuda), _t(C, cuda))
    torch.cuda.synchronize()
    assert row_rel_err(y.cpu().numpy(), ref) <= TOL_F32


def test_grouped_coefficients_reproduce_grouped_prefill(oal, cuda):
    """Expanding the grouped kernel into (a, b, C) gives the grouped prefill's output."""
    p = I.small_layer(511, B=1, T=260, Hq=4, Hkv=2, dtype="f32")
    a, b, C = (x.astype(np.float32) for x in oracle.grouped_coefficients(p.group_id, p.L, p.G,
                                                                         p.eps))
    q, k, v, g, L, G = dev_inputs(p, cuda)
    yg, _ = oal.prefill(q, k, v, g, L, G, p.eps, 64)
    yh, _ = oal.prefill_hadamard(q, k, v, _t(a, cuda), _t(b, cuda), _t(C, cuda), 64)
    torch.cuda.synchronize()
    assert row_rel_err(yh.cpu().numpy(), yg.cpu().numpy().astype(np.float64)) <= TOL_F32


def test_decode_continues_a_hadamard_prefill(oal, cuda):
    """The decode step reads only the packed coefficients and state, so it continues a
    sequence prefilled with the Hadamard form."""
    T0, n = 190, 3
    p = I.small_layer(512, B=2, T=T0 + n, Hq=4, Hkv=2, dtype="bf16")
    a, b, C = _coefs(9, 4)
    ref = oracle.hadamard_recurrent(p.q, p.k, p.v, a, b, C)
    q, k, v, *_ = dev_inputs(p, cuda)
    sl = lambda x, t0, t1: x[:, :, t0:t1].contiguous()  # noqa: E731
    _, state = oal.prefill_hadamard(sl(q, 0, T0), sl(k, 0, T0), sl(v, 0, T0), _t(a, cuda),
                                    _t(b, cuda), _t(C, cuda), 128)
    ws = oal.decode_workspace(2, 4, 2, cuda)
    for t in range(T0, T0 + n):
        y = oal.decode_step(sl(q, t, t + 1), sl(k, t, t + 1), sl(v, t, t + 1), state, ws)
        torch.cuda.synchronize()
        assert row_rel_err(y.cpu().numpy()[:, :, 0], ref[:, :, t]) <= TOL_F32
    assert oal.device_error() == 0


def test_negative_constant_kernel_is_running_mean(oal, cuda):
    """a = -1, b = 0, C = 0: every kernel value is -1 and every normaliser -(i + 1), so yhat
    is still the running mean of v."""
    T = 200
    p = I.small_layer(513, B=1, T=T, Hq=2, Hkv=1, dtype="f32")
    q, k, v, *_ = dev_inputs(p, cuda)
    a = torch.full((2,), -1.0, device=cuda)
    b = torch.zeros(2, 64, device=cuda)
    C = torch.zeros(2, 64, 64, device=cuda)
    y, _ = oal.prefill_hadamard(q, k, v, a, b, C, 64)
    torch.cuda.synchronize()
    vv = np.repeat(p.v.astype(np.float64), 2, axis=1)
    mean = np.cumsum(vv, axis=2) / np.arange(1, T + 1)[None, None, :, None]
    assert row_rel_err(y.cpu().numpy(), mean) <= TOL_F32
