"""The allocation-free decode entry point (oal_decode_step_noalloc) against the regular one.

Callers that cannot allocate device memory (a serving engine that owns all GPU memory, a
plugin interface that passes only inputs and outputs) use oal_decode_step_noalloc, whose
scratch lives in a fixed array inside the library."""
import ctypes

import numpy as np
import pytest

from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, row_rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _noalloc_fn():
    from positive_quadratic_b200 import build, oal
    build.build()
    fn = oal.lib().oal_decode_step_noalloc
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.POINTER(oal.Shape), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return oal, fn


def test_noalloc_decode_matches_workspace_decode(cuda):
    oal, noalloc = _noalloc_fn()
    T0 = 130
    p = I.small_layer(400, B=4, T=T0 + 2, Hq=14, Hkv=2, dtype="bf16")
    dt = torch.bfloat16
    q, k, v = (torch.from_numpy(x).to(cuda, dt) for x in (p.q, p.k, p.v))
    g, L, G = (torch.from_numpy(x).to(cuda) for x in (p.group_id, p.L, p.G))
    _, state = oal.prefill(q[:, :, :T0].contiguous(), k[:, :, :T0].contiguous(),
                           v[:, :, :T0].contiguous(), g, L, G, p.eps, 128)
    state_a, state_b = state.clone(), state.clone()
    ws = oal.decode_workspace(4, 14, 2, cuda)
    shape = oal.make_shape(4, 1, 14, 2, 128, oal.OAL_BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for t in (T0, T0 + 1):  # two calls in a row
        qt, kt, vt = (x[:, :, t:t + 1].contiguous() for x in (q, k, v))
        ya = oal.decode_step(qt, kt, vt, state_a, ws)
        yb = torch.full_like(ya, float("nan"))
        rc = noalloc(qt.data_ptr(), kt.data_ptr(), vt.data_ptr(), state_b.data_ptr(),
                     yb.data_ptr(), ctypes.byref(shape), stream)
        assert rc == 0, oal.status_string(rc)
        torch.cuda.synchronize()
        assert row_rel_err(yb.cpu().numpy(), ya.cpu().numpy()) <= TOL_BF16
    assert oal.device_error() == 0
    sa, sb = state_a.cpu().numpy(), state_b.cpu().numpy()
    assert np.array_equal(sa, sb)


def test_noalloc_rejects_too_large(cuda):
    oal, noalloc = _noalloc_fn()
    big = oal.make_shape(1024, 1, 8, 1, 128, oal.OAL_BF16)  # B*Hq = 8192
    # the call below passes fake pointers: make sure the size check rejects it before any
    # launch, i.e. that this shape really needs more than the library's 4 MiB of scratch
    need = ctypes.c_size_t()
    assert oal.lib().oal_decode_workspace_bytes(ctypes.byref(big), ctypes.byref(need)) == 0
    assert need.value > (4 << 20)
    P = ctypes.c_void_p(256)
    assert noalloc(P, P, P, P, P, ctypes.byref(big), None) == -3
