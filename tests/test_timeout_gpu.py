"""The failure path of the tensor-core kernels, made to run on a GPU without a fault.

Every wait of the tensor-core prefill kernels is bounded (about one second); a wait that runs
out sets OAL_ERR_TIMEOUT in the device error word and the kernel unwinds (copies drained, MMAs
committed, tensor memory freed) instead of hanging.  oal_set_debug_skip_copies makes the
inter-chunk readout issue none of its copies, so its waits wait for data that never comes:
the call must report the timeout, leave the context usable, and the next prefill must be
correct."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, row_rel_err
from tests.test_gpu_parity import dev_inputs, oal  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_bounded_wait_runs_out_and_context_survives(oal, cuda):
    p = I.small_layer(610, B=1, T=300, Hq=14, Hkv=2, dtype="bf16")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    assert oal.device_error() == 0
    prev = oal.set_debug_skip_copies(True)
    try:
        oal.prefill(q, k, v, g, L, G, p.eps, 128)
        torch.cuda.synchronize()
    finally:
        oal.set_debug_skip_copies(prev)
    assert oal.device_error() == -7      # OAL_ERR_TIMEOUT
    assert oal.device_error() == 0       # cleared by the read
    # the context is usable and the next call is correct
    y, _ = oal.prefill(q, k, v, g, L, G, p.eps, 128)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    assert row_rel_err(y.cpu().numpy(), ref) <= TOL_BF16
