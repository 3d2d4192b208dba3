"""CPU-side checks of the C ABI: the library loads without a GPU, exports every function the
header declares, and rejects bad arguments on the host before touching the device."""
import ctypes

import pytest

from positive_quadratic_b200 import build, oal


@pytest.fixture(scope="module")
def L():
    build.build()
    return oal.lib()


def test_exports_every_declared_symbol(L):
    names = oal.declared_symbols()
    assert {"oal_prefill", "oal_decode_step", "oal_dense_ref_gpu", "oal_state_bytes",
            "oal_prefill_workspace_bytes", "oal_decode_workspace_bytes", "oal_device_error",
            "oal_status_string", "oal_abi_version"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_abi_version_and_strings(L):
    assert L.oal_abi_version() == 1
    for code in oal.STATUS:
        assert oal.status_string(code) not in ("", "unknown status")


def test_state_bytes_layout():
    s = oal.make_shape(64, 1, 14, 2)
    per_unit = 2176 * 65 * 4
    coef = ((14 * 2176 * 4 + 255) // 256) * 256
    assert oal.state_bytes(s) == 256 + coef + 64 * 2 * per_unit


@pytest.mark.parametrize("field,value,code", [
    ("Hq", 0, -2), ("Hkv", 3, -2), ("B", -1, -2), ("T", -5, -2), ("dh", 32, -3),
    ("dv", 128, -3), ("chunk", 96, -3), ("dtype", 7, -3)])
def test_shape_validation(field, value, code):
    s = oal.make_shape(1, 256, 14, 2, 128, oal.OAL_BF16)
    setattr(s, field, value)
    n = ctypes.c_size_t()
    assert oal.lib().oal_prefill_workspace_bytes(ctypes.byref(s), ctypes.byref(n)) == code


def test_group_size_limit():
    s = oal.make_shape(1, 16, 16, 1)
    n = ctypes.c_size_t()
    assert oal.lib().oal_state_bytes(ctypes.byref(s), ctypes.byref(n)) == -3


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_prefill_host_side_errors(L):
    s = oal.make_shape(1, 256, 2, 1, 128, oal.OAL_F32)
    P = _fake(1 << 20)
    args = [P] * 6 + [ctypes.c_float(1e-6), P, P, P, ctypes.c_size_t(1 << 40), ctypes.byref(s),
                      None]
    bad = list(args)
    bad[0] = None
    assert L.oal_prefill(*bad) == -1
    mis = list(args)
    mis[1] = _fake((1 << 20) + 4)
    assert L.oal_prefill(*mis) == -4
    small = list(args)
    small[10] = ctypes.c_size_t(16)
    assert L.oal_prefill(*small) == -8
    assert L.oal_prefill(*args[:-2], None, None) == -1


def test_decode_and_dense_host_side_errors(L):
    s = oal.make_shape(2, 1, 14, 2, 128, oal.OAL_BF16)
    P = _fake(1 << 20)
    assert L.oal_decode_step(P, P, P, P, P, None, ctypes.c_size_t(0), ctypes.byref(s),
                             None) == -8
    assert L.oal_decode_step(P, None, P, P, P, P, ctypes.c_size_t(1 << 40), ctypes.byref(s),
                             None) == -1
    assert L.oal_dense_ref_gpu(P, P, P, P, P, P, ctypes.c_float(0.0), _fake(3),
                               ctypes.byref(s), None) == -4
    assert L.oal_device_error(None, None) == -1


def test_header_packed_order_is_complete():
    """The packed order written in include/oal.h covers every pair r <= t of 65 exactly once."""
    from tests._packed import packed_pairs
    p = packed_pairs()
    assert len({(int(r), int(t)) for r, t in p}) == 2145
    assert all(r <= t for r, t in p)


def test_decode_variant_switch():
    """The decode-kernel switch is host state only: it accepts 0 and 1, returns the previous
    value and refuses anything else without changing the setting."""
    prev = oal.set_decode_variant(1)
    try:
        assert prev == 0
        assert oal.set_decode_variant(1) == 1
        with pytest.raises(oal.OALError):
            oal.set_decode_variant(2)
        assert oal.set_decode_variant(0) == 1
    finally:
        oal.set_decode_variant(prev)
