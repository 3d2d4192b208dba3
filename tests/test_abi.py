"""CPU-side checks of the C ABI: the library loads without a GPU, exports every function the
header declares, and rejects bad arguments on the host before touching the device."""
import ctypes

import numpy as np
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


def test_prefill_path_query():
    assert oal.prefill_path(oal.make_shape(1, 4096, 14, 2, 128, oal.OAL_BF16)) == \
        oal.OAL_PATH_TENSOR
    for chunk, dt in ((64, oal.OAL_BF16), (256, oal.OAL_BF16), (128, oal.OAL_F32)):
        assert oal.prefill_path(oal.make_shape(1, 4096, 14, 2, chunk, dt)) == \
            oal.OAL_PATH_CUDA_CORE
    s = oal.make_shape(1, 256, 14, 2, 96, oal.OAL_BF16)
    p = ctypes.c_int()
    assert oal.lib().oal_prefill_path(ctypes.byref(s), ctypes.byref(p)) == -3
    s.chunk = 128
    assert oal.lib().oal_prefill_path(ctypes.byref(s), None) == -1


def test_packed_batch_host_checks():
    """The one-launch packed batch runs only on the tensor-core path; sizes and arguments are
    checked on the host before anything reaches the device."""
    lens = (ctypes.c_int32 * 3)(300, 0, 129)
    n = ctypes.c_size_t()
    s = oal.make_shape(1, 300, 14, 2, 128, oal.OAL_BF16)
    assert oal.lib().oal_prefill_packed_workspace_bytes(ctypes.byref(s), lens, 3,
                                                        ctypes.byref(n)) == 0
    chunks, toks = 3 + 0 + 2, 429
    tail = ((toks * 14 * 4 + 255) // 256 * 256 + 256 + (3 * 3 * 128 + 255) // 256 * 256)
    assert n.value == chunks * 2 * 913920 + 14 * 7680 + tail
    for chunk, dt in ((64, oal.OAL_BF16), (128, oal.OAL_F32)):
        s2 = oal.make_shape(1, 300, 14, 2, chunk, dt)
        assert oal.lib().oal_prefill_packed_workspace_bytes(ctypes.byref(s2), lens, 3,
                                                            ctypes.byref(n)) == -3
    bad = (ctypes.c_int32 * 2)(10, -1)
    assert oal.lib().oal_prefill_packed_workspace_bytes(ctypes.byref(s), bad, 2,
                                                        ctypes.byref(n)) == -2
    P = _fake(1 << 20)
    ws = _fake(1 << 24)
    # workspace too small, misaligned workspace, missing states
    assert oal.lib().oal_prefill_packed(P, P, P, P, P, P, 0.0, P, P, 1 << 21, ws, 256,
                                        ctypes.byref(s), lens, 3, None) == -8
    assert oal.lib().oal_prefill_packed(P, P, P, P, P, P, 0.0, P, P, 1 << 21, _fake(4096 + 16),
                                        1 << 40, ctypes.byref(s), lens, 3, None) == -4
    assert oal.lib().oal_prefill_packed(P, P, P, P, P, P, 0.0, P, None, 1 << 21, ws, 1 << 40,
                                        ctypes.byref(s), lens, 3, None) == -1


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


@pytest.mark.parametrize("B,Hq,Hkv", [(1, 14, 2), (64, 14, 2), (3, 8, 1), (5, 6, 3)])
def test_decode_workspace_size(B, Hq, Hkv):
    """The decode scratch is the reserved leading block plus one partial readout (65 fp32) per
    slab (9 of 240 packed rows) and query head: align256(4 B Hkv) + 2340 B Hq bytes, the
    size include/oal.h states for the no-alloc entry point."""
    n = oal.decode_workspace_bytes(oal.make_shape(B, 1, Hq, Hkv))
    assert n == (4 * B * Hkv + 255) // 256 * 256 + 2340 * B * Hq


def test_header_packed_order_is_complete():
    """The packed order written in include/oal.h covers every pair r <= t of 65 exactly once."""
    from tests._packed import packed_pairs
    p = packed_pairs()
    assert len({(int(r), int(t)) for r, t in p}) == 2145
    assert all(r <= t for r, t in p)


def _host_ws(L, s, segments):
    n = ctypes.c_size_t(0)
    rc = L.oal_prefill_host_workspace_bytes(ctypes.byref(s), segments, ctypes.byref(n))
    return rc, n.value


def _align256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("T,segments", [(4096, 4), (300, 4), (128, 3), (1000, 1), (0, 2)])
def test_prefill_host_workspace_layout(L, T, segments):
    """Staging for q, k, v (bf16) and yhat (fp32) of the whole call, then the prefill
    workspace of the longest segment: segments are whole chunks of 128 tokens."""
    B, Hq, Hkv = 2, 14, 2
    s = oal.make_shape(B, T, Hq, Hkv, 128, oal.OAL_BF16)
    rc, n = _host_ws(L, s, segments)
    assert rc == 0
    seg_len = 0 if T == 0 else -(-(-(-T // segments)) // 128) * 128
    seg = oal.make_shape(B, seg_len, Hq, Hkv, 128, oal.OAL_BF16)
    pws = oal.prefill_workspace_bytes(seg)
    staging = (_align256(B * Hq * T * 64 * 2) + 2 * _align256(B * Hkv * T * 64 * 2)
               + _align256(B * Hq * T * 64 * 4))
    assert n == staging + _align256(pws)


def test_prefill_host_side_argument_errors(L):
    s = oal.make_shape(1, 512, 2, 1, 128, oal.OAL_BF16)
    assert _host_ws(L, s, 0)[0] == -2                      # segments < 1
    f32 = oal.make_shape(1, 512, 2, 1, 128, oal.OAL_F32)
    assert _host_ws(L, f32, 2)[0] == -3                    # no continuation off the tc path
    assert _host_ws(L, f32, 1)[0] == 0
    assert L.oal_prefill_host_workspace_bytes(ctypes.byref(s), 2, None) == -1
    rc, need = _host_ws(L, s, 2)
    P = _fake(1 << 20)
    args = [P, P, P, P, P, P, ctypes.c_float(1e-6), P, P, _fake(1 << 24),
            ctypes.c_size_t(need), ctypes.byref(s), 2, None, None, None]
    bad = list(args)
    bad[8] = None                                           # no state
    assert L.oal_prefill_host(*bad) == -1
    small = list(args)
    small[10] = ctypes.c_size_t(need - 1)
    assert L.oal_prefill_host(*small) == -8
    mis = list(args)
    mis[9] = _fake((1 << 24) + 16)                          # workspace not 256-aligned
    assert L.oal_prefill_host(*mis) == -4
    nohost = list(args)
    nohost[0] = None
    assert L.oal_prefill_host(*nohost) == -1


def test_header_compiles_as_c_and_links(tmp_path):
    """include/oal.h is plain C: a C99 program includes it, links liboal.so and calls the
    host-only entry points (no GPU needed)."""
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(build.build())
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "oal.h"
int main(void) {
    oal_shape s = {1, 4096, 14, 2, OAL_HEAD_DIM, OAL_VALUE_DIM, 128, OAL_BF16};
    size_t n = 0;
    if (oal_abi_version() != OAL_ABI_VERSION) return 1;
    if (oal_state_bytes(&s, &n) != OAL_OK || n == 0) return 2;
    if (oal_prefill_workspace_bytes(&s, &n) != OAL_OK || n == 0) return 3;
    if (oal_prefill_host_workspace_bytes(&s, 4, &n) != OAL_OK || n == 0) return 4;
    s.chunk = 96;
    if (oal_prefill_workspace_bytes(&s, &n) != OAL_ERR_UNSUPPORTED) return 5;
    if (strlen(oal_status_string(OAL_ERR_ALIGN)) == 0) return 6;
    printf("ok\n");
    return 0;
}
''')
    exe = tmp_path / "abi"
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic",
                           "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-loal", "-Wl,-rpath," + libdir])
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_hadamard_host_side_errors(L):
    s = oal.make_shape(1, 256, 2, 1, 64, oal.OAL_F32)
    P = _fake(1 << 20)
    ws = ctypes.c_size_t(1 << 40)
    # q, k, v, a, b, C, out, state, workspace, bytes, shape, stream
    args = [P] * 9 + [ws, ctypes.byref(s), None]
    for i in (3, 4, 5, 7):                       # a, b, C, state
        bad = list(args)
        bad[i] = None
        assert L.oal_prefill_hadamard(*bad) == -1
    mis = list(args)
    mis[5] = _fake((1 << 20) + 8)                # C not 16-byte aligned
    assert L.oal_prefill_hadamard(*mis) == -4
    small = list(args)
    small[9] = ctypes.c_size_t(16)
    assert L.oal_prefill_hadamard(*small) == -8
    odd = oal.make_shape(1, 256, 2, 1, 96, oal.OAL_F32)
    assert L.oal_prefill_hadamard(*args[:10], ctypes.byref(odd), None) == -3
    assert L.oal_dense_hadamard_gpu(P, P, P, None, P, P, P, ctypes.byref(s), None) == -1


def test_varlen_host_side_errors(L):
    s = oal.make_shape(1, 0, 4, 2, 128, oal.OAL_BF16)
    lens = (ctypes.c_int32 * 3)(100, 0, 300)
    n = ctypes.c_size_t(0)
    assert L.oal_prefill_varlen_workspace_bytes(ctypes.byref(s), lens, 3, 2, ctypes.byref(n)) == 0
    one = oal.make_shape(1, 300, 4, 2, 128, oal.OAL_BF16)
    assert n.value == 2 * ((oal.prefill_workspace_bytes(one) + 255) // 256 * 256)
    bad = (ctypes.c_int32 * 2)(5, -1)
    assert L.oal_prefill_varlen_workspace_bytes(ctypes.byref(s), bad, 2, 1, ctypes.byref(n)) == -2
    assert L.oal_prefill_varlen_workspace_bytes(ctypes.byref(s), lens, 3, 0, ctypes.byref(n)) == -2
    P = _fake(1 << 20)
    sb = (oal.state_bytes(one) + 255) // 256 * 256
    streams = (ctypes.c_void_p * 1)(None)
    args = [P] * 6 + [ctypes.c_float(1e-6), P, _fake(1 << 24), ctypes.c_size_t(sb),
                      _fake(1 << 25), ctypes.c_size_t(1 << 40), ctypes.byref(s), lens, 3,
                      streams, 1]
    stride = list(args)
    stride[9] = ctypes.c_size_t(sb - 256)                 # smaller than one state
    assert L.oal_prefill_varlen(*stride) == -2
    nost = list(args)
    nost[8] = None
    assert L.oal_prefill_varlen(*nost) == -1
    mis = list(args)
    mis[10] = _fake((1 << 25) + 16)                       # workspace not 256-aligned
    assert L.oal_prefill_varlen(*mis) == -4


def test_dense_backward_host_side_errors(L):
    s = oal.make_shape(1, 64, 2, 1, 128, oal.OAL_F32)
    n = ctypes.c_size_t(0)
    assert L.oal_dense_backward_workspace_bytes(ctypes.byref(s), ctypes.byref(n)) == 0
    rows = 1 * 2 * 64
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert n.value == 2 * a256(rows * 4) + a256(rows * 64 * 4) + a256(rows * 81 * 4) + a256(8)
    P = _fake(1 << 20)
    # q k v gid L G eps dy dq dk dv dL deps ws bytes shape stream
    args = [P] * 6 + [ctypes.c_float(1e-6)] + [P] * 6 + [_fake(1 << 24), n, ctypes.byref(s),
                                                         None]
    for i in (3, 11, 12):                        # group_id, dL, deps
        bad = list(args)
        bad[i] = None
        assert L.oal_dense_backward_gpu(*bad) == -1
    small = list(args)
    small[14] = ctypes.c_size_t(n.value - 1)
    assert L.oal_dense_backward_gpu(*small) == -8
    mis = list(args)
    mis[13] = _fake((1 << 24) + 16)
    assert L.oal_dense_backward_gpu(*mis) == -4


@pytest.mark.parametrize("B,T,Hq,Hkv", [(1, 4096, 14, 2), (2, 100, 4, 2), (1, 64, 8, 1),
                                        (3, 0, 6, 3)])
def test_backward_workspace_size(L, B, T, Hq, Hkv):
    """The chunked backward's scratch as include/oal.h lists it, part by part."""
    s = oal.make_shape(B, T, Hq, Hkv, 128, oal.OAL_F32)
    n = ctypes.c_size_t(0)
    assert L.oal_backward_workspace_bytes(ctypes.byref(s), ctypes.byref(n)) == 0
    NC, rows = -(-T // 64), B * Hq * T
    parts = [oal.state_bytes(s), B * Hkv * NC * 565760, B * Hkv * NC * 565760, rows * 4,
             rows * 64 * 4, rows * 65 * 4, B * Hq * NC * 2176 * 4, rows * 81 * 4, rows * 4,
             Hq * 4]
    assert n.value == max(256, sum(_align256(x) for x in parts))
    assert L.oal_backward_workspace_bytes(ctypes.byref(s), None) == -1


def test_backward_host_side_errors(L):
    s = oal.make_shape(1, 64, 2, 1, 128, oal.OAL_F32)
    n = ctypes.c_size_t(0)
    assert L.oal_backward_workspace_bytes(ctypes.byref(s), ctypes.byref(n)) == 0
    P = _fake(1 << 20)
    # q k v gid L G eps dy dq dk dv dL deps ws bytes shape stream
    args = [P] * 6 + [ctypes.c_float(1e-6)] + [P] * 6 + [_fake(1 << 24), n, ctypes.byref(s),
                                                         None]
    for i in (0, 3, 4, 5, 7, 8, 9, 10, 11, 12):   # every pointer the call reads or writes
        bad = list(args)
        bad[i] = None
        assert L.oal_backward(*bad) == -1, i
    for i in (0, 7, 9, 11):                        # q, dy, dk, dL not 16-byte aligned
        mis = list(args)
        mis[i] = _fake((1 << 20) + 4)
        assert L.oal_backward(*mis) == -4, i
    small = list(args)
    small[14] = ctypes.c_size_t(n.value - 1)
    assert L.oal_backward(*small) == -8
    nows = list(args)
    nows[13] = None
    assert L.oal_backward(*nows) == -8
    mis_ws = list(args)
    mis_ws[13] = _fake((1 << 24) + 16)             # workspace not 256-byte aligned
    assert L.oal_backward(*mis_ws) == -4
    wide = oal.make_shape(1, 64, 18, 2, 128, oal.OAL_F32)   # 9 query heads per kv head
    assert L.oal_backward(*args[:15], ctypes.byref(wide), None) == -3


def test_prefill_continue_host_side_checks(L):
    """A continuation exists only on the tensor-core path (bf16, chunk 128); appending no
    tokens returns at once, before any device work."""
    P = _fake(1 << 20)
    ws = ctypes.c_size_t(1 << 40)
    for dtype, chunk in ((oal.OAL_F32, 128), (oal.OAL_BF16, 64), (oal.OAL_BF16, 256)):
        s = oal.make_shape(1, 256, 2, 1, chunk, dtype)
        assert L.oal_prefill_continue(*[P] * 6, ctypes.c_float(1e-6), P, P, P, ws,
                                      ctypes.byref(s), None) == -3
    s = oal.make_shape(1, 256, 2, 1, 128, oal.OAL_BF16)
    assert L.oal_prefill_continue(*[P] * 6, ctypes.c_float(1e-6), P, None, P, ws,
                                  ctypes.byref(s), None) == -1
    empty = oal.make_shape(1, 0, 2, 1, 128, oal.OAL_BF16)
    assert L.oal_prefill_continue(None, None, None, P, P, P, ctypes.c_float(1e-6), None, P, P,
                                  ws, ctypes.byref(empty), None) == 0
    odd = oal.make_shape(1, 256, 2, 1, 96, oal.OAL_BF16)
    assert L.oal_prefill_continue(*[P] * 6, ctypes.c_float(1e-6), P, P, P, ws,
                                  ctypes.byref(odd), None) == -3


def test_noalloc_decode_host_side_checks(L):
    """The allocation-free decode refuses a step whose scratch would exceed its fixed 4 MiB
    array before it touches the device; B*Hq = 1789 fits whatever Hkv."""
    fn = L.oal_decode_step_noalloc
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.POINTER(oal.Shape), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    P = _fake(1 << 20)
    assert _align256(4 * 1789) + 2340 * 1789 <= 4 << 20                 # Hkv = Hq, the worst
    assert _align256(4 * 128 * 2) + 2340 * 128 * 14 == 4 << 20          # exactly full
    for B, Hq, Hkv in ((129, 14, 2), (1790, 1, 1), (225, 8, 1)):
        need = _align256(4 * B * Hkv) + 2340 * B * Hq
        assert need > 4 << 20
        big = oal.make_shape(B, 1, Hq, Hkv, 128, oal.OAL_BF16)
        assert fn(P, P, P, P, P, ctypes.byref(big), None) == -3
    s = oal.make_shape(64, 1, 14, 2, 128, oal.OAL_BF16)
    assert fn(P, P, P, None, P, ctypes.byref(s), None) == -1      # no state
    assert fn(P, None, P, P, P, ctypes.byref(s), None) == -1      # no k
    assert fn(P, P, P, _fake((1 << 20) + 8), P, ctypes.byref(s), None) == -4
    assert fn(P, P, P, P, P, None, None) == -1


def test_contribution_stat_host_side_checks(L):
    P = _fake(1 << 20)
    s = oal.make_shape(2, 300, 14, 2, 128, oal.OAL_BF16)
    assert L.oal_contribution_stat(P, None, P, ctypes.byref(s), None) == -1
    assert L.oal_contribution_stat(P, P, _fake((1 << 20) + 4), ctypes.byref(s), None) == -4
    empty = oal.make_shape(2, 0, 14, 2, 128, oal.OAL_BF16)      # nothing to write
    assert L.oal_contribution_stat(None, None, None, ctypes.byref(empty), None) == 0
    bad = oal.make_shape(2, 300, 14, 3, 128, oal.OAL_BF16)      # Hq not a multiple of Hkv
    assert L.oal_contribution_stat(P, P, P, ctypes.byref(bad), None) == -2


def test_state_prefix_sum_host_side_checks(L):
    P = _fake(1 << 20)
    n = ctypes.c_size_t(1024)
    assert L.oal_state_prefix_sum(P, -1, n, P, None) == -2
    assert L.oal_state_prefix_sum(None, 2, ctypes.c_size_t(0), None, None) == 0
    assert L.oal_state_prefix_sum(None, 2, n, P, None) == -1
    assert L.oal_state_prefix_sum(P, 2, n, None, None) == -1
    assert L.oal_state_prefix_sum(P, 2, ctypes.c_size_t(1022), P, None) == -4
    assert L.oal_state_prefix_sum(_fake((1 << 20) + 4), 2, n, P, None) == -4


def test_overlap_switch_returns_previous_setting(L):
    prev = L.oal_set_prefill_overlap(0)
    try:
        assert prev in (0, 1)
        assert L.oal_set_prefill_overlap(7) == 0
        assert L.oal_set_prefill_overlap(1) == 1
    finally:
        L.oal_set_prefill_overlap(prev)


def test_binding_refuses_host_tensors():
    """The Python binding has no CPU path: host tensors are refused before the library is
    called, so nothing can silently compute elsewhere than in the CUDA kernels."""
    import torch
    B, Hq, Hkv, T = 1, 4, 2, 16
    q = torch.zeros(B, Hq, T, 64, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, T, 64, dtype=torch.bfloat16)
    v = torch.zeros(B, Hkv, T, 64, dtype=torch.bfloat16)
    gid = torch.zeros(Hq, 64, dtype=torch.int32)
    Lm = torch.eye(9, dtype=torch.float32).expand(Hq, 9, 9).contiguous()
    G = torch.ones(Hq, dtype=torch.int32)
    a, b, C = torch.ones(Hq), torch.zeros(Hq, 64), torch.zeros(Hq, 64, 64)
    calls = [
        lambda: oal.prefill(q, k, v, gid, Lm, G, 1e-6),
        lambda: oal.dense_ref(q, k, v, gid, Lm, G, 1e-6),
        lambda: oal.contribution_stat(q, k),
        lambda: oal.prefill_hadamard(q, k, v, a, b, C),
        lambda: oal.backward(q, k, v, gid, Lm, G, 1e-6, torch.zeros(B, Hq, T, 64)),
        lambda: oal.decode_step(q[:, :, :1].contiguous(), k[:, :, :1].contiguous(),
                                v[:, :, :1].contiguous(), torch.zeros(1 << 20, dtype=torch.uint8),
                                oal.decode_workspace(B, Hq, Hkv, "cpu")),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


def _ws(L, fn, s):
    n = ctypes.c_size_t(0)
    return getattr(L, fn)(ctypes.byref(s), ctypes.byref(n))


def test_grid_plane_limits():
    """Grids hold at most 65535 blocks in y and z: B*Hq for the CUDA-core kernels (prefill,
    Hadamard and dense forms, both backward passes), B*Hkv for the decode step and B*Hkv + 1
    for the tensor-core prefill's scan.  Larger problems are refused on the host with
    OAL_ERR_SHAPE, at the size query and at the call, before any device work.  The calls
    get NULL pointers, so a missing size check would show as OAL_ERR_NULL instead."""
    L = oal.lib()
    F32, BF16 = oal.OAL_F32, oal.OAL_BF16
    P = None
    eps = ctypes.c_float(1e-6)
    big = ctypes.c_size_t(1 << 45)
    # CUDA-core prefill: B*Hq planes
    assert _ws(L, "oal_prefill_workspace_bytes", oal.make_shape(13107, 1, 5, 5, 64, F32)) == 0
    over = oal.make_shape(6554, 1, 10, 2, 64, F32)                # 65540 planes
    assert _ws(L, "oal_prefill_workspace_bytes", over) == -2
    assert L.oal_prefill(None, None, None, None, None, None, eps, None, None, None, big,
                         ctypes.byref(over), None) == -2
    # tensor-core prefill: B*Hkv + 1 planes (B*Hq does not matter there)
    assert _ws(L, "oal_prefill_workspace_bytes", oal.make_shape(6554, 1, 10, 2, 128, BF16)) == 0
    assert _ws(L, "oal_prefill_workspace_bytes", oal.make_shape(32767, 1, 2, 2, 128, BF16)) == 0
    tc_over = oal.make_shape(32768, 1, 2, 2, 128, BF16)             # 65536 + 1 planes
    assert _ws(L, "oal_prefill_workspace_bytes", tc_over) == -2
    assert L.oal_prefill_continue(None, None, None, None, None, None, eps, None, None, None,
                                  big, ctypes.byref(tc_over), None) == -2
    assert _host_ws(L, tc_over, 1)[0] == -2
    # tensor-core prefill: the chunk-state images' 32-bit row coordinate (34 slices of 80 rows
    # per chunk and kv head)
    assert _ws(L, "oal_prefill_workspace_bytes", oal.make_shape(1, 98689 * 128, 8, 8, 128,
                                                                BF16)) == 0
    long_tc = oal.make_shape(1, 98690 * 128, 8, 8, 128, BF16)
    assert 8 * 98689 * 34 * 80 < 1 << 31 <= 8 * 98690 * 34 * 80
    assert _ws(L, "oal_prefill_workspace_bytes", long_tc) == -2
    assert L.oal_prefill(P, P, P, P, P, P, eps, P, P, P, big, ctypes.byref(long_tc), None) == -2
    # decode: B*Hkv planes, both entry points
    assert _ws(L, "oal_decode_workspace_bytes", oal.make_shape(32767, 1, 4, 2)) == 0
    dec_over = oal.make_shape(32768, 1, 4, 2)                       # 65536 planes
    assert _ws(L, "oal_decode_workspace_bytes", dec_over) == -2
    assert L.oal_decode_step(P, P, P, P, P, P, big, ctypes.byref(dec_over), None) == -2
    fn = L.oal_decode_step_noalloc
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.POINTER(oal.Shape), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    assert fn(P, P, P, P, P, ctypes.byref(dec_over), None) == -2
    # dense form, Hadamard forms, backward passes: B*Hq planes
    assert L.oal_dense_ref_gpu(P, P, P, P, P, P, eps, P, ctypes.byref(over), None) == -2
    assert L.oal_dense_hadamard_gpu(P, P, P, P, P, P, P, ctypes.byref(over), None) == -2
    assert L.oal_prefill_hadamard(P, P, P, P, P, P, P, P, P, big, ctypes.byref(over),
                                  None) == -2
    for name in ("oal_backward", "oal_dense_backward_gpu"):
        assert _ws(L, name.replace("_gpu", "") + "_workspace_bytes", over) == -2
        assert getattr(L, name)(*[P] * 6, eps, *[P] * 6, P, big, ctypes.byref(over),
                                None) == -2
    assert _ws(L, "oal_backward_workspace_bytes", oal.make_shape(13107, 1, 5, 5, 64, F32)) == 0
    # packed batch: every sequence's kv heads plus one plane
    lens = (ctypes.c_int32 * 32768)(*([1] * 32768))
    n = ctypes.c_size_t(0)
    s = oal.make_shape(1, 0, 2, 2, 128, BF16)
    assert L.oal_prefill_packed_workspace_bytes(ctypes.byref(s), lens, 32767,
                                                ctypes.byref(n)) == 0
    assert L.oal_prefill_packed_workspace_bytes(ctypes.byref(s), lens, 32768,
                                                ctypes.byref(n)) == -2


def test_library_packed_order_matches_header(tmp_path):
    """The library's packed feature order (its feature_rt, compiled for the host from the CUDA
    sources) is the order include/oal.h documents, row for row; the padding rows map past the
    last dimension (65, 65)."""
    import os
    import subprocess
    from tests._packed import F, FP, packed_pairs
    csrc = os.path.join(os.path.dirname(oal.LIB_PATH), "csrc")
    src = tmp_path / "rt.cu"
    src.write_text('#include "oal_common.cuh"\n#include <cstdio>\n'
                   "int main() {\n"
                   "    for (int f = 0; f < oal::kFP; ++f) {\n"
                   "        const oal::RT rt = oal::feature_rt(f);\n"
                   '        std::printf("%d %d\\n", rt.r, rt.t);\n'
                   "    }\n"
                   "    return 0;\n"
                   "}\n")
    exe = tmp_path / "rt"
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.check_call([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", csrc, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    rt = np.array([[int(x) for x in ln.split()] for ln in out.splitlines()])
    assert rt.shape == (FP, 2)
    assert np.array_equal(rt[:F], packed_pairs())
    assert np.all(rt[F:] == 65)
