"""Python binding of the OAL C ABI (include/oal.h): argument marshalling only.

Every step of the computation runs in the CUDA library liboal.so.  PyTorch supplies device
memory and streams.  The binding raises OALError on any non-zero status and refuses to run
when the library is missing.  There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboal.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "oal.h")

OAL_F32, OAL_BF16 = 0, 1
OAL_PATH_CUDA_CORE, OAL_PATH_TENSOR = 0, 1
HEAD_DIM = VALUE_DIM = 64
G_MAX = 8
FEATURES, FEATURES_PAD = 2145, 2176
STATUS = {0: "OAL_OK", -1: "OAL_ERR_NULL", -2: "OAL_ERR_SHAPE", -3: "OAL_ERR_UNSUPPORTED",
          -4: "OAL_ERR_ALIGN", -5: "OAL_ERR_GROUPS", -6: "OAL_ERR_CUDA", -7: "OAL_ERR_TIMEOUT",
          -8: "OAL_ERR_WORKSPACE", -9: "OAL_ERR_STATE"}


class Shape(ctypes.Structure):
    """oal_shape."""
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "Hq", "Hkv", "dh", "dv", "chunk",
                                               "dtype")]


class KernelStat(ctypes.Structure):
    """oal_kernel_stat."""
    _fields_ = [("name", ctypes.c_char * 40), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]


class OALError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = f"{what}: {STATUS.get(code, code)} ({status_string(code)})"
        if code == -6:
            msg += f" [{last_cuda_error()}]"
        super().__init__(msg)


_lock = threading.Lock()
_lib = None
_VP, _SZ, _PS = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Shape)


def lib() -> ctypes.CDLL:
    """The loaded liboal.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing; run "
                                   "python -m positive_quadratic_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            L.oal_abi_version.restype = ctypes.c_int
            L.oal_status_string.argtypes = [ctypes.c_int]
            L.oal_status_string.restype = ctypes.c_char_p
            for name in ("oal_state_bytes", "oal_prefill_workspace_bytes",
                         "oal_decode_workspace_bytes"):
                getattr(L, name).argtypes = [_PS, ctypes.POINTER(_SZ)]
            L.oal_prefill_path.argtypes = [_PS, ctypes.POINTER(ctypes.c_int)]
            L.oal_prefill_path.restype = ctypes.c_int
            L.oal_prefill.argtypes = [_VP] * 6 + [ctypes.c_float, _VP, _VP, _VP, _SZ, _PS, _VP]
            L.oal_prefill_continue.argtypes = L.oal_prefill.argtypes
            L.oal_decode_step.argtypes = [_VP] * 6 + [_SZ, _PS, _VP]
            L.oal_dense_ref_gpu.argtypes = [_VP] * 6 + [ctypes.c_float, _VP, _PS, _VP]
            L.oal_contribution_stat.argtypes = [_VP, _VP, _VP, _PS, _VP]
            L.oal_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), _VP]
            L.oal_launch_count.restype = ctypes.c_ulonglong
            L.oal_last_cuda_error.argtypes = [ctypes.c_char_p, ctypes.c_size_t]
            L.oal_last_cuda_error.restype = ctypes.c_int
            L.oal_set_prefill_overlap.argtypes = [ctypes.c_int]
            L.oal_set_prefill_overlap.restype = ctypes.c_int
            L.oal_set_debug_skip_copies.argtypes = [ctypes.c_int]
            L.oal_set_debug_skip_copies.restype = ctypes.c_int
            L.oal_prefill_host_workspace_bytes.argtypes = [_PS, ctypes.c_int,
                                                           ctypes.POINTER(_SZ)]
            L.oal_prefill_host.argtypes = [_VP] * 6 + [ctypes.c_float, _VP, _VP, _VP, _SZ, _PS,
                                                       ctypes.c_int, _VP, _VP, _VP]
            L.oal_prefill_hadamard.argtypes = [_VP] * 7 + [_VP, _VP, _SZ, _PS, _VP]
            L.oal_dense_hadamard_gpu.argtypes = [_VP] * 7 + [_PS, _VP]
            L.oal_prefill_varlen_workspace_bytes.argtypes = [_PS, _VP, ctypes.c_int,
                                                             ctypes.c_int, ctypes.POINTER(_SZ)]
            L.oal_prefill_varlen.argtypes = [_VP] * 6 + [ctypes.c_float, _VP, _VP, _SZ, _VP,
                                                         _SZ, _PS, _VP, ctypes.c_int, _VP,
                                                         ctypes.c_int]
            L.oal_prefill_packed_workspace_bytes.argtypes = [_PS, _VP, ctypes.c_int,
                                                             ctypes.POINTER(_SZ)]
            L.oal_prefill_packed_workspace_bytes.restype = ctypes.c_int
            L.oal_prefill_packed.argtypes = [_VP] * 6 + [ctypes.c_float, _VP, _VP, _SZ, _VP,
                                                         _SZ, _PS, _VP, ctypes.c_int, _VP]
            L.oal_prefill_packed.restype = ctypes.c_int
            L.oal_state_prefix_sum.argtypes = [_VP, ctypes.c_int, _SZ, _VP, _VP]
            L.oal_state_prefix_sum.restype = ctypes.c_int
            for pre in ("oal_dense_backward", "oal_backward"):
                getattr(L, pre + "_workspace_bytes").argtypes = [_PS, ctypes.POINTER(_SZ)]
                getattr(L, pre + "_workspace_bytes").restype = ctypes.c_int
            for name in ("oal_dense_backward_gpu", "oal_backward"):
                getattr(L, name).argtypes = [_VP] * 6 + [ctypes.c_float] + [_VP] * 7 + [
                    _SZ, _PS, _VP]
                getattr(L, name).restype = ctypes.c_int
            for name in ("oal_prefill_host_workspace_bytes", "oal_prefill_host",
                         "oal_prefill_hadamard", "oal_dense_hadamard_gpu",
                         "oal_prefill_varlen_workspace_bytes", "oal_prefill_varlen"):
                getattr(L, name).restype = ctypes.c_int
            L.oal_profile_enable.argtypes = [ctypes.c_int]
            L.oal_profile_enable.restype = ctypes.c_int
            L.oal_profile_read.argtypes = [ctypes.POINTER(KernelStat), ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int)]
            L.oal_profile_read.restype = ctypes.c_int
            for name in ("oal_state_bytes", "oal_prefill_workspace_bytes",
                         "oal_decode_workspace_bytes", "oal_prefill", "oal_decode_step",
                         "oal_dense_ref_gpu", "oal_device_error", "oal_contribution_stat",
                         "oal_prefill_continue"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def declared_symbols(header: str = HEADER):
    """Names of the functions include/oal.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*|unsigned long long)\s+(oal_\w+)\s*\(",
                                 text, re.M)))


def last_cuda_error() -> str:
    """Name and description of the CUDA error behind the most recent OAL_ERR_CUDA."""
    try:
        buf = ctypes.create_string_buffer(256)
        lib().oal_last_cuda_error(buf, 256)
        return buf.value.decode()
    except Exception:
        return "?"


def status_string(code: int) -> str:
    try:
        return lib().oal_status_string(int(code)).decode()
    except Exception:
        return "?"


def _check(rc: int, what: str):
    if rc != 0:
        raise OALError(rc, what)


def make_shape(B, T, Hq, Hkv, chunk=128, dtype=OAL_BF16, dh=HEAD_DIM, dv=VALUE_DIM) -> Shape:
    return Shape(int(B), int(T), int(Hq), int(Hkv), int(dh), int(dv), int(chunk), int(dtype))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return OAL_BF16
    if t.dtype == torch.float32:
        return OAL_F32
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def state_bytes(shape: Shape) -> int:
    n = _SZ()
    _check(lib().oal_state_bytes(ctypes.byref(shape), ctypes.byref(n)), "oal_state_bytes")
    return n.value


def prefill_workspace_bytes(shape: Shape) -> int:
    n = _SZ()
    _check(lib().oal_prefill_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)),
           "oal_prefill_workspace_bytes")
    return n.value


def prefill_path(shape: Shape) -> int:
    """OAL_PATH_TENSOR or OAL_PATH_CUDA_CORE: the kernels oal_prefill runs for `shape`."""
    p = ctypes.c_int()
    _check(lib().oal_prefill_path(ctypes.byref(shape), ctypes.byref(p)), "oal_prefill_path")
    return p.value


def decode_workspace_bytes(shape: Shape) -> int:
    n = _SZ()
    _check(lib().oal_decode_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)),
           "oal_decode_workspace_bytes")
    return n.value


def _shape_of(q, k, v, chunk):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, T, d]")
    B, Hq, T, dh = q.shape
    return make_shape(B, T, Hq, k.shape[1], chunk, _dtype_code(q), dh, v.shape[3])


def _contig_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def empty_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def prefill(q, k, v, group_id, L, G, eps: float, chunk: int = 128, out=None, state=None,
            workspace=None, stream=None):
    """oal_prefill on CUDA tensors.  Returns (out [B,Hq,T,dv] fp32, state uint8)."""
    shape = _shape_of(q, k, v, chunk)
    dev = q.device
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=torch.float32,
                          device=dev)
    if state is None:
        state = torch.empty(state_bytes(shape), dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = empty_workspace(prefill_workspace_bytes(shape), dev)
    _contig_cuda(q, k, v, group_id, L, G, out, state, workspace)
    rc = lib().oal_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                           float(eps), _ptr(out), _ptr(state), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), ctypes.byref(shape),
                           _stream(stream))
    _check(rc, "oal_prefill")
    return out, state


def prefill_state(k, v, group_id, L, G, eps: float, Hq: int, chunk: int = 128, state=None,
                  workspace=None, stream=None):
    """oal_prefill with out = NULL: the prefix state after the T tokens of k/v (and the
    coefficient tables of Hq query heads), without computing outputs."""
    B, Hkv, T, dh = k.shape
    shape = make_shape(B, T, Hq, Hkv, chunk, _dtype_code(k), dh, v.shape[3])
    dev = k.device
    if state is None:
        state = torch.empty(state_bytes(shape), dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = empty_workspace(prefill_workspace_bytes(shape), dev)
    _contig_cuda(k, v, group_id, L, G, state, workspace)
    rc = lib().oal_prefill(None, _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                           float(eps), None, _ptr(state), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), ctypes.byref(shape),
                           _stream(stream))
    _check(rc, "oal_prefill (state only)")
    return state


def state_body(state: torch.Tensor, B: int, Hq: int, Hkv: int) -> torch.Tensor:
    """fp32 view of the per-(b, kv) prefix states inside a state buffer (after the header and
    the coefficient tables): B*Hkv units of Hv[2176][64] then z[2176]."""
    off = 256 + ((Hq * FEATURES_PAD * 4 + 255) // 256) * 256
    n = B * Hkv * FEATURES_PAD * (VALUE_DIM + 1)
    return state[off:off + 4 * n].view(torch.float32)


def state_prefix_sum(parts: torch.Tensor, n_parts: int, out: torch.Tensor, stream=None):
    """oal_state_prefix_sum: out = parts[0] + ... + parts[n_parts - 1] (rows of a contiguous
    fp32 [rows, n] tensor, added in order)."""
    if parts.dim() != 2 or parts.dtype != torch.float32 or out.dtype != torch.float32:
        raise ValueError("parts [rows, n] and out [n] must be fp32")
    if not 0 <= n_parts <= parts.shape[0] or out.numel() != parts.shape[1]:
        raise ValueError("n_parts out of range or out of the wrong size")
    _contig_cuda(parts, out)
    _check(lib().oal_state_prefix_sum(_ptr(parts), int(n_parts), parts.shape[1], _ptr(out),
                                      _stream(stream)), "oal_state_prefix_sum")
    return out


def set_state_tokens(state: torch.Tensor, tokens: int) -> None:
    """Sets the token count in a state header (int64 at byte 32)."""
    state[32:40].copy_(torch.tensor([int(tokens)], dtype=torch.int64).view(torch.uint8))


def prefill_continue(q, k, v, group_id, L, G, eps: float, state, out=None, workspace=None,
                     stream=None):
    """oal_prefill_continue: appends the T tokens of q/k/v to the sequence held by `state`
    (bf16, chunk 128).  Returns out [B,Hq,T,dv] fp32; `state` is updated in place."""
    shape = _shape_of(q, k, v, 128)
    dev = q.device
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=torch.float32,
                          device=dev)
    if workspace is None:
        workspace = empty_workspace(prefill_workspace_bytes(shape), dev)
    _contig_cuda(q, k, v, group_id, L, G, out, state, workspace)
    rc = lib().oal_prefill_continue(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L),
                                    _ptr(G), float(eps), _ptr(out), _ptr(state),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    ctypes.byref(shape), _stream(stream))
    _check(rc, "oal_prefill_continue")
    return out


def decode_step(q, k, v, state, workspace, out=None, stream=None):
    """oal_decode_step on CUDA tensors q [B,Hq,1,dh], k/v [B,Hkv,1,d]; returns out."""
    shape = _shape_of(q, k, v, 128)
    shape.T = 1
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], 1, v.shape[3], dtype=torch.float32,
                          device=q.device)
    _contig_cuda(q, k, v, state, workspace, out)
    rc = lib().oal_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               ctypes.byref(shape), _stream(stream))
    _check(rc, "oal_decode_step")
    return out


def decode_workspace(B, Hq, Hkv, device) -> torch.Tensor:
    """Decode workspace (zero-filled; a step writes every scratch word before reading it)."""
    n = decode_workspace_bytes(make_shape(B, 1, Hq, Hkv))
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def dense_ref(q, k, v, group_id, L, G, eps: float, out=None, stream=None):
    """oal_dense_ref_gpu: the O(T^2) dense form."""
    shape = _shape_of(q, k, v, 128)
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=torch.float32,
                          device=q.device)
    _contig_cuda(q, k, v, group_id, L, G, out)
    rc = lib().oal_dense_ref_gpu(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                                 float(eps), _ptr(out), ctypes.byref(shape), _stream(stream))
    _check(rc, "oal_dense_ref_gpu")
    return out


def contribution_stat(q, k, out=None, stream=None):
    """oal_contribution_stat: eq. (1)'s chi per prompt (b, query head) and dimension, [B, Hq, 64]
    fp32; the page's chi_r is its mean over b."""
    if q.dim() != 4 or k.dim() != 4 or k.dtype != q.dtype:
        raise ValueError("q [B, Hq, T, d] and k [B, Hkv, T, d] of one dtype expected")
    B, Hq, T, d = q.shape
    shape = make_shape(B, T, Hq, k.shape[1], 128, _dtype_code(q), d)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    _contig_cuda(q, k, out)
    rc = lib().oal_contribution_stat(_ptr(q), _ptr(k), _ptr(out), ctypes.byref(shape),
                                     _stream(stream))
    _check(rc, "oal_contribution_stat")
    return out


def device_error(stream=None) -> int:
    """Reads and clears the device-side error word (0 = none)."""
    code = ctypes.c_int(0)
    _check(lib().oal_device_error(ctypes.byref(code), _stream(stream)), "oal_device_error")
    return code.value


def host_prefill_buffers(q, k, v, group_id, L, G, chunk: int = 128, segments: int = 4,
                         device="cuda") -> dict:
    """Device memory and copy streams for prefill_from_host: group ids, L and G copied once,
    the state, the oal_prefill_host workspace, and two copy streams."""
    shape = _shape_of(q, k, v, chunk)
    n = _SZ(0)
    _check(lib().oal_prefill_host_workspace_bytes(ctypes.byref(shape), int(segments),
                                                  ctypes.byref(n)),
           "oal_prefill_host_workspace_bytes")
    return dict(
        g=group_id.to(device=device, dtype=torch.int32).contiguous(),
        L=L.to(device=device, dtype=torch.float32).contiguous(),
        G=G.to(device=device, dtype=torch.int32).contiguous(),
        state=torch.empty(state_bytes(shape), dtype=torch.uint8, device=device),
        ws=empty_workspace(n.value, device), chunk=int(chunk), segments=int(segments),
        copy_in=torch.cuda.Stream(device=device), copy_out=torch.cuda.Stream(device=device))


def prefill_from_host(q, k, v, eps: float, bufs: dict, out_host=None, stream=None):
    """oal_prefill_host: q/k/v in (pinned) host memory, yhat back into host memory, with the
    copies of one segment overlapped with the kernels of the next.  ``bufs`` comes from
    host_prefill_buffers; the state ends in bufs["state"].  Returns the host output tensor,
    valid once ``stream`` (default: the current stream) is synchronised."""
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous host tensors")
    shape = _shape_of(q, k, v, bufs["chunk"])
    if out_host is None:
        out_host = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3],
                               dtype=torch.float32, pin_memory=True)
    ws = bufs["ws"]
    rc = lib().oal_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(bufs["g"]), _ptr(bufs["L"]),
                                _ptr(bufs["G"]), float(eps), _ptr(out_host),
                                _ptr(bufs["state"]), _ptr(ws), ws.numel() * ws.element_size(),
                                ctypes.byref(shape), bufs["segments"], _stream(stream),
                                ctypes.c_void_p(bufs["copy_in"].cuda_stream),
                                ctypes.c_void_p(bufs["copy_out"].cuda_stream))
    _check(rc, "oal_prefill_host")
    return out_host


def _hadamard_coefs(q, a, b, C):
    Hq = q.shape[1]
    a, b, C = (t.to(device=q.device, dtype=torch.float32).contiguous() for t in (a, b, C))
    if a.shape != (Hq,) or b.shape != (Hq, HEAD_DIM) or C.shape != (Hq, HEAD_DIM, HEAD_DIM):
        raise ValueError("a [Hq], b [Hq, 64], C [Hq, 64, 64] expected")
    return a, b, C


def prefill_hadamard(q, k, v, a, b, C, chunk: int = 128, out=None, state=None, workspace=None,
                     stream=None):
    """oal_prefill_hadamard: causal prefill with kappa = a + b.x + x^T C x, x = q*k/sqrt(64)
    (per query head a [Hq], b [Hq, 64], C [Hq, 64, 64]).  bf16 with chunk 128 (the default,
    as for prefill) runs on tensor cores.  Returns (out, state); the state continues with
    decode_step."""
    shape = _shape_of(q, k, v, chunk)
    dev = q.device
    a, b, C = _hadamard_coefs(q, a, b, C)
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=torch.float32,
                          device=dev)
    if state is None:
        state = torch.empty(state_bytes(shape), dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = empty_workspace(prefill_workspace_bytes(shape), dev)
    _contig_cuda(q, k, v, a, b, C, out, state, workspace)
    rc = lib().oal_prefill_hadamard(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(C),
                                    _ptr(out), _ptr(state), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    ctypes.byref(shape), _stream(stream))
    _check(rc, "oal_prefill_hadamard")
    return out, state


def dense_hadamard(q, k, v, a, b, C, out=None, stream=None):
    """oal_dense_hadamard_gpu: the O(T^2) causal form of the same kernel."""
    shape = _shape_of(q, k, v, 64)
    a, b, C = _hadamard_coefs(q, a, b, C)
    if out is None:
        out = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=torch.float32,
                          device=q.device)
    _contig_cuda(q, k, v, a, b, C, out)
    rc = lib().oal_dense_hadamard_gpu(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(C),
                                      _ptr(out), ctypes.byref(shape), _stream(stream))
    _check(rc, "oal_dense_hadamard_gpu")
    return out


def prefill_varlen(qs, ks, vs, group_id, L, G, eps: float, chunk: int = 128, streams=None,
                   states=None, workspace=None):
    """oal_prefill_varlen over a list of sequences: qs[i] [Hq, T_i, 64], ks[i] / vs[i]
    [Hkv, T_i, 64] (same dtype and device).  The blocks are packed back to back into one
    buffer per tensor (the layout the call reads).  Returns (outs, states): outs[i] [Hq, T_i,
    64] fp32, states [n, stride] uint8 with row i the state of sequence i (continue it with
    decode_step).  ``streams`` (torch streams) run sequences side by side; default: the
    current stream alone."""
    n = len(qs)
    if not (len(ks) == len(vs) == n) or n == 0:
        raise ValueError("qs, ks, vs: equal, non-zero numbers of sequences")
    seq = [int(t.shape[1]) for t in qs]
    Hq, Hkv, dev = qs[0].shape[0], ks[0].shape[0], qs[0].device
    pack = lambda ts: torch.cat([t.contiguous().reshape(-1) for t in ts])  # noqa: E731
    q, k, v = pack(qs), pack(ks), pack(vs)
    shape = make_shape(1, max(seq), Hq, Hkv, chunk, _dtype_code(q), qs[0].shape[-1],
                       vs[0].shape[-1])
    lens = (ctypes.c_int32 * n)(*seq)
    if streams is None:
        streams = [torch.cuda.current_stream(dev)]
    handles = (ctypes.c_void_p * len(streams))(*[st.cuda_stream for st in streams])
    nb = _SZ(0)
    _check(lib().oal_prefill_varlen_workspace_bytes(ctypes.byref(shape), lens, n, len(streams),
                                                    ctypes.byref(nb)),
           "oal_prefill_varlen_workspace_bytes")
    stride = (state_bytes(make_shape(1, 1, Hq, Hkv, chunk, _dtype_code(q))) + 255) // 256 * 256
    out = torch.empty(Hq * sum(seq) * vs[0].shape[-1], dtype=torch.float32, device=dev)
    if states is None:
        states = torch.empty(n, stride, dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = empty_workspace(nb.value, dev)
    _contig_cuda(q, k, v, group_id, L, G, out, states, workspace)
    cur = torch.cuda.current_stream(dev)
    streams[0].wait_stream(cur)  # the packed inputs were written on the current stream
    rc = lib().oal_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                                  float(eps), _ptr(out), _ptr(states), stride, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  ctypes.byref(shape), lens, n, handles, len(streams))
    _check(rc, "oal_prefill_varlen")
    cur.wait_stream(streams[0])  # streams[0] already waits for every other stream
    outs, off = [], 0
    for t in seq:
        outs.append(out[off * Hq * 64:(off + t) * Hq * 64].view(Hq, t, 64))
        off += t
    return outs, states


def pack_sequences(qs, ks, vs):
    """The packed layout of a variable-length batch: qs[i] [Hq, T_i, 64], ks[i] / vs[i]
    [Hkv, T_i, 64] concatenated block after block into flat q, k, v; returns (q, k, v, lens)."""
    n = len(qs)
    if not (len(ks) == len(vs) == n) or n == 0:
        raise ValueError("qs, ks, vs: equal, non-zero numbers of sequences")
    pack = lambda ts: torch.cat([t.contiguous().reshape(-1) for t in ts])  # noqa: E731
    return pack(qs), pack(ks), pack(vs), [int(t.shape[1]) for t in qs]


def prefill_packed(q, k, v, lens, Hq: int, Hkv: int, group_id, L, G, eps: float, out=None,
                   states=None, workspace=None, stream=None):
    """oal_prefill_packed: the variable-length batch (packed as pack_sequences lays it out)
    in one launch per tensor-core kernel.  bf16 only (chunk 128).  Returns (out, states):
    out flat fp32 [Hq * sum(lens) * 64] (sequence i's [Hq, T_i, 64] block after the blocks
    before it), states [n, stride] uint8."""
    n = len(lens)
    dev = q.device
    shape = make_shape(1, max(lens) if n else 0, Hq, Hkv, 128, _dtype_code(q))
    c_lens = (ctypes.c_int32 * max(n, 1))(*lens)
    nb = _SZ(0)
    _check(lib().oal_prefill_packed_workspace_bytes(ctypes.byref(shape), c_lens, n,
                                                    ctypes.byref(nb)),
           "oal_prefill_packed_workspace_bytes")
    stride = (state_bytes(make_shape(1, 1, Hq, Hkv, 128, _dtype_code(q))) + 255) // 256 * 256
    if out is None:
        out = torch.empty(Hq * sum(lens) * 64, dtype=torch.float32, device=dev)
    if states is None:
        states = torch.empty(n, stride, dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = empty_workspace(nb.value, dev)
    _contig_cuda(q, k, v, group_id, L, G, out, states, workspace)
    rc = lib().oal_prefill_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                                  float(eps), _ptr(out), _ptr(states), stride, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  ctypes.byref(shape), c_lens, n, _stream(stream))
    _check(rc, "oal_prefill_packed")
    return out, states


def backward(q, k, v, group_id, L, G, eps: float, dy, stream=None, workspace=None) -> dict:
    """oal_backward: the training-scale (chunked, O(T)) gradients for dy = dLoss/dyhat
    [B, Hq, T, 64] fp32.  Returns dict(dq, dk, dv, dL, deps) of fp32 device tensors."""
    return _backward("oal_backward", q, k, v, group_id, L, G, eps, dy, stream, workspace)


def dense_backward(q, k, v, group_id, L, G, eps: float, dy, stream=None) -> dict:
    """oal_dense_backward_gpu: gradients of the dense causal form for dy = dLoss/dyhat
    [B, Hq, T, 64] fp32.  Returns dict(dq, dk, dv, dL, deps) of fp32 device tensors."""
    return _backward("oal_dense_backward_gpu", q, k, v, group_id, L, G, eps, dy, stream, None)


def _backward(name, q, k, v, group_id, L, G, eps, dy, stream, ws) -> dict:
    shape = _shape_of(q, k, v, 64)
    dev = q.device
    dy = dy.to(device=dev, dtype=torch.float32).contiguous()
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv_ = torch.empty(v.shape, dtype=torch.float32, device=dev)
    dL = torch.empty(L.shape, dtype=torch.float32, device=dev)
    deps = torch.empty(4, dtype=torch.float32, device=dev)
    if ws is None:
        n = _SZ(0)
        query = "oal_backward_workspace_bytes" if name == "oal_backward" else \
            "oal_dense_backward_workspace_bytes"
        _check(getattr(lib(), query)(ctypes.byref(shape), ctypes.byref(n)), query)
        ws = empty_workspace(n.value, dev)
    _contig_cuda(q, k, v, group_id, L, G, dy, dq, dk, dv_, dL, deps, ws)
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(group_id), _ptr(L), _ptr(G),
                              float(eps), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv_), _ptr(dL),
                              _ptr(deps), _ptr(ws), ws.numel() * ws.element_size(),
                              ctypes.byref(shape), _stream(stream))
    _check(rc, name)
    return dict(dq=dq, dk=dk, dv=dv_, dL=dL, deps=deps[0])


def backward_workspace(q, k, v) -> torch.Tensor:
    """A workspace for backward() on inputs of these shapes (reusable across calls)."""
    n = _SZ(0)
    _check(lib().oal_backward_workspace_bytes(ctypes.byref(_shape_of(q, k, v, 64)),
                                              ctypes.byref(n)), "oal_backward_workspace_bytes")
    return empty_workspace(n.value, q.device)


def launch_count() -> int:
    """Kernels launched by the library since it was loaded."""
    return int(lib().oal_launch_count())


def profile_enable(on: bool = True):
    _check(lib().oal_profile_enable(1 if on else 0), "oal_profile_enable")


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since the previous read (waits for them)."""
    arr = (KernelStat * 64)()
    n = ctypes.c_int(0)
    _check(lib().oal_profile_read(arr, 64, ctypes.byref(n)), "oal_profile_read")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
            for i in range(n.value)}


def set_prefill_overlap(overlap: bool) -> bool:
    """Launch the tensor-core prefill's scan and readout kernels as programmatic dependents
    (True) or in plain stream order (False); returns the previous setting."""
    return bool(lib().oal_set_prefill_overlap(1 if overlap else 0))


def set_debug_skip_copies(on: bool) -> bool:
    """Test hook: while on, the tensor-core readout issues no copies, so its bounded waits run
    out and it reports OAL_ERR_TIMEOUT (see include/oal.h); returns the previous setting."""
    return bool(lib().oal_set_debug_skip_copies(1 if on else 0))
