"""fp64 CPU oracle for OAL causal grouped positive-quadratic attention.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU-baseline leg of the
benchmark are the only callers; the product path (the CUDA library and its binding) never
imports this package, and this package never imports the product.

The arithmetic lives in ``oal_oracle.c`` (plain C, fp64, OpenMP over (batch, query head));
this module compiles it with gcc on first use and marshals numpy arrays through ctypes.
Formulas follow "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of arXiv
2610.13674), section 核心公式, equations numbered in order of appearance:
(1) contribution statistic, (2) grouped score s_g, (3) kernel kappa, (4) prefix states
H0/H1/H2, (5) readout and normalisation.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oal_oracle.c")
_LIB = os.path.join(_HERE, "liboal_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile oal_oracle.c into liboal_oracle.so next to it (gcc -O2 -fno-fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-Wall",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oal_oracle_kappa.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _D, _D, _I,
                                             _D, ctypes.c_int, ctypes.c_int, ctypes.c_double, _D]
            lib.oal_oracle_dense.argtypes = [ctypes.c_int] * 6 + [_D, _D, _D, _I, _D, _I,
                                                                  ctypes.c_int, ctypes.c_double,
                                                                  _D, _D]
            lib.oal_oracle_recurrent.argtypes = [ctypes.c_int] * 6 + [_D, _D, _D, _I, _D, _I,
                                                                      ctypes.c_int,
                                                                      ctypes.c_double] + [_D] * 7
            lib.oal_oracle_dense_rows.argtypes = [ctypes.c_int] * 6 + [_D, _D, _D, _I, _D, _I,
                                                                       ctypes.c_int,
                                                                       ctypes.c_double,
                                                                       ctypes.c_int, _I, _I, _I,
                                                                       _D]
            lib.oal_oracle_chi.argtypes = [ctypes.c_int] * 5 + [_D, _D, _D]
            lib.oal_oracle_hadamard_recurrent.argtypes = [ctypes.c_int] * 6 + [_D] * 14
            lib.oal_oracle_hadamard_dense.argtypes = [ctypes.c_int] * 6 + [_D] * 8
            lib.oal_oracle_dense_backward.argtypes = [ctypes.c_int] * 6 + [
                _D, _D, _D, _I, _D, _I, ctypes.c_int, ctypes.c_double] + [_D] * 6
            for f in (lib.oal_oracle_kappa, lib.oal_oracle_dense, lib.oal_oracle_recurrent,
                      lib.oal_oracle_dense_rows, lib.oal_oracle_chi,
                      lib.oal_oracle_hadamard_recurrent, lib.oal_oracle_hadamard_dense,
                      lib.oal_oracle_dense_backward):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _d(a):
    return None if a is None else a.ctypes.data_as(_D)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc} (bad arguments or out of memory)")


def _common(q, k, v, group_id, L, G):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, T, d]")
    B, Hq, T, dh = q.shape
    Hkv, dv = k.shape[1], v.shape[3]
    if k.shape != (B, Hkv, T, dh) or v.shape != (B, Hkv, T, dv):
        raise ValueError("k/v shape mismatch")
    group_id, G, L = _i32(group_id), _i32(G), _f64(L)
    Gmax = L.shape[-1] - 1
    if group_id.shape != (Hq, dh) or G.shape != (Hq,) or L.shape != (Hq, Gmax + 1, Gmax + 1):
        raise ValueError("group_id [Hq, dh], G [Hq], L [Hq, Gmax+1, Gmax+1] expected")
    return q, k, v, group_id, L, G, (B, Hq, Hkv, T, dh, dv, Gmax)


def kappa(q, k, group_id, L, G, eps):
    """kappa(q_i, k_j) for one head over all (i, j), no causal mask (eqs. 2-3).

    q [Tq, dh], k [Tk, dh], group_id [dh], L [Gmax+1, Gmax+1], G int."""
    q, k, group_id, L = _f64(q), _f64(k), _i32(group_id), _f64(L)
    out = np.empty((q.shape[0], k.shape[0]), np.float64)
    rc = _load().oal_oracle_kappa(q.shape[0], k.shape[0], q.shape[1], _d(q), _d(k),
                                  group_id.ctypes.data_as(_I), _d(L), int(G), L.shape[0] - 1,
                                  float(eps), _d(out))
    _check(rc, "kappa")
    return out


def dense(q, k, v, group_id, L, G, eps, return_den: bool = False):
    """Dense causal definition: yhat_i = sum_{j<=i} kappa_ij v_j / sum_{j<=i} kappa_ij."""
    q, k, v, group_id, L, G, (B, Hq, Hkv, T, dh, dv, Gmax) = _common(q, k, v, group_id, L, G)
    y = np.empty((B, Hq, T, dv), np.float64)
    den = np.empty((B, Hq, T), np.float64) if return_den else None
    rc = _load().oal_oracle_dense(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v),
                                  group_id.ctypes.data_as(_I), _d(L), G.ctypes.data_as(_I), Gmax,
                                  float(eps), _d(y), _d(den))
    _check(rc, "dense")
    return (y, den) if return_den else y


def dense_rows(q, k, v, group_id, L, G, eps, rows):
    """Dense-definition outputs for selected (b, h, i) triples only -> [len(rows), dv]."""
    q, k, v, group_id, L, G, (B, Hq, Hkv, T, dh, dv, Gmax) = _common(q, k, v, group_id, L, G)
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    rb, rh, ri = (_i32(rows[:, c]) for c in range(3))
    y = np.empty((rows.shape[0], dv), np.float64)
    rc = _load().oal_oracle_dense_rows(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v),
                                       group_id.ctypes.data_as(_I), _d(L), G.ctypes.data_as(_I),
                                       Gmax, float(eps), rows.shape[0], rb.ctypes.data_as(_I),
                                       rh.ctypes.data_as(_I), ri.ctypes.data_as(_I), _d(y))
    _check(rc, "dense_rows")
    return y


class State:
    """Prefix state of eq. (4) per (batch, key/value head): H0 [B,Hkv,dv+1],
    H1 [B,Hkv,dh,dv+1], H2 [B,Hkv,dh,dh,dv+1] (fp64, full unpacked d_h x d_h)."""

    def __init__(self, H0, H1, H2):
        self.H0, self.H1, self.H2 = _f64(H0), _f64(H1), _f64(H2)

    @classmethod
    def zeros(cls, B, Hkv, dh, dv):
        w = dv + 1
        return cls(np.zeros((B, Hkv, w)), np.zeros((B, Hkv, dh, w)),
                   np.zeros((B, Hkv, dh, dh, w)))


def recurrent(q, k, v, group_id, L, G, eps, state: State | None = None,
              return_state: bool = False):
    """H0/H1/H2 recurrence (eqs. 4-5), token by token, continuing from ``state``."""
    q, k, v, group_id, L, G, (B, Hq, Hkv, T, dh, dv, Gmax) = _common(q, k, v, group_id, L, G)
    y = np.empty((B, Hq, T, dv), np.float64)
    out = State.zeros(B, Hkv, dh, dv) if return_state else None
    ins = (state.H0, state.H1, state.H2) if state is not None else (None, None, None)
    outs = (out.H0, out.H1, out.H2) if out is not None else (None, None, None)
    rc = _load().oal_oracle_recurrent(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v),
                                      group_id.ctypes.data_as(_I), _d(L), G.ctypes.data_as(_I),
                                      Gmax, float(eps), *[_d(a) for a in ins],
                                      *[_d(a) for a in outs], _d(y))
    _check(rc, "recurrent")
    return (y, out) if return_state else y


def chi(q, k):
    """Contribution statistic of eq. (1) per prompt (b, query head): [B, Hq, dh].  The
    statistic chi_r of the page is chi(q, k).mean(axis=0) for the prompts of a head."""
    q, k = _f64(q), _f64(k)
    if q.ndim != 4 or k.ndim != 4 or k.shape[0] != q.shape[0] or k.shape[2:] != q.shape[2:]:
        raise ValueError("q [B, Hq, T, dh] and k [B, Hkv, T, dh] expected")
    B, Hq, T, dh = q.shape
    out = np.zeros((B, Hq, dh), dtype=np.float64)
    _check(_load().oal_oracle_chi(B, Hq, k.shape[1], T, dh, _d(q), _d(k), _d(out)),
           "oal_oracle_chi")
    return out


def grouped_coefficients(group_id, L, G, eps):
    """Coefficients (a [Hq], b [Hq, dh], C [Hq, dh, dh]) of eq. (5) that the grouped kernel of
    eq. (3) expands into, with M = L L^T over each head's leading (G+1)x(G+1) block and
    sbar_0 = 1: a = eps + M_00, b_r = 2 M_{0,g(r)}, C_rt = M_{g(r),g(t)}."""
    group_id, G, L = _i32(group_id), _i32(G), _f64(L)
    Hq, dh = group_id.shape
    a, b, C = np.empty(Hq), np.empty((Hq, dh)), np.empty((Hq, dh, dh))
    for h in range(Hq):
        n = int(G[h]) + 1
        M = L[h, :n, :n] @ L[h, :n, :n].T
        g = group_id[h]
        a[h] = eps + M[0, 0]
        b[h] = 2.0 * M[0, g]
        C[h] = M[np.ix_(g, g)]
    return a, b, C


def _hadamard_common(q, k, v, a, b, C):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, T, d]")
    B, Hq, T, dh = q.shape
    Hkv, dv = k.shape[1], v.shape[3]
    if k.shape != (B, Hkv, T, dh) or v.shape != (B, Hkv, T, dv):
        raise ValueError("k/v shape mismatch")
    a, b, C = _f64(np.reshape(a, (Hq,))), _f64(b), _f64(C)
    if b.shape != (Hq, dh) or C.shape != (Hq, dh, dh):
        raise ValueError("a [Hq], b [Hq, dh], C [Hq, dh, dh] expected")
    return q, k, v, a, b, C, (B, Hq, Hkv, T, dh, dv)


def hadamard_dense(q, k, v, a, b, C, return_u: bool = False):
    """Ungrouped Hadamard form, dense: kappa = a + sum_r b_r x_r + sum_rt C_rt x_r x_t with
    x = q*k/sqrt(dh), u_i = sum_{j<=i} kappa_ij [v_j; 1], yhat_i = u_i[:dv] / u_i[dv]."""
    q, k, v, a, b, C, (B, Hq, Hkv, T, dh, dv) = _hadamard_common(q, k, v, a, b, C)
    y = np.empty((B, Hq, T, dv))
    u = np.empty((B, Hq, T, dv + 1)) if return_u else None
    _check(_load().oal_oracle_hadamard_dense(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v), _d(a),
                                             _d(b), _d(C), _d(y), _d(u)), "hadamard_dense")
    return (y, u) if return_u else y


def hadamard_recurrent(q, k, v, a, b, C, state: State | None = None,
                       return_state: bool = False, return_u: bool = False):
    """Ungrouped Hadamard form through eqs. (4)-(5) with the given a, b, C.  Returns y, then
    the state after the tokens (return_state) and u [B, Hq, T, dv+1] (return_u)."""
    q, k, v, a, b, C, (B, Hq, Hkv, T, dh, dv) = _hadamard_common(q, k, v, a, b, C)
    y = np.empty((B, Hq, T, dv))
    u = np.empty((B, Hq, T, dv + 1)) if return_u else None
    out = State.zeros(B, Hkv, dh, dv) if return_state else None
    ins = (state.H0, state.H1, state.H2) if state is not None else (None, None, None)
    outs = (out.H0, out.H1, out.H2) if out is not None else (None, None, None)
    _check(_load().oal_oracle_hadamard_recurrent(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v),
                                                 _d(a), _d(b), _d(C), *[_d(x) for x in ins],
                                                 *[_d(x) for x in outs], _d(y), _d(u)),
           "hadamard_recurrent")
    res = [y] + ([out] if return_state else []) + ([u] if return_u else [])
    return res[0] if len(res) == 1 else tuple(res)


def dense_backward(q, k, v, group_id, L, G, eps, dy):
    """Gradients of the dense grouped form for upstream dy = dLoss/dyhat [B, Hq, T, dv]:
    dict(dq, dk, dv, dL [Hq, Gmax+1, Gmax+1], deps)."""
    q, k, v, group_id, L, G, (B, Hq, Hkv, T, dh, dv, Gmax) = _common(q, k, v, group_id, L, G)
    dy = _f64(dy)
    if dy.shape != (B, Hq, T, dv):
        raise ValueError("dy must be [B, Hq, T, dv]")
    dq, dk, dvv = np.empty(q.shape), np.empty(k.shape), np.empty(v.shape)
    dL = np.empty(L.shape)
    deps = np.zeros(1)
    _check(_load().oal_oracle_dense_backward(B, Hq, Hkv, T, dh, dv, _d(q), _d(k), _d(v),
                                             group_id.ctypes.data_as(_I), _d(L),
                                             G.ctypes.data_as(_I), Gmax, float(eps), _d(dy),
                                             _d(dq), _d(dk), _d(dvv), _d(dL), _d(deps)),
           "dense_backward")
    return dict(dq=dq, dk=dk, dv=dvv, dL=dL, deps=float(deps[0]))


def threads() -> int:
    """Number of OpenMP threads the oracle will use (OMP_NUM_THREADS or all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else (os.cpu_count() or 1)
