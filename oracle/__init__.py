"""fp64 CPU oracle for the selective state-space scan (S6).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__.py and by the cpu_baseline / reference leg of bench.py, and by
nothing in the product package.  It shares no code with the CUDA library.

The arithmetic lives in ``ssm_oracle.c`` (plain C, fp64, OpenMP over the
independent (batch, channel) rows); this module only compiles it with gcc and
marshals numpy arrays to it.  Every array is converted to contiguous float64
first, so bf16 / fp32 inputs enter the oracle exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP); returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            lib.oracle_selective_scan_f64.argtypes = [vp] * 8 + [ci, vp, vp, vp, i64, i64, i64, i64]
            lib.oracle_selective_scan_f64.restype = ci
            lib.oracle_state_update_f64.argtypes = [vp] * 9 + [ci, vp, i64, i64, i64]
            lib.oracle_state_update_f64.restype = ci
            lib.oracle_selective_scan_zoh_f64.argtypes = [vp] * 8 + [ci, vp, vp, vp, i64, i64, i64, i64, ci]
            lib.oracle_selective_scan_zoh_f64.restype = ci
            lib.oracle_state_update_zoh_f64.argtypes = [vp] * 9 + [ci, vp, i64, i64, i64, ci]
            lib.oracle_state_update_zoh_f64.restype = ci
            lib.oracle_selective_scan_bwd_f64.argtypes = [vp] * 8 + [ci] + [vp] * 12 + [i64, i64, i64, i64]
            lib.oracle_selective_scan_bwd_f64.restype = ci
            lib.oracle_selective_scan_bwd_zoh_f64.argtypes = [vp] * 8 + [ci] + [vp] * 12 + [i64, i64, i64, i64, ci]
            lib.oracle_selective_scan_bwd_zoh_f64.restype = ci
            lib.oracle_causal_conv_silu_bwd_f64.argtypes = [vp] * 10 + [i64, i64, i64, i64]
            lib.oracle_causal_conv_silu_bwd_f64.restype = ci
            lib.oracle_causal_conv_silu_f64.argtypes = [vp] * 6 + [i64, i64, i64, i64]
            lib.oracle_causal_conv_silu_f64.restype = ci
            lib.oracle_num_threads.restype = ci
            lib.oracle_softplus_f64.argtypes = [ctypes.c_double]
            lib.oracle_softplus_f64.restype = ctypes.c_double
            lib.oracle_silu_f64.argtypes = [ctypes.c_double]
            lib.oracle_silu_f64.restype = ctypes.c_double
            _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> numpy, exact upcast
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def softplus(x: float) -> float:
    return float(_load().oracle_softplus_f64(float(x)))


def silu(x: float) -> float:
    return float(_load().oracle_silu_f64(float(x)))


def selective_scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, h0=None, zoh=False):
    """Forward scan.  Shapes: u/delta/z (b, d, L); B/C (b, N, L); A (d, N); D/delta_bias (d);
    h0 (b, d, N) or None; zoh: zero-order-hold input weight instead of Delta*B.
    Returns (y (b, d, L), last_state (b, d, N)) as float64 arrays."""
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    D, z, delta_bias, h0 = map(_f64, (D, z, delta_bias, h0))
    b, d, L = u.shape
    n = A.shape[1]
    assert delta.shape == u.shape and A.shape == (d, n) and B.shape == (b, n, L) and C.shape == (b, n, L)
    assert z is None or z.shape == u.shape
    assert h0 is None or h0.shape == (b, d, n)
    y = np.empty((b, d, L), dtype=np.float64)
    last = np.empty((b, d, n), dtype=np.float64)
    rc = _load().oracle_selective_scan_zoh_f64(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                               _ptr(z), _ptr(delta_bias), int(bool(softplus)), _ptr(h0),
                                               _ptr(y), _ptr(last), b, d, n, L, int(bool(zoh)))
    if rc != 0:
        raise ValueError("oracle_selective_scan_f64 rejected its arguments")
    return y, last


def state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, zoh=False):
    """One decode step.  state (b, d, N) is NOT modified; returns (y (b, d), new_state)."""
    st = _f64(state).copy()
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    D, z, delta_bias = map(_f64, (D, z, delta_bias))
    b, d, n = st.shape
    assert u.shape == (b, d) and delta.shape == (b, d) and A.shape == (d, n)
    assert B.shape == (b, n) and C.shape == (b, n)
    y = np.empty((b, d), dtype=np.float64)
    rc = _load().oracle_state_update_zoh_f64(_ptr(st), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                             _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
                                             _ptr(y), b, d, n, int(bool(zoh)))
    if rc != 0:
        raise ValueError("oracle_state_update_f64 rejected its arguments")
    return y, st


def selective_scan_bwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, h0=None, dy=None,
                       dlast=None, zoh=False):
    """Gradients of L = sum(dy * y) + sum(dlast * last_state) for the forward scan with these
    inputs (zoh: of the zero-order-hold scan).  Returns a dict of float64 arrays: du, ddelta
    (b, d, L); dA (d, N); dB, dC (b, N, L); dD, ddelta_bias (d) (always, as if D / delta_bias
    were given); dz (b, d, L) or None; dh0 (b, d, N) (the gradient with respect to the initial
    state, zero or h0)."""
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    D, z, delta_bias, h0, dy, dlast = map(_f64, (D, z, delta_bias, h0, dy, dlast))
    b, d, L = u.shape
    n = A.shape[1]
    assert dy is not None and dy.shape == u.shape
    assert dlast is None or dlast.shape == (b, d, n)
    out = dict(du=np.empty((b, d, L)), ddelta=np.empty((b, d, L)), dA=np.empty((d, n)),
               dB=np.empty((b, n, L)), dC=np.empty((b, n, L)), dD=np.empty(d), ddelta_bias=np.empty(d),
               dz=np.empty((b, d, L)) if z is not None else None, dh0=np.empty((b, d, n)))
    rc = _load().oracle_selective_scan_bwd_zoh_f64(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
        _ptr(h0), _ptr(dy), _ptr(dlast), _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]),
        _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dz"]), _ptr(out["ddelta_bias"]), _ptr(out["dh0"]), b, d, n, L,
        int(bool(zoh)))
    if rc != 0:
        raise ValueError("oracle_selective_scan_bwd_f64 rejected its arguments")
    return out


def causal_conv_silu(x, w, bias=None, x_prev=None):
    """u = silu(causal depthwise conv of x with w (dim, K) + bias), inputs before t = 0 taken
    from x_prev (batch, dim, K-1) or zero.  Returns (u (b, d, L), x_next (b, d, K-1)): the
    output and the last K-1 inputs (the state that continues the convolution)."""
    x, w, bias, x_prev = map(_f64, (x, w, bias, x_prev))
    b, d, L = x.shape
    K = w.shape[1]
    assert w.shape == (d, K) and (x_prev is None or x_prev.shape == (b, d, K - 1))
    u = np.empty((b, d, L))
    x_next = np.empty((b, d, max(K - 1, 0)))
    rc = _load().oracle_causal_conv_silu_f64(_ptr(x), _ptr(w), _ptr(bias), _ptr(x_prev), _ptr(u),
                                             _ptr(x_next) if K > 1 else None, b, d, L, K)
    if rc != 0:
        raise ValueError("oracle_causal_conv_silu_f64 rejected its arguments")
    return u, x_next


def causal_conv_silu_bwd(x, w, du, bias=None, x_prev=None, dx_next=None):
    """Gradients through causal_conv_silu, given du = dL/du (b, d, L) and optionally dx_next =
    dL/d x_next (b, d, K-1).  Returns a dict of float64 arrays: dx (b, d, L), dw (d, K),
    dbias (d) (always, as if bias were given), dx_prev (b, d, K-1)."""
    x, w, du, bias, x_prev, dx_next = map(_f64, (x, w, du, bias, x_prev, dx_next))
    b, d, L = x.shape
    K = w.shape[1]
    assert w.shape == (d, K) and du.shape == x.shape
    assert x_prev is None or x_prev.shape == (b, d, K - 1)
    assert dx_next is None or dx_next.shape == (b, d, K - 1)
    out = dict(dx=np.empty((b, d, L)), dw=np.empty((d, K)), dbias=np.empty(d), dx_prev=np.empty((b, d, K - 1)))
    rc = _load().oracle_causal_conv_silu_bwd_f64(_ptr(x), _ptr(w), _ptr(bias), _ptr(x_prev), _ptr(du),
                                                 _ptr(dx_next), _ptr(out["dx"]), _ptr(out["dw"]),
                                                 _ptr(out["dbias"]), _ptr(out["dx_prev"]) if K > 1 else None,
                                                 b, d, L, K)
    if rc != 0:
        raise ValueError("oracle_causal_conv_silu_bwd_f64 rejected its arguments")
    return out
