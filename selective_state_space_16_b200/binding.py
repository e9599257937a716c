"""ctypes binding of the C ABI in include/ssm_scan.h.

Argument marshalling only: every step of the scan runs in the CUDA kernels of
libssm_scan.so.  Tensors are torch tensors used purely as device memory; the
current torch CUDA stream is passed unless another stream is given.  If the
library has not been built this module raises on first use -- there is no CPU
fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_scan.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libssm_scan_debug.so")

(SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_LAUNCH, SSM_ERR_TIMEOUT, SSM_ERR_WORKSPACE,
 SSM_ERR_SCRATCH_LIMIT, SSM_ERR_BOUNDS) = range(8)
NOALLOC_SCRATCH_BYTES = 8 << 20
SSM_F32, SSM_BF16 = 0, 1
SSM_ALGO_AUTO, SSM_ALGO_SEQUENTIAL, SSM_ALGO_CHUNKED, SSM_ALGO_DIRECT = range(4)
ALGOS = {"auto": SSM_ALGO_AUTO, "sequential": SSM_ALGO_SEQUENTIAL, "chunked": SSM_ALGO_CHUNKED,
         "direct": SSM_ALGO_DIRECT}


class SsmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


SSM_DISC_SIMPLIFIED, SSM_DISC_ZOH = 0, 1


class FwdOptions(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int), ("lanes_per_channel", ctypes.c_int),
                ("spin_limit", ctypes.c_uint32), ("debug_skip_publish", ctypes.c_int),
                ("discretization", ctypes.c_int), ("checkpoints", ctypes.c_void_p)]


class ConvSpec(ctypes.Structure):
    """ssm_conv_t: causal conv1d + SiLU in front of the scan."""
    _fields_ = [("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("width", ctypes.c_int),
                ("state_in", ctypes.c_void_p), ("state_out", ctypes.c_void_p), ("u_out", ctypes.c_void_p)]


class BwdOptions(ctypes.Structure):
    """ssm_bwd_options_t: discretisation and conv prologue of a backward call."""
    _fields_ = [("discretization", ctypes.c_int), ("conv", ctypes.POINTER(ConvSpec)),
                ("dconv_weight", ctypes.c_void_p), ("dconv_bias", ctypes.c_void_p),
                ("dconv_state_in", ctypes.c_void_p), ("dconv_state_out", ctypes.c_void_p),
                ("checkpoints", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the argument and result types of every entry point of a loaded library."""
    vp, ci, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.ssm_abi_version.restype = ci
    lib.ssm_status_string.argtypes = [ci]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_selective_scan_workspace_size.argtypes = [ci, ci, ci, i64]
    lib.ssm_selective_scan_workspace_size.restype = sz
    lib.ssm_workspace_init.argtypes = [vp, sz, vp]
    lib.ssm_workspace_init.restype = ci
    fwd = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, ci, ci, ci, i64, ci, vp, sz]
    lib.ssm_selective_scan_fwd.argtypes = fwd + [vp]
    lib.ssm_selective_scan_fwd.restype = ci
    lib.ssm_selective_scan_fwd_ex.argtypes = fwd + [ctypes.POINTER(FwdOptions), vp]
    lib.ssm_selective_scan_fwd_ex.restype = ci
    lib.ssm_selective_scan_fwd_state.argtypes = fwd[:9] + [vp] + fwd[9:] + [ctypes.POINTER(FwdOptions), vp]
    lib.ssm_selective_scan_fwd_state.restype = ci
    lib.ssm_selective_scan_fwd_noalloc.argtypes = fwd[:16] + [vp]
    lib.ssm_selective_scan_fwd_noalloc.restype = ci
    lib.ssm_selective_scan_bwd_workspace_size.argtypes = [ci, ci, ci, i64]
    lib.ssm_selective_scan_bwd_workspace_size.restype = sz
    lib.ssm_selective_scan_bwd.argtypes = [vp] * 8 + [ci] + [vp] * 12 + [ci, ci, ci, i64, ci, vp, sz, vp]
    lib.ssm_selective_scan_bwd.restype = ci
    lib.ssm_selective_scan_bwd_ex.argtypes = ([vp] * 8 + [ci] + [vp] * 12 + [ci, ci, ci, i64, ci, vp, sz,
                                                                         ctypes.POINTER(BwdOptions), vp])
    lib.ssm_selective_scan_bwd_ex.restype = ci
    lib.ssm_state_update.argtypes = [vp] * 9 + [ci, vp, ci, ci, ci, ci, vp]
    lib.ssm_state_update.restype = ci
    lib.ssm_state_update_ex.argtypes = [vp] * 9 + [ci, vp, ci, ci, ci, ci, ci, vp]
    lib.ssm_state_update_ex.restype = ci
    lib.ssm_state_update_conv.argtypes = [vp] * 5 + [ci] + [vp] * 7 + [ci, vp, ci, ci, ci, ci, ci, vp]
    lib.ssm_state_update_conv.restype = ci
    lib.ssm_selective_scan_fwd_conv.argtypes = ([vp, ctypes.POINTER(ConvSpec)] + [vp] * 7 + [ci] +
                                                [vp] * 3 + [ci, ci, ci, i64, ci, vp, sz,
                                                            ctypes.POINTER(FwdOptions), vp])
    lib.ssm_selective_scan_fwd_conv.restype = ci
    lib.ssm_read_status.argtypes = [vp, vp]
    lib.ssm_read_status.restype = ci
    return lib


def load() -> ctypes.CDLL:
    """Load libssm_scan.so (raises if it was not built: run __graft_entry__.build())."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing; build it with selective_state_space_16_b200/build.py")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


@contextlib.contextmanager
def use_debug_library():
    """Route every call of this module through libssm_scan_debug.so (the range-checked
    build) inside the `with` block."""
    global _lib
    if not os.path.exists(DEBUG_LIB_PATH):
        raise ImportError(f"{DEBUG_LIB_PATH} is missing; build it with build.py --debug")
    debug = _declare(ctypes.CDLL(DEBUG_LIB_PATH))
    base = load()  # (before taking the lock, which load() takes itself)
    with _lock:
        saved = _lib if _lib is not None else base
        _lib = debug
    try:
        yield debug
    finally:
        with _lock:
            _lib = saved


def status_string(code: int) -> str:
    return load().ssm_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _io(t):
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"unsupported I/O dtype {t.dtype}")


def _check(code, where):
    if code != SSM_OK:
        raise SsmError(code, where)


def ssm_selective_scan_workspace_size(batch: int, dim: int, dstate: int, seqlen: int) -> int:
    return int(load().ssm_selective_scan_workspace_size(batch, dim, dstate, seqlen))


def ssm_workspace_init(workspace, stream=None):
    _check(load().ssm_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "ssm_workspace_init")


def new_workspace(batch, dim, dstate, seqlen, device="cuda", stream=None):
    """Allocate (with torch) and zero a workspace large enough for these sizes."""
    n = max(ssm_selective_scan_workspace_size(batch, dim, dstate, seqlen), 256)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ssm_workspace_init(ws, stream)
    return ws


def ssm_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, workspace,
                           stream=None, algo=None, lanes_per_channel=0, spin_limit=0, debug_skip_publish=-1,
                           check=True, initial_state=None, zoh=False, checkpoints=None):
    """Marshal a forward-scan call.  u/delta/z/y: (b, d, L); B/C: (b, N, L); A: (d, N) fp32;
    D/delta_bias: (d) fp32 or None; last_state: (b, d, N) fp32 or None; workspace: uint8;
    initial_state: (b, d, N) fp32 or None (zero), through ssm_selective_scan_fwd_state;
    zoh: zero-order-hold discretisation instead of the simplified one; checkpoints:
    (b, ceil(L/8), d, N) fp32 output for the backward, or None."""
    lib = load()
    b, d, L = u.shape
    n = A.shape[1]
    head = [_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus))]
    tail = [_ptr(y), _ptr(last_state), b, d, n, L, _io(u), _ptr(workspace),
            workspace.numel() * workspace.element_size()]
    default_opts = (algo is None and lanes_per_channel == 0 and spin_limit == 0 and debug_skip_publish < 0
                    and not zoh and checkpoints is None)
    if default_opts and initial_state is None:
        code = lib.ssm_selective_scan_fwd(*head, *tail, _stream(stream))
    else:
        a = ALGOS[algo] if isinstance(algo, str) else (algo or SSM_ALGO_AUTO)
        opts = FwdOptions(a, lanes_per_channel, spin_limit, debug_skip_publish,
                          SSM_DISC_ZOH if zoh else SSM_DISC_SIMPLIFIED, _ptr(checkpoints))
        if initial_state is None:
            code = lib.ssm_selective_scan_fwd_ex(*head, *tail, ctypes.byref(opts), _stream(stream))
        else:
            code = lib.ssm_selective_scan_fwd_state(*head, _ptr(initial_state), *tail, ctypes.byref(opts),
                                                    _stream(stream))
    if check:
        _check(code, "ssm_selective_scan_fwd")
    return code


def ssm_selective_scan_fwd_noalloc(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, stream=None,
                                   check=True):
    """Marshal a call of the forward scan that allocates nothing and takes no workspace
    (its scratch is a fixed array inside the library; see include/ssm_scan.h)."""
    b, d, L = u.shape
    n = A.shape[1]
    code = load().ssm_selective_scan_fwd_noalloc(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                                 _ptr(delta_bias), int(bool(softplus)), _ptr(y), _ptr(last_state),
                                                 b, d, n, L, _io(u), _stream(stream))
    if check:
        _check(code, "ssm_selective_scan_fwd_noalloc")
    return code


def ssm_selective_scan_bwd_workspace_size(batch: int, dim: int, dstate: int, seqlen: int) -> int:
    return int(load().ssm_selective_scan_bwd_workspace_size(batch, dim, dstate, seqlen))


def ssm_selective_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus, dy, du, ddelta, dA, dB, dC, dD, dz,
                           ddelta_bias, workspace, initial_state=None, dlast_state=None, dinitial_state=None,
                           stream=None, check=True):
    """Marshal a backward call (shapes as the forward; dA (d, N), dB/dC (b, N, L) fp32;
    dD/ddelta_bias (d) fp32 or None; dinitial_state (b, d, N) fp32 or None)."""
    b, d, L = u.shape
    n = A.shape[1]
    code = load().ssm_selective_scan_bwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
        _ptr(initial_state), _ptr(dy), _ptr(dlast_state), _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC),
        _ptr(dD), _ptr(dz), _ptr(ddelta_bias), _ptr(dinitial_state), b, d, n, L, _io(u), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    if check:
        _check(code, "ssm_selective_scan_bwd")
    return code


def ssm_selective_scan_bwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus, dy, du, ddelta, dA, dB, dC, dD, dz,
                              ddelta_bias, workspace, initial_state=None, dlast_state=None, dinitial_state=None,
                              zoh=False, conv_weight=None, conv_bias=None, conv_state_in=None, dconv_weight=None,
                              dconv_bias=None, dconv_state_in=None, dconv_state_out=None, checkpoints=None,
                              stream=None, check=True):
    """Marshal ssm_selective_scan_bwd_ex: as ssm_selective_scan_bwd, plus zoh and, when
    conv_weight (d, K) fp32 is given, the conv prologue: u is then x and du receives dx;
    dconv_weight (d, K), dconv_bias (d), dconv_state_in / dconv_state_out (b, d, K-1) fp32;
    checkpoints: the forward's (b, ceil(L/8), d, N) fp32, or None."""
    b, d, L = u.shape
    n = A.shape[1]
    spec = None
    if conv_weight is not None:
        spec = ConvSpec(_ptr(conv_weight), _ptr(conv_bias), int(conv_weight.shape[1]), _ptr(conv_state_in), None,
                        None)
    opts = BwdOptions(SSM_DISC_ZOH if zoh else SSM_DISC_SIMPLIFIED,
                      ctypes.pointer(spec) if spec is not None else None, _ptr(dconv_weight), _ptr(dconv_bias),
                      _ptr(dconv_state_in), _ptr(dconv_state_out), _ptr(checkpoints))
    code = load().ssm_selective_scan_bwd_ex(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
        _ptr(initial_state), _ptr(dy), _ptr(dlast_state), _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC),
        _ptr(dD), _ptr(dz), _ptr(ddelta_bias), _ptr(dinitial_state), b, d, n, L, _io(u), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(opts), _stream(stream))
    if check:
        _check(code, "ssm_selective_scan_bwd_ex")
    return code


def selective_scan_bwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, dy=None,
                       initial_state=None, dlast_state=None, workspace=None, stream=None, zoh=False,
                       conv_weight=None, conv_bias=None, conv_state_in=None, dconv_state_out=None,
                       checkpoints=None):
    """Convenience wrapper: allocates every gradient and, if not given, a workspace, then
    calls ssm_selective_scan_bwd (ssm_selective_scan_bwd_ex with zoh or a conv).  Returns a dict
    du, ddelta, dz (or None), dA, dB, dC, dD, ddelta_bias, dinitial_state; with conv_weight
    (u is then the conv input x) also dx (in place of du, which is then None), dconv_weight,
    dconv_bias and dconv_state_in (None for width 1)."""
    b, d, L = u.shape
    n = A.shape[1]
    f32 = dict(dtype=torch.float32, device=u.device)
    out = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u), dz=torch.empty_like(u) if z is not None else None,
               dA=torch.empty((d, n), **f32), dB=torch.empty((b, n, L), **f32), dC=torch.empty((b, n, L), **f32),
               dD=torch.empty(d, **f32), ddelta_bias=torch.empty(d, **f32),
               dinitial_state=torch.empty((b, d, n), **f32))
    if workspace is None:
        workspace = torch.empty(max(ssm_selective_scan_bwd_workspace_size(b, d, n, L), 256), dtype=torch.uint8,
                                device=u.device)
    if not zoh and conv_weight is None and checkpoints is None:
        ssm_selective_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus, dy, out["du"], out["ddelta"],
                               out["dA"], out["dB"], out["dC"], out["dD"], out["dz"], out["ddelta_bias"], workspace,
                               initial_state=initial_state, dlast_state=dlast_state,
                               dinitial_state=out["dinitial_state"], stream=stream)
        return out
    if conv_weight is not None:
        K = int(conv_weight.shape[1])
        out["dx"] = out.pop("du")
        out["du"] = None
        out["dconv_weight"] = torch.empty((d, K), **f32)
        out["dconv_bias"] = torch.empty(d, **f32)
        out["dconv_state_in"] = torch.empty((b, d, K - 1), **f32) if K > 1 else None
    ssm_selective_scan_bwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus, dy,
                              out["dx"] if conv_weight is not None else out["du"], out["ddelta"], out["dA"],
                              out["dB"], out["dC"], out["dD"], out["dz"], out["ddelta_bias"], workspace,
                              initial_state=initial_state, dlast_state=dlast_state,
                              dinitial_state=out["dinitial_state"], zoh=zoh, conv_weight=conv_weight,
                              conv_bias=conv_bias, conv_state_in=conv_state_in,
                              dconv_weight=out.get("dconv_weight"), dconv_bias=out.get("dconv_bias"),
                              dconv_state_in=out.get("dconv_state_in"), dconv_state_out=dconv_state_out,
                              checkpoints=checkpoints, stream=stream)
    return out


def ssm_selective_scan_fwd_conv(x, conv_weight, conv_bias, delta, A, B, C, D, z, delta_bias, softplus, y, last_state,
                                workspace, conv_state_in=None, conv_state_out=None, u_out=None, initial_state=None,
                                stream=None, algo=None, lanes_per_channel=0, zoh=False, check=True,
                                checkpoints=None):
    """Marshal a forward scan of u = silu(causal conv(x)): x (b, d, L) in the I/O dtype;
    conv_weight (d, K) fp32; conv_bias (d) fp32 or None; conv_state_in/out (b, d, K-1) fp32 or
    None; u_out (b, d, L) I/O dtype or None; checkpoints as ssm_selective_scan_fwd."""
    b, d, L = x.shape
    n = A.shape[1]
    spec = ConvSpec(_ptr(conv_weight), _ptr(conv_bias), int(conv_weight.shape[1]), _ptr(conv_state_in),
                    _ptr(conv_state_out), _ptr(u_out))
    a = ALGOS[algo] if isinstance(algo, str) else (algo or SSM_ALGO_AUTO)
    opts = FwdOptions(a, lanes_per_channel, 0, -1, SSM_DISC_ZOH if zoh else SSM_DISC_SIMPLIFIED, _ptr(checkpoints))
    code = load().ssm_selective_scan_fwd_conv(
        _ptr(x), ctypes.byref(spec), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        int(bool(softplus)), _ptr(initial_state), _ptr(y), _ptr(last_state), b, d, n, L, _io(x), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(opts), _stream(stream))
    if check:
        _check(code, "ssm_selective_scan_fwd_conv")
    return code


def ssm_state_update_conv(state, conv_state, x, conv_weight, conv_bias, delta, A, B, C, D, z, delta_bias, softplus,
                          y, zoh=False, stream=None, check=True):
    """Marshal a decode step with the conv prologue: conv_state (b, d, K-1) fp32 in/out."""
    b, d, n = state.shape
    code = load().ssm_state_update_conv(
        _ptr(state), _ptr(conv_state), _ptr(x), _ptr(conv_weight), _ptr(conv_bias), int(conv_weight.shape[1]),
        _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)), _ptr(y),
        b, d, n, _io(x), SSM_DISC_ZOH if zoh else SSM_DISC_SIMPLIFIED, _stream(stream))
    if check:
        _check(code, "ssm_state_update_conv")
    return code


def ssm_state_update(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, stream=None, check=True, zoh=False):
    """Marshal a decode call.  state: (b, d, N) fp32 in/out; u/delta/z/y: (b, d); B/C: (b, N);
    zoh: zero-order-hold discretisation (ssm_state_update_ex)."""
    b, d, n = state.shape
    args = [_ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)), _ptr(y), b, d, n, _io(u)]
    if zoh:
        code = load().ssm_state_update_ex(*args, SSM_DISC_ZOH, _stream(stream))
    else:
        code = load().ssm_state_update(*args, _stream(stream))
    if check:
        _check(code, "ssm_state_update")
    return code


def ssm_read_status(workspace, stream=None) -> int:
    return int(load().ssm_read_status(_ptr(workspace), _stream(stream)))


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                       return_last_state=True, workspace=None, stream=None, initial_state=None, **opts):
    """Convenience wrapper: allocates y (u's dtype), last_state (fp32) and, if not given,
    a workspace, then calls ssm_selective_scan_fwd (from initial_state when given).
    Returns (y, last_state)."""
    b, d, L = u.shape
    n = A.shape[1]
    y = torch.empty_like(u)
    last = torch.empty((b, d, n), dtype=torch.float32, device=u.device) if return_last_state else None
    if workspace is None:
        workspace = new_workspace(b, d, n, L, device=u.device, stream=stream)
    ssm_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, y, last, workspace,
                           stream=stream, initial_state=initial_state, **opts)
    return y, last
