"""CPU-only checks of the C ABI: the library loads, exports every entry point that
include/*.h declares, and rejects bad arguments before touching any device."""
import ctypes
import glob
import os
import re

import pytest

import selective_state_space_16_b200 as ssm
from selective_state_space_16_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(ssm_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_16_b200 import build as b
    b.build()
    return ssm.load()


def test_header_declares_entry_points():
    names = _declared_functions()
    for n in ["ssm_selective_scan_fwd", "ssm_state_update", "ssm_selective_scan_workspace_size",
              "ssm_read_status", "ssm_selective_scan_fwd_ex", "ssm_workspace_init",
              "ssm_selective_scan_fwd_state"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.ssm_abi_version() == 3


def test_status_strings(lib):
    for code in range(8):
        assert binding.status_string(code) != "unknown status"
    assert "workspace" in binding.status_string(binding.SSM_ERR_WORKSPACE)
    assert "range" in binding.status_string(binding.SSM_ERR_BOUNDS)


def test_debug_library_builds_and_exports_every_declared_symbol():
    """The range-checked build (-DSSM_DEBUG_CHECKS) compiles and offers the same C ABI."""
    from selective_state_space_16_b200 import build as b
    path = b.build(debug=True)
    import ctypes as ct
    dbg = ct.CDLL(path)
    missing = [n for n in _declared_functions() if not hasattr(dbg, n)]
    assert not missing, missing
    assert dbg.ssm_abi_version() == 3


def test_debug_library_switch_as_first_call():
    # Entering use_debug_library() before anything else has loaded the release library must
    # not deadlock (it loads that library too, and both take the module's lock); run in a
    # fresh process, bounded by a timeout.
    if not os.path.exists(binding.DEBUG_LIB_PATH):
        pytest.skip("debug library not built")
    import subprocess
    import sys
    code = ("from selective_state_space_16_b200 import binding\n"
            "with binding.use_debug_library() as lib:\n"
            "    assert binding.load() is lib\n"
            "assert binding.load() is not lib\n"
            "print('switched')\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "switched" in r.stdout, r.stderr


def test_workspace_size(lib):
    f = binding.ssm_selective_scan_workspace_size
    assert f(4, 5120, 16, 2048) % 256 == 0
    assert f(4, 5120, 16, 2048) >= 256 + 4 * 2048 * 128   # header + fp32 B/C rows
    assert f(4, 5120, 8, 2048) == 0                      # dstate not supported
    assert f(2, 64, 128, 100) >= 256 + 2 * 100 * 8 * 128 # wider state: B/C rows of 2N fp32
    assert f(2, 64, 48, 100) == 0
    assert f(-1, 5, 16, 5) == 0


P = ctypes.c_void_p


def _fwd(lib, **kw):
    args = dict(u=P(4096), delta=P(4096), A=P(4096), B=P(4096), C=P(4096), D=None, z=None, bias=None,
                softplus=1, y=P(4096), last=None, batch=1, dim=1, dstate=16, L=8, io=binding.SSM_BF16,
                ws=P(4096), wsb=1 << 20, stream=None)
    args.update(kw)
    return lib.ssm_selective_scan_fwd(*args.values())


def test_forward_argument_validation(lib):
    assert _fwd(lib, u=None) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, y=None) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, batch=-1) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, L=-3) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, io=7) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, dstate=8) == binding.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, dstate=48) == binding.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, u=P(4098)) == binding.SSM_ERR_INVALID_ARG      # not 16-byte aligned
    assert _fwd(lib, z=P(4100)) == binding.SSM_ERR_INVALID_ARG
    assert _fwd(lib, batch=0) == binding.SSM_OK                      # empty: nothing launched
    assert _fwd(lib, dim=0) == binding.SSM_OK
    assert _fwd(lib, ws=None) == binding.SSM_ERR_WORKSPACE
    assert _fwd(lib, wsb=16) == binding.SSM_ERR_WORKSPACE
    assert _fwd(lib, ws=P(4096 + 16)) == binding.SSM_ERR_WORKSPACE   # not 256-byte aligned


def test_forward_ex_rejects_unknown_algo(lib):
    opts = binding.FwdOptions(99, 0, 0, -1, 0)
    rc = lib.ssm_selective_scan_fwd_ex(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1,
                                       P(4096), None, 1, 1, 16, 8, binding.SSM_BF16, P(4096), 1 << 20,
                                       ctypes.byref(opts), None)
    assert rc == binding.SSM_ERR_INVALID_ARG


def test_forward_checkpoint_options_are_validated(lib):
    """Checkpoints (ABI 3) come from the sequential kernel only and must be 16-byte aligned;
    both are checked before anything touches the device."""
    def call(algo, ck, batch=1):
        opts = binding.FwdOptions(algo, 0, 0, -1, 0, ck)
        return lib.ssm_selective_scan_fwd_ex(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1,
                                             P(4096), None, batch, 1, 16, 8, binding.SSM_BF16, P(4096), 1 << 20,
                                             ctypes.byref(opts), None)
    assert call(binding.SSM_ALGO_CHUNKED, P(1 << 20)) == binding.SSM_ERR_UNSUPPORTED
    assert call(binding.SSM_ALGO_DIRECT, P(1 << 20)) == binding.SSM_ERR_UNSUPPORTED
    assert call(binding.SSM_ALGO_AUTO, P((1 << 20) + 8)) == binding.SSM_ERR_INVALID_ARG
    assert call(binding.SSM_ALGO_AUTO, P(1 << 20), batch=0) == binding.SSM_OK
    bopts = binding.BwdOptions(0, None, None, None, None, None, P((1 << 20) + 4))
    rc = lib.ssm_selective_scan_bwd_ex(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1, None,
                                       P(4096), None, P(4096), P(4096), P(4096), P(4096), P(4096), None, None,
                                       None, None, 2, 3, 16, 8, binding.SSM_BF16, P(4096), 1 << 30,
                                       ctypes.byref(bopts), None)
    assert rc == binding.SSM_ERR_INVALID_ARG


def test_forward_state_argument_validation(lib):
    def call(h0, last, batch=2, dim=3):
        return lib.ssm_selective_scan_fwd_state(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1,
                                                h0, P(4096), last, batch, dim, 16, 8, binding.SSM_BF16, P(4096),
                                                1 << 20, None, None)
    state_bytes = 2 * 3 * 16 * 4
    assert call(P(1 << 20), P(1 << 20)) == binding.SSM_ERR_INVALID_ARG                  # same buffer
    assert call(P(1 << 20), P((1 << 20) + state_bytes - 16)) == binding.SSM_ERR_INVALID_ARG  # overlap
    assert call(P((1 << 20) + state_bytes - 16), P(1 << 20)) == binding.SSM_ERR_INVALID_ARG
    assert call(P((1 << 20) + 8), None) == binding.SSM_ERR_INVALID_ARG                  # misaligned
    assert call(P(1 << 20), P((1 << 20) + state_bytes), batch=0) == binding.SSM_OK     # adjacent, empty


def test_decode_argument_validation(lib):
    def call(**kw):
        a = dict(state=P(4096), u=P(4096), delta=P(4096), A=P(4096), B=P(4096), C=P(4096), D=None, z=None,
                 bias=None, softplus=1, y=P(4096), batch=2, dim=3, dstate=16, io=binding.SSM_F32, stream=None)
        a.update(kw)
        return lib.ssm_state_update(*a.values())
    assert call(state=None) == binding.SSM_ERR_INVALID_ARG
    assert call(state=P(4100)) == binding.SSM_ERR_INVALID_ARG
    assert call(dstate=24) == binding.SSM_ERR_UNSUPPORTED
    assert call(io=3) == binding.SSM_ERR_INVALID_ARG
    assert call(batch=0) == binding.SSM_OK
    assert call(batch=65536) == binding.SSM_ERR_UNSUPPORTED  # the batch row is the grid's y index
    assert lib.ssm_state_update_ex(P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1,
                                   P(4096), 2, 3, 16, binding.SSM_F32, 5, None) == binding.SSM_ERR_INVALID_ARG


def test_read_status_needs_workspace(lib):
    assert lib.ssm_read_status(None, None) == binding.SSM_ERR_WORKSPACE


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        binding.load()


def test_product_package_does_not_import_oracle():
    pkg = os.path.join(ROOT, "selective_state_space_16_b200")
    for f in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if f.endswith((".py", ".cu", ".cuh", ".h")):
            txt = open(f).read()
            assert "import oracle" not in txt and "from oracle" not in txt and "ssm_oracle" not in txt, f


def test_backward_argument_validation(lib):
    def call(**kw):
        a = dict(u=P(4096), delta=P(4096), A=P(4096), B=P(4096), C=P(4096), D=None, z=None, bias=None, softplus=1,
                 h0=None, dy=P(4096), dlast=None, du=P(4096), ddelta=P(4096), dA=P(4096), dB=P(4096), dC=P(4096),
                 dD=None, dz=None, dbias=None, dh0=None, batch=2, dim=3, dstate=16, L=8, io=binding.SSM_BF16,
                 ws=P(4096), wsb=1 << 30, stream=None)
        a.update(kw)
        return lib.ssm_selective_scan_bwd(*a.values())
    assert call(dy=None) == binding.SSM_ERR_INVALID_ARG
    assert call(dB=None) == binding.SSM_ERR_INVALID_ARG
    assert call(z=P(4096)) == binding.SSM_ERR_INVALID_ARG            # z given, dz missing
    assert call(dA=P(4104)) == binding.SSM_ERR_INVALID_ARG           # misaligned
    assert call(dstate=32) == binding.SSM_ERR_UNSUPPORTED
    assert call(batch=0) == binding.SSM_OK
    assert call(ws=None) == binding.SSM_ERR_WORKSPACE
    assert call(wsb=64) == binding.SSM_ERR_WORKSPACE
    f = binding.ssm_selective_scan_bwd_workspace_size
    assert f(4, 5120, 16, 2048) % 256 == 0 and f(4, 5120, 16, 2048) > 4 * 2048 * 128
    assert f(1, 1, 8, 1) == 0


def test_backward_ex_argument_validation(lib):
    """ssm_selective_scan_bwd_ex rejects bad options before touching the device."""
    w = P(4096)
    def call(disc=binding.SSM_DISC_SIMPLIFIED, width=None, weight=w, dweight=P(4096), batch=2):
        spec = None if width is None else binding.ConvSpec(weight, None, width, None, None, None)
        opts = binding.BwdOptions(disc, ctypes.pointer(spec) if spec is not None else None, dweight, None, None, None)
        return lib.ssm_selective_scan_bwd_ex(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1, None,
                                             P(4096), None, P(4096), P(4096), P(4096), P(4096), P(4096), None, None,
                                             None, None, batch, 3, 16, 8, binding.SSM_BF16, P(4096), 1 << 30,
                                             ctypes.byref(opts), None)
    assert call(disc=7) == binding.SSM_ERR_INVALID_ARG
    assert call(width=0) == binding.SSM_ERR_INVALID_ARG
    assert call(width=5) == binding.SSM_ERR_INVALID_ARG
    assert call(width=4, weight=None) == binding.SSM_ERR_INVALID_ARG
    assert call(width=4, dweight=None) == binding.SSM_ERR_INVALID_ARG
    assert call(width=4, batch=0) == binding.SSM_OK
    assert call(disc=binding.SSM_DISC_ZOH, batch=0) == binding.SSM_OK


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="fake pointers: an accepted call would launch kernels on a real device")
def test_noalloc_scratch_limit_follows_its_formula(lib):
    """ssm_selective_scan_fwd_noalloc accepts every problem whose header + transposed B/C rows
    (256 + round_up(batch * seqlen * 128, 256) bytes) fit its 8 MiB scratch, whatever dim is.
    Without a device an accepted call stops at the device check (SSM_ERR_LAUNCH); a rejected
    one returns SSM_ERR_SCRATCH_LIMIT before that."""
    def call(batch, dim, L):
        return lib.ssm_selective_scan_fwd_noalloc(P(4096), P(4096), P(4096), P(4096), P(4096), None, None, None, 1,
                                                  P(4096), None, batch, dim, 16, L, binding.SSM_BF16, None)
    accepted = [(1, 5120, 2048), (4, 5120, 256), (8, 1536, 2048), (4, 5120, 2048), (1, 5120, 65534),
                (2, 5120, 32767)]
    for shape in accepted:
        assert call(*shape) == binding.SSM_ERR_LAUNCH, shape
    for shape in [(1, 64, 65536), (1, 5120, 65535), (4, 8, 1 << 15), (3, 5120, 21845)]:
        assert call(*shape) == binding.SSM_ERR_SCRATCH_LIMIT, shape
