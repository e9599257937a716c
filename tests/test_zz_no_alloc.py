"""The forward scan entry point that allocates nothing (ssm_selective_scan_fwd_noalloc).

Some callers cannot allocate device memory: a plugin that a host framework hands only
its input and output buffers, or a latency-critical loop that must not call cudaMalloc
(which can synchronise the whole device).  For them the library keeps its scratch in
one fixed array of its own device memory.  These tests call that entry point through
the C ABI and check it against the regular entry point (which uses a caller-supplied
workspace), twice in a row, since every call reuses the same array.

This file is named to be collected last, so that a run stopping at its first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import selective_state_space_16_b200 as ssm
import workloads
from parity import TOL, assert_close, oracle_forward, rel_err, to_dev
from selective_state_space_16_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io,shape", [("bf16", (2, 100, 1000)), ("f32", (1, 64, 256)), ("bf16", (1, 24, 7)),
                                      ("f32", (2, 40, 333))],
                         ids=["bf16_ragged", "f32_tiny", "bf16_unaligned_L", "f32_unaligned_L"])
def test_noalloc_matches_workspace_entry_twice(cuda_device, io, shape):
    # (rows that are not 16-byte multiples: this entry point gathers them in the kernel, the
    # regular one stages a padded copy at these small shapes)
    b, d, L = shape
    inp = to_dev(workloads.scan_inputs(b, d, L, io=io, seed=31), "cuda")
    y_ref, last_ref = ssm.selective_scan_fwd(**inp)          # regular entry point, own workspace
    torch.cuda.synchronize()
    for call in range(2):                                      # the scratch keeps the last call's contents
        y = torch.full_like(inp["u"], float("nan"))
        last = torch.full((b, d, 16), float("nan"), device="cuda")
        binding.ssm_selective_scan_fwd_noalloc(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                               inp["z"], inp["delta_bias"], True, y, last)
        torch.cuda.synchronize()
        e_y = rel_err(y, y_ref.double().cpu().numpy()).max()
        e_s = rel_err(last, last_ref.double().cpu().numpy()).max()
        assert np.isfinite(e_y) and e_y <= TOL[io], f"call {call}: y max rel err {e_y:.3e}"
        assert np.isfinite(e_s) and e_s <= TOL[io], f"call {call}: last_state max rel err {e_s:.3e}"


def test_noalloc_large_dim_matches_oracle(cuda_device):
    # The limit depends on batch * seqlen only (the B/C rows), not on dim: one batch row of the
    # Mamba-2.8B layer shape (d_inner 5120, L 2048, bf16) fits and is checked element by element
    # against the fp64 oracle, on two calls in a row.
    cpu = workloads.scan_inputs(1, 5120, 2048, io="bf16", seed=32)
    inp = to_dev(cpu, "cuda")
    y_ref, last_ref = oracle_forward(cpu)
    for call in range(2):
        y = torch.full_like(inp["u"], float("nan"))
        last = torch.full((1, 5120, 16), float("nan"), device="cuda")
        binding.ssm_selective_scan_fwd_noalloc(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                               inp["z"], inp["delta_bias"], True, y, last)
        torch.cuda.synchronize()
        assert_close(y, y_ref, "bf16", f"noalloc call {call}: y")
        assert_close(last, last_ref, "bf16", f"noalloc call {call}: last_state")


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    # 256 + batch * seqlen * 128 bytes of header and transposed B/C exceed the 8 MiB scratch:
    # rejected before any launch (fake pointers are never dereferenced).
    P = ctypes.c_void_p(4096)
    for batch, dim, L in [(4, 8, 1 << 15), (1, 64, 65536), (1, 5120, 65535)]:
        rc = binding.load().ssm_selective_scan_fwd_noalloc(P, P, P, P, P, None, None, None, 1, P, None,
                                                           batch, dim, 16, L, binding.SSM_BF16, None)
        assert rc == binding.SSM_ERR_SCRATCH_LIMIT, (batch, dim, L)
    assert "scratch" in binding.status_string(rc)
