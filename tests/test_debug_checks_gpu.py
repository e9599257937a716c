"""The range-checked debug library and the host-side launch-failure path (-m gpu).

libssm_scan_debug.so is the library compiled with -DSSM_DEBUG_CHECKS: its kernels check
their shared-memory offsets, TMA coordinates and global indices, and a failed check
records SSM_ERR_BOUNDS in the workspace status word instead of touching memory.  These
tests run the ragged parity shapes of every kernel through it: results must still match
the fp64 oracle and the status word must stay clean.

SSM_FAKE_LAUNCH_FAILURE makes every launching call return SSM_ERR_LAUNCH before anything
is launched; nothing here faults, traps or hangs the GPU.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, oracle_forward, to_dev
from selective_state_space_16_b200 import binding

pytestmark = pytest.mark.gpu

VARIANTS = [("sequential", 2), ("sequential", 4), ("sequential", 8), ("sequential", 42), ("chunked", 0),
            ("direct", 0)]


@pytest.fixture(scope="module")
def debug_lib():
    with binding.use_debug_library() as lib:
        yield lib


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("algo,lanes", VARIANTS, ids=[f"{a}{g}" for a, g in VARIANTS])
def test_debug_forward_ragged_clean(cuda_device, debug_lib, io, algo, lanes):
    if io == "f32" and lanes == 8:
        pytest.skip("8 lanes per channel needs 8 steps per 16-byte group (bf16)")
    cpu = workloads.scan_inputs(2, 100, 1000, io=io, seed=61)
    g = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(2, 100, 16, 1000)
    y, last = ssm.selective_scan_fwd(**g, workspace=ws, algo=algo, lanes_per_channel=lanes)
    assert ssm.ssm_read_status(ws) == binding.SSM_OK
    y_ref, last_ref = oracle_forward(cpu)
    assert_close(y, y_ref, io, f"debug {algo}/{lanes} y")
    assert_close(last, last_ref, io, f"debug {algo}/{lanes} last_state")


@pytest.mark.parametrize("L", [1, 63, 65, 2047])
def test_debug_forward_edge_lengths_clean(cuda_device, debug_lib, L):
    cpu = workloads.scan_inputs(3, 40, L, io="bf16", seed=62 + L)
    g = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(3, 40, 16, L)
    y, last = ssm.selective_scan_fwd(**g, workspace=ws)
    assert ssm.ssm_read_status(ws) == binding.SSM_OK
    y_ref, last_ref = oracle_forward(cpu)
    assert_close(y, y_ref, "bf16", f"debug L={L} y")
    assert_close(last, last_ref, "bf16", f"debug L={L} last_state")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_debug_backward_clean(cuda_device, debug_lib, io):
    b, d, L = 2, 48, 300
    cpu = workloads.scan_inputs(b, d, L, io=io, seed=63)
    g = to_dev(cpu, "cuda")
    dy = torch.randn(b, d, L, generator=torch.Generator().manual_seed(64)).to(cpu["u"].dtype)
    ws = torch.zeros(max(ssm.ssm_selective_scan_bwd_workspace_size(b, d, 16, L), 256), dtype=torch.uint8,
                     device="cuda")
    grads = ssm.selective_scan_bwd(**g, softplus=True, dy=dy.cuda(), workspace=ws)
    assert ssm.ssm_read_status(ws) == binding.SSM_OK
    ref = oracle.selective_scan_bwd(**cpu, softplus=True, dy=dy)
    for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias"):
        assert_close(grads[k], ref[k], "f32" if io == "f32" else "bf16", f"debug backward {k}")


def test_fake_launch_failure_returns_launch_error(cuda_device, monkeypatch):
    cpu = workloads.scan_inputs(1, 16, 64, io="bf16", seed=65)
    g = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(1, 16, 16, 64)
    y = torch.full_like(g["u"], float("nan"))
    last = torch.full((1, 16, 16), float("nan"), device="cuda")
    monkeypatch.setenv("SSM_FAKE_LAUNCH_FAILURE", "1")
    with pytest.raises(binding.SsmError) as e:
        ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                   True, y, last, ws)
    assert e.value.code == binding.SSM_ERR_LAUNCH
    code = ssm.ssm_state_update(torch.zeros(1, 16, 16, device="cuda"), g["u"][:, :, 0].contiguous(),
                                g["delta"][:, :, 0].contiguous(), g["A"], g["B"][:, :, 0].contiguous(),
                                g["C"][:, :, 0].contiguous(), g["D"], None, g["delta_bias"], True,
                                torch.empty(1, 16, dtype=torch.bfloat16, device="cuda"), check=False)
    assert code == binding.SSM_ERR_LAUNCH
    torch.cuda.synchronize()
    assert torch.isnan(y).all() and torch.isnan(last).all()      # nothing was launched
    monkeypatch.delenv("SSM_FAKE_LAUNCH_FAILURE")
    ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True, y,
                               last, ws)
    torch.cuda.synchronize()
    y_ref, _ = oracle_forward(cpu)
    assert_close(y, y_ref, "bf16", "after the injected failure")
    assert not os.environ.get("SSM_FAKE_LAUNCH_FAILURE")


def test_debug_status_reports_where(cuda_device, debug_lib):
    """A clean call leaves the whole status block (code and location) at zero."""
    cpu = workloads.scan_inputs(1, 24, 200, io="bf16", seed=66)
    g = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(1, 24, 16, 200)
    ssm.selective_scan_fwd(**g, workspace=ws)
    torch.cuda.synchronize()
    header = ws[:32].view(torch.int32).cpu().tolist()   # epoch, ticket, done, status, where[4]
    assert header[3] == 0 and header[4:8] == [0, 0, 0, 0], header


@pytest.mark.parametrize("zoh", [False, True])
def test_debug_backward_conv_clean(cuda_device, debug_lib, zoh):
    """The conv + ZOH backward through the range-checked library: clean status word."""
    b, d, L = 2, 40, 130
    cpu = workloads.scan_inputs(b, d, L, io="bf16", seed=67)
    conv = to_dev(workloads.conv_inputs(b, d, 4, seed=68, with_state=True), "cuda")
    g = to_dev(cpu, "cuda")
    dy = torch.randn(b, d, L, generator=torch.Generator().manual_seed(69)).to(torch.bfloat16).cuda()
    ws = torch.zeros(max(ssm.ssm_selective_scan_bwd_workspace_size(b, d, 16, L), 256), dtype=torch.uint8,
                     device="cuda")
    out = ssm.selective_scan_bwd(**g, softplus=True, dy=dy, workspace=ws, zoh=zoh, conv_weight=conv["conv_weight"],
                                 conv_bias=conv["conv_bias"], conv_state_in=conv["conv_state_in"],
                                 dconv_state_out=torch.ones(b, d, 3, device="cuda"))
    assert ssm.ssm_read_status(ws) == binding.SSM_OK
    assert torch.isfinite(out["dx"].float()).all() and torch.isfinite(out["dconv_weight"]).all()
