"""GPU parity of the backward (ssm_selective_scan_bwd) against the fp64 oracle backward,
whose gradients are pinned by finite differences of the forward scan.  Same seeded
inputs on both sides; tolerances as the forward: |x - x_ref| <= tol (1 + |x_ref|) with
tol 1e-4 for fp32 I/O and 2e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, io_of, to_dev

pytestmark = pytest.mark.gpu

OUT_KEYS = ["du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state"]


def _grad_inputs(b, d, L, io, seed, with_state=False):
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(b, d, L, generator=g).to(workloads.io_torch_dtype(io))
    dlast = torch.randn(b, d, 16, generator=g) if with_state else None
    h0 = workloads.initial_state(b, d, seed=seed + 1) if with_state else None
    return dy, dlast, h0


def check_backward(inp, dy, softplus=True, h0=None, dlast=None, what="backward", skip=()):
    io = io_of(inp["u"])
    g = to_dev(inp, "cuda")
    out = ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                 softplus=softplus, dy=dy.cuda(), initial_state=None if h0 is None else h0.cuda(),
                                 dlast_state=None if dlast is None else dlast.cuda())
    torch.cuda.synchronize()
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                    delta_bias=inp["delta_bias"], softplus=softplus, h0=h0, dy=dy, dlast=dlast)
    ref["dinitial_state"] = ref.pop("dh0")
    worst = {}
    for k in OUT_KEYS:
        if k in skip or ref[k] is None:
            continue
        worst[k] = assert_close(out[k], ref[k], io, f"{what} {k}")
    return worst


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_ragged(cuda_device, io):
    # 100 channels (not a multiple of a CTA's 64), L = 1000 (not a multiple of a segment)
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=41)
    dy, _, _ = _grad_inputs(2, 100, 1000, io, 42)
    check_backward(inp, dy, what=f"ragged {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_with_states(cuda_device, io):
    inp = workloads.scan_inputs(2, 70, 333, io=io, seed=43)
    dy, dlast, h0 = _grad_inputs(2, 70, 333, io, 44, with_state=True)
    check_backward(inp, dy, h0=h0, dlast=dlast, what=f"states {io}")


@pytest.mark.parametrize("flags", [dict(with_z=False), dict(with_D=False), dict(with_bias=False),
                                   dict(with_z=False, with_D=False, with_bias=False)],
                         ids=["no_gate", "no_D", "no_bias", "bare"])
def test_backward_optional_inputs(cuda_device, flags):
    inp = workloads.scan_inputs(1, 64, 256, io="f32", seed=45, **flags)
    dy, _, _ = _grad_inputs(1, 64, 256, "f32", 46)
    check_backward(inp, dy, what=str(flags))


def test_backward_softplus_off(cuda_device):
    inp = workloads.scan_inputs(1, 48, 256, io="f32", seed=47)
    inp["delta"] = (inp["delta"].float().abs() * 0.5 + 0.01).to(inp["delta"].dtype)
    inp["delta_bias"] = torch.linspace(0.0, 0.05, inp["delta_bias"].numel())
    dy, _, _ = _grad_inputs(1, 48, 256, "f32", 48)
    check_backward(inp, dy, softplus=False, what="softplus off")


@pytest.mark.parametrize("L", [1, 15, 16, 17, 64, 127])
def test_backward_edge_lengths(cuda_device, L):
    inp = workloads.scan_inputs(2, 20, L, io="f32", seed=49 + L)
    dy, dlast, h0 = _grad_inputs(2, 20, L, "f32", 50 + L, with_state=True)
    check_backward(inp, dy, h0=h0, dlast=dlast, what=f"L={L}")


def test_backward_empty_sequence(cuda_device):
    inp = to_dev(workloads.scan_inputs(2, 20, 0, io="bf16", seed=51), "cuda")
    dlast = torch.randn(2, 20, 16, device="cuda")
    dy = torch.empty(2, 20, 0, dtype=torch.bfloat16, device="cuda")
    out = ssm.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                                 inp["delta_bias"], dy=dy, dlast_state=dlast)
    torch.cuda.synchronize()
    assert torch.equal(out["dinitial_state"], dlast)
    assert torch.all(out["dA"] == 0) and torch.all(out["dD"] == 0) and torch.all(out["ddelta_bias"] == 0)


def test_backward_is_deterministic(cuda_device):
    inp = to_dev(workloads.scan_inputs(2, 96, 640, io="bf16", seed=52), "cuda")
    dy = torch.randn(2, 96, 640, device="cuda").to(torch.bfloat16)
    o1 = ssm.selective_scan_bwd(**inp, dy=dy)
    o2 = ssm.selective_scan_bwd(**inp, dy=dy)
    torch.cuda.synchronize()
    for k in OUT_KEYS:
        if o1[k] is not None:
            assert torch.equal(o1[k], o2[k]), k


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_backward_workload_full_size(cuda_device, idx):
    # The forward workloads (tiny fp32; Mamba-130M and Mamba-2.8B layer shapes, bf16) with
    # a seeded N(0, 1) output gradient, every gradient compared in full.
    w = workloads.WORKLOADS[idx]
    inp = workloads.workload_inputs(w)
    dy, _, _ = _grad_inputs(w.batch, w.dim, w.seqlen, w.io, 60 + idx)
    check_backward(inp, dy, what=w.name)
