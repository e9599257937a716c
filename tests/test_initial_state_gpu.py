"""GPU parity of the forward scan that starts from a given state (state continuation
across the blocks of a long sequence, [Eng] §7.2; reuse of a cached prefix state,
[Eng] §6.2), through ssm_selective_scan_fwd_state, against the fp64 oracle started
from the same state."""
import numpy as np
import pytest
import torch

import selective_state_space_16_b200 as ssm
import workloads
from parity import TOL, assert_close, check_forward, oracle_forward, to_dev

pytestmark = pytest.mark.gpu

VARIANTS = [("sequential", 2), ("sequential", 4), ("sequential", 8), ("sequential", 42), ("chunked", 0),
            ("direct", 0)]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("algo,lanes", VARIANTS, ids=[f"{a}{g or ''}" for a, g in VARIANTS])
def test_initial_state_variants_ragged(cuda_device, io, algo, lanes):
    if io == "f32" and lanes == 8:
        pytest.skip("8 lanes per channel needs 8 steps per 16-byte group (bf16)")
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=31)
    h0 = workloads.initial_state(2, 100, seed=32)
    check_forward(inp, h0=h0, algo=algo, lanes_per_channel=lanes, what=f"h0 {algo}/{lanes}/{io}")


def _slice(inp, t0, t1):
    """Steps [t0, t1) of a scan's inputs (per-step tensors sliced, parameters shared)."""
    out = dict(inp)
    for k in ("u", "delta", "z", "B", "C"):
        if inp[k] is not None:
            out[k] = inp[k][..., t0:t1].contiguous()
    return out


def _continued(inp, cuts, dev="cuda", **opts):
    """Scan block by block, each block starting from the previous block's last_state
    (two state buffers, so the initial and the final state never overlap)."""
    b, d, L = inp["u"].shape
    edges = [0] + list(cuts) + [L]
    ys = []
    state = None
    for t0, t1 in zip(edges[:-1], edges[1:]):
        g = to_dev(_slice(inp, t0, t1), dev)
        y, last = ssm.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                         g["delta_bias"], initial_state=state, **opts)
        ys.append(y)
        state = last
    torch.cuda.synchronize()
    return torch.cat(ys, dim=-1), state


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("cuts", [(512,), (64, 640), (333,), (1, 999)], ids=["half", "three", "odd", "edges"])
def test_state_continuation_equals_full_scan(cuda_device, io, cuts):
    # Odd cut points give blocks whose rows are not 16-byte multiples: those blocks take
    # the direct-load kernel, the others the staged one, and the state is handed across.
    inp = workloads.scan_inputs(2, 72, 1000, io=io, seed=33)
    y, last = _continued(inp, cuts)
    y_ref, last_ref = oracle_forward(inp)
    assert_close(y, y_ref, io, f"continued y {cuts}")
    assert_close(last, last_ref, io, f"continued last_state {cuts}")


@pytest.mark.parametrize("algo", ["sequential", "chunked"])
def test_long_sequence_in_blocks(cuda_device, algo):
    # 1 x 64 channels x 9000 steps in blocks of 2048 (+ a ragged tail), bf16.
    inp = workloads.scan_inputs(1, 64, 9000, io="bf16", dt_min=1e-4, dt_max=1e-2, seed=34)
    y, last = _continued(inp, [2048, 4096, 6144, 8192], algo=algo)
    y_ref, last_ref = oracle_forward(inp)
    assert_close(y, y_ref, "bf16", f"blocks/{algo} y")
    assert_close(last, last_ref, "bf16", f"blocks/{algo} last_state")


def test_empty_sequence_copies_initial_state(cuda_device):
    inp = workloads.scan_inputs(2, 20, 0, io="bf16", seed=35)
    h0 = workloads.initial_state(2, 20, seed=36).cuda()
    g = to_dev(inp, "cuda")
    y, last = ssm.selective_scan_fwd(**g, initial_state=h0)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(last, h0)


def test_overlapping_states_are_rejected(cuda_device):
    inp = to_dev(workloads.scan_inputs(1, 16, 64, io="bf16", seed=37), "cuda")
    state = torch.zeros(1, 16, 16, device="cuda")
    y = torch.empty_like(inp["u"])
    ws = ssm.new_workspace(1, 16, 16, 64)
    code = ssm.ssm_selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                                      inp["delta_bias"], True, y, state, ws, initial_state=state, check=False)
    assert code == ssm.binding.SSM_ERR_INVALID_ARG


def test_headline_from_state_sampled(cuda_device):
    # Mamba-2.8B layer shape (b4, d5120, L2048, bf16) on the default kernel, from a state
    # of scale 1; 512 sampled channels against the oracle.
    w = workloads.WORKLOADS[2]
    inp = workloads.workload_inputs(w)
    h0 = workloads.initial_state(w.batch, w.dim, seed=38)
    rng = np.random.default_rng(8)
    channels = np.sort(rng.choice(w.batch * w.dim, size=512, replace=False))
    check_forward(inp, h0=h0, channels=channels, what="headline from state")
