"""GPU parity of the zero-order-hold discretisation ([Eng] §2.2; SSM_DISC_ZOH) against the
fp64 oracle's hold weight expm1(Delta A)/A * B, which is pinned against an integrated ODE.
Tolerances as the forward scan."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, io_of, to_dev

pytestmark = pytest.mark.gpu


def check_zoh(inp, what, channels=None, **opts):
    io = io_of(inp["u"])
    g = to_dev(inp, "cuda")
    y, last = ssm.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                     zoh=True, **opts)
    torch.cuda.synchronize()
    if channels is None:
        y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                                z=inp["z"], delta_bias=inp["delta_bias"], zoh=True)
    else:
        b_, d_, L = inp["u"].shape
        y_ref, last_ref = [], []
        for c in channels:
            bi, di = divmod(int(c), d_)
            yy, ll = oracle.selective_scan(inp["u"][bi, di][None, None], inp["delta"][bi, di][None, None],
                                           inp["A"][di][None], inp["B"][bi][None], inp["C"][bi][None],
                                           D=inp["D"][di:di + 1], z=inp["z"][bi, di][None, None],
                                           delta_bias=inp["delta_bias"][di:di + 1], zoh=True)
            y_ref.append(yy[0, 0])
            last_ref.append(ll[0, 0])
        y_ref, last_ref = np.stack(y_ref), np.stack(last_ref)
        idx = torch.as_tensor(np.asarray(channels), device="cuda")
        y = y.reshape(b_ * d_, L).index_select(0, idx)
        last = last.reshape(b_ * d_, -1).index_select(0, idx)
    assert_close(y, y_ref, io, what + " y")
    assert_close(last, last_ref, io, what + " last_state")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("algo,lanes", [("sequential", 4), ("sequential", 8), ("direct", 0), (None, 0)],
                         ids=["seq4", "seq8", "direct", "auto"])
def test_zoh_forward_variants(cuda_device, io, algo, lanes):
    if io == "f32" and lanes == 8:
        pytest.skip("8 lanes per channel needs 8 steps per 16-byte group (bf16)")
    # step sizes from 1e-5 to 1: with A from -1 to -16, Delta A crosses the 1/16 switch
    # between the series and the exp(Delta A) - 1 forms of the hold weight
    inp = workloads.scan_inputs(2, 100, 1000, io=io, dt_min=1e-5, dt_max=1.0, seed=71)
    check_zoh(inp, f"zoh {algo}/{lanes}/{io}", algo=algo, lanes_per_channel=lanes)


@pytest.mark.parametrize("io,lanes", [("f32", 4), ("bf16", 4), ("bf16", 8)])
def test_zoh_unaligned_rows(cuda_device, io, lanes):
    # rows that are not 16-byte multiples: gathered by the sequential kernel itself, or (by
    # default at this small shape) staged from a padded copy
    inp = workloads.scan_inputs(2, 40, 333, io=io, dt_min=1e-5, dt_max=1.0, seed=90)
    check_zoh(inp, f"zoh gathered rows {io}/{lanes}", algo="sequential", lanes_per_channel=lanes)
    check_zoh(inp, f"zoh padded rows {io}", lanes_per_channel=lanes)


def test_zoh_tiny_steps_fp32(cuda_device):
    # every Delta A far below 1/16: the series branch only, where exp(Delta A) - 1 would cancel
    inp = workloads.scan_inputs(1, 64, 512, io="f32", dt_min=1e-7, dt_max=1e-5, seed=72)
    check_zoh(inp, "zoh tiny steps")


def test_zoh_with_initial_state_and_no_gate(cuda_device):
    inp = workloads.scan_inputs(2, 40, 333, io="f32", seed=73, with_z=False)
    h0 = workloads.initial_state(2, 40, seed=74)
    g = to_dev(inp, "cuda")
    y, last = ssm.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                     zoh=True, initial_state=h0.cuda())
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=None, delta_bias=inp["delta_bias"], h0=h0, zoh=True)
    assert_close(y, y_ref, "f32", "zoh h0 y")
    assert_close(last, last_ref, "f32", "zoh h0 last_state")


def test_zoh_headline_sampled(cuda_device):
    w = workloads.WORKLOADS[2]
    inp = workloads.workload_inputs(w)
    rng = np.random.default_rng(9)
    channels = np.sort(rng.choice(w.batch * w.dim, size=256, replace=False))
    check_zoh(inp, "zoh headline", channels=channels)


def test_zoh_chunked_is_unsupported(cuda_device):
    inp = to_dev(workloads.scan_inputs(1, 16, 256, io="bf16", seed=75), "cuda")
    y = torch.empty_like(inp["u"])
    ws = ssm.new_workspace(1, 16, 16, 256)
    code = ssm.ssm_selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                                      inp["delta_bias"], True, y, None, ws, algo="chunked", zoh=True, check=False)
    assert code == ssm.binding.SSM_ERR_UNSUPPORTED


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_decode_chain_equals_forward(cuda_device, io):
    b, d, L = 3, 50, 24
    inp = workloads.scan_inputs(b, d, L, io=io, dt_min=1e-4, dt_max=0.5, seed=76)
    g = to_dev(inp, "cuda")
    state = torch.zeros(b, d, 16, device="cuda")
    ys = []
    for t in range(L):
        y = torch.empty(b, d, dtype=g["u"].dtype, device="cuda")
        ssm.ssm_state_update(state, g["u"][..., t].contiguous(), g["delta"][..., t].contiguous(), g["A"],
                             g["B"][..., t].contiguous(), g["C"][..., t].contiguous(), g["D"],
                             g["z"][..., t].contiguous(), g["delta_bias"], True, y, zoh=True)
        ys.append(y)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], zoh=True)
    assert_close(torch.stack(ys, dim=-1), y_ref, io, "zoh decode y")
    assert_close(state, last_ref, io, "zoh decode state")
