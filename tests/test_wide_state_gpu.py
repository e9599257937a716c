"""GPU parity for the wider states d_state in {32, 64, 128, 256} (forward scan and decode)
against the fp64 oracle, which takes any d_state up to 256."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, check_forward, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("n", [32, 64, 128, 256])
def test_wide_forward(cuda_device, io, n):
    # 2 x 37 channels (not a multiple of a block's 8 warps), L = 300 (not a multiple of 32)
    inp = workloads.scan_inputs(2, 37, 300, dstate=n, io=io, seed=81 + n)
    check_forward(inp, what=f"N={n} {io}")


@pytest.mark.parametrize("n", [32, 256])
def test_wide_forward_zoh_and_state(cuda_device, n):
    inp = workloads.scan_inputs(1, 24, 200, dstate=n, io="f32", dt_min=1e-5, dt_max=1.0, seed=91 + n,
                                with_D=False)
    h0 = workloads.initial_state(1, 24, dstate=n, seed=92 + n)
    g = to_dev(inp, "cuda")
    y, last = ssm.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                     initial_state=h0.cuda(), zoh=True)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=None, z=inp["z"],
                                            delta_bias=inp["delta_bias"], h0=h0, zoh=True)
    assert_close(y, y_ref, "f32", f"N={n} zoh y")
    assert_close(last, last_ref, "f32", f"N={n} zoh last_state")


@pytest.mark.parametrize("L", [1, 31, 32, 33])
def test_wide_forward_edge_lengths(cuda_device, L):
    check_forward(workloads.scan_inputs(2, 9, L, dstate=64, io="bf16", seed=95 + L), what=f"N=64 L={L}")


def test_wide_forward_mamba_shape_sampled(cuda_device):
    # batch 4, d_inner 2048, L 2048, d_state 128, bf16: 128 sampled channels
    inp = workloads.scan_inputs(4, 2048, 2048, dstate=128, io="bf16", seed=99)
    rng = np.random.default_rng(10)
    channels = np.sort(rng.choice(4 * 2048, size=128, replace=False))
    check_forward(inp, channels=channels, what="N=128 b4 d2048 L2048")


def test_wide_chunked_is_unsupported(cuda_device):
    inp = to_dev(workloads.scan_inputs(1, 8, 64, dstate=32, io="bf16", seed=97), "cuda")
    y = torch.empty_like(inp["u"])
    ws = ssm.new_workspace(1, 8, 32, 64)
    code = ssm.ssm_selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                                      inp["delta_bias"], True, y, None, ws, algo="chunked", check=False)
    assert code == ssm.binding.SSM_ERR_UNSUPPORTED


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("n,zoh", [(32, False), (64, True), (128, False), (256, True)])
def test_wide_decode_chain_equals_forward(cuda_device, io, n, zoh):
    b, d, L = 3, 20, 12
    inp = workloads.scan_inputs(b, d, L, dstate=n, io=io, dt_min=1e-4, dt_max=0.5, seed=100 + n)
    g = to_dev(inp, "cuda")
    state = torch.zeros(b, d, n, device="cuda")
    ys = []
    for t in range(L):
        y = torch.empty(b, d, dtype=g["u"].dtype, device="cuda")
        ssm.ssm_state_update(state, g["u"][..., t].contiguous(), g["delta"][..., t].contiguous(), g["A"],
                             g["B"][..., t].contiguous(), g["C"][..., t].contiguous(), g["D"],
                             g["z"][..., t].contiguous(), g["delta_bias"], True, y, zoh=zoh)
        ys.append(y)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], zoh=zoh)
    assert_close(torch.stack(ys, dim=-1), y_ref, io, f"N={n} decode y")
    assert_close(state, last_ref, io, f"N={n} decode state")
