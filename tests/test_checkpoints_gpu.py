"""Forward checkpoints for the backward (ssm_fwd_options_t.checkpoints, ssm_bwd_options_t.checkpoints).

The forward may store the state at the start of every 8-step segment; checkpoint s must equal
the oracle's final state of the prefix [0, 8s) (from the same initial state).  A backward given
those checkpoints skips its own forward sweep; its gradients must match the oracle's as the
backward without them does.  Tolerances as the forward's: |x - x_ref| <= tol (1 + |x_ref|), tol
1e-4 for fp32 I/O and 2e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, to_dev
from selective_state_space_16_b200 import binding

pytestmark = pytest.mark.gpu


def _prefix_states(cpu, h0=None, zoh=False, u=None):
    """Oracle states at the start of every 8-step segment: (b, nseg, d, 16)."""
    b, d, L = cpu["u"].shape
    nseg = (L + 7) // 8
    out = np.zeros((b, nseg, d, 16))
    out[:, 0] = 0.0 if h0 is None else h0.double().numpy()
    uu = cpu["u"] if u is None else u
    for s in range(1, nseg):
        t = 8 * s
        _, last = oracle.selective_scan(uu[..., :t], cpu["delta"][..., :t], cpu["A"], cpu["B"][..., :t],
                                        cpu["C"][..., :t], D=cpu["D"], z=None if cpu["z"] is None else cpu["z"][..., :t],
                                        delta_bias=cpu["delta_bias"], h0=h0, zoh=zoh)
        out[:, s] = last
    return out


def _new_ckpt(b, d, L):
    return torch.full((b, (L + 7) // 8, d, 16), float("nan"), device="cuda")


@pytest.mark.parametrize("io,lanes", [("f32", 4), ("f32", 0), ("bf16", 4), ("bf16", 8), ("bf16", 0)])
def test_forward_checkpoints_are_prefix_states(cuda_device, io, lanes):
    b, d, L = 2, 100, 200
    cpu = workloads.scan_inputs(b, d, L, io=io, seed=400 + lanes)
    g = to_dev(cpu, "cuda")
    ck = _new_ckpt(b, d, L)
    algo = "sequential" if lanes else None
    y, last = ssm.selective_scan_fwd(**g, checkpoints=ck, algo=algo, lanes_per_channel=lanes)
    torch.cuda.synchronize()
    ref = _prefix_states(cpu)
    assert_close(ck, ref, io, f"checkpoints {io}/{lanes}")
    y_ref, last_ref = oracle.selective_scan(**cpu)
    assert_close(y, y_ref, io, "y with checkpoints")


@pytest.mark.parametrize("L", [1, 7, 9, 130, 203])
def test_forward_checkpoints_ragged_and_from_a_state(cuda_device, L):
    # L % 8 != 0 runs the padded-row path; checkpoint 0 is the initial state
    b, d = 2, 40
    cpu = workloads.scan_inputs(b, d, L, io="bf16", seed=410 + L)
    h0 = workloads.initial_state(b, d, seed=411 + L)
    g = to_dev(cpu, "cuda")
    ck = _new_ckpt(b, d, L)
    ssm.selective_scan_fwd(**g, checkpoints=ck, initial_state=h0.cuda())
    torch.cuda.synchronize()
    assert_close(ck, _prefix_states(cpu, h0=h0), "bf16", f"checkpoints L={L}")


def test_forward_checkpoints_zoh(cuda_device):
    b, d, L = 2, 64, 160
    cpu = workloads.scan_inputs(b, d, L, io="f32", seed=420)
    g = to_dev(cpu, "cuda")
    ck = _new_ckpt(b, d, L)
    ssm.selective_scan_fwd(**g, checkpoints=ck, zoh=True)
    torch.cuda.synchronize()
    assert_close(ck, _prefix_states(cpu, zoh=True), "f32", "zoh checkpoints")


@pytest.mark.parametrize("L", [160, 157])
def test_forward_checkpoints_conv(cuda_device, L):
    # (L = 157: x staged in padded rows)
    b, d = 2, 64
    cpu = workloads.scan_inputs(b, d, L, io="bf16", seed=430)
    conv = workloads.conv_inputs(b, d, 4, seed=431, with_state=True)
    g, c = to_dev(cpu, "cuda"), to_dev(conv, "cuda")
    ck = _new_ckpt(b, d, L)
    y = torch.empty_like(g["u"])
    last = torch.empty(b, d, 16, device="cuda")
    ssm.ssm_selective_scan_fwd_conv(g["u"], c["conv_weight"], c["conv_bias"], g["delta"], g["A"], g["B"], g["C"],
                                    g["D"], g["z"], g["delta_bias"], True, y, last, ssm.new_workspace(b, d, 16, L),
                                    conv_state_in=c["conv_state_in"], checkpoints=ck)
    torch.cuda.synchronize()
    u, _ = oracle.causal_conv_silu(cpu["u"], conv["conv_weight"], conv["conv_bias"], conv["conv_state_in"])
    u_io = torch.from_numpy(u).to(torch.bfloat16)   # the kernel scans u rounded to the I/O type
    assert_close(ck, _prefix_states(cpu, u=u_io), "bf16", "conv checkpoints")


BWD_KEYS = ["ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state"]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh,conv", [(False, False), (True, False), (False, True), (True, True)],
                         ids=["plain", "zoh", "conv", "zoh_conv"])
def test_backward_with_forward_checkpoints(cuda_device, io, zoh, conv):
    b, d, L = 2, 70, 333
    cpu = workloads.scan_inputs(b, d, L, io=io, seed=440)
    g = to_dev(cpu, "cuda")
    h0 = workloads.initial_state(b, d, seed=441)
    gen = torch.Generator().manual_seed(442)
    dy = torch.randn(b, d, L, generator=gen).to(cpu["u"].dtype)
    dlast = torch.randn(b, d, 16, generator=gen)
    cv = workloads.conv_inputs(b, d, 4, seed=443, with_state=True) if conv else None
    c = to_dev(cv, "cuda") if conv else {}
    ck = _new_ckpt(b, d, L)
    ws = ssm.new_workspace(b, d, 16, L)
    y, last = torch.empty_like(g["u"]), torch.empty(b, d, 16, device="cuda")
    if conv:
        ssm.ssm_selective_scan_fwd_conv(g["u"], c["conv_weight"], c["conv_bias"], g["delta"], g["A"], g["B"],
                                        g["C"], g["D"], g["z"], g["delta_bias"], True, y, last, ws,
                                        conv_state_in=c["conv_state_in"], initial_state=h0.cuda(), zoh=zoh,
                                        checkpoints=ck)
    else:
        ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                                   y, last, ws, initial_state=h0.cuda(), zoh=zoh, checkpoints=ck)
    kw = dict(softplus=True, dy=dy.cuda(), initial_state=h0.cuda(), dlast_state=dlast.cuda(), zoh=zoh,
              conv_weight=c.get("conv_weight"), conv_bias=c.get("conv_bias"), conv_state_in=c.get("conv_state_in"))
    with_ck = ssm.selective_scan_bwd(**g, checkpoints=ck, **kw)
    without = ssm.selective_scan_bwd(**g, **kw)
    torch.cuda.synchronize()
    u = cpu["u"]
    if conv:
        uf, _ = oracle.causal_conv_silu(cpu["u"], cv["conv_weight"], cv["conv_bias"], cv["conv_state_in"])
        u = torch.from_numpy(uf).to(cpu["u"].dtype)
    ref = oracle.selective_scan_bwd(u, cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                                    delta_bias=cpu["delta_bias"], h0=h0, dy=dy, dlast=dlast, zoh=zoh)
    ref["dinitial_state"] = ref.pop("dh0")
    keys = BWD_KEYS + (["dx", "dconv_weight", "dconv_bias", "dconv_state_in"] if conv else ["du"])
    if conv:
        cg = oracle.causal_conv_silu_bwd(cpu["u"], cv["conv_weight"], ref["du"], cv["conv_bias"], cv["conv_state_in"])
        ref.update(dx=cg["dx"], dconv_weight=cg["dw"], dconv_bias=cg["dbias"], dconv_state_in=cg["dx_prev"])
    tag = f"{io} zoh={zoh} conv={conv}"
    for k in keys:
        assert_close(with_ck[k], ref[k], io, f"with checkpoints {k} ({tag})")
        a, bb = with_ck[k].double().cpu(), without[k].double().cpu()
        assert torch.allclose(a, bb, rtol=1e-3, atol=1e-3 * (1 + float(bb.abs().max()))), f"{k} vs recomputed ({tag})"


def test_checkpoints_unsupported_paths(cuda_device):
    b, d, L = 1, 16, 64
    cpu = workloads.scan_inputs(b, d, L, io="bf16", seed=450)
    g = to_dev(cpu, "cuda")
    ck = _new_ckpt(b, d, L)
    y, last = torch.empty_like(g["u"]), torch.empty(b, d, 16, device="cuda")
    ws = ssm.new_workspace(b, d, 16, L)
    for algo in ("chunked", "direct"):
        code = ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                          g["delta_bias"], True, y, last, ws, algo=algo, checkpoints=ck, check=False)
        assert code == binding.SSM_ERR_UNSUPPORTED, algo
    # the checkpoint-storing kernels exist for 4 and 8 lanes per channel
    for lanes in (2, 42):
        code = ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                          g["delta_bias"], True, y, last, ws, algo="sequential",
                                          lanes_per_channel=lanes, checkpoints=ck, check=False)
        assert code == binding.SSM_ERR_UNSUPPORTED, lanes
    wide = workloads.scan_inputs(b, d, L, dstate=32, io="bf16", seed=451)
    gw = to_dev(wide, "cuda")
    code = ssm.ssm_selective_scan_fwd(gw["u"], gw["delta"], gw["A"], gw["B"], gw["C"], gw["D"], gw["z"],
                                      gw["delta_bias"], True, y, torch.empty(b, d, 32, device="cuda"),
                                      ssm.new_workspace(b, d, 32, L), checkpoints=torch.zeros(b, 8, d, 32, device="cuda"),
                                      check=False)
    assert code == binding.SSM_ERR_UNSUPPORTED


def test_backward_with_checkpoints_headline_shape(cuda_device):
    # The Mamba-2.8B layer workload (batch 4, d_inner 5120, L 2048, bf16): the backward reading the
    # forward's checkpoints agrees with the backward that recomputes them, every gradient, to the
    # rounding of the fp32 states (the two forwards may split the chains over lanes differently).
    w = workloads.WORKLOADS[2]
    cpu = workloads.workload_inputs(w)
    g = to_dev(cpu, "cuda")
    dy = torch.randn(w.batch, w.dim, w.seqlen, generator=torch.Generator().manual_seed(460)).to(torch.bfloat16).cuda()
    ck = _new_ckpt(w.batch, w.dim, w.seqlen)
    ssm.selective_scan_fwd(**g, checkpoints=ck)
    with_ck = ssm.selective_scan_bwd(**g, dy=dy, checkpoints=ck)
    without = ssm.selective_scan_bwd(**g, dy=dy)
    torch.cuda.synchronize()
    assert torch.isfinite(ck).all()
    for k in ["du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state"]:
        a, b = with_ck[k].double(), without[k].double()
        err = float(((a - b).abs() / (1 + b.abs())).max())
        assert err <= 2e-2, (k, err)
