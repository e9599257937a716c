"""GPU parity of ssm_selective_scan_bwd_ex -- the backward of the zero-order-hold scan and of
the scan with the causal conv1d + SiLU prologue -- against the fp64 oracle backward (pinned by
finite differences of the RK4-pinned ZOH forward and of the numpy.convolve-pinned conv).

With the conv, the kernel recomputes u = silu(conv(x)) rounded to the I/O type (as the forward
feeds the scan) and takes the gradient through that rounding unchanged; the reference does the
same: the oracle's u rounded to the I/O type enters the oracle scan backward, whose du then
enters the oracle conv backward in fp64.  Tolerances as the forward: |x - x_ref| <= tol
(1 + |x_ref|), tol 1e-4 for fp32 I/O and 2e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, io_of, to_dev

pytestmark = pytest.mark.gpu

SCAN_KEYS = ["ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state"]


def _grads_in(b, d, L, io, seed, with_state=False):
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(b, d, L, generator=g).to(workloads.io_torch_dtype(io))
    dlast = torch.randn(b, d, 16, generator=g) if with_state else None
    h0 = workloads.initial_state(b, d, seed=seed + 1) if with_state else None
    return dy, dlast, h0


def _reference(inp, dy, zoh, conv=None, h0=None, dlast=None, dconv_out=None, softplus=True):
    u = inp["u"]
    if conv is not None:
        u_f64, _ = oracle.causal_conv_silu(inp["u"], conv["conv_weight"], conv["conv_bias"], conv["conv_state_in"])
        u = torch.from_numpy(u_f64).to(inp["u"].dtype)   # the scan sees u rounded to the I/O type
    ref = oracle.selective_scan_bwd(u, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                    delta_bias=inp["delta_bias"], softplus=softplus, h0=h0, dy=dy, dlast=dlast,
                                    zoh=zoh)
    ref["dinitial_state"] = ref.pop("dh0")
    if conv is not None:
        c = oracle.causal_conv_silu_bwd(inp["u"], conv["conv_weight"], ref["du"], conv["conv_bias"],
                                        conv["conv_state_in"], dx_next=dconv_out)
        ref.update(dx=c["dx"], dconv_weight=c["dw"], dconv_bias=c["dbias"], dconv_state_in=c["dx_prev"])
    return ref


def check(inp, dy, zoh=False, conv=None, h0=None, dlast=None, dconv_out=None, softplus=True, what=""):
    io = io_of(inp["u"])
    g = to_dev(inp, "cuda")
    c = to_dev(conv, "cuda") if conv is not None else {}
    out = ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                 softplus=softplus, dy=dy.cuda(), initial_state=None if h0 is None else h0.cuda(),
                                 dlast_state=None if dlast is None else dlast.cuda(), zoh=zoh,
                                 conv_weight=c.get("conv_weight"), conv_bias=c.get("conv_bias"),
                                 conv_state_in=c.get("conv_state_in"),
                                 dconv_state_out=None if dconv_out is None else dconv_out.cuda())
    torch.cuda.synchronize()
    ref = _reference(inp, dy, zoh, conv, h0, dlast, dconv_out, softplus)
    keys = SCAN_KEYS + (["dx", "dconv_weight", "dconv_bias"] if conv is not None else ["du"])
    if conv is not None and conv["conv_weight"].shape[1] > 1:
        keys.append("dconv_state_in")
    worst = {}
    for k in keys:
        if ref[k] is None:
            continue
        worst[k] = assert_close(out[k], ref[k], io, f"{what} {k}")
    return worst


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_backward_ragged(cuda_device, io):
    # 100 channels (not a multiple of a CTA's 32), L = 1000 (not a multiple of a segment);
    # Delta A spans both regimes of the ZOH weight (|Delta A| below and above 1/16)
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=201)
    dy, _, _ = _grads_in(2, 100, 1000, io, 202)
    check(inp, dy, zoh=True, what=f"zoh {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_backward_states_and_zero_A(cuda_device, io):
    inp = workloads.scan_inputs(2, 70, 333, io=io, seed=203)
    inp["A"][:, 0] = 0.0          # the ZOH weight's limit Delta B, and its A-derivative Delta^2 / 2
    inp["A"][:, 1] = -1e-4
    dy, dlast, h0 = _grads_in(2, 70, 333, io, 204, with_state=True)
    check(inp, dy, zoh=True, h0=h0, dlast=dlast, what=f"zoh states {io}")


def test_zoh_backward_softplus_off(cuda_device):
    inp = workloads.scan_inputs(1, 40, 257, io="f32", seed=205)
    inp["delta"] = inp["delta"].abs() + 0.01
    inp["delta_bias"] = torch.zeros(40)
    dy, _, _ = _grads_in(1, 40, 257, "f32", 206)
    check(inp, dy, zoh=True, softplus=False, what="zoh softplus off")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_conv_backward_widths(cuda_device, io, K):
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=210 + K)
    conv = workloads.conv_inputs(2, 100, K, seed=220 + K, with_state=K > 1)
    dy, _, _ = _grads_in(2, 100, 1000, io, 230 + K)
    check(inp, dy, conv=conv, what=f"conv K={K} {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_backward_all_inputs(cuda_device, io):
    # carried-in conv state and its gradient, gradient reaching the carried-out inputs,
    # initial SSM state and dlast, no conv bias
    b, d, L = 2, 70, 333
    inp = workloads.scan_inputs(b, d, L, io=io, seed=240)
    conv = workloads.conv_inputs(b, d, 4, seed=241, with_bias=False, with_state=True)
    dy, dlast, h0 = _grads_in(b, d, L, io, 242, with_state=True)
    dconv_out = torch.randn(b, d, 3, generator=torch.Generator().manual_seed(243))
    check(inp, dy, conv=conv, h0=h0, dlast=dlast, dconv_out=dconv_out, what=f"conv full {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_zoh_backward(cuda_device, io):
    inp = workloads.scan_inputs(2, 64, 520, io=io, seed=250)
    conv = workloads.conv_inputs(2, 64, 4, seed=251, with_state=True)
    dy, _, _ = _grads_in(2, 64, 520, io, 252)
    check(inp, dy, zoh=True, conv=conv, what=f"conv+zoh {io}")


@pytest.mark.parametrize("L", [1, 2, 3, 7, 9, 17])
def test_conv_backward_short_sequences(cuda_device, L):
    # L < width - 1: the carried-out inputs (and their gradient) reach back into the state
    inp = workloads.scan_inputs(2, 36, L, io="f32", seed=260 + L)
    conv = workloads.conv_inputs(2, 36, 4, seed=270 + L, with_state=True)
    dy, _, _ = _grads_in(2, 36, L, "f32", 280 + L)
    dconv_out = torch.randn(2, 36, 3, generator=torch.Generator().manual_seed(290 + L))
    check(inp, dy, conv=conv, dconv_out=dconv_out, what=f"conv L={L}")


def test_conv_backward_empty_sequence(cuda_device):
    b, d, K = 2, 8, 4
    inp = workloads.scan_inputs(b, d, 0, io="f32", seed=300)
    conv = to_dev(workloads.conv_inputs(b, d, K, seed=301, with_state=True), "cuda")
    g = to_dev(inp, "cuda")
    dconv_out = torch.randn(b, d, K - 1, generator=torch.Generator().manual_seed(302)).cuda()
    out = ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                 dy=torch.empty_like(g["u"]), conv_weight=conv["conv_weight"],
                                 conv_bias=conv["conv_bias"], conv_state_in=conv["conv_state_in"],
                                 dconv_state_out=dconv_out)
    torch.cuda.synchronize()
    assert torch.all(out["dconv_weight"] == 0) and torch.all(out["dconv_bias"] == 0)
    assert torch.equal(out["dconv_state_in"], dconv_out)


def test_conv_backward_is_deterministic(cuda_device):
    inp = workloads.scan_inputs(2, 96, 700, io="bf16", seed=310)
    conv = to_dev(workloads.conv_inputs(2, 96, 4, seed=311, with_state=True), "cuda")
    g = to_dev(inp, "cuda")
    dy = torch.randn(2, 96, 700, generator=torch.Generator().manual_seed(312)).to(torch.bfloat16).cuda()
    outs = [ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                   dy=dy, zoh=True, conv_weight=conv["conv_weight"], conv_bias=conv["conv_bias"],
                                   conv_state_in=conv["conv_state_in"]) for _ in range(2)]
    torch.cuda.synchronize()
    for k, v in outs[0].items():
        if v is not None:
            assert torch.equal(v, outs[1][k]), k


def test_conv_backward_mamba_layer_sampled(cuda_device):
    # A Mamba-130M-like layer (bf16, d_inner 1536, L 2048, conv width 4, ZOH) on one batch
    # row; the per-channel gradients compared on 48 sampled channels (dB and dC, sums over
    # all channels, are covered by the full comparisons above).
    b, d, L = 1, 1536, 2048
    inp = workloads.scan_inputs(b, d, L, io="bf16", seed=320)
    conv = workloads.conv_inputs(b, d, 4, seed=321, with_state=False)
    dy, _, _ = _grads_in(b, d, L, "bf16", 322)
    g = to_dev(inp, "cuda")
    c = to_dev(conv, "cuda")
    out = ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                 dy=dy.cuda(), zoh=True, conv_weight=c["conv_weight"], conv_bias=c["conv_bias"])
    torch.cuda.synchronize()
    ch = np.sort(np.random.default_rng(323).choice(d, 48, replace=False))
    sub = {k: (v[:, ch] if k in ("u", "delta", "z") else v[ch] if k in ("A", "D", "delta_bias") else v)
           for k, v in inp.items()}
    subconv = dict(conv_weight=conv["conv_weight"][ch], conv_bias=conv["conv_bias"][ch], conv_state_in=None)
    ref = _reference(sub, dy[:, ch], True, subconv)
    for k in ("dx", "ddelta", "dz"):
        assert_close(out[k][:, ch], ref[k], "bf16", f"mamba layer {k}")
    for k in ("dA", "dD", "ddelta_bias", "dconv_weight", "dconv_bias"):
        assert_close(out[k][ch], ref[k], "bf16", f"mamba layer {k}")
