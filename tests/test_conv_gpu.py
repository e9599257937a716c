"""GPU parity of the causal conv1d + SiLU prologue fused into the scan
(ssm_selective_scan_fwd_conv, ssm_state_update_conv) against the fp64 oracle's convolution
(pinned by numpy.convolve) followed by its scan.  The kernels round u to the I/O type before
the scan (as a separate conv kernel storing u would); the oracle's u is rounded the same way."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import assert_close, io_of, to_dev

pytestmark = pytest.mark.gpu


def _oracle_conv_scan(inp, conv, h0=None, zoh=False):
    dt = inp["u"].dtype
    u, x_next = oracle.causal_conv_silu(inp["u"], conv["conv_weight"], conv["conv_bias"], conv["conv_state_in"])
    u_io = torch.from_numpy(u).to(dt)   # the kernels feed the scan u rounded to the I/O type
    y, last = oracle.selective_scan(u_io, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                    delta_bias=inp["delta_bias"], h0=h0, zoh=zoh)
    return y, last, u, x_next


def _gpu_conv_scan(inp, conv, h0=None, **opts):
    g = to_dev(inp, "cuda")
    c = to_dev(conv, "cuda")
    b, d, L = inp["u"].shape
    K = conv["conv_weight"].shape[1]
    y = torch.empty_like(g["u"])
    last = torch.empty(b, d, 16, device="cuda")
    u_out = torch.empty_like(g["u"])
    state_out = torch.empty(b, d, K - 1, device="cuda") if K > 1 else None
    ws = ssm.new_workspace(b, d, 16, L)
    ssm.ssm_selective_scan_fwd_conv(g["u"], c["conv_weight"], c["conv_bias"], g["delta"], g["A"], g["B"], g["C"],
                                    g["D"], g["z"], g["delta_bias"], True, y, last, ws,
                                    conv_state_in=c["conv_state_in"], conv_state_out=state_out, u_out=u_out,
                                    initial_state=None if h0 is None else h0.cuda(), **opts)
    torch.cuda.synchronize()
    return y, last, u_out, state_out


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("algo,lanes", [("sequential", 4), ("sequential", 8), ("direct", 0), (None, 0)],
                         ids=["seq4", "seq8", "direct", "auto"])
def test_conv_scan_variants(cuda_device, io, algo, lanes):
    if io == "f32" and lanes == 8:
        pytest.skip("8 lanes per channel needs 8 steps per 16-byte group (bf16)")
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=111)
    conv = workloads.conv_inputs(2, 100, 4, seed=112, with_state=True)
    y, last, u_out, st = _gpu_conv_scan(inp, conv, algo=algo, lanes_per_channel=lanes)
    y_ref, last_ref, u_ref, x_next = _oracle_conv_scan(inp, conv)
    assert_close(u_out, u_ref, io, f"conv {algo}/{lanes} u")
    assert_close(y, y_ref, io, f"conv {algo}/{lanes} y")
    assert_close(last, last_ref, io, f"conv {algo}/{lanes} last_state")
    assert torch.equal(st.cpu().double(), torch.from_numpy(x_next)), "conv state out"


@pytest.mark.parametrize("io,L", [("bf16", 63), ("bf16", 1001), ("f32", 1001), ("bf16", 2047)])
def test_conv_scan_unaligned_rows(cuda_device, io, L):
    # rows of x that are not 16-byte multiples: x is staged like u, by a padded copy (the
    # default at this shape) or gathered by the kernel itself (the sequential kernel asked for
    # explicitly); u_out and y are stored element by element, the conv state out read from the
    # caller's x
    inp = workloads.scan_inputs(2, 72, L, io=io, seed=140 + L)
    conv = workloads.conv_inputs(2, 72, 4, seed=141, with_state=True)
    y_ref, last_ref, u_ref, x_next = _oracle_conv_scan(inp, conv)
    for opts in (dict(), dict(algo="sequential")):
        y, last, u_out, st = _gpu_conv_scan(inp, conv, **opts)
        assert_close(u_out, u_ref, io, f"conv L={L} {opts} u")
        assert_close(y, y_ref, io, f"conv L={L} {opts} y")
        assert_close(last, last_ref, io, f"conv L={L} {opts} last_state")
        assert torch.equal(st.cpu().double(), torch.from_numpy(x_next)), f"conv state out {opts}"


@pytest.mark.parametrize("K", [1, 2, 3])
def test_conv_widths_no_bias_no_state(cuda_device, K):
    inp = workloads.scan_inputs(1, 48, 300, io="f32", seed=113 + K)
    conv = workloads.conv_inputs(1, 48, K, seed=114 + K, with_bias=False)
    y, last, u_out, st = _gpu_conv_scan(inp, conv)
    y_ref, last_ref, u_ref, x_next = _oracle_conv_scan(inp, conv)
    assert_close(u_out, u_ref, "f32", f"K={K} u")
    assert_close(y, y_ref, "f32", f"K={K} y")
    if K > 1:
        assert torch.equal(st.cpu().double(), torch.from_numpy(x_next))


def test_conv_continuation_equals_whole(cuda_device):
    # blocks [0, 700) and [700, 1000), handing over both the conv state and the scan state
    b, d, L, cut = 2, 64, 1000, 704
    inp = workloads.scan_inputs(b, d, L, io="bf16", seed=115)
    conv = workloads.conv_inputs(b, d, 4, seed=116)
    first = {k: (v[..., :cut].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in inp.items()}
    second = {k: (v[..., cut:].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in inp.items()}
    y1, last1, _, st1 = _gpu_conv_scan(first, conv)
    conv2 = dict(conv, conv_state_in=st1.cpu())
    y2, last2, _, _ = _gpu_conv_scan(second, conv2, h0=last1.cpu())
    y_ref, last_ref, _, _ = _oracle_conv_scan(inp, conv)
    assert_close(torch.cat([y1, y2], dim=-1), y_ref, "bf16", "conv continuation y")
    assert_close(last2, last_ref, "bf16", "conv continuation last_state")


def test_conv_headline_sampled(cuda_device):
    w = workloads.WORKLOADS[2]
    inp = workloads.workload_inputs(w)
    conv = workloads.conv_inputs(w.batch, w.dim, 4, seed=117)
    y, last, u_out, _ = _gpu_conv_scan(inp, conv)
    rng = np.random.default_rng(11)
    chans = np.sort(rng.choice(w.batch * w.dim, size=128, replace=False))
    for c in chans:
        bi, di = divmod(int(c), w.dim)
        sub = dict(u=inp["u"][bi:bi + 1, di:di + 1], delta=inp["delta"][bi:bi + 1, di:di + 1],
                   A=inp["A"][di:di + 1], B=inp["B"][bi:bi + 1], C=inp["C"][bi:bi + 1], D=inp["D"][di:di + 1],
                   z=inp["z"][bi:bi + 1, di:di + 1], delta_bias=inp["delta_bias"][di:di + 1])
        sc = dict(conv_weight=conv["conv_weight"][di:di + 1], conv_bias=conv["conv_bias"][di:di + 1],
                  conv_state_in=None)
        y_ref, last_ref, u_ref, _ = _oracle_conv_scan(sub, sc)
        assert_close(y[bi, di], y_ref[0, 0], "bf16", f"conv headline y ch {c}")
        assert_close(last[bi, di], last_ref[0, 0], "bf16", f"conv headline state ch {c}")


def test_conv_unsupported_paths(cuda_device):
    inp = to_dev(workloads.scan_inputs(1, 16, 256, io="bf16", seed=118), "cuda")
    conv = to_dev(workloads.conv_inputs(1, 16, 4, seed=119), "cuda")
    y = torch.empty_like(inp["u"])
    ws = ssm.new_workspace(1, 16, 16, 256)
    code = ssm.ssm_selective_scan_fwd_conv(inp["u"], conv["conv_weight"], conv["conv_bias"], inp["delta"], inp["A"],
                                           inp["B"], inp["C"], inp["D"], inp["z"], inp["delta_bias"], True, y, None,
                                           ws, algo="chunked", check=False)
    assert code == ssm.binding.SSM_ERR_UNSUPPORTED


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_decode_chain_equals_forward(cuda_device, io):
    b, d, L = 3, 40, 20
    inp = workloads.scan_inputs(b, d, L, io=io, seed=120)
    conv = workloads.conv_inputs(b, d, 4, seed=121, with_state=True)
    g = to_dev(inp, "cuda")
    c = to_dev(conv, "cuda")
    state = torch.zeros(b, d, 16, device="cuda")
    cst = c["conv_state_in"].clone()
    ys = []
    for t in range(L):
        y = torch.empty(b, d, dtype=g["u"].dtype, device="cuda")
        ssm.ssm_state_update_conv(state, cst, g["u"][..., t].contiguous(), c["conv_weight"], c["conv_bias"],
                                  g["delta"][..., t].contiguous(), g["A"], g["B"][..., t].contiguous(),
                                  g["C"][..., t].contiguous(), g["D"], g["z"][..., t].contiguous(), g["delta_bias"],
                                  True, y)
        ys.append(y)
    torch.cuda.synchronize()
    y_ref, last_ref, _, x_next = _oracle_conv_scan(inp, conv)
    assert_close(torch.stack(ys, dim=-1), y_ref, io, "conv decode y")
    assert_close(state, last_ref, io, "conv decode state")
    assert torch.equal(cst.cpu().double(), torch.from_numpy(x_next))
