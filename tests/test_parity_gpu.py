"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs, element by element, with the spec's tolerances:
  fp32 I/O: |x - x_ref| <= 1e-4 (1 + |x_ref|);  bf16 I/O: |x - x_ref| <= 2e-2 (1 + |x_ref|).
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_16_b200 as ssm
import workloads
from parity import TOL, assert_close, check_forward, gpu_forward, oracle_forward, to_dev

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ kernel variants, ragged sizes
VARIANTS = [("sequential", 2), ("sequential", 4), ("sequential", 8), ("sequential", 42), ("chunked", 0),
            ("direct", 0)]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("algo,lanes", VARIANTS, ids=[f"{a}{g or ''}" for a, g in VARIANTS])
def test_forward_variants_ragged(cuda_device, io, algo, lanes):
    # lanes: lanes per channel; 42 = 4 lanes per channel, each lane carrying two channels
    if io == "f32" and lanes == 8:
        pytest.skip("8 lanes per channel needs 8 steps per 16-byte group (bf16)")
    # 100 channels: not a multiple of any channel tile; L = 1000: not a multiple of a stage.
    inp = workloads.scan_inputs(2, 100, 1000, io=io, seed=11)
    check_forward(inp, algo=algo, lanes_per_channel=lanes, what=f"{algo}/{lanes}/{io}")


@pytest.mark.parametrize("flags", [dict(with_z=False), dict(with_D=False), dict(with_bias=False),
                                   dict(with_z=False, with_D=False, with_bias=False)],
                         ids=["no_gate", "no_D", "no_bias", "bare"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_forward_optional_inputs(cuda_device, flags, io):
    inp = workloads.scan_inputs(2, 64, 512, io=io, seed=12, **flags)
    check_forward(inp, what=str(flags))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_forward_softplus_off(cuda_device, io):
    inp = workloads.scan_inputs(1, 48, 256, io=io, seed=13)
    # With softplus off the step is delta + bias itself, so both are made positive here
    # (the workload's bias is an inverse softplus, i.e. negative).
    inp["delta"] = (inp["delta"].float().abs() * 0.5 + 0.01).to(inp["delta"].dtype)
    inp["delta_bias"] = torch.linspace(0.0, 0.05, inp["delta_bias"].numel())
    check_forward(inp, softplus=False, what="softplus off")


@pytest.mark.parametrize("L", [1, 7, 8, 9, 63, 64, 65, 4095, 4096])
def test_forward_edge_lengths(cuda_device, L):
    inp = workloads.scan_inputs(2, 20, L, io="bf16", seed=14 + L)
    check_forward(inp, what=f"L={L}")


@pytest.mark.parametrize("io,L", [("f32", 1001), ("f32", 1002), ("bf16", 1001), ("bf16", 1004)])
def test_forward_unaligned_rows(cuda_device, io, L):
    # L * sizeof(element) not a multiple of 16 (every row a different offset from the 16-byte
    # grid): at this small shape the default copies u, delta, z into padded rows in the
    # workspace; the sequential kernel requested explicitly gathers the rows itself (4 and 8
    # lanes per channel), and 2 lanes per channel fall back to the padded copy.
    inp = workloads.scan_inputs(2, 100, L, io=io, seed=70 + L)
    check_forward(inp, what=f"padded rows {io} L={L}")
    check_forward(inp, algo="sequential", lanes_per_channel=4, what=f"gathered rows {io} L={L} 4 lanes")
    check_forward(inp, algo="sequential", what=f"gathered rows {io} L={L}")
    if io == "bf16":
        check_forward(inp, algo="sequential", lanes_per_channel=8, what=f"gathered rows {io} L={L} 8 lanes")
    check_forward(inp, algo="sequential", lanes_per_channel=2, what=f"padded rows {io} L={L} 2 lanes")


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("L", [160, 131])
def test_forward_more_tiles_than_one_round(cuda_device, io, L):
    # b8 d5120 (40960 channels): more 8-channel tiles than the CTAs' warps hold at once, so each
    # CTA stages them in several rounds; TMA-staged rows (L 160) and gathered rows (L 131, the
    # row words set up again for every round); checked on sampled channels
    inp = workloads.scan_inputs(8, 5120, L, io=io, seed=95)
    rng = np.random.default_rng(95)
    channels = np.sort(rng.choice(8 * 5120, 512, replace=False))
    check_forward(inp, channels=channels, what=f"b8 d5120 L{L} {io}, several rounds")


@pytest.mark.parametrize("L", [1, 7, 9, 63, 65, 127, 129, 193])
def test_forward_gathered_rows_short_and_ragged(cuda_device, L):
    # gathered rows around the stage length (64 bf16 steps) and the copies one stage past
    # the last; 20 channels (a partial 8-channel tile), with and without the z gate
    for with_z in (True, False):
        inp = workloads.scan_inputs(3, 20, L, io="bf16", seed=80 + L, with_z=with_z)
        check_forward(inp, algo="sequential", what=f"gathered rows L={L} z={with_z}")


def test_forward_unaligned_headline_full_size(cuda_device):
    # the Mamba-2.8B layer shape one step short of 2048: every row starts 2 bytes off the last.
    # The default gathers the rows in the kernel at this shape.  Storing checkpoints takes the
    # padded copy instead; with the same lanes per channel both stage the same values and run
    # the same arithmetic, so y and the final state agree bit for bit.
    inp = workloads.scan_inputs(4, 5120, 2047, io="bf16", seed=71)
    check_forward(inp, what="b4 d5120 L2047")
    y_ga, last_ga = gpu_forward(inp, lanes_per_channel=4)
    ck = torch.empty(4, (2047 + 7) // 8, 5120, 16, device="cuda")
    y_pad, last_pad = gpu_forward(inp, lanes_per_channel=4, checkpoints=ck)
    assert torch.equal(y_ga, y_pad) and torch.equal(last_ga, last_pad)


def test_forward_empty_sequence_gives_zero_state(cuda_device):
    inp = workloads.scan_inputs(2, 20, 0, io="bf16", seed=15)
    y, last = gpu_forward(inp)
    assert y.numel() == 0 and torch.all(last == 0)


def test_forward_single_channel(cuda_device):
    check_forward(workloads.scan_inputs(1, 1, 300, io="f32", seed=16), what="b1 d1")


def test_workspace_reuse_is_deterministic(cuda_device):
    inp = workloads.scan_inputs(2, 96, 640, io="bf16", seed=17)
    g = to_dev(inp, "cuda")
    ws = ssm.new_workspace(2, 96, 16, 640)
    y1, l1 = ssm.selective_scan_fwd(**g, workspace=ws)
    y2, l2 = ssm.selective_scan_fwd(**g, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(l1, l2)
    assert ssm.ssm_read_status(ws) == 0


# ------------------------------------------------------------------ the five workloads, full size
@pytest.mark.parametrize("idx", [0, 1, 2])
def test_workload_full_size(cuda_device, idx):
    w = workloads.WORKLOADS[idx]
    check_forward(workloads.workload_inputs(w), what=w.name)


def test_workload_long_sequence_sampled(cuda_device):
    w = workloads.WORKLOADS[3]
    inp = workloads.workload_inputs(w)
    rng = np.random.default_rng(3)
    channels = np.sort(rng.choice(w.batch * w.dim, size=384, replace=False))
    check_forward(inp, channels=channels, what=w.name + " (sampled channels)")


# ------------------------------------------------------------------ chunked scan (look-back)
def test_chunked_headline_full_size(cuda_device):
    w = workloads.WORKLOADS[2]
    check_forward(workloads.workload_inputs(w), algo="chunked", what=w.name + " chunked")


def test_chunked_long_sequence_sampled(cuda_device):
    # the long workload (L 32768, decay persisting across chunks) through the look-back
    # kernel, every output of 384 sampled channels against the oracle
    w = workloads.WORKLOADS[3]
    inp = workloads.workload_inputs(w)
    rng = np.random.default_rng(33)
    channels = np.sort(rng.choice(w.batch * w.dim, size=384, replace=False))
    check_forward(inp, channels=channels, algo="chunked", what=w.name + " chunked (sampled channels)")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_chunked_many_chunks_few_channels(cuda_device, io):
    # one tile, 70+ chunks: the look-back chain is long and the ragged last chunk is partial
    inp = workloads.scan_inputs(1, 8, 4600 if io == "bf16" else 2300, io=io, seed=41)
    check_forward(inp, algo="chunked", what=f"chunked long chain {io}")


def test_chunked_workspace_reuse(cuda_device):
    # Consecutive launches on one workspace (flag epochs and the ticket counter are reset
    # by each launch).  The look-back combines a unit's predecessors in whatever order
    # their states are published, so floating-point rounding may differ between launches:
    # every launch must match the oracle, and launches must agree to rounding.
    cpu = workloads.scan_inputs(2, 40, 1024, io="f32", seed=42)
    inp = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(2, 40, 16, 1024)
    outs = [ssm.selective_scan_fwd(**inp, workspace=ws, algo="chunked") for _ in range(3)]
    torch.cuda.synchronize()
    y_ref, last_ref = oracle_forward(cpu)
    for y, last in outs:
        assert_close(y, y_ref, "f32", "chunked relaunch y")
        assert_close(last, last_ref, "f32", "chunked relaunch last_state")
        assert torch.allclose(y, outs[0][0], rtol=1e-5, atol=1e-6)
    assert ssm.ssm_read_status(ws) == 0


def test_chunked_lookback_wait_is_bounded(cuda_device):
    """Units of chunk 3 never publish: their successors' look-back waits must run out,
    record SSM_ERR_TIMEOUT and let the kernel finish; the workspace then still serves
    a normal call."""
    cpu = workloads.scan_inputs(1, 16, 1024, io="bf16", seed=43)
    inp = to_dev(cpu, "cuda")
    ws = ssm.new_workspace(1, 16, 16, 1024)
    ssm.selective_scan_fwd(**inp, workspace=ws, algo="chunked", spin_limit=2000, debug_skip_publish=3)
    assert ssm.ssm_read_status(ws) == 4          # SSM_ERR_TIMEOUT, read back and cleared
    assert ssm.ssm_read_status(ws) == 0
    y, last = ssm.selective_scan_fwd(**inp, workspace=ws, algo="chunked")
    torch.cuda.synchronize()
    y_ref, last_ref = oracle_forward(cpu)
    assert_close(y, y_ref, "bf16", "after timeout: y")
    assert_close(last, last_ref, "bf16", "after timeout: last_state")


# ------------------------------------------------------------------ decode
def _decode_gpu_step(state, s, dec, y):
    ssm.ssm_state_update(state, s["u"], s["delta"], dec["A"], s["B"], s["C"], dec["D"], s["z"],
                         dec["delta_bias"], True, y)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_small_chain(cuda_device, io):
    dec = workloads.decode_inputs(3, 50, io=io, seed=21, pool=4)
    g = dict(A=dec["A"].cuda(), D=dec["D"].cuda(), delta_bias=dec["delta_bias"].cuda())
    state = dec["state0"].cuda()
    st_ref = dec["state0"].double().numpy()
    for step in range(12):
        s = dec["sets"][step % 4]
        sg = {k: v.cuda() for k, v in s.items()}
        y = torch.empty_like(sg["u"])
        _decode_gpu_step(state, sg, g, y)
        y_ref, st_ref = oracle.state_update(st_ref, s["u"], s["delta"], dec["A"], s["B"], s["C"], D=dec["D"],
                                            z=s["z"], delta_bias=dec["delta_bias"])
        torch.cuda.synchronize()
        assert_close(y, y_ref, io, f"decode y step {step}")
        assert_close(state, st_ref, io, f"decode state step {step}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_unaligned_bc(cuda_device, io):
    # B and C one element past a 16-byte boundary: the step reads them element by element
    dec = workloads.decode_inputs(2, 37, io=io, seed=23, pool=1)
    s = dec["sets"][0]
    sg = {k: v.cuda() for k, v in s.items()}
    for k in ("B", "C"):
        buf = torch.zeros(sg[k].numel() + 1, dtype=sg[k].dtype, device="cuda")
        buf[1:] = sg[k].reshape(-1)
        sg[k] = buf[1:].view(sg[k].shape)
        assert sg[k].data_ptr() % 16 != 0
    g = dict(A=dec["A"].cuda(), D=dec["D"].cuda(), delta_bias=dec["delta_bias"].cuda())
    state = dec["state0"].cuda()
    y = torch.empty_like(sg["u"])
    _decode_gpu_step(state, sg, g, y)
    y_ref, st_ref = oracle.state_update(dec["state0"], s["u"], s["delta"], dec["A"], s["B"], s["C"], D=dec["D"],
                                        z=s["z"], delta_bias=dec["delta_bias"])
    torch.cuda.synchronize()
    assert_close(y, y_ref, io, "decode y, unaligned B/C")
    assert_close(state, st_ref, io, "decode state, unaligned B/C")


def test_decode_chain_equals_forward(cuda_device):
    inp = workloads.scan_inputs(2, 40, 64, io="f32", seed=22)
    y_fwd, last_fwd = gpu_forward(inp)
    g = to_dev(inp, "cuda")
    state = torch.zeros(2, 40, 16, device="cuda")
    ys = []
    for t in range(64):
        y = torch.empty(2, 40, device="cuda")
        ssm.ssm_state_update(state, g["u"][:, :, t].contiguous(), g["delta"][:, :, t].contiguous(), g["A"],
                             g["B"][:, :, t].contiguous(), g["C"][:, :, t].contiguous(), g["D"],
                             g["z"][:, :, t].contiguous(), g["delta_bias"], True, y)
        ys.append(y)
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=2)
    assert_close(y_dec, y_fwd.double().cpu().numpy(), "f32", "decode chain vs forward y")
    assert_close(state, last_fwd.double().cpu().numpy(), "f32", "decode chain vs forward state")


def test_decode_workload_full_size_sampled(cuda_device):
    w = workloads.WORKLOADS[4]
    dec = workloads.workload_decode_inputs(w)
    g = dict(A=dec["A"].cuda(), D=dec["D"].cuda(), delta_bias=dec["delta_bias"].cuda())
    sets = [{k: v.cuda() for k, v in s.items()} for s in dec["sets"]]
    state = dec["state0"].cuda()
    y = torch.empty(w.batch, w.dim, dtype=torch.bfloat16, device="cuda")
    d0, k = 1234, 8  # sampled channels: every batch row, d in [d0, d0+k)
    sl = slice(d0, d0 + k)
    st_ref = dec["state0"][:, sl].double().numpy()
    A, D, bias = dec["A"][sl], dec["D"][sl], dec["delta_bias"][sl]
    for step in range(w.decode_steps):
        s = dec["sets"][step % workloads.POOL]
        _decode_gpu_step(state, sets[step % workloads.POOL], g, y)
        y_ref, st_ref = oracle.state_update(st_ref, s["u"][:, sl], s["delta"][:, sl], A, s["B"], s["C"], D=D,
                                            z=s["z"][:, sl], delta_bias=bias)
        if step + 1 in (1, 10, w.decode_steps):
            torch.cuda.synchronize()
            assert_close(y[:, sl], y_ref, "bf16", f"decode y after {step + 1} steps")
            assert_close(state[:, sl], st_ref, "bf16", f"decode state after {step + 1} steps")
