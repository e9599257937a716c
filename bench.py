#!/usr/bin/env python
"""Benchmark of the selective scan (S6) on B200: Gelem/s (B*D*L per second).

A step is one forward scan (the whole hot path: B/C staging, step sizes,
discretisation, scan, output contraction, D skip, silu gate, final state) over the
Mamba-2.8B-shaped layer workload (batch 4, d_inner 5120, d_state 16, L 2048, bf16
I/O, fp32 state), inputs resident in HBM.  Inputs are synthetic and seeded.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One JSON line is printed by rank 0.  With N > 1 (torchrun, one rank per GPU) every
rank scans its own batch (independent sequences, no collective on the data path):
weak scaling, value = elements of all ranks / max-over-ranks time.
`--impl reference` times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "selective-scan Gelem/s (B*D*L per second), 1xB200"
UNIT = "Gelem/s"
SM_COUNT_NOMINAL = 148
MUFU_EX2_PER_CLK_PER_SM = 16     # special-function unit lanes per SM per clock
EXPS_PER_ELEMENT = 16            # exp(Delta*A[d,n]) for n = 0..15 per (b, d, t)
SM_MAX_MHZ_FALLBACK = 1965.0
HBM_GBS_FALLBACK = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=float(j["hbm_gbs"]), sm_max_mhz=float(j.get("sm_max_mhz", SM_MAX_MHZ_FALLBACK)),
                    source="measured")
    return dict(hbm_gbs=HBM_GBS_FALLBACK, sm_max_mhz=SM_MAX_MHZ_FALLBACK, source="fallback")


def scan_algorithmic_bytes(w: workloads.Workload) -> int:
    """Bytes the method must move once: u, delta, z read and y written ((b,d,L) each),
    B and C read ((b,16,L) each), final state written ((b,d,16) fp32), A/D/bias read."""
    e = 2 if w.io == "bf16" else 4
    bdl = w.batch * w.dim * w.seqlen
    return (4 * bdl * e + 2 * w.batch * w.dstate * w.seqlen * e + w.batch * w.dim * w.dstate * 4
            + w.dim * w.dstate * 4 + 2 * w.dim * 4)


def decode_algorithmic_bytes(w: workloads.Workload) -> int:
    """Per decode step: fp32 state read + written, u/delta/z read, y written ((b,d) each),
    B/C read ((b,16) each), A/D/bias read."""
    e = 2 if w.io == "bf16" else 4
    bd = w.batch * w.dim
    return (2 * bd * w.dstate * 4 + 4 * bd * e + 2 * w.batch * w.dstate * e + w.dim * w.dstate * 4 + 2 * w.dim * 4)


# ----------------------------------------------------------------------------- clocks (NVML)
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            dom, bus, devn = (getattr(props, k, None) for k in ("pci_domain_id", "pci_bus_id", "pci_device_id"))
            if all(isinstance(v, int) for v in (dom, bus, devn)):
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08X}:{bus:02X}:{devn:02X}.0".encode())
            else:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._sample()  # the first queries of a process are slow: make them before timing
            self.samples, self.reasons = [], set()
        except Exception:
            self._h = None

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()
            if not self.samples:
                self._sample()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*): NCCL over
    NVLink on GPUs; gloo when no GPU is visible (the CPU tests of this plumbing)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The job's time is the slowest rank's (every rank calls this, in the same order)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(elements_per_rank: int, world: int, steps: int, t_max: float) -> float:
    """Whole-job G elements/s: every rank scans its own full workload (weak scaling: one
    independent batch per GPU, no data-path collective), timed by the slowest rank."""
    return elements_per_rank * world * steps / t_max / 1e9


# ----------------------------------------------------------------------------- measurements
# The device sources each kernel family is compiled from (its traffic record stays valid
# while these files are unchanged).
KERNEL_SOURCES = {
    "scan_fwd_seq_kernel": ["common.cuh", "scan_math.cuh", "poly_coeffs.cuh", "scan_fwd_seq.cuh"],
    "scan_fwd_chunked_kernel": ["common.cuh", "scan_math.cuh", "poly_coeffs.cuh", "scan_fwd_seq.cuh",
                                "scan_fwd_chunked.cuh"],
    "state_update_kernel": ["common.cuh", "scan_math.cuh", "poly_coeffs.cuh", "aux_kernels.cuh"],
    "scan_bwd_kernel": ["common.cuh", "scan_math.cuh", "poly_coeffs.cuh", "scan_fwd_seq.cuh", "scan_bwd.cuh"],
    "scan_fwd_wide_kernel": ["common.cuh", "scan_math.cuh", "poly_coeffs.cuh", "scan_fwd_wide.cuh"],
}


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code (comments stripped, whitespace runs collapsed) of the device sources a
    kernel family is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_16_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            code = re.sub(r"\s+", " ", _COMMENT.sub("", fh.read())).strip()
        h.update(f.encode() + code.encode())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on the
    current sources of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    for r in recs:
        if (r.get("kernel") == kernel and r.get("workload") == workload and
                r.get("src_sha") == kernel_source_hash(kernel)):
            return r.get("dram_bytes_per_launch")
    return None


def time_forward(ssm, g, ws, steps, warmup, world, stream, clocks=None, opts=None):
    opts = opts or {}

    def call():
        ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                   True, g["y"], g["last"], ws, stream=stream, **opts)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            call()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        ev0.record(stream)
        for _ in range(steps):
            call()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) / 1e3  # seconds


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def forward_buffers(w, dev):
    inp = workloads.workload_inputs(w)
    g = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    g["y"] = torch.empty_like(g["u"])
    g["last"] = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32, device=dev)
    return inp, g


def time_calls(fn, stream, steps, warmup=3):
    """Milliseconds per call of fn() (which launches on `stream`): `warmup` untimed calls, then
    `steps` calls between two CUDA events recorded on that stream."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            fn()
        ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) / steps


def e2e_forward(ssm, w, inp, y_ref, steps, stream, nstreams=4, chunks_per_row=1):
    """Same metric through the public C-ABI call with HOST (pinned) buffers: every step
    copies all inputs host->device, runs the scan and copies y and the final state back.
    A step is cut into batch * chunks_per_row independent channel chunks; chunk c always
    runs on stream c % nstreams with private device buffers (its own copy of its batch row's
    B/C rows and of its slices of A, D, delta_bias), so uploads, scans and downloads of
    different chunks -- and of consecutive steps -- overlap without any cross-stream wait."""
    names = ["u", "delta", "z"]
    host = {k: inp[k].pin_memory() for k in names + ["B", "C", "A", "D", "delta_bias"]}
    y_h = torch.empty_like(host["u"]).pin_memory()
    last_h = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32).pin_memory()
    cw = (w.dim + chunks_per_row - 1) // chunks_per_row
    chunks = []
    for bb in range(w.batch):
        for c in range(chunks_per_row):
            d0, d1 = c * cw, min(w.dim, (c + 1) * cw)
            if d0 < d1:
                chunks.append((bb, d0, d1))
    streams = [torch.cuda.Stream() for _ in range(nstreams)]
    bufs = []
    for i, (bb, d0, d1) in enumerate(chunks):
        n = d1 - d0
        bufs.append(dict(
            u=torch.empty(1, n, w.seqlen, dtype=host["u"].dtype, device="cuda"),
            delta=torch.empty(1, n, w.seqlen, dtype=host["u"].dtype, device="cuda"),
            z=torch.empty(1, n, w.seqlen, dtype=host["u"].dtype, device="cuda"),
            B=torch.empty(1, w.dstate, w.seqlen, dtype=host["B"].dtype, device="cuda"),
            C=torch.empty(1, w.dstate, w.seqlen, dtype=host["C"].dtype, device="cuda"),
            A=torch.empty(n, w.dstate, dtype=torch.float32, device="cuda"),
            D=torch.empty(n, dtype=torch.float32, device="cuda"),
            delta_bias=torch.empty(n, dtype=torch.float32, device="cuda"),
            y=torch.empty(1, n, w.seqlen, dtype=host["u"].dtype, device="cuda"),
            last=torch.empty(1, n, w.dstate, dtype=torch.float32, device="cuda"),
            ws=ssm.new_workspace(1, n, w.dstate, w.seqlen)))
    h2d = sum(host[k].numel() * host[k].element_size() for k in names + ["A", "D", "delta_bias"])
    h2d += len(chunks) * 2 * w.dstate * w.seqlen * host["B"].element_size()   # each chunk's B/C rows
    d2h = y_h.numel() * y_h.element_size() + last_h.numel() * 4

    def step():
        for i, (bb, d0, d1) in enumerate(chunks):
            g = bufs[i]
            st = streams[i % nstreams]
            with torch.cuda.stream(st):
                for k in names:
                    g[k].copy_(host[k][bb:bb + 1, d0:d1], non_blocking=True)
                g["B"].copy_(host["B"][bb:bb + 1], non_blocking=True)
                g["C"].copy_(host["C"][bb:bb + 1], non_blocking=True)
                for k in ("A", "D", "delta_bias"):
                    g[k].copy_(host[k][d0:d1], non_blocking=True)
                ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                           g["delta_bias"], True, g["y"], g["last"], g["ws"], stream=st)
                y_h[bb:bb + 1, d0:d1].copy_(g["y"], non_blocking=True)
                last_h[bb:bb + 1, d0:d1].copy_(g["last"], non_blocking=True)

    step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for st in streams:
        st.wait_event(ev0)
    for _ in range(steps):
        step()
    for st in streams:
        stream.wait_stream(st)
    ev1.record(stream)
    torch.cuda.synchronize()
    t = ev0.elapsed_time(ev1) / 1e3
    # the downloaded result is the device-resident call's result (to bf16 rounding: the chunks
    # may take another lane split, which orders the chain sums differently)
    assert torch.allclose(y_h.float(), y_ref.float().cpu(), rtol=2e-2, atol=2e-2)
    return {"value": w.elements * steps / t / 1e9, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "pipeline": (f"pinned host buffers; {len(chunks)} channel chunks per step, each: H2D of its inputs, "
                         f"scan, D2H of y and last_state, on {nstreams} streams; steps overlap")}


def measure_long(ssm, stream, pk, steps=5):
    """Long-sequence workload (batch 1, d_inner 5120, L 32768): the default kernel choice
    and the chunked kernel (sequence split across CTAs, decoupled look-back)."""
    w = workloads.WORKLOADS[3]
    _, g = forward_buffers(w, "cuda")
    ws = ssm.new_workspace(w.batch, w.dim, w.dstate, w.seqlen)
    out = {"workload": w.name, "unit": UNIT}
    for name, opts in (("default", {}), ("chunked_lookback", {"algo": "chunked"})):
        t = time_forward(ssm, g, ws, steps, 2, 1, stream, opts=opts)
        ms = t / steps * 1e3
        out[name] = {"value": w.elements / (ms / 1e3) / 1e9, "ms_per_step": ms,
                     "hbm_frac": scan_algorithmic_bytes(w) / (ms / 1e3) / 1e9 / pk["hbm_gbs"]}
    out["chunked_lookback"]["traffic"] = traffic_record("scan_fwd_chunked_kernel", w.name)
    assert ssm.ssm_read_status(ws) == 0
    del g
    return out


def measure_decode(ssm, stream, pk, steps=None):
    w = workloads.WORKLOADS[4]
    nsteps = steps or w.decode_steps
    dec = workloads.workload_decode_inputs(w)
    A, D, bias = dec["A"].cuda(), dec["D"].cuda(), dec["delta_bias"].cuda()
    sets = [{k: v.cuda() for k, v in s.items()} for s in dec["sets"]]
    state = dec["state0"].cuda()
    y = torch.empty(w.batch, w.dim, dtype=torch.bfloat16, device="cuda")

    def chain(n):
        for i in range(n):
            s = sets[i % workloads.POOL]
            ssm.ssm_state_update(state, s["u"], s["delta"], A, s["B"], s["C"], D, s["z"], bias, True, y,
                                 stream=stream)

    with torch.cuda.stream(stream):
        chain(20)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        chain(nsteps)
    # replay() launches on the current stream, which time_calls makes `stream`
    per_step = time_calls(graph.replay, stream, 1, warmup=1) / 1e3 / nsteps
    gbs = decode_algorithmic_bytes(w) / per_step / 1e9
    del graph
    return {"workload": w.name, "value": w.batch * w.dim / per_step / 1e9, "unit": "Gelem/s (B*D per step)",
            "us_per_step": per_step * 1e6, "steps": nsteps, "launch": f"one CUDA graph of {nsteps} steps",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "note": "state is 84 MB < 126 MB L2: see ncu dram bytes",
                         "traffic": traffic_record("state_update_kernel", w.name)}}


def measure_unaligned(ssm, stream, pk, steps=10):
    """Headline shape at L = 2047 (rows not a multiple of 16 bytes, which TMA cannot address:
    at this shape the sequential kernel gathers them itself) against L = 2048 on the same
    inputs' distribution."""
    out = {"workload": "mamba2p8b_b4_d5120", "unit": UNIT}
    for L in (2048, 2047):
        inp = workloads.scan_inputs(4, 5120, L, io="bf16", seed=1002)
        g = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        g["y"] = torch.empty_like(g["u"])
        g["last"] = torch.empty(4, 5120, 16, dtype=torch.float32, device="cuda")
        ws = ssm.new_workspace(4, 5120, 16, L)
        t = time_forward(ssm, g, ws, steps, 3, 1, stream)
        ms = t / steps * 1e3
        assert ssm.ssm_read_status(ws) == 0
        out[f"L{L}"] = {"value": 4 * 5120 * L / (ms / 1e3) / 1e9, "ms_per_step": ms}
        # the same from x through the fused conv1d (width 4) + SiLU
        conv = {k: (v.cuda() if v is not None else None) for k, v in workloads.conv_inputs(4, 5120, 4, seed=5).items()}

        def call():
            ssm.ssm_selective_scan_fwd_conv(g["u"], conv["conv_weight"], conv["conv_bias"], g["delta"], g["A"], g["B"],
                                            g["C"], g["D"], g["z"], g["delta_bias"], True, g["y"], g["last"], ws,
                                            stream=stream)

        out[f"conv_L{L}"] = {"ms_per_step": time_calls(call, stream, steps)}
        del g, ws
    out["ratio_2047_to_2048"] = out["L2047"]["ms_per_step"] / out["L2048"]["ms_per_step"]
    out["conv_ratio_2047_to_2048"] = out["conv_L2047"]["ms_per_step"] / out["conv_L2048"]["ms_per_step"]
    return out


def measure_zoh(ssm, stream, pk, steps=10):
    """Headline workload with the zero-order-hold discretisation (sequential kernel)."""
    w = workloads.WORKLOADS[workloads.HEADLINE]
    _, g = forward_buffers(w, "cuda")
    ws = ssm.new_workspace(w.batch, w.dim, w.dstate, w.seqlen)
    t = time_forward(ssm, g, ws, steps, 3, 1, stream, opts={"zoh": True})
    ms = t / steps * 1e3
    assert ssm.ssm_read_status(ws) == 0
    del g
    return {"workload": w.name, "discretization": "zero-order hold", "value": w.elements / (ms / 1e3) / 1e9,
            "unit": UNIT, "ms_per_step": ms}


def measure_conv(ssm, stream, pk, steps=10):
    """Headline workload scanned from x through the fused causal conv1d (width 4) + SiLU."""
    w = workloads.WORKLOADS[workloads.HEADLINE]
    _, g = forward_buffers(w, "cuda")
    conv = {k: (v.cuda() if v is not None else None) for k, v in workloads.conv_inputs(w.batch, w.dim, 4, seed=5).items()}
    ws = ssm.new_workspace(w.batch, w.dim, w.dstate, w.seqlen)

    def call():
        ssm.ssm_selective_scan_fwd_conv(g["u"], conv["conv_weight"], conv["conv_bias"], g["delta"], g["A"], g["B"],
                                        g["C"], g["D"], g["z"], g["delta_bias"], True, g["y"], g["last"], ws,
                                        stream=stream)

    ms = time_calls(call, stream, steps)
    del g
    return {"workload": w.name, "prologue": "causal conv1d width 4 + SiLU, fused", "value": w.elements / (ms / 1e3) / 1e9,
            "unit": UNIT, "ms_per_step": ms}


WIDE_SHAPE = (4, 2048, 2048)   # batch, d_inner, L of the wider-state measurements (bf16 I/O)


def measure_wide(ssm, stream, pk, steps=5, only=None):
    """Forward scan with d_state 32, 64, 128 and 256 (batch 4, d_inner 2048, L 2048, bf16 I/O;
    inputs above L2 except B/C), timed per call with CUDA events on the launching stream.  With
    N exponentials per element the bound is the special-function unit: roofline Gelem/s =
    ex2 peak / N."""
    bsz, dim, L = WIDE_SHAPE
    sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    ex2_peak = sm_count * MUFU_EX2_PER_CLK_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e9
    out = {"workload": f"b{bsz}_d{dim}_L{L}_bf16", "unit": UNIT, "ex2_peak_gex2s": ex2_peak}
    for n in (only,) if only else (32, 64, 128, 256):
        inp = workloads.scan_inputs(bsz, dim, L, dstate=n, io="bf16", seed=900 + n)
        g = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        y = torch.empty_like(g["u"])
        last = torch.empty(bsz, dim, n, dtype=torch.float32, device="cuda")
        ws = ssm.new_workspace(bsz, dim, n, L)

        def call():
            ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                       True, y, last, ws, stream=stream)

        ms = time_calls(call, stream, steps)
        assert ssm.ssm_read_status(ws) == 0
        rate = bsz * dim * L / (ms / 1e3) / 1e9
        out[f"N{n}"] = {"ms_per_step": ms, "value": rate, "roofline_value": ex2_peak / n,
                        "ex2_frac": rate * n / ex2_peak,
                        "traffic": traffic_record("scan_fwd_wide_kernel", f"N{n}_b{bsz}_d{dim}_L{L}")}
        del g, y, last, ws
    return out


def measure_backward(ssm, stream, pk, steps=5):
    """Backward of the headline workload (gradients of every input for a seeded N(0, 1) dy),
    timed with CUDA events on the launching stream; inputs larger than L2."""
    w = workloads.WORKLOADS[workloads.HEADLINE]
    _, g = forward_buffers(w, "cuda")
    gen = torch.Generator().manual_seed(77)
    dy = torch.randn(w.batch, w.dim, w.seqlen, generator=gen).to(torch.bfloat16).cuda()
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(w.batch, w.dim, w.dstate, w.seqlen),
                     dtype=torch.uint8, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    du, ddelta, dz = torch.empty_like(g["u"]), torch.empty_like(g["u"]), torch.empty_like(g["u"])
    dA, dD, dbias = torch.empty(w.dim, w.dstate, **f32), torch.empty(w.dim, **f32), torch.empty(w.dim, **f32)
    dB, dC = torch.empty(w.batch, w.dstate, w.seqlen, **f32), torch.empty(w.batch, w.dstate, w.seqlen, **f32)

    def call():
        ssm.ssm_selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                                   dy, du, ddelta, dA, dB, dC, dD, dz, dbias, ws, stream=stream)

    def timed(fn):
        return time_calls(fn, stream, steps, warmup=2)

    ms = timed(call)
    # the same with the zero-order hold and the conv prologue (width 4, carried-in state):
    # u is then the conv input x and du receives dx
    conv = {k: (v.cuda() if v is not None else None)
            for k, v in workloads.conv_inputs(w.batch, w.dim, 4, seed=5, with_state=True).items()}
    dcw, dcb = torch.empty(w.dim, 4, **f32), torch.empty(w.dim, **f32)
    dcs = torch.empty(w.batch, w.dim, 3, **f32)

    def call_ex():
        ssm.ssm_selective_scan_bwd_ex(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                      True, dy, du, ddelta, dA, dB, dC, dD, dz, dbias, ws, zoh=True,
                                      conv_weight=conv["conv_weight"], conv_bias=conv["conv_bias"],
                                      conv_state_in=conv["conv_state_in"], dconv_weight=dcw, dconv_bias=dcb,
                                      dconv_state_in=dcs, stream=stream)

    ms_ex = timed(call_ex)
    # the forward storing its 8-step checkpoints, and the backward reading them instead of
    # recomputing them (a training step's pair of calls)
    ck = torch.empty(w.batch, (w.seqlen + 7) // 8, w.dim, w.dstate, **f32)
    fws = ssm.new_workspace(w.batch, w.dim, w.dstate, w.seqlen)

    def fwd_ck():
        ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                                   g["y"], g["last"], fws, stream=stream, checkpoints=ck)

    def bwd_ck():
        ssm.ssm_selective_scan_bwd_ex(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                      True, dy, du, ddelta, dA, dB, dC, dD, dz, dbias, ws, checkpoints=ck,
                                      stream=stream)

    ms_fwd_ck = timed(fwd_ck)
    ms_bwd_ck = timed(bwd_ck)
    # algorithmic bytes: u, delta, z, dy read and du, ddelta, dz written (2 B each), B/C read,
    # dB/dC written (fp32), A/D/bias and their gradients
    nbytes = w.elements * 14 + w.batch * w.dstate * w.seqlen * (2 * 2 + 2 * 4) + w.dim * (w.dstate + 2) * 8
    gbs = nbytes / (ms / 1e3) / 1e9
    del g
    return {"workload": w.name, "value": w.elements / (ms / 1e3) / 1e9, "unit": UNIT, "ms_per_step": ms,
            "zoh_conv": {"value": w.elements / (ms_ex / 1e3) / 1e9, "ms_per_step": ms_ex,
                         "what": "ssm_selective_scan_bwd_ex: zero-order hold + conv1d width 4 (dx, conv gradients)"},
            "with_forward_checkpoints": {"value": w.elements / (ms_bwd_ck / 1e3) / 1e9, "ms_per_step": ms_bwd_ck,
                                         "forward_ms_with_checkpoints": ms_fwd_ck,
                                         "what": "backward reading the forward's 8-step checkpoints (no forward "
                                                 "sweep); the forward call that stores them"},
            "gradients": "du, ddelta, dz, dA, dB, dC, dD, ddelta_bias", "launches_per_step": 4,
            "hbm": {"achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                    "algorithmic_bytes_per_step": nbytes,
                    "traffic": traffic_record("scan_bwd_kernel", w.name)},
            "ex2_per_element": "32 (the forward once with checkpoints, each segment once more) + 2 sigmoid + 2 softplus"}


def _oracle_sample(inp, w, channels):
    """The workload restricted to its first `channels` flat (batch, channel) rows, as a list
    of per-batch-row oracle calls (whole batch rows first)."""
    calls, left = [], channels
    for b in range(w.batch):
        if left <= 0:
            break
        c = min(left, w.dim)
        calls.append(dict(u=inp["u"][b, :c][None], delta=inp["delta"][b, :c][None], A=inp["A"][:c],
                          B=inp["B"][b][None], C=inp["C"][b][None], D=inp["D"][:c], z=inp["z"][b, :c][None],
                          delta_bias=inp["delta_bias"][:c]))
        left -= c
    return calls


def _plan_oracle_sample(inp, w, budget_s):
    """Pick a sample of about `budget_s` seconds of oracle work: the whole workload repeated
    `reps` times, or (when one pass is longer) its first `channels` rows once."""
    import oracle
    n_probe = min(w.batch * w.dim, 1024)  # enough rows to keep every oracle thread busy
    probe = _oracle_sample(inp, w, n_probe)
    for c in probe:  # untimed first call: thread-pool start-up and first-touch page faults
        oracle.selective_scan(**c)
    t0 = time.perf_counter()
    for c in probe:
        oracle.selective_scan(**c)
    per_row = (time.perf_counter() - t0) / n_probe
    rows = w.batch * w.dim
    if per_row * rows <= budget_s:
        return rows, max(1, int(budget_s / (per_row * rows)))
    return max(1, int(budget_s / per_row)), 1


def cpu_oracle_rate(w, budget_s: float):
    """Time the fp64 oracle on a bounded sample of the workload.
    Returns (Gelem/s, seconds, description, threads)."""
    import oracle
    inp = workloads.workload_inputs(w)
    rows, reps = _plan_oracle_sample(inp, w, budget_s)
    calls = _oracle_sample(inp, w, rows)
    t0 = time.perf_counter()
    for _ in range(reps):
        for c in calls:
            oracle.selective_scan(**c)
    dt = time.perf_counter() - t0
    elems = rows * w.seqlen * reps
    what = "the whole workload" if rows == w.batch * w.dim else f"its first {rows} of {w.batch * w.dim} channels"
    desc = f"{what} (L={w.seqlen}), {reps} pass(es): {elems} elements in {dt:.1f} s"
    return elems / dt / 1e9, dt, desc, oracle.num_threads()


# ----------------------------------------------------------------------------- arms
def run_reference(args, world, rank):
    """The fp64 CPU oracle on the host cores, on the headline workload: each step is a
    bounded sample of it (the whole workload when K+W steps of it fit in ~2 minutes)."""
    if rank != 0:
        return
    w = workloads.WORKLOADS[workloads.HEADLINE]
    import oracle
    oracle.build()
    inp = workloads.workload_inputs(w)
    budget_per_step = max(0.02, 120.0 / max(1, args.steps + args.warmup))
    rows, _ = _plan_oracle_sample(inp, w, budget_per_step)
    calls = _oracle_sample(inp, w, rows)
    for _ in range(args.warmup):
        for c in calls:
            oracle.selective_scan(**c)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for c in calls:
            oracle.selective_scan(**c)
    dt = time.perf_counter() - t0
    val = rows * w.seqlen * args.steps / dt / 1e9
    what = "the whole workload" if rows == w.batch * w.dim else f"its first {rows} of {w.batch * w.dim} channels"
    desc = f"{what} (L={w.seqlen}) per step"
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "impl": "reference",
            "config": {"workload": w.name, "batch": w.batch, "d_inner": w.dim, "d_state": w.dstate,
                       "seq_len": w.seqlen, "io": w.io, "sample": desc},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gpu(args, world, rank, local):
    import selective_state_space_16_b200 as ssm
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    w = workloads.WORKLOADS[workloads.HEADLINE]
    inp, g = forward_buffers(w, dev)
    ws = ssm.new_workspace(w.batch, w.dim, w.dstate, w.seqlen)
    stream = torch.cuda.Stream()
    clocks = ClockSampler(local)
    t = time_forward(ssm, g, ws, args.steps, args.warmup, world, stream, clocks)
    t = max_over_ranks(t, world)
    per_call = t / args.steps
    value = job_throughput(w.elements, world, args.steps, t)
    assert ssm.ssm_read_status(ws) == 0

    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    ex2_peak = sm_count * MUFU_EX2_PER_CLK_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e9  # G ex2 / s
    achieved_ex2 = EXPS_PER_ELEMENT * w.elements / per_call / 1e9
    hbm_achieved = scan_algorithmic_bytes(w) / per_call / 1e9
    clk = clocks.summary()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 I/O, fp32 state and arithmetic)",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "batch": w.batch, "d_inner": w.dim, "d_state": w.dstate,
                       "seq_len": w.seqlen, "io": w.io, "per_rank": "one full batch per GPU",
                       "l2": "inputs larger than L2 (338 MB per step vs 126 MB L2)", "parallelism": f"dp{world}"},
            "roofline": {"bound": "alu", "achieved": achieved_ex2, "peak": ex2_peak, "unit": "Gex2/s",
                         "frac": achieved_ex2 / ex2_peak,
                         "traffic": traffic_record("scan_fwd_seq_kernel", w.name),
                         "peak_source": f"{sm_count} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x "
                                        f"{pk['sm_max_mhz']:.0f} MHz ({pk['source']} max clock)",
                         "timed": "whole C-ABI call (B/C pack + scan kernels) per launch"},
            "roofline_hbm": {"achieved": hbm_achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": hbm_achieved / pk["hbm_gbs"], "peak_source": pk["source"],
                             "algorithmic_bytes_per_step": scan_algorithmic_bytes(w)},
            "clocks": clk,
            "gpu_launches": 2 * args.steps}
    if rank == 0:
        e2e_steps = max(3, min(args.steps, 10))
        line["e2e"] = e2e_forward(ssm, w, inp, g["y"], e2e_steps, stream)
    if world == 1 and not args.skip_extra:
        line["also"] = {"long": measure_long(ssm, stream, pk), "decode": measure_decode(ssm, stream, pk),
                        "backward": measure_backward(ssm, stream, pk), "zoh": measure_zoh(ssm, stream, pk),
                        "conv": measure_conv(ssm, stream, pk), "unaligned": measure_unaligned(ssm, stream, pk),
                        "wide": measure_wide(ssm, stream, pk)}
    if rank == 0 and world == 1 and not args.skip_cpu:
        rate, secs, desc, cores = cpu_oracle_rate(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_profile_workload(args):
    """Run only one of the extra workloads (for profiler captures)."""
    import selective_state_space_16_b200 as ssm
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    pk = peaks()
    if args.workload == "long":
        out = measure_long(ssm, stream, pk, steps=args.steps)
    elif args.workload == "backward":
        out = measure_backward(ssm, stream, pk, steps=args.steps)
    elif args.workload == "wide":
        out = measure_wide(ssm, stream, pk, steps=args.steps, only=args.dstate)
    elif args.workload == "unaligned":
        out = measure_unaligned(ssm, stream, pk, steps=args.steps)
    else:
        w = workloads.WORKLOADS[4]
        out = measure_decode(ssm, stream, pk, steps=args.steps)
    print(json.dumps({"workload": args.workload, "result": out}), flush=True)


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-extra", action="store_true")
    ap.add_argument("--workload", default="headline",
                    choices=["headline", "long", "decode", "backward", "wide", "unaligned"],
                    help="profiling runs: 'long' / 'decode' / 'backward' / 'wide' / 'unaligned' run only that "
                         "workload a few times")
    ap.add_argument("--dstate", type=int, default=None, choices=[32, 64, 128, 256],
                    help="with --workload wide: that d_state only")
    args = ap.parse_args()
    world, rank, local = dist_setup(args.gpus) if args.impl == "native" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload != "headline":
            run_profile_workload(args)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "native":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
