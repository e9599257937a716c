"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same seeded inputs, and compare with the tolerances of the spec:
    fp32 I/O:            max |x - x_ref| <= 1e-4 * (1 + |x_ref|)
    bf16 I/O, fp32 state: max |x - x_ref| <= 2e-2 * (1 + |x_ref|)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import selective_state_space_16_b200 as ssm

TOL = {"f32": 1e-4, "bf16": 2e-2}


def io_of(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


def to_dev(inputs, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def rel_err(x, ref):
    x = x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, dtype=np.float64)
    return np.abs(x - ref) / (1.0 + np.abs(ref))


def assert_close(x, ref, io, what):
    e = rel_err(x, ref)
    worst = float(e.max()) if e.size else 0.0
    assert np.isfinite(worst) and worst <= TOL[io], f"{what}: max rel err {worst:.3e} > {TOL[io]} ({io})"
    return worst


def gpu_forward(inp, dev="cuda", softplus=True, h0=None, **opts):
    g = to_dev(inp, dev)
    y, last = ssm.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                     g["delta_bias"], softplus=softplus,
                                     initial_state=None if h0 is None else h0.to(dev), **opts)
    torch.cuda.synchronize()
    return y, last


def oracle_forward(inp, softplus=True, channels=None, h0=None):
    """Full oracle, or only the listed flat channels (b*dim + d) when `channels` is given;
    returns (y, last) restricted to those channels in that order.  h0: initial state
    (b, d, N) or None (zero)."""
    if channels is None:
        return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                     z=inp["z"], delta_bias=inp["delta_bias"], softplus=softplus, h0=h0)
    b_, d_, L = inp["u"].shape
    ys, lasts = [], []
    channels = np.asarray(channels)
    for bi in np.unique(channels // d_):
        ds = channels[channels // d_ == bi] % d_
        sub = dict(u=inp["u"][bi, ds][None], delta=inp["delta"][bi, ds][None], A=inp["A"][ds],
                   B=inp["B"][bi][None], C=inp["C"][bi][None],
                   D=None if inp["D"] is None else inp["D"][ds],
                   z=None if inp["z"] is None else inp["z"][bi, ds][None],
                   delta_bias=None if inp["delta_bias"] is None else inp["delta_bias"][ds],
                   h0=None if h0 is None else h0[bi, ds][None])
        y, last = oracle.selective_scan(**sub, softplus=softplus)
        ys.append((bi, ds, y[0], last[0]))
    order = {(int(bi), int(d)): (y[i], last[i]) for bi, ds, y, last in ys for i, d in enumerate(ds)}
    yy = np.stack([order[(int(c // d_), int(c % d_))][0] for c in channels])
    ll = np.stack([order[(int(c // d_), int(c % d_))][1] for c in channels])
    return yy, ll


def check_forward(inp, softplus=True, channels=None, what="forward", h0=None, **opts):
    io = io_of(inp["u"])
    y, last = gpu_forward(inp, softplus=softplus, h0=h0, **opts)
    y_ref, last_ref = oracle_forward(inp, softplus=softplus, channels=channels, h0=h0)
    if channels is not None:
        b_, d_, L = inp["u"].shape
        idx = torch.as_tensor(np.asarray(channels), device=y.device)
        y = y.reshape(b_ * d_, L).index_select(0, idx)
        last = last.reshape(b_ * d_, -1).index_select(0, idx)
    e1 = assert_close(y, y_ref, io, what + " y")
    e2 = assert_close(last, last_ref, io, what + " last_state")
    return e1, e2
