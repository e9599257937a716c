"""Every entry point over a grid of shapes, through the C ABI: each call must succeed, leave the
device status clean and give finite outputs.  (Values are checked against the oracle in the
parity tests; this sweep is about launch planning and staging across shapes: one channel to
tens of thousands, sequences from one step to 2048 with rows that are and are not 16-byte
multiples, tiles that need several rounds per CTA.)"""
import numpy as np
import pytest
import torch

import selective_state_space_16_b200 as ssm
import workloads

pytestmark = pytest.mark.gpu

MAX_ELEMENTS = 24 << 20  # per (batch, dim, L) tensor
GRID = [(b, d, L)
        for b, d in [(1, 1), (1, 7), (3, 20), (1, 1536), (2, 5120), (8, 5120), (16, 2048), (64, 256), (200, 64),
                     (1, 8192), (2, 12288)]
        for L in (1, 63, 129, 2047, 2048)
        if b * d * L <= MAX_ELEMENTS]


def _finite(t):
    return bool(torch.isfinite(t.float()).all())


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("b,d,L", GRID, ids=[f"b{b}_d{d}_L{L}" for b, d, L in GRID])
def test_shape_sweep(cuda_device, b, d, L, io):
    g = {k: (v.cuda() if v is not None else None)
         for k, v in workloads.scan_inputs(b, d, L, io=io, seed=7).items()}
    ws = ssm.new_workspace(b, d, 16, L)
    y = torch.empty_like(g["u"])
    last = torch.empty(b, d, 16, device="cuda")
    variants = {"default": {}, "sequential": dict(algo="sequential"), "zoh": dict(zoh=True),
                "checkpoints": dict(checkpoints=torch.empty(b, (L + 7) // 8, d, 16, device="cuda"))}
    for name, opts in variants.items():
        ssm.ssm_selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                                   y, last, ws, **opts)
        assert ssm.ssm_read_status(ws) == 0, name
        assert _finite(y) and _finite(last), name
    cw = torch.from_numpy(np.random.default_rng(7).normal(0, 0.3, (d, 4)).astype(np.float32)).cuda()
    ssm.ssm_selective_scan_fwd_conv(g["u"], cw, None, g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                    g["delta_bias"], True, y, last, ws)
    assert ssm.ssm_read_status(ws) == 0, "conv"
    assert _finite(y) and _finite(last), "conv"
    if b * d * L <= (8 << 20):
        dy = torch.randn(b, d, L, generator=torch.Generator().manual_seed(8)).to(g["u"].dtype).cuda()
        out = ssm.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                     dy=dy)
        torch.cuda.synchronize()
        for k in ("du", "ddelta", "dA", "dB", "dC"):
            assert _finite(out[k]), f"backward {k}"
