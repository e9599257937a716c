"""Pins for the fp64 oracle: each checks it against something other than itself
(hand-derived worked examples, closed forms, library routines, brute force), so
that a dropped term, a wrong sign or index, or a transposed operand fails here.

Pages cited (sections as printed):
  [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
  [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
  [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
  [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
  [Tech] "Transformer架构遭遇颠覆性突破：Mamba模型如何用状态空间重新定义序列建模效率？"
"""
import glob
import math
import os
import random

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _selective_case(rng, b=2, d=3, n=4, L=17, softplus=True, with_z=True, with_D=True, with_bias=True):
    """Fully time-varying inputs; A varies in both d and n (d != n) so that a transposed
    A index cannot pass."""
    u = rng.standard_normal((b, d, L))
    delta = 0.5 * rng.standard_normal((b, d, L))
    A = -rng.uniform(0.1, 2.0, (d, n))
    B = rng.standard_normal((b, n, L))
    C = rng.standard_normal((b, n, L))
    D = rng.standard_normal(d) if with_D else None
    z = rng.standard_normal((b, d, L)) if with_z else None
    bias = rng.uniform(-3, 0.5, d) if with_bias else None
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=D, z=z, delta_bias=bias, softplus=softplus)


def _step_sizes(case):
    x = case["delta"] + (0 if case["delta_bias"] is None else case["delta_bias"][None, :, None])
    return np.logaddexp(0.0, x) if case["softplus"] else x


# ---------------------------------------------------------------------------------------------
# Worked examples derived by hand (tests/golden/*.txt, each with its citation)
# ---------------------------------------------------------------------------------------------
def _parse_golden(path):
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split(":", 1)
            v = v.split()
            out[k.strip()] = v[0] if k.strip() == "kind" else [float(x) for x in v]
    return out


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "worked_*.txt"))),
                         ids=lambda p: os.path.basename(p))
def test_worked_examples(path):
    g = _parse_golden(path)
    n = int(g["dstate"][0])
    sp = bool(g["softplus"][0])
    A = np.array(g["A"]).reshape(1, n)
    D = np.array(g["D"]) if "D" in g else None
    bias = np.array(g["bias"]) if "bias" in g else None
    if g["kind"] == "scan":
        L = int(g["L"][0])
        u = np.array(g["u"]).reshape(1, 1, L)
        delta = np.array(g["delta"]).reshape(1, 1, L)
        B = np.array([g[f"B{i}"] for i in range(n)]).reshape(1, n, L)
        C = np.array([g[f"C{i}"] for i in range(n)]).reshape(1, n, L)
        z = np.array(g["z"]).reshape(1, 1, L) if "z" in g else None
        y, last = oracle.selective_scan(u, delta, A, B, C, D=D, z=z, delta_bias=bias, softplus=sp)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(last.ravel(), g["last_state"], rtol=1e-14, atol=1e-14)
    else:
        st = np.array(g["state"]).reshape(1, 1, n)
        y, new = oracle.state_update(st, np.array(g["u"]).reshape(1, 1), np.array(g["delta"]).reshape(1, 1),
                                     A, np.array(g["B"]).reshape(1, n), np.array(g["C"]).reshape(1, n),
                                     D=D, delta_bias=bias, softplus=sp)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-14)
        np.testing.assert_allclose(new.ravel(), g["last_state"], rtol=1e-14)


# ---------------------------------------------------------------------------------------------
# Elementwise helpers against library routines
# ---------------------------------------------------------------------------------------------
def test_softplus_matches_logaddexp():
    # softplus(x) = log(1 + e^x) = logaddexp(0, x)   ([Card] 选择性机制: Delta = Softplus(.))
    xs = [-745.0, -200.0, -40.0, -20.0, -5.0, -1e-3, 0.0, 1e-8, 0.3, 5.0, 20.0, 40.0, 200.0, 700.0]
    for x in xs:
        assert oracle.softplus(x) == pytest.approx(float(np.logaddexp(0.0, x)), rel=1e-15, abs=1e-300)


def test_silu_matches_expit():
    # silu(z) = z * sigmoid(z)   ([Hist] Mamba Block 数据流)
    for zv in [-700.0, -30.0, -2.5, -1e-6, 0.0, 1e-6, 0.7, 3.0, 30.0, 700.0]:
        assert oracle.silu(zv) == pytest.approx(zv * float(scipy.special.expit(zv)), rel=1e-14, abs=1e-300)


# ---------------------------------------------------------------------------------------------
# P-A: A = 0 and constant Delta, B, C  =>  scaled prefix sum  ([Card] 离散化变换 / 线性扫描算法)
# ---------------------------------------------------------------------------------------------
def test_prefix_sum_when_A_is_zero():
    rng = _rng(1)
    b, d, n, L = 2, 3, 5, 300
    u = rng.standard_normal((b, d, L))
    c = 0.37
    delta = np.full((b, d, L), c)
    Bv = rng.standard_normal((b, n))
    Cv = rng.standard_normal((b, n))
    B = np.repeat(Bv[:, :, None], L, axis=2)
    C = np.repeat(Cv[:, :, None], L, axis=2)
    D = rng.standard_normal(d)
    A = np.zeros((d, n))
    y, last = oracle.selective_scan(u, delta, A, B, C, D=D, softplus=False)
    cb = (Cv * Bv).sum(axis=1)  # (b,)
    expect = c * cb[:, None, None] * np.cumsum(u, axis=2) + D[None, :, None] * u
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(last, c * Bv[:, None, :] * u.sum(axis=2)[:, :, None], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# P-B: LTI case  =>  y = K * u + D u,  K_j = sum_n C_n Abar_n^j Bbar_n
#      ([Eng] §2.3; [S4M] 2.1; [Tech] 二.3 with kernel length L)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("L", [1, 64, 1000, 4096])
def test_lti_equals_convolution(L):
    rng = _rng(2 + L)
    d, n = 3, 16
    u = rng.standard_normal((1, d, L))
    dt = np.array([0.003, 0.02, 0.15])
    delta = np.repeat(dt[None, :, None], L, axis=2)
    A = -np.arange(1, n + 1, dtype=np.float64)[None, :] * rng.uniform(0.5, 1.5, (d, 1))
    Bv, Cv = rng.standard_normal(n), rng.standard_normal(n)
    B = np.repeat(Bv[None, :, None], L, axis=2)
    C = np.repeat(Cv[None, :, None], L, axis=2)
    D = rng.standard_normal(d)
    y, _ = oracle.selective_scan(u, delta, A, B, C, D=D, softplus=False)
    j = np.arange(L)
    for di in range(d):
        abar = np.exp(dt[di] * A[di])                       # (n,)
        K = (Cv[None, :] * abar[None, :] ** j[:, None] * (dt[di] * Bv)[None, :]).sum(axis=1)
        direct = np.convolve(u[0, di], K)[:L]
        m = 1 << (2 * L - 1).bit_length()
        viafft = np.fft.irfft(np.fft.rfft(u[0, di], m) * np.fft.rfft(K, m), m)[:L]
        np.testing.assert_allclose(y[0, di], direct + D[di] * u[0, di], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(y[0, di], viafft + D[di] * u[0, di], rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------------------------------------
# P-C / P-D: brute-force closed form  h_t = sum_{s<=t} (prod_{r=s+1..t} Abar_r) Bbar_s u_s,
#            y_t = C_t h_t  ([Card] Mamba架构设计 closed form, with the C_t read-out)
# ---------------------------------------------------------------------------------------------
def _brute_force(case):
    u, A, B, C = case["u"], case["A"], case["B"], case["C"]
    b, d, L = u.shape
    n = A.shape[1]
    dt = _step_sizes(case)
    y = np.zeros((b, d, L))
    hL = np.zeros((b, d, n))
    for bi in range(b):
        for di in range(d):
            abar = np.exp(dt[bi, di][:, None] * A[di][None, :])       # (L, n)
            for t in range(L):
                h = np.zeros(n)
                for s in range(t + 1):
                    decay = np.prod(abar[s + 1:t + 1], axis=0) if s < t else np.ones(n)
                    h += decay * dt[bi, di, s] * B[bi, :, s] * u[bi, di, s]
                yt = float(C[bi, :, t] @ h)
                if case["D"] is not None:
                    yt += case["D"][di] * u[bi, di, t]
                if case["z"] is not None:
                    zt = case["z"][bi, di, t]
                    yt *= zt * scipy.special.expit(zt)
                y[bi, di, t] = yt
                if t == L - 1:
                    hL[bi, di] = h
    return y, hL


@pytest.mark.parametrize("flags", [dict(), dict(with_z=False), dict(with_D=False, with_z=False, with_bias=False),
                                   dict(softplus=False, with_bias=False)],
                         ids=["full", "no_gate", "bare", "no_softplus"])
def test_brute_force_closed_form(flags):
    rng = _rng(3)
    case = _selective_case(rng, **flags)
    y, last = oracle.selective_scan(**case)
    y_bf, h_bf = _brute_force(case)
    np.testing.assert_allclose(y, y_bf, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(last, h_bf, rtol=1e-11, atol=1e-12)


def test_initial_state_enters_as_decayed_carry():
    # h_t = (prod_{r<=t} Abar_r) h_init + (zero-start scan)_t: the state continuation of [Eng] §7.2.
    rng = _rng(4)
    case = _selective_case(rng, with_z=False, with_D=False)
    b, d, L = case["u"].shape
    n = case["A"].shape[1]
    h0 = rng.standard_normal((b, d, n))
    y0, last0 = oracle.selective_scan(**case)
    y1, last1 = oracle.selective_scan(**case, h0=h0)
    dt = _step_sizes(case)
    P = np.exp(np.cumsum(dt, axis=2)[:, :, :, None] * case["A"][None, :, None, :])  # (b,d,L,n)
    extra_y = np.einsum("bdtn,bnt,bdn->bdt", P, case["C"], h0)
    np.testing.assert_allclose(y1, y0 + extra_y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(last1, last0 + P[:, :, -1, :] * h0, rtol=1e-11, atol=1e-12)


def test_block_continuation_equals_whole_scan():
    # Scanning [0, L1) and then [L1, L) from the first block's final state is the scan of
    # [0, L) ([Eng] §7.2): the block split is invisible in y and in the final state.
    rng = _rng(41)
    case = _selective_case(rng)
    L = case["u"].shape[2]
    y, last = oracle.selective_scan(**case)
    for cut in (1, L // 3, L - 1):
        first = {k: (v[..., :cut] if k in ("u", "delta", "z", "B", "C") and v is not None else v)
                 for k, v in case.items()}
        second = {k: (v[..., cut:] if k in ("u", "delta", "z", "B", "C") and v is not None else v)
                  for k, v in case.items()}
        y1, h1 = oracle.selective_scan(**first)
        y2, h2 = oracle.selective_scan(**second, h0=h1)
        np.testing.assert_allclose(np.concatenate([y1, y2], axis=2), y, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(h2, last, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------------------------
# P-E: two-step identity with constant Abar  ([Card] 线性扫描算法)
# ---------------------------------------------------------------------------------------------
def test_two_step_identity():
    rng = _rng(5)
    b, d, n = 2, 3, 4
    A = -rng.uniform(0.1, 2.0, (d, n))
    h0 = rng.standard_normal((b, d, n))
    dt = 0.3
    delta = np.full((b, d), dt)
    x1, x2 = rng.standard_normal((b, d)), rng.standard_normal((b, d))
    B1, B2 = rng.standard_normal((b, n)), rng.standard_normal((b, n))
    C1 = rng.standard_normal((b, n))
    _, h1 = oracle.state_update(h0, x1, delta, A, B1, C1, softplus=False)
    _, h2 = oracle.state_update(h1, x2, delta, A, B2, C1, softplus=False)
    abar = np.exp(dt * A)[None]
    expect = abar ** 2 * h0 + abar * (dt * B1[:, None, :]) * x1[..., None] + (dt * B2[:, None, :]) * x2[..., None]
    np.testing.assert_allclose(h2, expect, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------------------------
# P-F: the associative pair operator (a1,b1) (x) (a2,b2) = (a2 a1, a2 b1 + b2)  ([Eng] §4.1)
#      folded under random bracketings equals the sequential recurrence's final state.
# ---------------------------------------------------------------------------------------------
def _combine(p, q):
    return (q[0] * p[0], q[0] * p[1] + q[1])


def _random_tree_fold(pairs, rnd):
    items = list(pairs)
    while len(items) > 1:
        i = rnd.randrange(len(items) - 1)
        items[i:i + 2] = [_combine(items[i], items[i + 1])]
    return items[0]


def test_pair_operator_bracketings_match_scan():
    rng = _rng(6)
    case = _selective_case(rng, b=1, d=2, n=4, L=41, with_z=False, with_D=False)
    _, last = oracle.selective_scan(**case)
    dt = _step_sizes(case)
    rnd = random.Random(7)
    for di in range(2):
        a = np.exp(dt[0, di][:, None] * case["A"][di][None, :])                  # (L, n)
        bb = dt[0, di][:, None] * case["B"][0].T * case["u"][0, di][:, None]     # (L, n)
        pairs = [(a[t], bb[t]) for t in range(41)]
        for _ in range(5):
            P, H = _random_tree_fold(pairs, rnd)
            np.testing.assert_allclose(H, last[0, di], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(P, np.exp(dt[0, di].sum() * case["A"][di]), rtol=1e-12)


# ---------------------------------------------------------------------------------------------
# P-G: L chained decode steps from zero state equal the forward scan  ([Card] 线性扫描算法;
#      [Eng] §6.2 incremental one-step recurrence)
# ---------------------------------------------------------------------------------------------
def test_decode_chain_equals_scan():
    rng = _rng(8)
    case = _selective_case(rng, b=2, d=3, n=16, L=25)
    y, last = oracle.selective_scan(**case)
    b, d, L = case["u"].shape
    st = np.zeros((b, d, 16))
    for t in range(L):
        yt, st = oracle.state_update(st, case["u"][:, :, t], case["delta"][:, :, t], case["A"],
                                     case["B"][:, :, t], case["C"][:, :, t], D=case["D"],
                                     z=case["z"][:, :, t], delta_bias=case["delta_bias"], softplus=True)
        np.testing.assert_allclose(yt, y[:, :, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st, last, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# P-H: limits  ([Eng] §3.2; [Card] 离散化变换 / 选择性机制)
# ---------------------------------------------------------------------------------------------
def test_small_delta_freezes_state():
    rng = _rng(9)
    b, d, n = 2, 3, 8
    A = -rng.uniform(0.1, 2.0, (d, n))
    h0 = rng.standard_normal((b, d, n))
    delta = np.full((b, d), -60.0)  # softplus(-60) ~ 8.8e-27
    x = rng.standard_normal((b, d))
    Bv, Cv = rng.standard_normal((b, n)), rng.standard_normal((b, n))
    y, h1 = oracle.state_update(h0, x, delta, A, Bv, Cv, softplus=True)
    np.testing.assert_allclose(h1, h0, rtol=1e-20, atol=1e-24)
    np.testing.assert_allclose(y, np.einsum("bn,bdn->bd", Cv, h0), rtol=1e-14)


def test_large_delta_resets_state():
    rng = _rng(10)
    case = _selective_case(rng, b=1, d=2, n=4, L=30, softplus=False, with_bias=False, with_z=False)
    case["delta"] = np.full_like(case["delta"], 60.0)
    case["A"] = -np.abs(case["A"]) - 1.0  # Abar <= e^-60
    y, _ = oracle.selective_scan(**case)
    expect = 60.0 * np.einsum("bnt,bnt,bdt->bdt", case["C"], case["B"], case["u"]) + case["D"][None, :, None] * case["u"]
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# P-I: epilogue special cases  ([Eng] §2.2 D skip; [Hist] Mamba Block gate)
# ---------------------------------------------------------------------------------------------
def test_zero_B_gives_gated_skip():
    rng = _rng(11)
    case = _selective_case(rng, b=2, d=3, n=16, L=50)
    case["B"] = np.zeros_like(case["B"])
    case["D"] = np.ones(3)
    y, last = oracle.selective_scan(**case)
    z = case["z"]
    np.testing.assert_allclose(y, case["u"] * z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    assert np.all(last == 0.0)


def test_empty_and_degenerate_shapes():
    rng = _rng(12)
    case = _selective_case(rng, b=1, d=2, n=3, L=0)
    y, last = oracle.selective_scan(**case)
    assert y.shape == (1, 2, 0) and np.all(last == 0.0)
    case = _selective_case(rng, b=0, d=2, n=3, L=5)
    y, last = oracle.selective_scan(**case)
    assert y.shape == (0, 2, 5)


# ---------------------------------------------------------------------------------------------
# Backward: gradients of L = sum(dy * y) + sum(dlast * last_state) against central finite
# differences of the forward scan (itself pinned above).  A dropped term, a wrong sign or a
# transposed index in any gradient fails one element here.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("flags", [dict(), dict(softplus=False), dict(with_z=False, with_D=False, with_bias=False)],
                         ids=["full", "softplus_off", "bare"])
def test_backward_matches_finite_differences(flags):
    rng = _rng(51)
    case = _selective_case(rng, b=2, d=3, n=4, L=9, **flags)
    if not case["softplus"]:  # keep the step positive (a decaying state) without softplus
        case["delta"] = np.abs(case["delta"]) + 0.05
        case["delta_bias"] = rng.uniform(0.0, 0.05, case["delta_bias"].shape)
    b, d, L = case["u"].shape
    n = case["A"].shape[1]
    h0 = rng.standard_normal((b, d, n))
    dy = rng.standard_normal((b, d, L))
    dlast = rng.standard_normal((b, d, n))
    grads = oracle.selective_scan_bwd(**case, h0=h0, dy=dy, dlast=dlast)

    def loss(name, value):
        c = dict(case, h0=h0)
        c[name] = value
        y, last = oracle.selective_scan(**c)
        return float((dy * y).sum() + (dlast * last).sum())

    eps = 1e-6
    names = [("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("h0", "dh0")]
    names += [(k, "d" + k) for k in ("D", "z", "delta_bias") if case[k] is not None]
    for name, key in names:
        base = h0 if name == "h0" else case[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            hi, lo = base.copy(), base.copy()
            hi[idx] += eps
            lo[idx] -= eps
            fd[idx] = (loss(name, hi) - loss(name, lo)) / (2 * eps)
        np.testing.assert_allclose(grads[key], fd, rtol=1e-6, atol=1e-7 * (1 + np.abs(fd).max()), err_msg=name)
    if case["z"] is None:
        assert grads["dz"] is None


def test_backward_is_linear_in_the_output_gradient():
    rng = _rng(52)
    case = _selective_case(rng)
    b, d, L = case["u"].shape
    dy1, dy2 = rng.standard_normal((b, d, L)), rng.standard_normal((b, d, L))
    g1 = oracle.selective_scan_bwd(**case, dy=dy1)
    g2 = oracle.selective_scan_bwd(**case, dy=dy2)
    g12 = oracle.selective_scan_bwd(**case, dy=dy1 - 3.0 * dy2)
    for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias", "dh0"):
        np.testing.assert_allclose(g12[k], g1[k] - 3.0 * g2[k], rtol=1e-11, atol=1e-12, err_msg=k)


# ---------------------------------------------------------------------------------------------
# Zero-order hold ([Eng] §2.2): the discretisation of h' = A h + B x with the input held over
# each step.  Pinned against a fine fourth-order Runge-Kutta integration of that ODE.
# ---------------------------------------------------------------------------------------------
def _rk4_zoh_reference(case):
    u, A, B, C = case["u"], case["A"], case["B"], case["C"]
    b, d, L = u.shape
    n = A.shape[1]
    dt = _step_sizes(case)
    y = np.zeros((b, d, L))
    last = np.zeros((b, d, n))
    sub = 400
    for bi in range(b):
        for di in range(d):
            h = np.zeros(n)
            a = A[di]
            for t in range(L):
                drive = B[bi, :, t] * u[bi, di, t]           # held over the step
                f = lambda hh: a * hh + drive
                step = dt[bi, di, t] / sub
                for _ in range(sub):
                    k1 = f(h)
                    k2 = f(h + 0.5 * step * k1)
                    k3 = f(h + 0.5 * step * k2)
                    k4 = f(h + step * k3)
                    h = h + step / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
                yt = C[bi, :, t] @ h + (case["D"][di] if case["D"] is not None else 0.0) * u[bi, di, t]
                if case["z"] is not None:
                    zt = case["z"][bi, di, t]
                    yt *= zt / (1.0 + np.exp(-zt))
                y[bi, di, t] = yt
            last[bi, di] = h
    return y, last


def test_zoh_matches_integrated_ode():
    rng = _rng(61)
    case = _selective_case(rng, b=1, d=2, n=3, L=6)
    y, last = oracle.selective_scan(**case, zoh=True)
    y_ref, last_ref = _rk4_zoh_reference(case)
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(last, last_ref, rtol=1e-9, atol=1e-11)
    # ... and it is not the simplified discretisation
    y_s, _ = oracle.selective_scan(**case)
    assert np.abs(y_s - y).max() > 1e-3


def test_zoh_limits():
    rng = _rng(62)
    case = _selective_case(rng)
    # A = 0: the hold weight is exactly Delta*B, as the simplified discretisation
    c0 = dict(case, A=np.zeros_like(case["A"]))
    np.testing.assert_array_equal(oracle.selective_scan(**c0, zoh=True)[0], oracle.selective_scan(**c0)[0])
    # small Delta A: ZOH -> simplified, with a relative gap of order Delta*|A|
    cs = dict(case, delta=np.full_like(case["delta"], -20.0), delta_bias=None)   # softplus(-20) ~ 2e-9
    y_z, h_z = oracle.selective_scan(**cs, zoh=True)
    y_s, h_s = oracle.selective_scan(**cs)
    np.testing.assert_allclose(h_z, h_s, rtol=1e-7, atol=1e-20)


def test_zoh_decode_chain_equals_scan():
    rng = _rng(63)
    case = _selective_case(rng, L=8)
    y, last = oracle.selective_scan(**case, zoh=True)
    b, d, L = case["u"].shape
    state = np.zeros((b, d, case["A"].shape[1]))
    for t in range(L):
        yt, state = oracle.state_update(state, case["u"][..., t], case["delta"][..., t], case["A"], case["B"][..., t],
                                        case["C"][..., t], D=case["D"], z=case["z"][..., t],
                                        delta_bias=case["delta_bias"], softplus=case["softplus"], zoh=True)
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(state, last, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------------------------
# Causal depthwise conv1d + SiLU before the scan ([Hist] Mamba Block 数据流): against
# numpy.convolve per channel and scipy's expit, with and without a carried-in state.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("K", [1, 2, 4])
def test_causal_conv_matches_numpy_convolve(K):
    from scipy.special import expit
    rng = _rng(70 + K)
    b, d, L = 2, 3, 11
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, K))
    bias = rng.standard_normal(d)
    prev = rng.standard_normal((b, d, K - 1))
    for with_prev in (False, True):
        u, x_next = oracle.causal_conv_silu(x, w, bias, prev if with_prev else None)
        for bi in range(b):
            for di in range(d):
                head = prev[bi, di] if with_prev else np.zeros(K - 1)
                full = np.concatenate([head, x[bi, di]])
                # causal: output t uses full[t .. t+K-1] with w in order (oldest first)
                conv = np.convolve(full, w[di][::-1], mode="valid")
                pre = conv + bias[di]
                np.testing.assert_allclose(u[bi, di], pre * expit(pre), rtol=1e-13, atol=1e-14)
                np.testing.assert_array_equal(x_next[bi, di], full[len(full) - (K - 1):] if K > 1 else [])


def test_causal_conv_continuation():
    # converting [0, L1) then [L1, L) with the carried-in inputs equals converting [0, L)
    rng = _rng(75)
    x = rng.standard_normal((2, 3, 13))
    w = rng.standard_normal((3, 4))
    u, _ = oracle.causal_conv_silu(x, w)
    u1, s1 = oracle.causal_conv_silu(x[..., :5], w)
    u2, _ = oracle.causal_conv_silu(x[..., 5:], w, x_prev=s1)
    np.testing.assert_allclose(np.concatenate([u1, u2], axis=2), u, rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------------------------
# Backward of the zero-order-hold scan and of the conv prologue, against central finite
# differences of the forward functions pinned above (the RK4-pinned ZOH scan and the
# numpy.convolve-pinned conv).  A dropped or mis-signed term in any gradient fails here.
# ---------------------------------------------------------------------------------------------
def _central_fd(loss, base, eps=1e-6):
    fd = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        hi, lo = base.copy(), base.copy()
        hi[idx] += eps
        lo[idx] -= eps
        fd[idx] = (loss(hi) - loss(lo)) / (2 * eps)
    return fd


def _assert_fd(got, fd, what):
    np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7 * (1 + np.abs(fd).max()), err_msg=what)


@pytest.mark.parametrize("flags", [dict(), dict(softplus=False), dict(with_z=False, with_D=False, with_bias=False)],
                         ids=["full", "softplus_off", "bare"])
def test_backward_zoh_matches_finite_differences(flags):
    rng = _rng(81)
    case = _selective_case(rng, b=2, d=3, n=4, L=9, **flags)
    if not case["softplus"]:
        case["delta"] = np.abs(case["delta"]) + 0.05
        case["delta_bias"] = rng.uniform(0.0, 0.05, case["delta_bias"].shape)
    # both regimes of the ZOH weight's A-derivative: |Delta A| < 1e-3 (series) and A = 0
    case["A"][0, 1] = -2e-5
    case["A"][1, 2] = 0.0
    case["A"][2, 0] = 3e-4
    b, d, L = case["u"].shape
    n = case["A"].shape[1]
    h0 = rng.standard_normal((b, d, n))
    dy = rng.standard_normal((b, d, L))
    dlast = rng.standard_normal((b, d, n))
    grads = oracle.selective_scan_bwd(**case, h0=h0, dy=dy, dlast=dlast, zoh=True)
    plain = oracle.selective_scan_bwd(**case, h0=h0, dy=dy, dlast=dlast)
    assert np.abs(grads["dA"] - plain["dA"]).max() > 1e-3   # the ZOH weight does depend on A

    def loss_of(name):
        def loss(value):
            c = dict(case, h0=h0)
            c[name] = value
            y, last = oracle.selective_scan(**c, zoh=True)
            return float((dy * y).sum() + (dlast * last).sum())
        return loss

    names = [("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("h0", "dh0")]
    names += [(k, "d" + k) for k in ("D", "z", "delta_bias") if case[k] is not None]
    for name, key in names:
        base = h0 if name == "h0" else case[name]
        _assert_fd(grads[key], _central_fd(loss_of(name), base), f"zoh {name}")


def test_backward_zoh_tends_to_simplified_for_small_steps():
    # For Delta A -> 0 the ZOH weight expm1(Delta A)/A B approaches Delta B, and so do the
    # gradients (to first order in Delta A).
    rng = _rng(82)
    case = _selective_case(rng, b=1, d=2, n=3, L=6, softplus=False)
    case["delta"] = np.full_like(case["delta"], 1e-7)
    case["delta_bias"] = np.zeros(2)
    dy = rng.standard_normal(case["u"].shape)
    gz = oracle.selective_scan_bwd(**case, dy=dy, zoh=True)
    gs = oracle.selective_scan_bwd(**case, dy=dy)
    for k in ("du", "ddelta", "dB", "dC", "dD", "dz"):
        np.testing.assert_allclose(gz[k], gs[k], rtol=1e-5, atol=1e-12, err_msg=k)


@pytest.mark.parametrize("K,L,with_prev,with_bias", [(1, 7, False, True), (2, 7, True, False), (4, 9, True, True),
                                                     (4, 2, True, True), (4, 9, False, False), (3, 1, True, True)],
                         ids=["K1", "K2_prev", "K4_prev", "K4_shortL", "K4_bare", "K3_L1"])
def test_conv_backward_matches_finite_differences(K, L, with_prev, with_bias):
    rng = _rng(90 + 7 * K + L)
    b, d = 2, 3
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, K))
    bias = rng.standard_normal(d) if with_bias else None
    prev = rng.standard_normal((b, d, K - 1)) if with_prev else None
    du = rng.standard_normal((b, d, L))
    dxn = rng.standard_normal((b, d, K - 1))
    g = oracle.causal_conv_silu_bwd(x, w, du, bias, prev, dx_next=dxn)

    def loss(xx=x, ww=w, bb=bias, pp=prev):
        u, x_next = oracle.causal_conv_silu(xx, ww, bb, pp)
        return float((du * u).sum() + (dxn * x_next).sum())

    _assert_fd(g["dx"], _central_fd(lambda v: loss(xx=v), x), "conv dx")
    _assert_fd(g["dw"], _central_fd(lambda v: loss(ww=v), w), "conv dw")
    _assert_fd(g["dbias"], _central_fd(lambda v: loss(bb=v), bias if with_bias else np.zeros(d)), "conv dbias")
    if K > 1:
        _assert_fd(g["dx_prev"], _central_fd(lambda v: loss(pp=v), prev if with_prev else np.zeros((b, d, K - 1))),
                   "conv dx_prev")
    # without dx_next the state output carries no gradient
    g0 = oracle.causal_conv_silu_bwd(x, w, du, bias, prev)
    _assert_fd(g0["dx"], _central_fd(lambda v: float((du * oracle.causal_conv_silu(v, w, bias, prev)[0]).sum()), x),
               "conv dx (no dx_next)")


@pytest.mark.parametrize("zoh", [False, True], ids=["simplified", "zoh"])
def test_conv_scan_chain_matches_finite_differences(zoh):
    # the whole Mamba x branch: u = silu(conv(x)), then the scan; gradients with respect to
    # x and the conv weight through both backward functions
    rng = _rng(95)
    b, d, n, L, K = 2, 3, 4, 8, 4
    case = _selective_case(rng, b=b, d=d, n=n, L=L)
    x = rng.standard_normal((b, d, L))
    w = 0.5 * rng.standard_normal((d, K))
    cb = rng.standard_normal(d)
    prev = rng.standard_normal((b, d, K - 1))
    dy = rng.standard_normal((b, d, L))
    u, _ = oracle.causal_conv_silu(x, w, cb, prev)
    gs = oracle.selective_scan_bwd(**dict(case, u=u), dy=dy, zoh=zoh)
    gc = oracle.causal_conv_silu_bwd(x, w, gs["du"], cb, prev)

    def loss(xx=x, ww=w):
        uu, _ = oracle.causal_conv_silu(xx, ww, cb, prev)
        y, _ = oracle.selective_scan(**dict(case, u=uu), zoh=zoh)
        return float((dy * y).sum())

    _assert_fd(gc["dx"], _central_fd(lambda v: loss(xx=v), x), "chain dx")
    _assert_fd(gc["dw"], _central_fd(lambda v: loss(ww=v), w), "chain dw")
