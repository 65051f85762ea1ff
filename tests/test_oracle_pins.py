"""Pins for the CPU oracle, checked against things other than itself.

Each test ties one oracle routine to a fact fixed by the pages or by mathematics:
hand-worked examples (tests/golden/hand_examples.json), closed forms, geometric
sums, brute-force unrolled recurrences, a library conv, finite differences and
autograd of an independent formulation, and the structural claims of the pages
(folding with reset equals the per-sample run; samples never leak into each other).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from selective_scan_sfm_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def small_case(B=3, D=4, L=7, N=3, seed=0, softplus=True):
    r = np.random.default_rng(seed)
    d = dict(u=r.standard_normal((B, D, L)), dt=0.5 * r.standard_normal((B, D, L)) - 2.0,
             z=r.standard_normal((B, D, L)), Bm=r.standard_normal((B, N, L)),
             Cm=r.standard_normal((B, N, L)), A=-np.exp(r.standard_normal((D, N))),
             Dskip=r.standard_normal(D), dt_bias=0.3 * r.standard_normal(D))
    if not softplus:
        d["dt"] = np.abs(d["dt"]) * 0.3
    return d


# ---------------------------------------------------------------- scalar functions

def test_softplus_silu_special_values(ora):
    assert ora.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert ora.softplus(30.0) == 30.0
    assert ora.softplus(-30.0) == pytest.approx(math.exp(-30.0), rel=1e-12)
    assert ora.silu(0.0) == 0.0
    assert ora.silu(50.0) == pytest.approx(50.0, rel=1e-15)
    assert abs(ora.silu(-50.0)) < 1e-19
    v = torch.linspace(-15, 25, 81, dtype=torch.float64)
    sp = torch.nn.functional.softplus(v)  # library routine, threshold 20 like the oracle
    si = torch.nn.functional.silu(v)
    for a, b, c in zip(v.tolist(), sp.tolist(), si.tolist()):
        assert ora.softplus(a) == pytest.approx(b, rel=1e-14, abs=1e-300)
        assert ora.silu(a) == pytest.approx(c, rel=1e-14, abs=1e-300)


# ---------------------------------------------------------------- aux tokens

def test_aux_hand_examples(ora):
    g = json.load(open(GOLD))
    x = np.array(g["aux_init"]["x"]).reshape(1, 1, -1)
    np.testing.assert_array_equal(ora.aux_init(x).ravel(), g["aux_init"]["xa"])
    y = np.array(g["aux_swap"]["y"]).reshape(1, 1, -1)
    np.testing.assert_array_equal(ora.aux_swap(y).ravel(), g["aux_swap"]["swapped"])


def test_aux_init_invariants(ora):
    x = rnd((3, 5, 11), 1)
    xa = ora.aux_init(x)
    assert xa.shape == (3, 5, 13)
    np.testing.assert_array_equal(xa[..., 1:-1], x)                      # middle tokens untouched
    np.testing.assert_allclose(xa[..., 0], x.mean(-1), rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(xa[..., 0], xa[..., -1])
    c = np.full((2, 3, 9), 0.37)
    np.testing.assert_allclose(ora.aux_init(c)[..., [0, -1]], 0.37, rtol=1e-15)  # constant sample


def test_aux_swap_invariants(ora):
    y = rnd((2, 3, 6), 2)
    s = ora.aux_swap(y)
    np.testing.assert_array_equal(s[..., 1:-1], y[..., 1:-1])
    np.testing.assert_array_equal(s[..., 0], y[..., -1])
    np.testing.assert_array_equal(s[..., -1], y[..., 0])
    np.testing.assert_array_equal(ora.aux_swap(s), y)                      # swap o swap = id


# ---------------------------------------------------------------- boundary-safe conv

@pytest.mark.parametrize("name", ["conv_same", "conv_causal"])
def test_conv_hand_examples(ora, name):
    g = json.load(open(GOLD))[name]
    xa = np.array(g["xa"]).reshape(1, 1, -1)
    w = np.array(g["w"]).reshape(1, -1)
    u = ora.conv1d(xa, w, None, K=4, pad_left=g["pad_left"], silu=False)
    np.testing.assert_array_equal(u.ravel(), g["u"])


@pytest.mark.parametrize("K,pad_left", [(4, 1), (4, 3), (4, 0), (3, 1), (2, 0), (1, 0)])
def test_conv_matches_library_conv_per_sample(ora, K, pad_left):
    B, D, L = 3, 5, 9
    xa, w, b = rnd((B, D, L), 3), rnd((D, K), 4), rnd(D, 5)
    u = ora.conv1d(xa, w, b, K=K, pad_left=pad_left, silu=False)
    t = torch.from_numpy(xa)
    t = torch.nn.functional.pad(t, (pad_left, K - 1 - pad_left))        # zeros per sample
    ref = torch.nn.functional.conv1d(t, torch.from_numpy(w).unsqueeze(1), torch.from_numpy(b), groups=D)
    np.testing.assert_allclose(u, ref.numpy(), rtol=1e-13, atol=1e-13)
    us = ora.conv1d(xa, w, b, K=K, pad_left=pad_left, silu=True)
    np.testing.assert_allclose(us, torch.nn.functional.silu(ref).numpy(), rtol=1e-13, atol=1e-13)


def test_conv_delta_kernel_is_shift_and_edges_are_partial_sums(ora):
    B, D, L, K = 2, 3, 8, 4
    xa = rnd((B, D, L), 6)
    for k in range(K):
        w = np.zeros((D, K)); w[:, k] = 1.0
        u = ora.conv1d(xa, w, None, K=K, pad_left=1)
        shift = k - 1
        for t in range(L):
            s = t + shift
            exp = xa[..., s] if 0 <= s < L else np.zeros((B, D))
            np.testing.assert_array_equal(u[..., t], exp)
    w = rnd((D, K), 7)
    u = ora.conv1d(np.ones((B, D, L)), w, None, K=K, pad_left=1)
    np.testing.assert_allclose(u[..., 0], np.broadcast_to(w[:, 1:].sum(1), (B, D)), rtol=1e-14)
    np.testing.assert_allclose(u[..., 3], np.broadcast_to(w.sum(1), (B, D)), rtol=1e-14)
    np.testing.assert_allclose(u[..., L - 2], np.broadcast_to(w[:, :3].sum(1), (B, D)), rtol=1e-14)
    np.testing.assert_allclose(u[..., L - 1], np.broadcast_to(w[:, :2].sum(1), (B, D)), rtol=1e-14)


def test_conv_sample_isolation(ora):
    B, D, L, K = 4, 3, 6, 4
    xa, w, b = rnd((B, D, L), 8), rnd((D, K), 9), rnd(D, 10)
    u0 = ora.conv1d(xa, w, b, K=K, pad_left=1, silu=True)
    xb = xa.copy(); xb[2] = np.inf
    u1 = ora.conv1d(xb, w, b, K=K, pad_left=1, silu=True)
    for s in (0, 1, 3):
        np.testing.assert_array_equal(u1[s], u0[s])


# ---------------------------------------------------------------- the scan

def test_scan_hand_example_two_folded_samples(ora):
    g = json.load(open(GOLD))["scan_folded_two_samples"]
    u = np.array(g["u"]).reshape(2, 1, 4)
    dt = np.ones((2, 1, 4))
    Bm = np.ones((2, 1, 4)); Cm = np.ones((2, 1, 4))
    A = np.array([[-math.log(2.0)]])
    Dskip = np.array([0.5])
    want = np.array(g["y"]).reshape(2, 1, 4)
    y = ora.scan(u, dt, Bm, Cm, A, Dskip, None, None, dt_softplus=False)
    np.testing.assert_allclose(y, want, rtol=1e-15)
    yf = ora.scan_folded(u, dt, Bm, Cm, A, 2, Dskip, None, None, dt_softplus=False)
    np.testing.assert_allclose(yf, want, rtol=1e-15)


def test_scan_closed_form_constant_inputs(ora):
    """h_t = Delta*B*u0*(1 - a^(t+1))/(1 - a), a = exp(Delta*A); t restarts in every sample."""
    B, D, L, N = 3, 2, 11, 4
    delta = np.array([0.05, 0.3])                       # per channel, no softplus
    A = -np.array([[0.5, 1.0, 2.0, 7.0], [0.1, 0.2, 3.0, 0.01]])
    Bc = np.array([[1.0, -0.5, 2.0, 0.3], [0.7, 0.1, -1.0, 2.0], [1.5, 1.5, 0.2, -0.2]])  # per sample
    Cc = np.array([[0.2, 1.0, -1.0, 0.5], [1.0, 1.0, 1.0, 1.0], [-0.3, 0.4, 0.9, 2.0]])
    u0 = np.array([[1.0, -2.0], [0.5, 3.0], [2.0, 0.1]])
    Dskip = np.array([0.25, -1.5])
    u = np.broadcast_to(u0[:, :, None], (B, D, L)).copy()
    dt = np.broadcast_to(delta[None, :, None], (B, D, L)).copy()
    Bm = np.broadcast_to(Bc[:, :, None], (B, N, L)).copy()
    Cm = np.broadcast_to(Cc[:, :, None], (B, N, L)).copy()
    want = np.zeros((B, D, L))
    for b in range(B):
        for d in range(D):
            a = np.exp(delta[d] * A[d])
            for t in range(L):
                h = delta[d] * Bc[b] * u0[b, d] * (1 - a ** (t + 1)) / (1 - a)
                want[b, d, t] = (Cc[b] * h).sum() + Dskip[d] * u0[b, d]
    y = ora.scan(u, dt, Bm, Cm, A, Dskip, None, None, dt_softplus=False)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-13)
    yf = ora.scan_folded(u, dt, Bm, Cm, A, 3, Dskip, None, None, dt_softplus=False)
    np.testing.assert_allclose(yf, want, rtol=1e-12, atol=1e-13)


def test_scan_n1_geometric_limits(ora):
    B, D, L = 2, 3, 9
    r = np.random.default_rng(11)
    u, dt = r.standard_normal((B, D, L)), np.abs(r.standard_normal((B, D, L))) + 0.1
    Bm, Cm = r.standard_normal((B, 1, L)), r.standard_normal((B, 1, L))
    # A = 0: Abar = 1, the state is a prefix sum of Delta*B*u within each sample
    y = ora.scan(u, dt, Bm, np.ones_like(Cm), np.zeros((D, 1)), dt_softplus=False)
    np.testing.assert_allclose(y, np.cumsum(dt * Bm * u, axis=-1), rtol=1e-13, atol=1e-13)
    # A << 0: Abar underflows to 0, the scan is memoryless
    y = ora.scan(u, dt, Bm, Cm, np.full((D, 1), -1e6), dt_softplus=False)
    np.testing.assert_allclose(y, Cm * dt * Bm * u, rtol=1e-14, atol=1e-300)


def brute_force(u, dt, z, Bm, Cm, A, Dskip, dt_bias, softplus=True):
    """y_t = sum_{s<=t} C_t (prod_{r=s+1..t} Abar_r) Delta_s B_s u_s + D u_t, then the gate."""
    B, D, L = u.shape
    N = A.shape[1]
    delta = dt + dt_bias[None, :, None]
    if softplus:
        delta = np.where(delta > 20, delta, np.log1p(np.exp(delta)))
    y = np.zeros((B, D, L))
    for b in range(B):
        for d in range(D):
            for t in range(L):
                acc = 0.0
                for n in range(N):
                    for s in range(t + 1):
                        prod = 1.0
                        for r in range(s + 1, t + 1):
                            prod *= math.exp(delta[b, d, r] * A[d, n])
                        acc += Cm[b, n, t] * prod * delta[b, d, s] * Bm[b, n, s] * u[b, d, s]
                acc += Dskip[d] * u[b, d, t]
                y[b, d, t] = acc * (z[b, d, t] / (1 + math.exp(-z[b, d, t])))
    return y


@pytest.mark.parametrize("L", [1, 2, 3, 6])
def test_scan_brute_force_tiny(ora, L):
    c = small_case(B=2, D=3, L=L, N=3, seed=12 + L)
    y = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"])
    want = brute_force(c["u"], c["dt"], c["z"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"])
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-14)


def materialised(u, dt, z, Bm, Cm, A, Dskip, dt_bias, softplus=True, lib=np):
    """O(L^2) kernel form with cumulative log-decays S_t = sum_{r<=t} Delta_r A:
    prod_{r=s+1..t} Abar_r = exp(S_t - S_s); works on numpy or torch arrays."""
    if lib is np:
        delta = dt + dt_bias[None, :, None]
        if softplus:
            delta = np.where(delta > 20, delta, np.log1p(np.exp(np.minimum(delta, 20))))
        S = np.cumsum(delta[..., None] * A[None, :, None, :], axis=2)            # [B,D,L,N]
        diff = S[:, :, :, None, :] - S[:, :, None, :, :]                           # [B,D,t,s,N]
        L = u.shape[-1]
        mask = np.tril(np.ones((L, L), bool))[None, None, :, :, None]
        Kts = np.where(mask, np.exp(np.where(mask, diff, 0.0)), 0.0)
        w = delta * u                                                              # [B,D,L]
        inner = np.einsum("bdtsn,bds,bns->bdtn", Kts, w, Bm)
        y = np.einsum("bdtn,bnt->bdt", inner, Cm) + Dskip[None, :, None] * u
        return y * (z / (1 + np.exp(-z)))
    delta = dt + dt_bias[None, :, None]
    if softplus:
        delta = torch.nn.functional.softplus(delta)
    S = torch.cumsum(delta[..., None] * A[None, :, None, :], dim=2)
    diff = S[:, :, :, None, :] - S[:, :, None, :, :]
    L = u.shape[-1]
    mask = torch.tril(torch.ones(L, L, dtype=torch.bool))[None, None, :, :, None]
    Kts = torch.where(mask, torch.exp(torch.where(mask, diff, torch.zeros_like(diff))), torch.zeros_like(diff))
    inner = torch.einsum("bdtsn,bds,bns->bdtn", Kts, delta * u, Bm)
    y = torch.einsum("bdtn,bnt->bdt", inner, Cm) + Dskip[None, :, None] * u
    return y * torch.nn.functional.silu(z)


def test_scan_materialised_form_moderate(ora):
    c = small_case(B=2, D=5, L=51, N=8, seed=21)
    y = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"])
    want = materialised(c["u"], c["dt"], c["z"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"])
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("B", [4, 6, 12])
def test_fold_equals_unfolded_bitwise(ora, B):
    """Folding [B,D,L] -> [B1,D,B2*L] with the reset equals the per-sample runs exactly."""
    c = small_case(B=B, D=3, L=8, N=4, seed=30 + B)
    y0, s0 = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"],
                      want_state=True)
    for B2 in [b2 for b2 in range(1, B + 1) if B % b2 == 0]:
        y1, s1 = ora.scan_folded(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], B2, c["Dskip"],
                                 c["dt_bias"], c["z"], want_state=True)
        np.testing.assert_array_equal(y1, y0)
        np.testing.assert_array_equal(s1, s0)


def test_folding_without_reset_would_leak(ora):
    """Guard against a reset that does nothing: one long recurrence WITHOUT the reset
    differs from the per-sample result in every sample after the first."""
    c = small_case(B=2, D=2, L=6, N=2, seed=40)
    y0 = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"])
    cat = lambda a: np.concatenate([a[0], a[1]], axis=-1)[None]
    yl = ora.scan(cat(c["u"]), cat(c["dt"]), cat(c["Bm"]), cat(c["Cm"]), c["A"], c["Dskip"],
                  c["dt_bias"], cat(c["z"]))
    np.testing.assert_array_equal(yl[0, :, :6], y0[0])
    assert np.abs(yl[0, :, 6:] - y0[1]).max() > 1e-6


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
@pytest.mark.parametrize("field", ["u", "dt", "z", "Bm", "Cm"])
def test_sample_isolation_with_nonfinite(ora, bad, field):
    c = small_case(B=4, D=3, L=6, N=3, seed=50)
    y0 = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"])
    p = {k: v.copy() for k, v in c.items()}
    p[field][1] = bad
    y1 = ora.scan(p["u"], p["dt"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"], p["z"])
    y2 = ora.scan_folded(p["u"], p["dt"], p["Bm"], p["Cm"], p["A"], 4, p["Dskip"], p["dt_bias"], p["z"])
    for s in (0, 2, 3):
        np.testing.assert_array_equal(y1[s], y0[s])
        np.testing.assert_array_equal(y2[s], y0[s])


def test_final_state_is_last_state(ora):
    c = small_case(B=2, D=3, L=5, N=2, seed=60, softplus=False)
    _, fs = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], want_state=True, dt_softplus=False)
    # with C = e_n and no skip/gate, y_{L-1} reads state n directly
    for n in range(2):
        Cm = np.zeros_like(c["Cm"]); Cm[:, n, :] = 1.0
        y = ora.scan(c["u"], c["dt"], c["Bm"], Cm, c["A"], dt_softplus=False)
        np.testing.assert_allclose(fs[..., n], y[..., -1], rtol=1e-15)


# ---------------------------------------------------------------- backward

def _loss(ora, c, dout):
    y = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"])
    return float((y * dout).sum())


def test_backward_finite_differences(ora):
    c = small_case(B=2, D=2, L=5, N=2, seed=70)
    dout = rnd(c["u"].shape, 71)
    g = ora.scan_bwd(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], dout, c["Dskip"], c["dt_bias"], c["z"])
    names = {"u": "du", "dt": "ddt", "z": "dz", "Bm": "dB", "Cm": "dC", "A": "dA",
             "Dskip": "dDskip", "dt_bias": "ddt_bias"}
    h = 1e-6
    for f, gname in names.items():
        arr = c[f]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            keep = arr[idx]
            arr[idx] = keep + h; lp = _loss(ora, c, dout)
            arr[idx] = keep - h; lm = _loss(ora, c, dout)
            arr[idx] = keep
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-8, err_msg=gname)


def test_backward_matches_autograd_of_materialised_form(ora):
    c = small_case(B=3, D=4, L=13, N=4, seed=80)
    dout = rnd(c["u"].shape, 81)
    g = ora.scan_bwd(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], dout, c["Dskip"], c["dt_bias"], c["z"])
    T = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in c.items()}
    y = materialised(T["u"], T["dt"], T["z"], T["Bm"], T["Cm"], T["A"], T["Dskip"], T["dt_bias"], lib=torch)
    (y * torch.from_numpy(dout)).sum().backward()
    pairs = {"u": "du", "dt": "ddt", "z": "dz", "Bm": "dB", "Cm": "dC", "A": "dA",
             "Dskip": "dDskip", "dt_bias": "ddt_bias"}
    for f, gname in pairs.items():
        np.testing.assert_allclose(g[gname], T[f].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=gname)


# ---------------------------------------------------------------- the mixer layer and chain

def torch_mixer(x, p, aux_init, swap_out, pad_left=1):
    """Independent fp64 composition with library ops: pad+conv1d, silu, materialised scan."""
    xt = torch.from_numpy(x)
    if aux_init:
        m = xt.mean(-1, keepdim=True)
        xt = torch.cat([m, xt, m], -1)
    K = p["conv_w"].shape[1]
    xp = torch.nn.functional.pad(xt, (pad_left, K - 1 - pad_left))
    u = torch.nn.functional.silu(torch.nn.functional.conv1d(
        xp, torch.from_numpy(p["conv_w"]).unsqueeze(1), torch.from_numpy(p["conv_b"]), groups=xt.shape[1]))
    y = materialised(u.numpy(), p["dt"], p["z"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"])
    if swap_out:
        y = y.copy(); y[..., [0, -1]] = y[..., [-1, 0]]
    return y


def test_mixer_layer_matches_library_composition(ora):
    B, D, T, N, K = 3, 4, 9, 4, 4
    d = synth.make_inputs(B, D, T, N, K=K, dtype="f32", seed=3, random_A=True)
    p = {k: d[k].double().numpy() for k in ("z", "dt", "Bm", "Cm", "A", "Dskip", "dt_bias", "conv_w", "conv_b")}
    x = d["x"].double().numpy()
    for aux, swap in [(True, False), (True, True)]:
        y = ora.mixer_layer(x, p["dt"], p["z"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"],
                            p["conv_w"], p["conv_b"], aux_init_in=aux, swap_out=swap)
        np.testing.assert_allclose(y, torch_mixer(x, p, aux, swap), rtol=1e-10, atol=1e-12)


def test_threads_do_not_change_results(ora):
    c = small_case(B=7, D=3, L=9, N=3, seed=90)
    y1 = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"], threads=1)
    y4 = ora.scan(c["u"], c["dt"], c["Bm"], c["Cm"], c["A"], c["Dskip"], c["dt_bias"], c["z"], threads=4)
    np.testing.assert_array_equal(y1, y4)


# ---------------------------------------------------------------- the mixer layer backward

def test_conv_and_aux_backward_are_adjoints(ora):
    """For the linear parts, <f(a), v> = <a, f^T(v)>: conv without bias/SiLU and aux init."""
    B, D, L, K = 2, 3, 9, 4
    xa, w, v = rnd((B, D, L), 100), rnd((D, K), 101), rnd((B, D, L), 102)
    for pl in (0, 1, 3):
        u = ora.conv1d(xa, w, None, K=K, pad_left=pl, silu=False)
        dxa, dw, _ = ora.conv1d_bwd(xa, w, None, v, pad_left=pl, silu=False)
        assert float((u * v).sum()) == pytest.approx(float((xa * dxa).sum()), rel=1e-12)
        # dw from the library conv's autograd
        t = torch.tensor(xa, requires_grad=False)
        wt = torch.tensor(w, requires_grad=True)
        out = torch.nn.functional.conv1d(torch.nn.functional.pad(t, (pl, K - 1 - pl)), wt.unsqueeze(1), groups=D)
        (out * torch.from_numpy(v)).sum().backward()
        np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-12, atol=1e-13)
    x, g = rnd((B, D, 7), 103), rnd((B, D, 9), 104)
    assert float((ora.aux_init(x) * g).sum()) == pytest.approx(float((x * ora.aux_init_bwd(g)).sum()), rel=1e-12)


def _mixer_loss(ora, p, dout, aux, swap):
    y = ora.mixer_layer(p["x"], p["dt"], p["z"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"], p["conv_w"],
                        p["conv_b"], aux_init_in=aux, swap_out=swap)
    return float((y * dout).sum())


@pytest.mark.parametrize("aux,swap", [(True, True), (False, False)])
def test_mixer_backward_finite_differences(ora, aux, swap):
    d = synth.make_inputs(B=2, D=2, T=5, N=2, dtype="f32", seed=110, aux=aux, random_A=True)
    p = {k: d[k].double().numpy().copy() for k in ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias",
                                                   "conv_w", "conv_b")}
    L = p["dt"].shape[-1]
    dout = rnd((2, 2, L), 111)
    g = ora.mixer_layer_bwd(p["x"], p["dt"], p["z"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"],
                            p["conv_w"], p["conv_b"], dout, aux_init_in=aux, swap_out=swap)
    names = {"x": "dx", "conv_w": "dconv_w", "conv_b": "dconv_b", "dt": "ddt", "z": "dz", "Bm": "dB",
             "A": "dA", "dt_bias": "ddt_bias"}
    h = 1e-6
    for f, gname in names.items():
        arr = p[f]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            keep = arr[idx]
            arr[idx] = keep + h; lp = _mixer_loss(ora, p, dout, aux, swap)
            arr[idx] = keep - h; lm = _mixer_loss(ora, p, dout, aux, swap)
            arr[idx] = keep
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-8, err_msg=gname)


def test_mixer_backward_matches_autograd_of_library_composition(ora):
    d = synth.make_inputs(B=3, D=4, T=11, N=4, dtype="f32", seed=120, random_A=True)
    names = ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "conv_w", "conv_b")
    p = {k: d[k].double().numpy() for k in names}
    dout = rnd((3, 4, 13), 121)
    g = ora.mixer_layer_bwd(p["x"], p["dt"], p["z"], p["Bm"], p["Cm"], p["A"], p["Dskip"], p["dt_bias"],
                            p["conv_w"], p["conv_b"], dout, aux_init_in=True, swap_out=True)
    T = {k: torch.tensor(v, requires_grad=True) for k, v in p.items()}
    xt = T["x"]
    m = xt.mean(-1, keepdim=True)
    xa = torch.cat([m, xt, m], -1)
    u = torch.nn.functional.silu(torch.nn.functional.conv1d(
        torch.nn.functional.pad(xa, (1, 2)), T["conv_w"].unsqueeze(1), T["conv_b"], groups=4))
    y = materialised(u, T["dt"], T["z"], T["Bm"], T["Cm"], T["A"], T["Dskip"], T["dt_bias"], lib=torch)
    y = torch.cat([y[..., -1:], y[..., 1:-1], y[..., :1]], -1)  # swap
    (y * torch.from_numpy(dout)).sum().backward()
    pairs = {"x": "dx", "conv_w": "dconv_w", "conv_b": "dconv_b", "dt": "ddt", "z": "dz", "Bm": "dB", "Cm": "dC",
             "A": "dA", "Dskip": "dDskip", "dt_bias": "ddt_bias"}
    for f, gname in pairs.items():
        np.testing.assert_allclose(g[gname], T[f].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=gname)
