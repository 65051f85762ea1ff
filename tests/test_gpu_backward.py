"""GPU parity of the scan backward against the fp64 oracle's reverse sweep.

Per-element gradients (du, ddt, dz, dB, dC) use the metric of tests/parity.py; the
reduced parameter gradients (dA, dDskip, ddt_bias) use the norm-wise ||g-r||_inf/||r||_inf."""
import numpy as np
import pytest
import torch

import oracle
from selective_scan_sfm_b200 import SfmError, sfm_selective_scan_fold_bwd, synth

from parity import TOL, rel_err, to_cuda

pytestmark = pytest.mark.gpu

PER_ELEMENT = ("du", "ddt", "dz", "dB", "dC")
REDUCED = ("dA", "dDskip", "ddt_bias")


def normwise(g, r):
    g, r = np.asarray(g, np.float64), np.asarray(r, np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


def run_both(d, dout, samples=None):
    dc = to_cuda(d)
    g = sfm_selective_scan_fold_bwd(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dout.cuda(), z=dc["z"],
                                    Dskip=dc["Dskip"], dt_bias=dc["dt_bias"])
    torch.cuda.synchronize()
    f = lambda t: t.double().numpy()
    ref = oracle.scan_bwd(f(d["x"]), f(d["dt"]), f(d["Bm"]), f(d["Cm"]), f(d["A"]), f(dout), f(d["Dskip"]),
                          f(d["dt_bias"]), f(d["z"]))
    return {k: v.double().cpu().numpy() for k, v in g.items()}, ref


def check_grads(g, ref, tol_elem, tol_red):
    errs = {}
    for k in PER_ELEMENT:
        errs[k] = rel_err(g[k], ref[k])
    for k in REDUCED:
        errs[k] = normwise(g[k], ref[k])
    bad = {k: e for k, e in errs.items() if e > (tol_elem if k in PER_ELEMENT else tol_red)}
    assert not bad, "gradient errors above bound: %s (all: %s)" % (bad, errs)
    return errs


def test_backward_small_fp32():
    d = synth.make_inputs(B=3, D=70, T=40, N=8, dtype="f32", seed=31, aux=False, random_A=True)
    dout = synth.make_dout(3, 70, 40, seed=31, dtype="f32")
    g, ref = run_both(d, dout)
    check_grads(g, ref, TOL["f32"], TOL["f32"])


def test_backward_is_bitwise_reproducible():
    d = synth.make_inputs(B=4, D=130, T=51, N=16, dtype="bf16", seed=32, aux=False)
    dc = to_cuda(d)
    dout = synth.make_dout(4, 130, 51, seed=32).cuda()
    run = lambda: sfm_selective_scan_fold_bwd(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dout, z=dc["z"],
                                              Dskip=dc["Dskip"], dt_bias=dc["dt_bias"])
    a, b = run(), run()
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_sample_isolation():
    d = synth.make_inputs(B=4, D=64, T=30, N=8, dtype="f32", seed=33, aux=False)
    dc = to_cuda(d)
    dout = synth.make_dout(4, 64, 30, seed=33, dtype="f32").cuda()
    run = lambda o: sfm_selective_scan_fold_bwd(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], o, z=dc["z"],
                                                Dskip=dc["Dskip"], dt_bias=dc["dt_bias"])
    g0 = run(dout)
    o2 = dout.clone()
    o2[1] = float("nan")
    g1 = run(o2)
    keep = [0, 2, 3]
    for k in PER_ELEMENT:
        assert torch.equal(g1[k][keep], g0[k][keep]), k


def test_backward_workspace_errors():
    d = to_cuda(synth.make_inputs(B=2, D=32, T=20, N=4, dtype="f32", seed=34, aux=False))
    dout = torch.randn(2, 32, 20, device="cuda")
    args = (d["x"], d["dt"], d["Bm"], d["Cm"], d["A"], dout)
    with pytest.raises(SfmError, match="INVALID"):
        sfm_selective_scan_fold_bwd(*args, workspace=torch.empty(64, dtype=torch.uint8, device="cuda"))
    big = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    with pytest.raises(SfmError, match="MISALIGNED"):
        sfm_selective_scan_fold_bwd(*args, workspace=big[16:])


def test_backward_chain_stage3_shape_bf16():
    """The backward at the four-layer chain's shape (B=64, D=640, L=198, N=16, bf16 inputs),
    every gradient against the fp64 oracle on the full tensors."""
    w = synth.WORKLOADS["chain4_stage3"]
    d = synth.make_inputs(B=w["B"], D=w["D"], T=w["T"] + 2, N=w["N"], dtype="bf16", seed=4000, aux=False)
    dout = synth.make_dout(w["B"], w["D"], w["T"] + 2, seed=4000)
    g, ref = run_both(d, dout)
    errs = check_grads(g, ref, TOL["bf16"], TOL["bf16"])
    # fp32 arithmetic on exact bf16 inputs: far inside the bf16 bound
    assert max(errs.values()) < 1e-3, errs


# ------------------------------------------------------------------ the whole mixer layer

from selective_scan_sfm_b200 import sfm_mixer_bwd  # noqa: E402

MIXER_ELEM = ("dx", "ddt", "dz", "dB", "dC")
MIXER_RED = ("dconv_w", "dconv_b", "dA", "dDskip", "ddt_bias")


def run_mixer_both(d, dout, aux, swap, pad_left=1, bias=True):
    dc = to_cuda(d)
    kw = dict(z=dc["z"], Dskip=dc["Dskip"], dt_bias=dc["dt_bias"], conv_w=dc["conv_w"],
              conv_b=dc["conv_b"] if bias else None, pad_left=pad_left, aux_init=aux, swap_out=swap)
    g = sfm_mixer_bwd(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dout.cuda(), **kw)
    torch.cuda.synchronize()
    f = lambda t: t.double().numpy()
    ref = oracle.mixer_layer_bwd(f(d["x"]), f(d["dt"]), f(d["z"]), f(d["Bm"]), f(d["Cm"]), f(d["A"]),
                                 f(d["Dskip"]), f(d["dt_bias"]), f(d["conv_w"]),
                                 f(d["conv_b"]) if bias else None, f(dout), aux_init_in=aux, swap_out=swap,
                                 pad_left=pad_left)
    return {k: v.double().cpu().numpy() for k, v in g.items()}, ref


def check_mixer(g, ref, tol):
    errs = {}
    for k in ref:
        errs[k] = rel_err(g[k], ref[k]) if k in MIXER_ELEM else normwise(g[k], ref[k])
    assert set(g) == set(ref), (sorted(g), sorted(ref))
    bad = {k: e for k, e in errs.items() if e > tol}
    assert not bad, "mixer gradient errors above bound: %s (all: %s)" % (bad, errs)
    return errs


@pytest.mark.parametrize("aux,swap,pad_left,bias", [(True, True, 1, True), (False, False, 3, True),
                                                    (True, False, 0, False), (False, True, 2, True)])
def test_mixer_backward_small_fp32(aux, swap, pad_left, bias):
    B, D, T, N = 3, 70, 33, 8
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype="f32", seed=4100 + pad_left, aux=aux, random_A=True)
    L = T + 2 if aux else T
    dout = synth.make_dout(B, D, L, seed=4100, dtype="f32")
    g, ref = run_mixer_both(d, dout, aux, swap, pad_left, bias)
    check_mixer(g, ref, TOL["f32"])


def test_mixer_backward_chain_stage3_bf16():
    """The stage-entry layer of the four-layer chain (aux init, swapped output) at full size."""
    w = synth.WORKLOADS["chain4_stage3"]
    d = synth.make_inputs(**w, seed=0)
    dout = synth.make_dout(w["B"], w["D"], w["T"] + 2, seed=9)
    g, ref = run_mixer_both(d, dout, True, True)
    errs = check_mixer(g, ref, TOL["bf16"])
    assert max(errs.values()) < 1e-3, errs


def test_mixer_backward_is_bitwise_reproducible():
    d = to_cuda(synth.make_inputs(B=4, D=96, T=49, N=16, dtype="bf16", seed=4200))
    dout = synth.make_dout(4, 96, 51, seed=4200).cuda()
    run = lambda: sfm_mixer_bwd(d["x"], d["dt"], d["Bm"], d["Cm"], d["A"], dout, z=d["z"], Dskip=d["Dskip"],
                                dt_bias=d["dt_bias"], conv_w=d["conv_w"], conv_b=d["conv_b"], aux_init=True,
                                swap_out=True)
    a, b = run(), run()
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_large_state_size():
    d = synth.make_inputs(B=2, D=40, T=30, N=32, dtype="f32", seed=4300, aux=False, random_A=True)
    dout = synth.make_dout(2, 40, 30, seed=4300, dtype="f32")
    g, ref = run_both(d, dout)
    check_grads(g, ref, TOL["f32"], TOL["f32"])
    d2 = synth.make_inputs(B=2, D=40, T=30, N=32, dtype="f32", seed=4301, random_A=True)
    g2, ref2 = run_mixer_both(d2, synth.make_dout(2, 40, 32, seed=4301, dtype="f32"), True, True)
    check_mixer(g2, ref2, TOL["f32"])


@pytest.mark.parametrize("N", [1, 3, 5, 15])
def test_backward_odd_state_sizes(N):
    """Odd N splits the states unequally between a channel's two threads (the second half
    one state short, empty at N = 1); D = 70 leaves a partial last channel tile."""
    d = synth.make_inputs(B=3, D=70, T=37, N=N, dtype="f32", seed=4400 + N, aux=False, random_A=True)
    dout = synth.make_dout(3, 70, 37, seed=4400 + N, dtype="f32")
    g, ref = run_both(d, dout)
    check_grads(g, ref, TOL["f32"], TOL["f32"])


@pytest.mark.parametrize("N", [1, 7])
def test_mixer_backward_odd_state_sizes(N):
    B, D, T = 2, 70, 33
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype="f32", seed=4500 + N, random_A=True)
    dout = synth.make_dout(B, D, T + 2, seed=4500 + N, dtype="f32")
    g, ref = run_mixer_both(d, dout, True, True, 1, True)
    check_mixer(g, ref, TOL["f32"])
