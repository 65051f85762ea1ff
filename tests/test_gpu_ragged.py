"""GPU parity of the ragged (variable-length) folded scan against the oracle's definition:
every packed sample computed on its own (oracle.mixer_layer_varlen), element by element,
with the metric and bounds of tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
from selective_scan_sfm_b200 import (SfmError, sfm_get_device_error, sfm_selective_scan_fold,
                                     sfm_selective_scan_fold_varlen, synth)

from parity import TOL, bf16_round, rel_err, to_cuda

pytestmark = pytest.mark.gpu


def run_gpu(dc, aux, swap, conv=True, gate=True, skip=True, bias=True, pad_left=None, y=None, final_state=None,
            out_dtype=None, **launch):
    return sfm_selective_scan_fold_varlen(
        dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dc["cu_seqlens"], z=dc["z"] if gate else None,
        Dskip=dc["Dskip"] if skip else None, dt_bias=dc["dt_bias"] if bias else None,
        conv_w=dc["conv_w"] if conv else None, conv_b=dc["conv_b"] if conv else None, pad_left=pad_left,
        aux_init=aux, swap_out=swap, y=y, final_state=final_state, out_dtype=out_dtype, **launch)


def run_oracle(d, aux, swap, conv=True, gate=True, skip=True, bias=True, pad_left=None, want_state=False):
    f = lambda t: None if t is None else t.double().numpy()
    return oracle.mixer_layer_varlen(
        f(d["x"]), f(d["dt"]), f(d["z"]) if gate else None, f(d["Bm"]), f(d["Cm"]), f(d["A"]),
        f(d["Dskip"]) if skip else None, f(d["dt_bias"]) if bias else None, f(d["conv_w"]) if conv else None,
        f(d["conv_b"]) if conv else None, d["cu_seqlens"].numpy(), aux_init_in=aux, swap_out=swap,
        pad_left=pad_left, want_state=want_state)


def covered(d):
    cu = d["cu_seqlens"].tolist()
    m = np.zeros(d["Ltot"], bool)
    for a, e in zip(cu[:-1], cu[1:]):
        m[a:e] = True
    return m


def check(y, ref, dtype, mask=None, label=""):
    g = y.double().cpu().numpy()
    if mask is not None:
        g, ref = g[:, mask], ref[:, mask]
    if y.dtype == torch.bfloat16:
        ref_cmp = bf16_round(ref)
    else:
        ref_cmp = ref
    e = rel_err(g, ref_cmp)
    assert e <= TOL[dtype], "%s: max rel err %.3g > %.3g" % (label, e, TOL[dtype])
    return e


CASES = [
    # lens (tokens per sample incl. aux), aux, swap, dtype, N, D, launch overrides
    ([51, 3, 200, 77, 130, 9], True, True, "f32", 8, 70, {}),
    ([1, 0, 64, 65, 0, 129, 2], False, True, "f32", 16, 70, dict(chunk=16, B1=1)),
    ([30, 31, 5, 90, 17, 48], True, False, "bf16", 16, 130, dict(B1=2)),
    ([300, 7, 45, 3], True, True, "bf16", 16, 64, dict(chunk=32, d_tile=32)),
    ([12, 0, 0, 33, 8], False, False, "bf16", 4, 96, {}),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_ragged_grid(case):
    lens, aux, swap, dtype, N, D, launch = CASES[case]
    d = synth.make_ragged_inputs(lens, D=D, N=N, dtype=dtype, seed=500 + case, aux=aux, random_A=True)
    dc = to_cuda(d)
    y = run_gpu(dc, aux, swap, **launch)
    torch.cuda.synchronize()
    assert sfm_get_device_error(clear=True) == 0
    check(y, run_oracle(d, aux, swap), dtype, covered(d), "case %d" % case)


@pytest.mark.parametrize("opts", [dict(pad_left=3), dict(pad_left=0), dict(conv=False), dict(gate=False),
                                  dict(skip=False, bias=False)])
def test_ragged_layer_options(opts):
    lens = [40, 9, 71, 26]
    aux = opts.get("conv", True)  # aux tokens belong to the conv input
    d = synth.make_ragged_inputs(lens, D=48, N=8, dtype="f32", seed=520, aux=aux)
    y = run_gpu(to_cuda(d), aux, aux, **opts)
    check(y, run_oracle(d, aux, aux, **opts), "f32", covered(d), str(opts))


def test_ragged_bf16_in_f32_out_and_final_states():
    lens = [60, 14, 101, 33, 5]
    d = synth.make_ragged_inputs(lens, D=80, N=16, dtype="bf16", seed=530, aux=True)
    dc = to_cuda(d)
    fs = torch.empty(len(lens), 80, 16, device="cuda")
    y = run_gpu(dc, True, True, final_state=fs, out_dtype=torch.float32, chunk=24)
    ref, ref_fs = run_oracle(d, True, True, want_state=True)
    assert y.dtype == torch.float32
    check(y, ref, "bf16", covered(d), "bf16 in, f32 out")
    e = rel_err(fs.double().cpu().numpy(), ref_fs)
    assert e <= TOL["bf16"], e


def test_ragged_gaps_are_not_written():
    """Positions that belong to no sample keep what y held."""
    D, N, Lt = 32, 8, 52
    g = torch.Generator().manual_seed(540)
    cu = torch.tensor([5, 20, 20, 47], dtype=torch.int32)
    d = dict(x=torch.randn(D, Lt, generator=g), dt=0.5 * torch.randn(D, Lt, generator=g),
             z=torch.randn(D, Lt, generator=g), Bm=torch.randn(N, Lt, generator=g), Cm=torch.randn(N, Lt, generator=g),
             A=-torch.exp(torch.randn(D, N, generator=g)), Dskip=torch.randn(D, generator=g),
             dt_bias=torch.full((D,), -3.0), conv_w=torch.rand(D, 4, generator=g) - 0.5,
             conv_b=torch.rand(D, generator=g) - 0.5, cu_seqlens=cu, Ltot=Lt)
    dc = to_cuda(d)
    y = torch.full((D, Lt), 7.0, device="cuda")
    run_gpu(dc, False, True, y=y)
    yc = y.cpu()
    assert torch.all(yc[:, :5] == 7.0) and torch.all(yc[:, 47:] == 7.0)
    check(y, run_oracle(d, False, True), "f32", covered(d), "gaps")


def test_ragged_sample_isolation():
    lens = [33, 20, 45, 12]
    d = synth.make_ragged_inputs(lens, D=64, N=16, dtype="bf16", seed=550, aux=True)
    dc = to_cuda(d)
    y0 = run_gpu(dc, True, True).clone()
    cu = d["cu_seqlens"].tolist()
    j = 2
    a, e = cu[j], cu[j + 1]
    for k in ("dt", "z"):
        dc[k][:, a:e] = float("nan")
    dc["Bm"][:, a:e] = float("inf")
    dc["x"][:, a - 2 * j:e - 2 * j - 2] = float("nan")
    y1 = run_gpu(dc, True, True)
    keep = torch.ones(d["Ltot"], dtype=torch.bool)
    keep[a:e] = False
    assert torch.equal(y1[:, keep.cuda()], y0[:, keep.cuda()])


def test_ragged_invalid_offsets_are_reported_and_skipped():
    """Offsets past the packed end, or an aux sample without a patch token: the sample is
    skipped (nothing of it read or written), the others are computed, and the device
    error word says SFM_ERR_INVALID_ARG."""
    sfm_get_device_error(clear=True)
    D, N = 32, 8
    # (a) no aux: sample 1 ends past the packed length 20
    d = synth.make_ragged_inputs([10, 10], D=D, N=N, dtype="f32", seed=560, aux=False)
    dc = to_cuda(d)
    good = d["cu_seqlens"].clone()
    dc["cu_seqlens"] = torch.tensor([0, 10, 40], dtype=torch.int32, device="cuda")
    y = torch.full((D, 20), 7.0, device="cuda")
    run_gpu(dc, False, False, y=y)
    assert sfm_get_device_error(clear=True) == 1  # SFM_ERR_INVALID_ARG
    d["cu_seqlens"] = good
    ref = run_oracle(d, False, False)
    check(y[:, :10], ref[:, :10], "f32", None, "valid sample next to an invalid one")
    assert torch.all(y[:, 10:].cpu() == 7.0)
    # (b) aux: sample 1 has 2 tokens (no patch token)
    lens = [12, 2, 16]
    d = synth.make_ragged_inputs(lens, D=D, N=N, dtype="f32", seed=561, aux=True)
    dc = to_cuda(d)
    y = torch.full((D, 30), 7.0, device="cuda")
    run_gpu(dc, True, True, y=y)
    assert sfm_get_device_error(clear=True) == 1
    assert torch.all(y[:, 12:14].cpu() == 7.0)
    f = lambda t: t.double().numpy()
    for s, (a, e) in ((0, (0, 12)), (2, (14, 30))):
        xs = d["x"][:, a - 2 * s:e - 2 * s - 2]
        r = oracle.mixer_layer(f(xs)[None], f(d["dt"][:, a:e])[None], f(d["z"][:, a:e])[None],
                               f(d["Bm"][:, a:e])[None], f(d["Cm"][:, a:e])[None], f(d["A"]), f(d["Dskip"]),
                               f(d["dt_bias"]), f(d["conv_w"]), f(d["conv_b"]), aux_init_in=True, swap_out=True)[0]
        check(y[:, a:e], r, "f32", None, "sample %d" % s)
    assert sfm_get_device_error(clear=True) == 0


def test_ragged_host_validation():
    d = to_cuda(synth.make_ragged_inputs([10, 12], D=16, N=4, dtype="f32", seed=570, aux=False))
    with pytest.raises(SfmError, match="UNSUPPORTED"):
        sfm_selective_scan_fold_varlen(d["x"], d["dt"], d["Bm"], d["Cm"], d["A"], d["cu_seqlens"], z=d["z"],
                                       chunk=12)  # not a multiple of 8
    with pytest.raises(ValueError):
        sfm_selective_scan_fold_varlen(d["x"], d["dt"], d["Bm"], d["Cm"], d["A"], d["cu_seqlens"].long())


def test_ragged_equal_lengths_match_the_fixed_layout():
    B, D, T, N = 8, 96, 49, 16
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype="bf16", seed=580)
    dc = to_cuda(d)
    L = T + 2
    yf = sfm_selective_scan_fold(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], z=dc["z"], Dskip=dc["Dskip"],
                                 dt_bias=dc["dt_bias"], conv_w=dc["conv_w"], conv_b=dc["conv_b"], aux_init=True,
                                 swap_out=True)
    pk = lambda t: t.permute(1, 0, 2).reshape(t.shape[1], -1).contiguous()
    cu = torch.arange(0, (B + 1) * L, L, dtype=torch.int32, device="cuda")
    yv = sfm_selective_scan_fold_varlen(pk(dc["x"]), pk(dc["dt"]), pk(dc["Bm"]), pk(dc["Cm"]), dc["A"], cu,
                                        z=pk(dc["z"]), Dskip=dc["Dskip"], dt_bias=dc["dt_bias"], conv_w=dc["conv_w"],
                                        conv_b=dc["conv_b"], aux_init=True, swap_out=True)
    e = rel_err(yv.double().cpu().numpy(), pk(yf).double().cpu().numpy())
    assert e <= 2e-2, e  # both within the bf16 bound of the same exact result; usually bitwise equal


def test_ragged_full_size_sampled():
    """The ragged workload at full size (128 samples of 49..196 patch tokens, D = 640,
    N = 16, bf16) in the benchmark's launch shape; six samples against the oracle."""
    w = synth.WORKLOADS["ragged_t49_196"]
    lens = synth.ragged_lengths(w["S"], w["T_lo"], w["T_hi"], seed=0)
    d = synth.make_ragged_inputs(lens, D=w["D"], N=w["N"], dtype=w["dtype"], seed=0)
    dc = to_cuda(d)
    y = run_gpu(dc, True, True)
    torch.cuda.synchronize()
    assert sfm_get_device_error(clear=True) == 0
    cu = d["cu_seqlens"].tolist()
    f = lambda t: t.double().numpy()
    for s in synth.sample_indices(w["S"], 6, seed=1):
        a, e = cu[s], cu[s + 1]
        xs = d["x"][:, a - 2 * s:e - 2 * s - 2]
        r = oracle.mixer_layer(f(xs)[None], f(d["dt"][:, a:e])[None], f(d["z"][:, a:e])[None],
                               f(d["Bm"][:, a:e])[None], f(d["Cm"][:, a:e])[None], f(d["A"]), f(d["Dskip"]),
                               f(d["dt_bias"]), f(d["conv_w"]), f(d["conv_b"]), aux_init_in=True, swap_out=True,
                               threads=4)[0]
        check(y[:, a:e], r, "bf16", None, "sample %d" % s)
