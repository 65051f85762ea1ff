"""The allocation-free scan backward (sfm_selective_scan_fold_bwd_noalloc).

Some callers cannot call cudaMalloc: a plug-in whose host application owns every byte of
device memory, a deployment that fixes its memory budget at start-up, or a loop that
cannot afford cudaMalloc's implicit device synchronisation.  For them the library keeps
a workspace of its own (a 64 MiB device array); the caller passes only inputs and outputs.

This file is named to be collected last, so that a run stopping at the first failure has
already run every other test.  It passes on its own in a fresh process too: the first
call on the device sets up the array's address itself."""
import ctypes

import pytest
import torch

from selective_scan_sfm_b200 import (SfmError, _abi, sfm_selective_scan_fold_bwd,
                                     sfm_selective_scan_fold_bwd_noalloc, synth)

from parity import TOL, rel_err, to_cuda

pytestmark = pytest.mark.gpu


def _grads_like(B, D, L, N):
    f = dict(dtype=torch.float32, device="cuda")
    return dict(du=torch.empty(B, D, L, **f), ddt=torch.empty(B, D, L, **f), dz=torch.empty(B, D, L, **f),
                dA=torch.empty(D, N, **f), dDskip=torch.empty(D, **f), ddt_bias=torch.empty(D, **f),
                dB=torch.empty(B, N, L, **f), dC=torch.empty(B, N, L, **f))


def _case(B, D, T, N, dtype, seed):
    d = to_cuda(synth.make_inputs(B=B, D=D, T=T, N=N, dtype=dtype, seed=seed, aux=False, random_A=True))
    dout = synth.make_dout(B, D, T, seed=seed, dtype=dtype).cuda()
    return d, dout


def _run_both(d, dout):
    kw = dict(z=d["z"], Dskip=d["Dskip"], dt_bias=d["dt_bias"])
    args = (d["x"], d["dt"], d["Bm"], d["Cm"], d["A"], dout)
    ref = sfm_selective_scan_fold_bwd(*args, **kw)  # existing entry point, caller workspace
    B, D, L = d["x"].shape
    got = sfm_selective_scan_fold_bwd_noalloc(*args, _grads_like(B, D, L, d["A"].shape[1]), **kw)
    torch.cuda.synchronize()
    return got, ref


def test_noalloc_backward_matches_the_workspace_entry_point_on_two_calls():
    # two calls in a row with different shapes and inputs: the second reuses the built-in
    # workspace left over from the first and must not depend on its contents
    for (B, D, T, N, dtype, seed, tol) in [(4, 130, 51, 16, "bf16", 301, TOL["bf16"]),
                                           (3, 70, 40, 8, "f32", 302, TOL["f32"])]:
        d, dout = _case(B, D, T, N, dtype, seed)
        got, ref = _run_both(d, dout)
        for k in ref:
            e = rel_err(got[k].double().cpu().numpy(), ref[k].double().cpu().numpy())
            assert e <= tol, "%s differs from the workspace entry point: %.3g" % (k, e)


def test_noalloc_backward_rejects_problems_beyond_its_workspace():
    # B*D*L = 8*1024*1024 fp32 elements need > 64 MiB of workspace; rejected before launch
    B, D, L, N = 8, 1024, 1024, 16
    a = _abi.ScanArgs()
    a.size = ctypes.sizeof(_abi.ScanArgs)
    fake = 0x7F0000000000  # validation fails on the size first: nothing is dereferenced
    for i, k in enumerate(("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias")):
        setattr(a, k, fake + (i << 32))
    a.B, a.D, a.L, a.N, a.reset_period, a.dt_softplus = B, D, L, N, L, 1
    a.in_dtype = a.out_dtype = _abi.SFM_F32
    g = _abi.ScanGrads()
    g.size = ctypes.sizeof(_abi.ScanGrads)
    for i, k in enumerate(("dout", "du", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC")):
        setattr(g, k, fake + ((i + 16) << 32))
    need = ctypes.c_size_t(0)
    assert _abi.lib().sfm_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(need)) == _abi.SFM_OK
    assert need.value > _abi.NOALLOC_SCRATCH_BYTES
    rc = _abi.lib().sfm_selective_scan_fold_bwd_noalloc(ctypes.byref(a), ctypes.byref(g), None)
    assert rc == _abi.SFM_ERR_UNSUPPORTED
    with pytest.raises(SfmError, match="UNSUPPORTED"):
        _abi.check(rc, "sfm_selective_scan_fold_bwd_noalloc")
