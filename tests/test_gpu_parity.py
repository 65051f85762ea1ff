"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the same
seeded inputs, element by element, with the bound stated in tests/parity.py."""
import numpy as np
import pytest
import torch

from selective_scan_sfm_b200 import (SfmError, sfm_aux_init, sfm_aux_swap, sfm_fold_conv1d,
                                     sfm_selective_scan_fold, synth)

from parity import TOL, bf16_round, fused, oracle_layer, rel_err, to_cuda

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def check(got, ref, dtype, what=""):
    e = rel_err(got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got, ref)
    assert e <= TOL[dtype], "%s max rel err %.3g > %.1g" % (what, e, TOL[dtype])
    return e


# ------------------------------------------------------------------ the tiny fp32 folded case

@pytest.mark.parametrize("B1", [1, 2, 4])
@pytest.mark.parametrize("swap", [False, True])
def test_tiny_fp32_every_fold(B1, swap):
    d = synth.make_inputs(**synth.WORKLOADS["tiny_fp32"], seed=0)
    dc = to_cuda(d)
    y = fused(dc, B1=B1, swap_out=swap)
    ref = oracle_layer(d, swap_out=swap)
    check(y, ref, "f32", "tiny B1=%d" % B1)


def test_fold_choice_is_bitwise_invariant():
    """The reset makes samples independent: B1, the channel tile and the LUT choice only
    change the schedule; each channel's arithmetic is identical, so outputs match bitwise."""
    d = synth.make_inputs(B=8, D=96, T=49, N=16, dtype="bf16", seed=3)
    dc = to_cuda(d)
    base = fused(dc, B1=8, d_tile=32)
    for kw in (dict(B1=1), dict(B1=2, d_tile=64), dict(B1=4, d_tile=128), dict(B1=0)):
        assert torch.equal(fused(dc, **kw), base), kw


# ------------------------------------------------------------------ shapes spanning tiles and ragged tails

GRID = [
    # B, D, T, N, K, pad_left, dtype, d_tile, chunk
    (6, 200, 75, 16, 4, 1, "bf16", 64, 32),
    (6, 200, 75, 16, 4, 3, "bf16", 128, 16),
    (5, 70, 40, 8, 4, 1, "f32", 32, 8),
    (3, 33, 30, 3, 3, 1, "f32", 64, 24),
    (4, 40, 17, 1, 2, 0, "bf16", 32, 8),
    (2, 129, 61, 5, 1, 0, "f32", 128, 64),
    (7, 64, 120, 16, 4, 0, "bf16", 64, 40),
    (2, 48, 254, 12, 4, 2, "f32", 32, 128),
]


@pytest.mark.parametrize("B,D,T,N,K,pl,dtype,d_tile,chunk", GRID)
def test_grid_against_oracle(B, D, T, N, K, pl, dtype, d_tile, chunk):
    d = synth.make_inputs(B=B, D=D, T=T, N=N, K=K, dtype=dtype, seed=B * 1000 + D + T, random_A=True)
    dc = to_cuda(d)
    for swap in (False, True):
        y = fused(dc, pad_left=pl, swap_out=swap, d_tile=d_tile, chunk=chunk, B1=1 if B % 2 else 2)
        ref = oracle_layer(d, pad_left=pl, swap_out=swap)
        check(y, ref, dtype, "grid swap=%s" % swap)


@pytest.mark.parametrize("conv,gate,skip,bias,softplus,aux", [
    (False, False, False, False, False, False),
    (False, True, True, True, True, False),
    (True, False, True, True, True, True),
    (True, True, False, True, True, True),
    (True, True, True, False, True, True),
    (True, True, True, True, False, True),
    (False, True, True, True, True, True),
    (True, True, True, True, True, False),
])
def test_optional_parts(conv, gate, skip, bias, softplus, aux):
    B, D, T, N = 4, 72, 60, 16
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype="f32", seed=11, aux=aux)
    if not softplus:
        # Delta = dt + dt_bias used as given: keep both positive and small
        d["dt"] = d["dt"].abs() * 0.1
        d["dt_bias"] = torch.nn.functional.softplus(d["dt_bias"])
    dc = to_cuda(d)
    y = sfm_selective_scan_fold(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], z=dc["z"] if gate else None,
                                Dskip=dc["Dskip"] if skip else None, dt_bias=dc["dt_bias"] if bias else None,
                                conv_w=dc["conv_w"] if conv else None, conv_b=dc["conv_b"] if conv else None,
                                dt_softplus=softplus, aux_init=aux, chunk=24)
    ref = oracle_layer(d, aux_init=aux, conv=conv, gate=gate, skip=skip, bias=bias, dt_softplus=softplus)
    check(y, ref, "f32")


def test_final_state_and_bf16_to_f32():
    d = synth.make_inputs(B=4, D=80, T=47, N=16, dtype="bf16", seed=5)
    dc = to_cuda(d)
    fs = torch.full((4, 80, 16), float("nan"), device="cuda")
    y = fused(dc, final_state=fs, out_dtype=torch.float32, chunk=16)
    ref, ref_state = oracle_layer(d, want_state=True)
    assert y.dtype == torch.float32
    # output not rounded to bf16: the bound is set by the bf16 inputs and fp32 arithmetic
    assert rel_err(y.double().cpu().numpy(), ref) <= 2e-3
    assert rel_err(fs.double().cpu().numpy(), ref_state) <= 2e-3


def test_edge_sizes():
    for (B, D, T, N, aux) in [(1, 1, 1, 1, True), (1, 3, 2, 2, True), (2, 1, 1, 4, False), (3, 5, 9, 16, True),
                              (1, 1, 300, 16, True)]:
        d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype="f32", seed=7 + T, aux=aux)
        dc = to_cuda(d)
        for swap in (False, True):
            L = T + 2 if aux else T
            if swap and L < 2:
                continue
            y = fused(dc, aux_init=aux, swap_out=swap)
            check(y, oracle_layer(d, aux_init=aux, swap_out=swap), "f32", "edge %s" % ((B, D, T, N, aux),))


@pytest.mark.parametrize("bad", [float("inf"), float("nan")])
def test_sample_isolation(bad):
    d = synth.make_inputs(B=6, D=64, T=49, N=16, dtype="bf16", seed=13)
    dc = to_cuda(d)
    y0 = fused(dc, B1=1, chunk=24)  # all six samples in one folded row
    for field in ("x", "dt", "z", "Bm", "Cm"):
        p = dict(dc)
        p[field] = dc[field].clone()
        p[field][2] = bad
        y1 = fused(p, B1=1, chunk=24)
        keep = [0, 1, 3, 4, 5]
        assert torch.equal(y1[keep], y0[keep]), field


def test_random_A_and_canaries():
    d = synth.make_inputs(B=4, D=130, T=49, N=16, dtype="bf16", seed=17, random_A=True)
    dc = to_cuda(d)
    B, D, L = 4, 130, 51
    guard = 4096
    buf = torch.full((guard * 2 + B * D * L,), 1234.0, dtype=torch.bfloat16, device="cuda")
    y = buf[guard:guard + B * D * L].view(B, D, L)
    fused(dc, y=y)
    assert torch.all(buf[:guard] == 1234.0) and torch.all(buf[guard + B * D * L:] == 1234.0)
    check(y, oracle_layer(d), "bf16")


def test_misaligned_pointer_is_rejected():
    d = to_cuda(synth.make_inputs(B=2, D=16, T=49, N=8, dtype="bf16", seed=1))
    big = torch.empty(2 * 16 * 51 + 1, dtype=torch.bfloat16, device="cuda")
    y = big[1:].view(2, 16, 51)  # 2-byte offset
    with pytest.raises(SfmError, match="MISALIGNED"):
        fused(d, y=y)


# ------------------------------------------------------------------ the standalone steps

def test_standalone_aux_and_conv():
    import oracle
    d = synth.make_inputs(B=3, D=40, T=49, N=4, dtype="bf16", seed=19)
    dc = to_cuda(d)
    xa = sfm_aux_init(dc["x"])
    ref_xa = bf16_round(oracle.aux_init(d["x"].double().numpy()))  # xa is a bf16 tensor on both sides
    assert torch.equal(xa[..., 1:-1], dc["x"])
    check(xa, ref_xa, "bf16", "aux_init")
    for pl in (0, 1, 3):
        for silu in (False, True):
            u = sfm_fold_conv1d(xa, dc["conv_w"], dc["conv_b"], pad_left=pl, B2=3, silu=silu)
            ref = oracle.conv1d(ref_xa, d["conv_w"].double().numpy(),
                                d["conv_b"].double().numpy(), K=4, pad_left=pl, silu=silu)
            check(u, ref, "bf16", "conv pl=%d" % pl)
    y = xa.clone()
    sfm_aux_swap(y)
    assert torch.equal(y[..., 0], xa[..., -1]) and torch.equal(y[..., -1], xa[..., 0])
    assert torch.equal(y[..., 1:-1], xa[..., 1:-1])


def test_unfused_pipeline_matches_fused():
    """aux_init -> conv -> scan(u) -> swap as four launches equals the fused launch."""
    d = synth.make_inputs(B=4, D=96, T=49, N=16, dtype="f32", seed=23)
    dc = to_cuda(d)
    xa = sfm_aux_init(dc["x"])
    u = sfm_fold_conv1d(xa, dc["conv_w"], dc["conv_b"], silu=True)
    y = sfm_selective_scan_fold(u, dc["dt"], dc["Bm"], dc["Cm"], dc["A"], z=dc["z"], Dskip=dc["Dskip"],
                                dt_bias=dc["dt_bias"])
    sfm_aux_swap(y)
    yf = fused(dc, swap_out=True)
    check(y, oracle_layer(d, swap_out=True), "f32", "unfused")
    assert rel_err(y.double().cpu().numpy(), yf.double().cpu().numpy()) <= 1e-5


# ------------------------------------------------------------------ full sizes, in the benchmark's launch shape

@pytest.mark.parametrize("name", ["stage4_t49", "stage3_t196", "long_t784"])
def test_full_size_sampled(name):
    w = synth.WORKLOADS[name]
    d = synth.make_inputs(**w, seed=0)
    dc = to_cuda(d)
    y = fused(dc, B1=0)  # the look-up-table choice, as the benchmark runs it
    samples = synth.sample_indices(w["B"], 6, seed=1)
    ref = oracle_layer(d, samples=samples)
    check(y[samples], ref, w["dtype"], name)


def test_chain_of_four_layers():
    """Four mixer layers at the stage-3 shape: aux init on layer 0, head<->tail swap between
    layers, bf16 between layers on both sides; sampled samples through the whole chain."""
    w = synth.WORKLOADS["chain4_stage3"]
    layers = synth.make_chain(**w, seed=0)
    samples = synth.sample_indices(w["B"], 4, seed=2)
    x = layers[0]["x"].cuda()
    xo = layers[0]["x"][samples]
    for i, d in enumerate(layers):
        last = i == len(layers) - 1
        dc = to_cuda(d)
        dc["x"] = x
        y = fused(dc, aux_init=(i == 0), swap_out=not last)
        dd = dict(d)
        dd["x"] = xo
        ref = oracle_layer({k: (v[samples] if k in ("dt", "z", "Bm", "Cm") else v) for k, v in dd.items()},
                           aux_init=(i == 0), swap_out=not last)
        check(y[samples], ref, "bf16", "chain layer %d" % i)
        x = y
        xo = torch.from_numpy(bf16_round(ref)).to(torch.bfloat16)


# ------------------------------------------------------------------ lanes mode: P lanes split a channel's tokens

LANES_GRID = [
    # B, D, T, N, dtype, lanes, d_tile
    (2, 40, 300, 16, "bf16", 8, 16),
    (3, 20, 130, 8, "f32", 4, 8),
    (2, 33, 100, 5, "f32", 16, 2),
    (1, 8, 500, 16, "bf16", 32, 4),
    (4, 64, 75, 16, "bf16", 2, 64),
    (2, 10, 17, 1, "f32", 8, 4),
    (2, 12, 61, 3, "f32", 32, 8),
]


@pytest.mark.parametrize("B,D,T,N,dtype,lanes,d_tile", LANES_GRID)
def test_lanes_against_oracle(B, D, T, N, dtype, lanes, d_tile):
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype=dtype, seed=7000 + T + lanes, random_A=True)
    dc = to_cuda(d)
    for swap in (False, True):
        fs = torch.full((B, D, N), float("nan"), device="cuda")
        y = fused(dc, swap_out=swap, lanes=lanes, d_tile=d_tile, B1=B, final_state=fs)
        ref, ref_state = oracle_layer(d, swap_out=swap, want_state=True)
        check(y, ref, dtype, "lanes=%d swap=%s" % (lanes, swap))
        assert rel_err(fs.double().cpu().numpy(), ref_state) <= TOL[dtype]


@pytest.mark.parametrize("conv,gate,aux", [(False, False, False), (True, False, True), (False, True, True)])
def test_lanes_optional_parts(conv, gate, aux):
    d = synth.make_inputs(B=2, D=24, T=90, N=8, dtype="f32", seed=7100, aux=aux)
    dc = to_cuda(d)
    y = sfm_selective_scan_fold(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], z=dc["z"] if gate else None,
                                Dskip=dc["Dskip"], dt_bias=dc["dt_bias"], conv_w=dc["conv_w"] if conv else None,
                                conv_b=dc["conv_b"] if conv else None, aux_init=aux, lanes=8, d_tile=8)
    check(y, oracle_layer(d, aux_init=aux, conv=conv, gate=gate), "f32")


def test_lanes_sample_isolation():
    d = synth.make_inputs(B=4, D=16, T=200, N=16, dtype="bf16", seed=7200)
    dc = to_cuda(d)
    y0 = fused(dc, lanes=8, d_tile=16, B1=1)
    for field in ("x", "dt", "Bm"):
        p = dict(dc)
        p[field] = dc[field].clone()
        p[field][1] = float("nan")
        y1 = fused(p, lanes=8, d_tile=16, B1=1)
        assert torch.equal(y1[[0, 2, 3]], y0[[0, 2, 3]]), field


# ------------------------------------------------------------------ two channels per thread

CPT2_GRID = [
    # B, D, T, N, dtype, d_tile, chunk (chunk >= L: whole-sample staging)
    (4, 128, 49, 16, "bf16", 64, 56),
    (3, 70, 49, 12, "f32", 32, 56),
    (2, 96, 120, 16, "bf16", 64, 32),
    (2, 34, 75, 16, "f32", 32, 24),
]


@pytest.mark.parametrize("B,D,T,N,dtype,d_tile,chunk", CPT2_GRID)
def test_two_channels_per_thread(B, D, T, N, dtype, d_tile, chunk):
    d = synth.make_inputs(B=B, D=D, T=T, N=N, dtype=dtype, seed=8000 + D + T, random_A=True)
    dc = to_cuda(d)
    for swap in (False, True):
        fs = torch.full((B, D, N), float("nan"), device="cuda")
        y = fused(dc, swap_out=swap, d_tile=d_tile, chunk=chunk, chans_per_thread=2, B1=B, final_state=fs)
        ref, ref_state = oracle_layer(d, swap_out=swap, want_state=True)
        check(y, ref, dtype, "cpt=2 swap=%s" % swap)
        assert rel_err(fs.double().cpu().numpy(), ref_state) <= TOL[dtype]
        y1 = fused(dc, swap_out=swap, d_tile=d_tile, chunk=chunk, chans_per_thread=1, B1=B)
        assert rel_err(y.double().cpu().numpy(), y1.double().cpu().numpy()) <= TOL[dtype]


# ------------------------------------------------------------------ state sizes above 16 (lanes mode)

@pytest.mark.parametrize("N,dtype", [(24, "f32"), (32, "bf16"), (64, "f32")])
def test_large_state_sizes(N, dtype):
    d = synth.make_inputs(B=3, D=40, T=70, N=N, dtype=dtype, seed=9000 + N, random_A=True)
    dc = to_cuda(d)
    fs = torch.full((3, 40, N), float("nan"), device="cuda")
    y = fused(dc, swap_out=True, final_state=fs)  # routed to lanes mode automatically
    ref, ref_state = oracle_layer(d, swap_out=True, want_state=True)
    check(y, ref, dtype, "N=%d" % N)
    assert rel_err(fs.double().cpu().numpy(), ref_state) <= TOL[dtype]
    with pytest.raises(SfmError, match="UNSUPPORTED"):
        fused(dc, lanes=1, d_tile=32)  # one thread per channel holds at most 16 states
