"""GPU parity of the tcgen05 projection GEMM against the oracle's fp64 matmul.

Bounds from the arithmetic: bf16 x bf16 products are exact in fp32 and the tensor core
accumulates in fp32, so |g - r| <= K * 2^-23 * sum_k |W||X| before the output rounding;
fp32 outputs are held to 4e-6 of sum_k |W||X| (K <= 1280), bf16 outputs to that plus the
round-to-nearest error of an 8-bit significand (half an ulp: at most 2^-8 of the value)."""
import numpy as np
import pytest
import torch

import oracle
from selective_scan_sfm_b200 import SfmError, sfm_get_device_error, sfm_proj_gemm

pytestmark = pytest.mark.gpu


def draw(M, K, Ntok, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(M, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    X = torch.randn(Ntok, K, generator=g).to(torch.bfloat16)
    return W, X


def bound(W, X, L, M0, token_major):
    aw, ax = np.abs(W.double().numpy()), np.abs(X.double().numpy())
    return oracle.proj(aw, ax, L, M0=M0, token_major=token_major)


def check(got, ref, mag, dtype):
    g = got.double().cpu().numpy()
    if dtype == torch.float32:
        err = np.max(np.abs(g - ref) / (mag + 1e-30))
        assert err <= 4e-6, err
    else:
        err = np.max(np.abs(g - ref) / (4e-6 * mag + 2.0 ** -8 * np.abs(ref) + 1e-30))
        assert err <= 1.0, err


SCHEDULES = (1, 2)  # one CTA per tile; persistent


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("M,K,B,L,M0,tile_n,dt", [
    (128, 64, 2, 64, 128, 128, torch.float32),        # one CTA, one K step
    (256, 320, 4, 51, 128, 256, torch.bfloat16),      # in_proj shape: x and z split, ragged token tail
    (200, 72, 3, 37, 70, 128, torch.float32),         # M, K and token tails; split inside a tile
    (1280, 640, 8, 198, 640, 0, torch.bfloat16),      # stage-3 in_proj rows, automatic tile
    (64, 1280, 2, 51, 64, 256, torch.float32),        # long K (20 stages through a 4-stage ring)
])
def test_channel_major(M, K, B, L, M0, tile_n, dt, schedule):
    W, X = draw(M, K, B * L, seed=M + K + L)
    o0, o1 = sfm_proj_gemm(W.cuda(), X.cuda(), L, M0=M0, out_dtype=dt, tile_n=tile_n, schedule=schedule)
    torch.cuda.synchronize()
    assert sfm_get_device_error(clear=True) == 0
    r0, r1 = oracle.proj(W.double().numpy(), X.double().numpy(), L, M0=M0)
    m0, m1 = bound(W, X, L, M0, False)
    check(o0, r0, m0, dt)
    if M0 < M:
        check(o1, r1, m1, dt)
    else:
        assert o1 is None


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("M,K,Ntok,dt", [(40, 640, 198 * 3, torch.bfloat16), (72, 320, 300, torch.float32)])
def test_token_major(M, K, Ntok, dt, schedule):
    W, X = draw(M, K, Ntok, seed=M * 7 + K)
    o, none = sfm_proj_gemm(W.cuda(), X.cuda(), 1, token_major=True, out_dtype=dt, schedule=schedule)
    assert none is None
    ref = oracle.proj(W.double().numpy(), X.double().numpy(), 1, token_major=True)
    check(o, ref, bound(W, X, 1, None, True), dt)


def test_rows_past_the_ends_are_not_written():
    M, K, B, L = 70, 64, 2, 45
    W, X = draw(M, K, B * L, seed=9)
    o0 = torch.full((B, 30, L), 5.0, device="cuda")
    o1 = torch.full((B, 40, L), 5.0, device="cuda")
    big = torch.full((B * 40 * L + 64,), 7.0, device="cuda")
    o1 = big[:B * 40 * L].view(B, 40, L)
    sfm_proj_gemm(W.cuda(), X.cuda(), L, M0=30, out_dtype=torch.float32, out0=o0, out1=o1)
    torch.cuda.synchronize()
    assert torch.all(big[B * 40 * L:] == 7.0)  # nothing past out1
    r0, r1 = oracle.proj(W.double().numpy(), X.double().numpy(), L, M0=30)
    m0, m1 = bound(W, X, L, 30, False)
    check(o0, r0, m0, torch.float32)
    check(o1, r1, m1, torch.float32)


def test_validation():
    W, X = draw(128, 60, 64, seed=3)  # K = 60: row pitch 120 bytes, not a multiple of 16
    with pytest.raises(SfmError, match="UNSUPPORTED"):
        sfm_proj_gemm(W.cuda(), X.cuda(), 64)
    W, X = draw(128, 64, 64, seed=3)
    with pytest.raises(ValueError):
        sfm_proj_gemm(W.cuda(), X.cuda(), 48)  # 64 tokens are not whole samples of 48


# ------------------------------------------------------------------ the path around the scan

from selective_scan_sfm_b200 import sfm_conv1d_tokens, sfm_selective_scan_fold  # noqa: E402

from parity import TOL, bf16_round, rel_err  # noqa: E402


@pytest.mark.parametrize("dt,pad_left", [(torch.float32, 1), (torch.bfloat16, 3), (torch.bfloat16, 0)])
def test_conv1d_tokens(dt, pad_left):
    g = torch.Generator().manual_seed(70 + pad_left)
    B, D, L = 3, 100, 77
    x = torch.randn(B, D, L, generator=g).to(dt)
    w = torch.rand(D, 4, generator=g) - 0.5
    bias = torch.rand(D, generator=g) - 0.5
    u = sfm_conv1d_tokens(x.cuda(), w.cuda(), bias.cuda(), pad_left=pad_left)
    ref = oracle.conv1d(x.double().numpy(), w.double().numpy(), bias.double().numpy(), pad_left=pad_left, silu=True)
    ref = ref.transpose(0, 2, 1).reshape(B * L, D)
    got = u.double().cpu().numpy()
    if dt == torch.float32:
        assert rel_err(got, ref) <= TOL["f32"]
    else:
        assert rel_err(got, bf16_round(ref)) <= 2.0 ** -7  # bf16 RN on both sides, fp32 vs fp64 sums


def test_projections_feed_the_scan():
    """tokens -> in_proj (x, z) -> conv (token-major u) -> x_proj (dt_low, B, C) -> dt_proj
    (dt) -> the fused scan, all on the GPU, against the same chain in the oracle (fp64,
    rounded to bf16 at the same stage boundaries, on its own values)."""
    g = torch.Generator().manual_seed(77)
    B, L, C, D, N, R = 4, 51, 160, 320, 16, 24
    bf = torch.bfloat16
    tok = torch.randn(B * L, C, generator=g).to(bf)
    W_in = (torch.randn(2 * D, C, generator=g) / C ** 0.5).to(bf)
    W_x = (torch.randn(R + 2 * N, D, generator=g) / D ** 0.5).to(bf)
    W_dt = (0.5 * torch.randn(D, R, generator=g) / R ** 0.5).to(bf)
    conv_w = torch.rand(D, 4, generator=g) - 0.5
    conv_b = torch.rand(D, generator=g) - 0.5
    A = -torch.exp(torch.randn(D, N, generator=g))
    Dskip = torch.randn(D, generator=g)
    dt_bias = torch.log(torch.expm1(1e-3 + torch.rand(D, generator=g, dtype=torch.float64) * (1e-1 - 1e-3))).float()
    c = lambda t: t.cuda()
    x, z = sfm_proj_gemm(c(W_in), c(tok), L, M0=D)
    u_tok = sfm_conv1d_tokens(x, c(conv_w), c(conv_b))
    dt_low, _ = sfm_proj_gemm(c(W_x[:R].contiguous()), u_tok, L, token_major=True)
    Bm, Cm = sfm_proj_gemm(c(W_x[R:].contiguous()), u_tok, L, M0=N)
    dt, _ = sfm_proj_gemm(c(W_dt), dt_low, L)
    y = sfm_selective_scan_fold(x, dt, Bm, Cm, c(A), z=z, Dskip=c(Dskip), dt_bias=c(dt_bias), conv_w=c(conv_w),
                                conv_b=c(conv_b))
    torch.cuda.synchronize()
    assert sfm_get_device_error(clear=True) == 0

    f = lambda t: t.double().numpy()
    r16 = bf16_round
    xr, zr = oracle.proj(f(W_in), f(tok), L, M0=D)
    xr, zr = r16(xr), r16(zr)
    ur = r16(oracle.conv1d(xr, f(conv_w), f(conv_b), silu=True).transpose(0, 2, 1).reshape(B * L, D))
    dlr = r16(oracle.proj(f(W_x[:R]), ur, L, token_major=True))
    br, cr = oracle.proj(f(W_x[R:]), ur, L, M0=N)
    br, cr = r16(br), r16(cr)
    dtr, _ = oracle.proj(f(W_dt), dlr, L)
    dtr = r16(dtr)
    yr = oracle.mixer_layer(xr, dtr, zr, br, cr, f(A), f(Dskip), f(dt_bias), f(conv_w), f(conv_b))
    e = rel_err(y.double().cpu().numpy(), yr)
    assert e <= TOL["bf16"], e
