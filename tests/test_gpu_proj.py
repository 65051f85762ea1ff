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


@pytest.mark.parametrize("M,K,B,L,M0,tile_n,dt", [
    (128, 64, 2, 64, 128, 128, torch.float32),        # one CTA, one K step
    (256, 320, 4, 51, 128, 256, torch.bfloat16),      # in_proj shape: x and z split, ragged token tail
    (200, 72, 3, 37, 70, 128, torch.float32),         # M, K and token tails; split inside a tile
    (1280, 640, 8, 198, 640, 0, torch.bfloat16),      # stage-3 in_proj rows, automatic tile
    (64, 1280, 2, 51, 64, 256, torch.float32),        # long K (20 stages through a 4-stage ring)
])
def test_channel_major(M, K, B, L, M0, tile_n, dt):
    W, X = draw(M, K, B * L, seed=M + K + L)
    o0, o1 = sfm_proj_gemm(W.cuda(), X.cuda(), L, M0=M0, out_dtype=dt, tile_n=tile_n)
    torch.cuda.synchronize()
    assert sfm_get_device_error(clear=True) == 0
    r0, r1 = oracle.proj(W.double().numpy(), X.double().numpy(), L, M0=M0)
    m0, m1 = bound(W, X, L, M0, False)
    check(o0, r0, m0, dt)
    if M0 < M:
        check(o1, r1, m1, dt)
    else:
        assert o1 is None


@pytest.mark.parametrize("M,K,Ntok,dt", [(40, 640, 198 * 3, torch.bfloat16), (72, 320, 300, torch.float32)])
def test_token_major(M, K, Ntok, dt):
    W, X = draw(M, K, Ntok, seed=M * 7 + K)
    o, none = sfm_proj_gemm(W.cuda(), X.cuda(), 1, token_major=True, out_dtype=dt)
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
