"""Seeded synthetic inputs for the folded selective scan (no arithmetic of the method).

Shared by the tests, the smoke check and the benchmark; it only draws random numbers.
Draws use a CPU ``torch.Generator`` seeded per call, in fp32, in this fixed order:
x ~ N(0,1) [B,D,T] (the mixer input before the conv), z ~ N(0,1) [B,D,L],
dt = 0.5*N(0,1) [B,D,L], dt_bias = log(expm1(U(1e-3,1e-1))) [D] (so that
softplus(dt_bias) is uniform on [1e-3, 1e-1]), B ~ N(0,1) [B,N,L], C ~ N(0,1) [B,N,L],
Dskip ~ N(0,1) [D], conv_w ~ U(-0.5,0.5) [D,K], conv_b ~ U(-0.5,0.5) [D].
A[d,n] = -(n+1) (S4D-real), or A = -exp(N(0,1)) with ``random_A`` so no structure
of A can be relied on.  x, z, dt, B, C are then cast to the I/O dtype; A, Dskip,
dt_bias, conv_w and conv_b stay fp32.

The shapes stand in for MambaVision stage-3 / stage-4 token sequences at 224x224
(T = 196 / 49 patch tokens, plus the two auxiliary tokens).
"""
from __future__ import annotations

import math

import torch

#: Workloads by name: the shapes and dtypes of the five cases of the hot path.
WORKLOADS = {
    # tiny folded scan, fp32 I/O: B=4 folded as B1=1 x B2=4
    "tiny_fp32": dict(B=4, D=16, T=49, N=8, K=4, dtype="f32", B2=4),
    # MambaVision stage-4 shaped: 7x7 tokens
    "stage4_t49": dict(B=256, D=1280, T=49, N=16, K=4, dtype="bf16"),
    # MambaVision stage-3 shaped: 14x14 tokens
    "stage3_t196": dict(B=128, D=640, T=196, N=16, K=4, dtype="bf16"),
    # longer sequences (28x28 tokens) where folding matters less
    "long_t784": dict(B=16, D=320, T=784, N=16, K=4, dtype="bf16"),
    # ragged batch: 128 samples of 49..196 patch tokens (windowed / detection-like mix of
    # the stage-4 and stage-3 token counts) packed along time, stage-3 channels
    "ragged_t49_196": dict(S=128, T_lo=49, T_hi=196, D=640, N=16, K=4, dtype="bf16", ragged=True),
    # four mixer layers in a chain at the stage-3 shape
    "chain4_stage3": dict(B=64, D=640, T=196, N=16, K=4, dtype="bf16", layers=4),
}

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DT[name]


def make_inputs(B: int, D: int, T: int, N: int, K: int = 4, dtype: str = "bf16", seed: int = 0,
                random_A: bool = False, aux: bool = True, **_ignored) -> dict:
    """Draw one layer's inputs on the CPU.

    With ``aux`` the conv input x has T tokens (the kernel adds the two auxiliary
    tokens, L = T + 2); without it x already has L = T tokens."""
    g = torch.Generator().manual_seed(int(seed))
    L = T + 2 if aux else T
    io = _TORCH_DT[dtype]
    x = torch.randn(B, D, T, generator=g)
    z = torch.randn(B, D, L, generator=g)
    dt = 0.5 * torch.randn(B, D, L, generator=g)
    u01 = torch.rand(D, generator=g, dtype=torch.float64)
    dt_bias = torch.log(torch.expm1(1e-3 + u01 * (1e-1 - 1e-3))).float()
    Bm = torch.randn(B, N, L, generator=g)
    Cm = torch.randn(B, N, L, generator=g)
    Dskip = torch.randn(D, generator=g)
    conv_w = torch.rand(D, K, generator=g) - 0.5
    conv_b = torch.rand(D, generator=g) - 0.5
    if random_A:
        A = -torch.exp(torch.randn(D, N, generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(D, 1)
    return dict(x=x.to(io), z=z.to(io), dt=dt.to(io), Bm=Bm.to(io), Cm=Cm.to(io),
                A=A.contiguous(), Dskip=Dskip, dt_bias=dt_bias, conv_w=conv_w.contiguous(),
                conv_b=conv_b, B=B, D=D, T=T, L=L, N=N, K=K, dtype=dtype)


def ragged_lengths(S: int, T_lo: int, T_hi: int, seed: int = 0, aux: bool = True) -> list:
    """Per-sample token counts L_s for a ragged batch: T_s uniform on {T_lo..T_hi} patch
    tokens (plus the two aux tokens with ``aux``)."""
    g = torch.Generator().manual_seed(int(seed) + 991)
    T = torch.randint(T_lo, T_hi + 1, (S,), generator=g)
    return [int(t) + (2 if aux else 0) for t in T]


def make_ragged_inputs(lens, D: int, N: int, K: int = 4, dtype: str = "bf16", seed: int = 0,
                       random_A: bool = False, aux: bool = True) -> dict:
    """One layer's inputs for S samples of lengths ``lens`` (tokens per sample, aux tokens
    included) packed along time, drawn like ``make_inputs``: x [D, Ltot - 2S] with ``aux``
    (else [D, Ltot]), z and dt [D, Ltot], Bm and Cm [N, Ltot], cu_seqlens int32 [S+1]."""
    g = torch.Generator().manual_seed(int(seed))
    S = len(lens)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    Lt = cu[-1]
    io = _TORCH_DT[dtype]
    x = torch.randn(D, Lt - 2 * S if aux else Lt, generator=g)
    z = torch.randn(D, Lt, generator=g)
    dt = 0.5 * torch.randn(D, Lt, generator=g)
    u01 = torch.rand(D, generator=g, dtype=torch.float64)
    dt_bias = torch.log(torch.expm1(1e-3 + u01 * (1e-1 - 1e-3))).float()
    Bm = torch.randn(N, Lt, generator=g)
    Cm = torch.randn(N, Lt, generator=g)
    Dskip = torch.randn(D, generator=g)
    conv_w = torch.rand(D, K, generator=g) - 0.5
    conv_b = torch.rand(D, generator=g) - 0.5
    if random_A:
        A = -torch.exp(torch.randn(D, N, generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(D, 1)
    return dict(x=x.to(io), z=z.to(io), dt=dt.to(io), Bm=Bm.to(io), Cm=Cm.to(io), A=A.contiguous(), Dskip=Dskip,
                dt_bias=dt_bias, conv_w=conv_w.contiguous(), conv_b=conv_b,
                cu_seqlens=torch.tensor(cu, dtype=torch.int32), S=S, D=D, Ltot=Lt, N=N, K=K, dtype=dtype)


def make_chain(B: int, D: int, T: int, N: int, layers: int = 4, K: int = 4, dtype: str = "bf16",
               seed: int = 0, **_ignored) -> list:
    """Per-layer inputs of a mixer chain: layer 0 draws x [B,D,T]; every layer draws its
    own z, dt, B, C and parameters from seed + 1000*layer."""
    out = []
    for i in range(layers):
        d = make_inputs(B, D, T, N, K=K, dtype=dtype, seed=seed + 1000 * i)
        if i > 0:
            d["x"] = None
        out.append(d)
    return out


def make_dout(B: int, D: int, L: int, seed: int = 0, dtype: str = "bf16") -> torch.Tensor:
    """Upstream gradient for the backward check: N(0,1)."""
    g = torch.Generator().manual_seed(int(seed) + 77)
    return torch.randn(B, D, L, generator=g).to(_TORCH_DT[dtype])


def sample_indices(B: int, k: int, seed: int = 0) -> list:
    """k distinct sample indices spread over the batch, always including 0 and B-1."""
    if k >= B:
        return list(range(B))
    g = torch.Generator().manual_seed(int(seed) + 5)
    mid = torch.randperm(B - 2, generator=g)[: max(0, k - 2)] + 1
    return sorted(set([0, B - 1] + mid.tolist()))


def elements(B: int, D: int, L: int) -> int:
    return B * D * L


def inv_softplus(v: float) -> float:
    return math.log(math.expm1(v))
