"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare element by element.

Error metric (the pages give none): per element |g - r| / (|r| + rms(r)), rms over the
whole compared tensor, maximum over elements.  Pure relative error is undefined where
y crosses zero; scaling by the tensor's rms keeps the bound meaningful there.
Bounds: 1e-5 for fp32 I/O, 2e-2 for bf16 I/O (fp32 state and accumulation in both)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_scan_sfm_b200 import sfm_selective_scan_fold

TOL = {"f32": 1e-5, "bf16": 2e-2}
PARAMS = ("A", "Dskip", "dt_bias", "conv_w", "conv_b")
ACTS = ("x", "z", "dt", "Bm", "Cm")


def rel_err(got, ref) -> float:
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    return float(np.max(np.abs(g - r) / (np.abs(r) + rms + 1e-300)))


def to_cuda(d: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def fused(dc: dict, **kw) -> torch.Tensor:
    """One launch of the fused forward on CUDA inputs produced by synth.make_inputs."""
    args = dict(z=dc["z"], Dskip=dc["Dskip"], dt_bias=dc["dt_bias"], conv_w=dc["conv_w"], conv_b=dc["conv_b"],
                aux_init=True)
    args.update(kw)
    return sfm_selective_scan_fold(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], **args)


def oracle_layer(d: dict, samples=None, aux_init=True, swap_out=False, conv=True, gate=True, skip=True, bias=True,
                 pad_left=None, dt_softplus=True, want_state=False, threads=4):
    """The oracle on CPU copies of the same inputs, optionally on a subset of samples."""
    sel = (lambda t: t) if samples is None else (lambda t: t[samples])
    f = lambda t: None if t is None else sel(t).double().numpy()
    p = lambda t: None if t is None else t.double().numpy()
    return oracle.mixer_layer(
        f(d["x"]), f(d["dt"]), f(d["z"]) if gate else None, f(d["Bm"]), f(d["Cm"]), p(d["A"]),
        p(d["Dskip"]) if skip else None, p(d["dt_bias"]) if bias else None,
        p(d["conv_w"]) if conv else None, p(d["conv_b"]) if conv else None,
        aux_init_in=aux_init, swap_out=swap_out, pad_left=pad_left, dt_softplus=dt_softplus,
        want_state=want_state, threads=threads)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (round-to-nearest-even) and widen back."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()
