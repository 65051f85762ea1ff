"""CPU oracle for the SF-Mamba folded selective scan hot path (fp64).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py``; never by the product package.  It shares no code
with the CUDA library.  ``sfm_oracle.c`` holds the arithmetic; this module compiles it
with gcc (``build()``), marshals numpy fp64 arrays through ctypes and composes the
mixer layer from the single steps in the order the pages give:

    aux init (first layer of a stage) or head<->tail swap of the previous output
    -> depthwise conv1d with per-sample zero padding -> SiLU
    -> Delta = softplus(dt + dt_bias) -> selective scan with D skip -> y * SiLU(z)
    -> head<->tail swap of the output for the next layer.

Sources: "SF-Mamba：重新思考视觉 Mamba 的信息流与并行效率" (techloop.online), sections on
Auxiliary Patch Swapping and Batch Folding with Periodic State Reset;
"Seeing Both Ways, Running One Way" (sungsoo.github.io), section 3.1-3.3 equations and
section 8.1 items 1-5.  Pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_l = ctypes.c_long
_i = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile sfm_oracle.c into liboracle.so (plain gcc, IEEE fp64, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.ora_softplus.restype = ctypes.c_double
        lib.ora_softplus.argtypes = [ctypes.c_double]
        lib.ora_silu.restype = ctypes.c_double
        lib.ora_silu.argtypes = [ctypes.c_double]
        lib.ora_aux_init.argtypes = [_dp, _dp, _l, _l, _l]
        lib.ora_aux_swap.argtypes = [_dp, _l, _l, _l]
        lib.ora_conv1d.argtypes = [_dp, _dp, _dp, _dp, _l, _l, _l, _i, _i, _i]
        scan_args = [_dp] * 10 + [_l, _l, _l, _l, _i]
        lib.ora_scan.argtypes = scan_args + [_l, _l]
        lib.ora_scan_folded.argtypes = scan_args + [_l]
        lib.ora_scan_bwd.argtypes = [_dp] * 17 + [_l, _l, _l, _l, _i]
        lib.ora_conv1d_bwd.argtypes = [_dp] * 7 + [_l, _l, _l, _i, _i, _i]
        lib.ora_aux_init_bwd.argtypes = [_dp, _dp, _l, _l, _l]
        for f in ("ora_aux_init", "ora_aux_swap", "ora_conv1d", "ora_scan", "ora_scan_folded", "ora_scan_bwd",
                  "ora_conv1d_bwd", "ora_aux_init_bwd"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: exact widening of the stored values
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(_dp)


def softplus(v: float) -> float:
    return _load().ora_softplus(float(v))


def silu(v: float) -> float:
    return _load().ora_silu(float(v))


def aux_init(x):
    """[B,D,T] -> [B,D,T+2] with head = tail = mean over the T tokens."""
    x = _f64(x)
    B, D, T = x.shape
    xa = np.empty((B, D, T + 2), np.float64)
    _load().ora_aux_init(_p(x), _p(xa), B, D, T)
    return xa


def aux_swap(y):
    """Returns a copy of y [B,D,L] with tokens 0 and L-1 exchanged."""
    y = _f64(y).copy()
    B, D, L = y.shape
    _load().ora_aux_swap(_p(y), B, D, L)
    return y


def conv1d(xa, w, bias, K=None, pad_left=None, silu=False):
    """Depthwise conv1d, zero padding per sample; pad_left defaults to (K-1)//2."""
    xa, w, bias = _f64(xa), _f64(w), _f64(bias)
    B, D, L = xa.shape
    K = w.shape[1] if K is None else K
    pad_left = (K - 1) // 2 if pad_left is None else pad_left
    u = np.empty_like(xa)
    _load().ora_conv1d(_p(xa), _p(w), _p(bias), _p(u), B, D, L, K, pad_left, int(silu))
    return u


def _scan_common(u, dt, z, Bm, Cm, A, Dskip, dt_bias):
    u, dt, z, Bm, Cm, A = _f64(u), _f64(dt), _f64(z), _f64(Bm), _f64(Cm), _f64(A)
    return u, dt, z, Bm, Cm, A, _f64(Dskip), _f64(dt_bias)


def scan(u, dt, Bm, Cm, A, Dskip=None, dt_bias=None, z=None, dt_softplus=True,
         want_state=False, threads=1):
    """Per-sample selective scan (+ D skip, + SiLU(z) gate when z is given).

    threads > 1 splits the samples across host threads (ctypes drops the GIL); the
    arithmetic of every sample is unchanged."""
    u, dt, z, Bm, Cm, A, Dskip, dt_bias = _scan_common(u, dt, z, Bm, Cm, A, Dskip, dt_bias)
    B, D, L = u.shape
    N = A.shape[1]
    y = np.empty_like(u)
    fs = np.empty((B, D, N), np.float64) if want_state else None
    lib = _load()

    def run(lo, hi):
        lib.ora_scan(_p(u), _p(dt), _p(z), _p(Bm), _p(Cm), _p(A), _p(Dskip), _p(dt_bias),
                     _p(y), _p(fs), B, D, L, N, int(dt_softplus), lo, hi)

    threads = max(1, min(int(threads), B))
    if threads == 1:
        run(0, B)
    else:
        edges = [B * i // threads for i in range(threads + 1)]
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(edges[i], edges[i + 1]), range(threads)))
    return (y, fs) if want_state else y


def scan_folded(u, dt, Bm, Cm, A, B2, Dskip=None, dt_bias=None, z=None, dt_softplus=True,
                want_state=False):
    """Literal folded scan: one recurrence over [B1, D, B2*L] with the reset select."""
    u, dt, z, Bm, Cm, A, Dskip, dt_bias = _scan_common(u, dt, z, Bm, Cm, A, Dskip, dt_bias)
    B, D, L = u.shape
    N = A.shape[1]
    if B % B2:
        raise ValueError("B2 must divide B")
    y = np.empty_like(u)
    fs = np.empty((B, D, N), np.float64) if want_state else None
    _load().ora_scan_folded(_p(u), _p(dt), _p(z), _p(Bm), _p(Cm), _p(A), _p(Dskip), _p(dt_bias),
                            _p(y), _p(fs), B, D, L, N, int(dt_softplus), B2)
    return (y, fs) if want_state else y


def scan_bwd(u, dt, Bm, Cm, A, dout, Dskip=None, dt_bias=None, z=None, dt_softplus=True):
    """Gradients of the gated scan output w.r.t. its inputs, as a dict of fp64 arrays."""
    u, dt, z, Bm, Cm, A, Dskip, dt_bias = _scan_common(u, dt, z, Bm, Cm, A, Dskip, dt_bias)
    dout = _f64(dout)
    B, D, L = u.shape
    N = A.shape[1]
    g = {k: np.zeros((B, D, L)) for k in ("du", "ddt", "dz")}
    g["dA"] = np.zeros((D, N))
    g["dDskip"] = np.zeros(D)
    g["ddt_bias"] = np.zeros(D)
    g["dB"] = np.zeros((B, N, L))
    g["dC"] = np.zeros((B, N, L))
    _load().ora_scan_bwd(_p(u), _p(dt), _p(z), _p(Bm), _p(Cm), _p(A), _p(Dskip), _p(dt_bias), _p(dout),
                         _p(g["du"]), _p(g["ddt"]), _p(g["dz"]), _p(g["dA"]),
                         _p(g["dDskip"] if Dskip is not None else None),
                         _p(g["ddt_bias"] if dt_bias is not None else None),
                         _p(g["dB"]), _p(g["dC"]), B, D, L, N, int(dt_softplus))
    if z is None:
        del g["dz"]
    if Dskip is None:
        del g["dDskip"]
    if dt_bias is None:
        del g["ddt_bias"]
    return g


def mixer_layer(x, dt, z, Bm, Cm, A, Dskip, dt_bias, conv_w, conv_b, *, aux_init_in=False,
                swap_out=False, pad_left=None, dt_softplus=True, want_state=False,
                round_out=None, threads=1):
    """One SF-Mamba mixer layer on fp64 values.

    x is [B,D,T] when aux_init_in (stage-entry layer), else [B,D,L].  conv_w None
    means x is already the scan input u.  round_out, if given, is applied to the
    gated output before the swap (the layer-boundary dtype of a chain)."""
    xa = aux_init(x) if aux_init_in else _f64(x)
    if conv_w is not None:
        K = np.asarray(conv_w).shape[1] if not hasattr(conv_w, "shape") else conv_w.shape[1]
        u = conv1d(xa, conv_w, conv_b, K=K, pad_left=pad_left, silu=True)
    else:
        u = xa
    res = scan(u, dt, Bm, Cm, A, Dskip, dt_bias, z, dt_softplus, want_state, threads)
    y, fs = res if want_state else (res, None)
    if round_out is not None:
        y = round_out(y)
    if swap_out:
        y = aux_swap(y)
    return (y, fs) if want_state else y


def conv1d_bwd(xa, w, bias, du, pad_left=None, silu=True):
    """Gradients of conv1d(+SiLU) w.r.t. its input, weights and bias, given dLoss/du."""
    xa, w, bias, du = _f64(xa), _f64(w), _f64(bias), _f64(du)
    B, D, L = xa.shape
    K = w.shape[1]
    pad_left = (K - 1) // 2 if pad_left is None else pad_left
    dxa = np.empty_like(xa)
    dw = np.zeros((D, K))
    db = np.zeros(D) if bias is not None else None
    _load().ora_conv1d_bwd(_p(xa), _p(w), _p(bias), _p(du), _p(dxa), _p(dw), _p(db), B, D, L, K, pad_left, int(silu))
    return dxa, dw, db


def aux_init_bwd(dxa):
    """dLoss/dx from dLoss/dxa for xa = [mean(x), x, mean(x)]."""
    dxa = _f64(dxa)
    B, D, L = dxa.shape
    dx = np.empty((B, D, L - 2))
    _load().ora_aux_init_bwd(_p(dxa), _p(dx), B, D, L - 2)
    return dx


def mixer_layer_bwd(x, dt, z, Bm, Cm, A, Dskip, dt_bias, conv_w, conv_b, dout, *, aux_init_in=False,
                    swap_out=False, pad_left=None, dt_softplus=True):
    """Gradients of mixer_layer's output w.r.t. every input and parameter, composed from
    the single-step backwards in reverse order: swap, gate + scan, SiLU + conv, aux init."""
    dout = _f64(dout)
    if swap_out:
        dout = aux_swap(dout)  # the swap is its own inverse
    xa = aux_init(x) if aux_init_in else _f64(x)
    K = conv_w.shape[1]
    u = conv1d(xa, conv_w, conv_b, K=K, pad_left=pad_left, silu=True)
    g = scan_bwd(u, dt, Bm, Cm, A, dout, Dskip, dt_bias, z, dt_softplus)
    dxa, dw, db = conv1d_bwd(xa, conv_w, conv_b, g.pop("du"), pad_left=pad_left, silu=True)
    g["dx"] = aux_init_bwd(dxa) if aux_init_in else dxa
    g["dconv_w"] = dw
    if db is not None:
        g["dconv_b"] = db
    return g


# ---------------------------------------------------------------- ragged (variable-length) folding
#
# S samples of different lengths packed along time: sample s holds packed positions
# [cu[s], cu[s+1]) of dt, z, Bm, Cm (rows [D, Ltot] and [N, Ltot]) and of the output; with
# aux init its T_s = L_s - 2 patch tokens sit at x positions [cu[s] - 2s, cu[s+1] - 2s - 2).
# The fold's reset and boundary-safe conv (techloop.online, Batch Folding with Periodic
# State Reset and the convolution-boundary paragraph; sungsoo.github.io section 3.3) with
# the fixed period replaced by the offsets.

def _x_span(cu, s, aux):
    a, e = int(cu[s]), int(cu[s + 1])
    return (a - 2 * s, e - 2 * s - 2) if aux else (a, e)


def mixer_layer_varlen(x, dt, z, Bm, Cm, A, Dskip, dt_bias, conv_w, conv_b, cu_seqlens, *, aux_init_in=False,
                       swap_out=False, pad_left=None, dt_softplus=True, want_state=False):
    """The ragged layer by its definition: every sample is mixer_layer run on its own slice.

    Positions that belong to no sample stay 0.  Returns y [D, Ltot] (and the final states
    [S, D, N] with want_state)."""
    dt = _f64(dt)
    D, Lt = dt.shape
    cu = [int(v) for v in np.asarray(cu_seqlens).reshape(-1)]
    S = len(cu) - 1
    N = np.asarray(Bm).shape[0]
    y = np.zeros((D, Lt))
    fs = np.zeros((S, D, N))
    xf, zf, Bf, Cf = _f64(x), _f64(z), _f64(Bm), _f64(Cm)
    for s in range(S):
        a, e = cu[s], cu[s + 1]
        if e == a:
            continue
        xa, xe = _x_span(cu, s, aux_init_in)
        res = mixer_layer(xf[None, :, xa:xe], dt[None, :, a:e], None if zf is None else zf[None, :, a:e],
                          Bf[None, :, a:e], Cf[None, :, a:e], A, Dskip, dt_bias, conv_w, conv_b,
                          aux_init_in=aux_init_in, swap_out=swap_out, pad_left=pad_left, dt_softplus=dt_softplus,
                          want_state=want_state)
        if want_state:
            y[:, a:e], fs[s] = res[0][0], res[1][0]
        else:
            y[:, a:e] = res[0]
    return (y, fs) if want_state else y


def mixer_layer_packed_literal(x, dt, z, Bm, Cm, A, Dskip, dt_bias, conv_w, conv_b, cu_seqlens, *,
                               aux_init_in=False, swap_out=False, pad_left=None, dt_softplus=True):
    """The ragged fold read literally, written apart from the C routines: ONE recurrence
    along each packed row with the transition Abar = 0 at every offset cu[s], conv taps
    that read zero wherever they leave the sample of the tap's centre, aux tokens (the
    mean of each sample's own x tokens) placed at every sample's ends, and each sample's
    first and last outputs exchanged.  numpy fp64; small sizes only."""
    dt, xf = _f64(dt), _f64(x)
    D, Lt = dt.shape
    cu = [int(v) for v in np.asarray(cu_seqlens).reshape(-1)]
    S = len(cu) - 1
    owner = np.full(Lt, -1)  # sample of each packed position, -1 for none
    for s in range(S):
        owner[cu[s]:cu[s + 1]] = s
    # the conv input along the packed row (aux tokens filled in)
    xa = np.zeros((D, Lt))
    for s in range(S):
        a, e = cu[s], cu[s + 1]
        if e == a:
            continue
        if aux_init_in:
            xs, xe = a - 2 * s, e - 2 * s - 2
            m = xf[:, xs:xe].sum(axis=1) / (xe - xs)
            xa[:, a], xa[:, e - 1] = m, m
            xa[:, a + 1:e - 1] = xf[:, xs:xe]
        else:
            xa[:, a:e] = xf[:, a:e]
    if conv_w is not None:
        w = _f64(conv_w)
        K = w.shape[1]
        pl = (K - 1) // 2 if pad_left is None else pad_left
        pre = np.zeros((D, Lt)) + (0.0 if conv_b is None else _f64(conv_b)[:, None])
        for p in range(Lt):
            for k in range(K):
                q = p + k - pl
                if 0 <= q < Lt and owner[q] == owner[p] and owner[p] >= 0:
                    pre[:, p] += w[:, k] * xa[:, q]
        u = pre / (1.0 + np.exp(-pre))
    else:
        u = xa
    v = dt + (0.0 if dt_bias is None else _f64(dt_bias)[:, None])
    if dt_softplus:
        delta = np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))
    else:
        delta = v
    Af, Bf, Cf = _f64(A), _f64(Bm), _f64(Cm)
    starts = set(cu[s] for s in range(S) if cu[s + 1] > cu[s])
    h = np.zeros(Af.shape)  # [D, N]
    y = np.zeros((D, Lt))
    for p in range(Lt):
        if owner[p] < 0:
            h[:] = 0.0
            continue
        # the reset is a select, not a multiplication by 0, so nothing of the previous
        # sample (not even inf or nan) enters this one
        carried = np.zeros_like(h) if p in starts else np.exp(delta[:, p:p + 1] * Af) * h
        h = carried + (delta[:, p] * u[:, p])[:, None] * Bf[None, :, p]
        y[:, p] = h @ Cf[:, p]
        if Dskip is not None:
            y[:, p] += _f64(Dskip) * u[:, p]
    if z is not None:
        zf = _f64(z)
        y = y * (zf / (1.0 + np.exp(-zf)))
    if swap_out:
        for s in range(S):
            a, e = cu[s], cu[s + 1]
            if e > a:
                y[:, [a, e - 1]] = y[:, [e - 1, a]]
    return y


# ---------------------------------------------------------------- per-token projections
#
# The dense maps around the scan (the Mamba block's input, state and step-size
# projections; background of sungsoo.github.io, Sources and Evidence Notes, items 4-5):
# P[m, n] = sum_k W[m, k] X[n, k] over tokens n = b*L + t.

def proj(W, X, L, M0=None, token_major=False):
    """P = W X^T in fp64 (numpy matmul), laid out as the projection kernel writes it:
    token-major [Ntok, M], or channel-major ([B, M0, L], [B, M - M0, L]) with rows split
    at M0 (the second part None when M0 == M)."""
    W, X = _f64(W), _f64(X)
    M = W.shape[0]
    Ntok = X.shape[0]
    P = W @ X.T  # [M, Ntok]
    if token_major:
        return P.T.copy()
    M0 = M if M0 is None else M0
    B = Ntok // L
    cm = P.reshape(M, B, L).transpose(1, 0, 2)  # [B, M, L]
    return cm[:, :M0].copy(), (cm[:, M0:].copy() if M0 < M else None)
