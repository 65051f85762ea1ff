"""selective_scan_sfm_b200 -- the batch-folded selective scan of SF-Mamba on B200.

A thin PyTorch-facing binding over the C ABI in include/sfm.h (libsfm.so, hand-written
sm_100a CUDA).  Every function here only checks and marshals arguments: all steps of
the path run inside the library's kernels; PyTorch provides device memory and streams.
Names follow the C entry points.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import SFM_BF16, SFM_F32, SfmError

__all__ = [
    "sfm_aux_init", "sfm_aux_swap", "sfm_fold_conv1d", "sfm_selective_scan_fold", "sfm_selective_scan_fold_varlen",
    "sfm_selective_scan_fold_bwd", "sfm_selective_scan_fold_bwd_noalloc", "sfm_mixer_bwd", "sfm_choose_b1", "sfm_choose_variant", "sfm_get_device_error",
    "sfm_proj_gemm", "sfm_conv1d_tokens", "SfmError", "library_path",
]

_DT = {torch.float32: SFM_F32, torch.bfloat16: SFM_BF16}


def library_path() -> str:
    return _abi.LIB_PATH


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype=None, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError("%s is required" % name)
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _code(dtype) -> int:
    if dtype not in _DT:
        raise ValueError("unsupported dtype %s (float32 or bfloat16)" % dtype)
    return _DT[dtype]


def sfm_aux_init(x, xa=None, stream=None):
    """x [B,D,T] -> xa [B,D,T+2] with head = tail = mean over the T tokens."""
    _dev(x, "x")
    B, D, T = x.shape
    if xa is None:
        xa = torch.empty(B, D, T + 2, dtype=x.dtype, device=x.device)
    _dev(xa, "xa", x.dtype, (B, D, T + 2))
    _abi.check(_abi.lib().sfm_aux_init(_ptr(x), _ptr(xa), B, D, T, _code(x.dtype), _stream(stream)), "sfm_aux_init")
    return xa


def sfm_aux_swap(y, stream=None):
    """In place: y[..., 0] <-> y[..., L-1]."""
    _dev(y, "y")
    B, D, L = y.shape
    _abi.check(_abi.lib().sfm_aux_swap(_ptr(y), B, D, L, _code(y.dtype), _stream(stream)), "sfm_aux_swap")
    return y


def sfm_fold_conv1d(x, w, bias=None, u=None, pad_left=None, B2=1, silu=False, stream=None):
    """Depthwise conv1d with zero padding per sample; x, u [B,D,L]; w [D,K] fp32."""
    _dev(x, "x")
    B, D, L = x.shape
    _dev(w, "w", torch.float32)
    K = w.shape[1]
    _dev(w, "w", torch.float32, (D, K))
    _dev(bias, "bias", torch.float32, (D,), optional=True)
    if u is None:
        u = torch.empty_like(x)
    _dev(u, "u", x.dtype, (B, D, L))
    pl = (K - 1) // 2 if pad_left is None else int(pad_left)
    _abi.check(_abi.lib().sfm_fold_conv1d(_ptr(x), _ptr(w), _ptr(bias), _ptr(u), B, D, L, K, pl, int(B2),
                                          int(bool(silu)), _code(x.dtype), _stream(stream)), "sfm_fold_conv1d")
    return u


def _scan_args(x, dt, Bm, Cm, A, z, Dskip, dt_bias, conv_w, conv_b, y, final_state, B1, pad_left, dt_softplus,
               aux_init, swap_out, out_dtype, lanes, d_tile, chunk, need_y=True, exp2_split=0, chans_per_thread=0):
    _dev(dt, "dt")
    B, D, L = dt.shape
    io = dt.dtype
    T = L - 2 if aux_init else L
    _dev(x, "x", io, (B, D, T))
    N = Bm.shape[1] if isinstance(Bm, torch.Tensor) and Bm.dim() == 3 else -1
    _dev(Bm, "Bm", io, (B, N, L))
    _dev(Cm, "Cm", io, (B, N, L))
    _dev(z, "z", io, (B, D, L), optional=True)
    _dev(A, "A", torch.float32, (D, N))
    _dev(Dskip, "Dskip", torch.float32, (D,), optional=True)
    _dev(dt_bias, "dt_bias", torch.float32, (D,), optional=True)
    K = 0
    if conv_w is not None:
        _dev(conv_w, "conv_w", torch.float32)
        K = conv_w.shape[1]
        _dev(conv_w, "conv_w", torch.float32, (D, K))
    _dev(conv_b, "conv_b", torch.float32, (D,), optional=True)
    od = io if out_dtype is None else out_dtype
    if need_y:
        if y is None:
            y = torch.empty(B, D, L, dtype=od, device=dt.device)
        _dev(y, "y", od, (B, D, L))
    _dev(final_state, "final_state", torch.float32, (B, D, N), optional=True)
    a = _abi.ScanArgs()
    a.size = ctypes.sizeof(_abi.ScanArgs)
    a.x, a.dt, a.z, a.Bm, a.Cm = (t.data_ptr() if t is not None else None for t in (x, dt, z, Bm, Cm))
    a.A, a.Dskip, a.dt_bias, a.conv_w, a.conv_b = (t.data_ptr() if t is not None else None
                                                   for t in (A, Dskip, dt_bias, conv_w, conv_b))
    a.y = y.data_ptr() if y is not None else None
    a.final_state = final_state.data_ptr() if final_state is not None else None
    a.B, a.D, a.L, a.N = B, D, L, N
    a.K = K
    a.pad_left = ((K - 1) // 2 if pad_left is None else int(pad_left)) if K else 0
    a.B1 = int(B1)
    a.reset_period = L
    a.dt_softplus, a.aux_init, a.swap_out = int(bool(dt_softplus)), int(bool(aux_init)), int(bool(swap_out))
    a.in_dtype, a.out_dtype = _code(io), _code(od)
    a.lanes, a.d_tile, a.chunk, a.exp2_split = int(lanes), int(d_tile), int(chunk), int(exp2_split)
    a.chans_per_thread = int(chans_per_thread)
    return a, y


def sfm_selective_scan_fold(x, dt, Bm, Cm, A, *, z=None, Dskip=None, dt_bias=None, conv_w=None, conv_b=None,
                            y=None, final_state=None, B1=0, pad_left=None, dt_softplus=True, aux_init=False,
                            swap_out=False, out_dtype=None, lanes=0, d_tile=0, chunk=0, exp2_split=0,
                            chans_per_thread=0, stream=None):
    """Fused forward: [aux init] -> conv+SiLU -> folded scan with reset -> D skip ->
    SiLU(z) gate -> [aux swap].  Returns y [B,D,L].  B1, lanes, d_tile, chunk, exp2_split,
    chans_per_thread: launch-shape overrides (0 = the look-up table's choice)."""
    a, y = _scan_args(x, dt, Bm, Cm, A, z, Dskip, dt_bias, conv_w, conv_b, y, final_state, B1, pad_left,
                      dt_softplus, aux_init, swap_out, out_dtype, lanes, d_tile, chunk, exp2_split=exp2_split,
                      chans_per_thread=chans_per_thread)
    _abi.check(_abi.lib().sfm_selective_scan_fold(ctypes.byref(a), _stream(stream)), "sfm_selective_scan_fold")
    return y


def _varlen_args(x, dt, Bm, Cm, A, cu_seqlens, z, Dskip, dt_bias, conv_w, conv_b, y, final_state, B1, pad_left,
                 dt_softplus, aux_init, swap_out, out_dtype, d_tile=0, chunk=0, exp2_split=0, chans_per_thread=0):
    _dev(dt, "dt")
    if dt.dim() != 2:
        raise ValueError("dt must be [D, Ltot] (packed), got %s" % (tuple(dt.shape),))
    D, Lt = dt.shape
    io = dt.dtype
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be [S+1] with S >= 1")
    S = cu_seqlens.numel() - 1
    _dev(x, "x", io, (D, Lt - 2 * S if aux_init else Lt))
    N = Bm.shape[0] if isinstance(Bm, torch.Tensor) and Bm.dim() == 2 else -1
    _dev(Bm, "Bm", io, (N, Lt))
    _dev(Cm, "Cm", io, (N, Lt))
    _dev(z, "z", io, (D, Lt), optional=True)
    _dev(A, "A", torch.float32, (D, N))
    _dev(Dskip, "Dskip", torch.float32, (D,), optional=True)
    _dev(dt_bias, "dt_bias", torch.float32, (D,), optional=True)
    K = 0
    if conv_w is not None:
        _dev(conv_w, "conv_w", torch.float32)
        K = conv_w.shape[1]
        _dev(conv_w, "conv_w", torch.float32, (D, K))
    _dev(conv_b, "conv_b", torch.float32, (D,), optional=True)
    od = io if out_dtype is None else out_dtype
    if y is None:
        y = torch.empty(D, Lt, dtype=od, device=dt.device)
    _dev(y, "y", od, (D, Lt))
    _dev(final_state, "final_state", torch.float32, (S, D, N), optional=True)
    a = _abi.ScanArgs()
    a.size = ctypes.sizeof(_abi.ScanArgs)
    a.x, a.dt, a.z, a.Bm, a.Cm = (t.data_ptr() if t is not None else None for t in (x, dt, z, Bm, Cm))
    a.A, a.Dskip, a.dt_bias, a.conv_w, a.conv_b = (t.data_ptr() if t is not None else None
                                                   for t in (A, Dskip, dt_bias, conv_w, conv_b))
    a.y = y.data_ptr()
    a.final_state = final_state.data_ptr() if final_state is not None else None
    a.B, a.D, a.L, a.N = S, D, Lt, N
    a.K = K
    a.pad_left = ((K - 1) // 2 if pad_left is None else int(pad_left)) if K else 0
    a.B1 = int(B1)
    a.reset_period = 0
    a.dt_softplus, a.aux_init, a.swap_out = int(bool(dt_softplus)), int(bool(aux_init)), int(bool(swap_out))
    a.in_dtype, a.out_dtype = _code(io), _code(od)
    a.lanes, a.d_tile, a.chunk, a.exp2_split = 0, int(d_tile), int(chunk), int(exp2_split)
    a.chans_per_thread = int(chans_per_thread)
    return a, y


def sfm_selective_scan_fold_varlen(x, dt, Bm, Cm, A, cu_seqlens, *, z=None, Dskip=None, dt_bias=None, conv_w=None,
                                   conv_b=None, y=None, final_state=None, B1=0, pad_left=None, dt_softplus=True,
                                   aux_init=False, swap_out=False, out_dtype=None, d_tile=0, chunk=0, exp2_split=0,
                                   chans_per_thread=0, stream=None):
    """Ragged fused forward: S samples of different lengths packed along time, the state
    reset at every offset of cu_seqlens (int32 [S+1] on the device).  dt, z: [D, Ltot];
    Bm, Cm: [N, Ltot]; x: [D, Ltot - 2S] with aux_init, else [D, Ltot]; final_state
    [S, D, N].  Returns y [D, Ltot].  Offsets are checked on the device (see
    sfm_get_device_error)."""
    a, y = _varlen_args(x, dt, Bm, Cm, A, cu_seqlens, z, Dskip, dt_bias, conv_w, conv_b, y, final_state, B1, pad_left,
                        dt_softplus, aux_init, swap_out, out_dtype, d_tile, chunk, exp2_split, chans_per_thread)
    _abi.check(_abi.lib().sfm_selective_scan_fold_varlen(ctypes.byref(a), ctypes.c_void_p(cu_seqlens.data_ptr()),
                                                         _stream(stream)), "sfm_selective_scan_fold_varlen")
    return y


def sfm_conv1d_tokens(x, w, bias=None, *, pad_left=None, silu=True, u=None, stream=None):
    """Boundary-safe depthwise conv (+SiLU) of x [B,D,L], written token-major u [B*L, D]."""
    _dev(x, "x")
    B, D, L = x.shape
    K = w.shape[1]
    _dev(w, "w", torch.float32, (D, K))
    _dev(bias, "bias", torch.float32, (D,), optional=True)
    if u is None:
        u = torch.empty(B * L, D, dtype=x.dtype, device=x.device)
    _dev(u, "u", x.dtype, (B * L, D))
    pl = (K - 1) // 2 if pad_left is None else int(pad_left)
    _abi.check(_abi.lib().sfm_conv1d_tokens(_ptr(x), _ptr(w), _ptr(bias), _ptr(u), B, D, L, K, pl, int(bool(silu)),
                                            _code(x.dtype), _stream(stream)), "sfm_conv1d_tokens")
    return u


def _proj_args(W, X, L, M0, token_major, out_dtype, out0, out1, tile_n, schedule=0):
    _dev(W, "W", torch.bfloat16)
    _dev(X, "X", torch.bfloat16)
    if W.dim() != 2 or X.dim() != 2 or W.shape[1] != X.shape[1]:
        raise ValueError("W must be [M, K] and X [Ntok, K], got %s and %s" % (tuple(W.shape), tuple(X.shape)))
    M, K = W.shape
    Ntok = X.shape[0]
    if L < 1 or Ntok % L:
        raise ValueError("Ntok = %d is not a multiple of L = %d" % (Ntok, L))
    B = Ntok // L
    M0 = M if (M0 is None or token_major) else int(M0)
    od = torch.bfloat16 if out_dtype is None else out_dtype
    if token_major:
        if out0 is None:
            out0 = torch.empty(Ntok, M, dtype=od, device=X.device)
        _dev(out0, "out0", od, (Ntok, M))
        out1 = None
    else:
        if out0 is None:
            out0 = torch.empty(B, M0, L, dtype=od, device=X.device)
        _dev(out0, "out0", od, (B, M0, L))
        if M0 < M:
            if out1 is None:
                out1 = torch.empty(B, M - M0, L, dtype=od, device=X.device)
            _dev(out1, "out1", od, (B, M - M0, L))
        else:
            out1 = None
    a = _abi.ProjArgs()
    a.size = ctypes.sizeof(_abi.ProjArgs)
    a.W, a.X = W.data_ptr(), X.data_ptr()
    a.out0 = out0.data_ptr()
    a.out1 = out1.data_ptr() if out1 is not None else None
    a.M, a.K, a.Ntok, a.M0, a.L = M, K, Ntok, M0, int(L)
    a.token_major, a.out_dtype, a.tile_n = int(bool(token_major)), _code(od), int(tile_n)
    a.schedule = int(schedule)
    return a, out0, out1


def sfm_proj_gemm(W, X, L, *, M0=None, token_major=False, out_dtype=None, out0=None, out1=None, tile_n=0,
                  schedule=0, stream=None):
    """P[m, n] = sum_k W[m, k] X[n, k] on the tensor cores (bf16 in, fp32 accumulation).
    W: [M, K] bf16; X: [Ntok, K] bf16 (tokens sample-major, L per sample).  Channel-major
    (default): returns (out0 [B, M0, L], out1 [B, M-M0, L] or None); token-major: returns
    (out0 [Ntok, M], None)."""
    a, out0, out1 = _proj_args(W, X, L, M0, token_major, out_dtype, out0, out1, tile_n, schedule)
    _abi.check(_abi.lib().sfm_proj_gemm(ctypes.byref(a), _stream(stream)), "sfm_proj_gemm")
    return out0, out1


def sfm_selective_scan_fold_bwd(u, dt, Bm, Cm, A, dout, *, z=None, Dskip=None, dt_bias=None, B1=0,
                                dt_softplus=True, workspace=None, grads=None, stream=None):
    """Backward of the gated scan (input u, no conv).  Returns a dict of fp32 grads."""
    a, _ = _scan_args(u, dt, Bm, Cm, A, z, Dskip, dt_bias, None, None, None, None, B1, None, dt_softplus,
                      False, False, None, 0, 0, 0, need_y=False)
    B, D, L, N = a.B, a.D, a.L, a.N
    _dev(dout, "dout", dt.dtype, (B, D, L))
    dev = dt.device
    f32 = torch.float32
    if grads is None:
        grads = dict(du=torch.empty(B, D, L, dtype=f32, device=dev), ddt=torch.empty(B, D, L, dtype=f32, device=dev),
                     dA=torch.empty(D, N, dtype=f32, device=dev), dB=torch.empty(B, N, L, dtype=f32, device=dev),
                     dC=torch.empty(B, N, L, dtype=f32, device=dev))
        if z is not None:
            grads["dz"] = torch.empty(B, D, L, dtype=f32, device=dev)
        if Dskip is not None:
            grads["dDskip"] = torch.empty(D, dtype=f32, device=dev)
        if dt_bias is not None:
            grads["ddt_bias"] = torch.empty(D, dtype=f32, device=dev)
    g = _abi.ScanGrads()
    g.size = ctypes.sizeof(_abi.ScanGrads)
    g.dout = dout.data_ptr()
    for k in ("du", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC"):
        t = grads.get(k)
        setattr(g, k, None if t is None else _dev(t, k, f32).data_ptr())
    need = ctypes.c_size_t(0)
    _abi.check(_abi.lib().sfm_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(need)),
               "sfm_scan_bwd_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(int(need.value), 1), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8)
    _abi.check(_abi.lib().sfm_selective_scan_fold_bwd(ctypes.byref(a), ctypes.byref(g),
                                                      ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                                      _stream(stream)), "sfm_selective_scan_fold_bwd")
    return grads


def sfm_selective_scan_fold_bwd_noalloc(u, dt, Bm, Cm, A, dout, grads, *, z=None, Dskip=None, dt_bias=None,
                                        dt_softplus=True, stream=None):
    """The scan backward with the workspace built into the library, for callers that
    cannot allocate device memory (see include/sfm.h).  `grads` is a dict of
    caller-allocated fp32 tensors (du, ddt, dA, dB, dC, and dz / dDskip / ddt_bias when
    z / Dskip / dt_bias are given); it is filled in and returned."""
    a, _ = _scan_args(u, dt, Bm, Cm, A, z, Dskip, dt_bias, None, None, None, None, 0, None, dt_softplus,
                      False, False, None, 0, 0, 0, need_y=False)
    _dev(dout, "dout", dt.dtype, (a.B, a.D, a.L))
    g = _abi.ScanGrads()
    g.size = ctypes.sizeof(_abi.ScanGrads)
    g.dout = dout.data_ptr()
    for k in ("du", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC"):
        t = grads.get(k)
        setattr(g, k, None if t is None else _dev(t, k, torch.float32).data_ptr())
    _abi.check(_abi.lib().sfm_selective_scan_fold_bwd_noalloc(ctypes.byref(a), ctypes.byref(g), _stream(stream)),
               "sfm_selective_scan_fold_bwd_noalloc")
    return grads


def _mixer_bwd_args(x, dt, Bm, Cm, A, dout, z, Dskip, dt_bias, conv_w, conv_b, pad_left, dt_softplus, aux_init,
                    swap_out, workspace):
    a, _ = _scan_args(x, dt, Bm, Cm, A, z, Dskip, dt_bias, conv_w, conv_b, None, None, 0, pad_left, dt_softplus,
                      aux_init, swap_out, None, 0, 0, 0, need_y=False)
    B, D, L, N = a.B, a.D, a.L, a.N
    _dev(dout, "dout", dt.dtype, (B, D, L))
    dev, f32 = dt.device, torch.float32
    e = lambda *shape: torch.empty(*shape, dtype=f32, device=dev)
    grads = dict(dx=e(*x.shape), ddt=e(B, D, L), dA=e(D, N), dB=e(B, N, L), dC=e(B, N, L))
    if conv_w is not None:
        grads["dconv_w"] = e(*conv_w.shape)
        if conv_b is not None:
            grads["dconv_b"] = e(D)
    if z is not None:
        grads["dz"] = e(B, D, L)
    if Dskip is not None:
        grads["dDskip"] = e(D)
    if dt_bias is not None:
        grads["ddt_bias"] = e(D)
    g = _abi.MixerGrads()
    g.size = ctypes.sizeof(_abi.MixerGrads)
    g.dout = dout.data_ptr()
    for k in ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC"):
        t = grads.get(k)
        setattr(g, k, None if t is None else t.data_ptr())
    need = ctypes.c_size_t(0)
    _abi.check(_abi.lib().sfm_mixer_bwd_workspace_size(ctypes.byref(a), ctypes.byref(need)),
               "sfm_mixer_bwd_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(int(need.value), 1), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8)
    return a, g, grads, workspace


def sfm_mixer_bwd(x, dt, Bm, Cm, A, dout, *, z=None, Dskip=None, dt_bias=None, conv_w=None, conv_b=None,
                  pad_left=None, dt_softplus=True, aux_init=False, swap_out=False, workspace=None, stream=None):
    """Backward of the whole fused layer (same arguments as sfm_selective_scan_fold).
    dout is the gradient of the stored output (after the swap).  Returns fp32 grads:
    dx, dconv_w, dconv_b, ddt, dz, dA, dDskip, ddt_bias, dB, dC (those that apply)."""
    a, g, grads, workspace = _mixer_bwd_args(x, dt, Bm, Cm, A, dout, z, Dskip, dt_bias, conv_w, conv_b, pad_left,
                                             dt_softplus, aux_init, swap_out, workspace)
    _abi.check(_abi.lib().sfm_mixer_bwd(ctypes.byref(a), ctypes.byref(g), ctypes.c_void_p(workspace.data_ptr()),
                                        workspace.numel(), _stream(stream)), "sfm_mixer_bwd")
    return grads


def sfm_choose_variant(B: int, T: int, D: int, N: int) -> dict:
    v = _abi.Variant()
    _abi.check(_abi.lib().sfm_choose_variant(int(B), int(T), int(D), int(N), ctypes.byref(v)), "sfm_choose_variant")
    return dict(B1=v.B1, lanes=v.lanes, d_tile=v.d_tile, chunk=v.chunk, exp2_pairs=v.exp2_pairs,
                chans_per_thread=v.chans_per_thread)


def sfm_choose_b1(B: int, T: int, D: int, N: int) -> int:
    out = ctypes.c_int(0)
    _abi.check(_abi.lib().sfm_choose_b1(int(B), int(T), int(D), int(N), ctypes.byref(out)), "sfm_choose_b1")
    return out.value


def sfm_get_device_error(clear: bool = True, stream=None) -> int:
    code = ctypes.c_int(0)
    _abi.check(_abi.lib().sfm_get_device_error(_stream(stream), int(bool(clear)), ctypes.byref(code)),
               "sfm_get_device_error")
    return code.value
