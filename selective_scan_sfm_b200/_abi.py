"""ctypes view of the libsfm C ABI (include/sfm.h).  Marshalling only: no arithmetic.

The shared library is the in-tree ``libsfm.so`` built by ``selective_scan_sfm_b200.build``;
there is no fallback of any kind -- if it is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsfm.so")

SFM_OK, SFM_ERR_INVALID_ARG, SFM_ERR_MISALIGNED, SFM_ERR_UNSUPPORTED, SFM_ERR_CUDA, SFM_ERR_TIMEOUT = range(6)
SFM_F32, SFM_BF16 = 0, 1

#: Every entry point declared in include/sfm.h.
ENTRY_POINTS = (
    "sfm_status_string", "sfm_abi_version", "sfm_last_cuda_error", "sfm_aux_init", "sfm_aux_swap", "sfm_fold_conv1d",
    "sfm_selective_scan_fold", "sfm_scan_bwd_workspace_size", "sfm_selective_scan_fold_bwd",
    "sfm_choose_b1", "sfm_choose_variant", "sfm_get_device_error", "sfm_selective_scan_fold_bwd_noalloc",
    "sfm_mixer_bwd_workspace_size", "sfm_mixer_bwd", "sfm_selective_scan_fold_varlen", "sfm_proj_gemm",
    "sfm_conv1d_tokens", "sfm_selftest_wait_timeout",
)

#: Size of the workspace built into the library for sfm_selective_scan_fold_bwd_noalloc.
NOALLOC_SCRATCH_BYTES = 64 << 20

_vp = ctypes.c_void_p
_i = ctypes.c_int


class ScanArgs(ctypes.Structure):
    """Mirror of sfm_scan_args."""
    _fields_ = [
        ("size", ctypes.c_uint32),
        ("x", _vp), ("dt", _vp), ("z", _vp), ("Bm", _vp), ("Cm", _vp),
        ("A", _vp), ("Dskip", _vp), ("dt_bias", _vp), ("conv_w", _vp), ("conv_b", _vp),
        ("y", _vp), ("final_state", _vp),
        ("B", _i), ("D", _i), ("L", _i), ("N", _i),
        ("K", _i), ("pad_left", _i),
        ("B1", _i), ("reset_period", _i),
        ("dt_softplus", _i), ("aux_init", _i), ("swap_out", _i),
        ("in_dtype", _i), ("out_dtype", _i),
        ("lanes", _i), ("d_tile", _i), ("chunk", _i), ("exp2_split", _i), ("chans_per_thread", _i),
    ]


class ProjArgs(ctypes.Structure):
    """Mirror of sfm_proj_args."""
    _fields_ = [
        ("size", ctypes.c_uint32),
        ("W", _vp), ("X", _vp), ("out0", _vp), ("out1", _vp),
        ("M", _i), ("K", _i), ("Ntok", _i), ("M0", _i), ("L", _i),
        ("token_major", _i), ("out_dtype", _i), ("tile_n", _i), ("schedule", _i),
    ]


class ScanGrads(ctypes.Structure):
    """Mirror of sfm_scan_grads."""
    _fields_ = [
        ("size", ctypes.c_uint32),
        ("dout", _vp), ("du", _vp), ("ddt", _vp), ("dz", _vp), ("dA", _vp),
        ("dDskip", _vp), ("ddt_bias", _vp), ("dB", _vp), ("dC", _vp),
    ]


class MixerGrads(ctypes.Structure):
    """Mirror of sfm_mixer_grads."""
    _fields_ = [
        ("size", ctypes.c_uint32),
        ("dout", _vp), ("dx", _vp), ("dconv_w", _vp), ("dconv_b", _vp), ("ddt", _vp), ("dz", _vp),
        ("dA", _vp), ("dDskip", _vp), ("ddt_bias", _vp), ("dB", _vp), ("dC", _vp),
    ]


class Variant(ctypes.Structure):
    """Mirror of sfm_variant."""
    _fields_ = [("B1", _i), ("lanes", _i), ("d_tile", _i), ("chunk", _i), ("exp2_pairs", _i),
                ("chans_per_thread", _i)]


_lib = None


def lib():
    """The loaded libsfm (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libsfm.so is not built (python -m selective_scan_sfm_b200.build); "
                               "there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        L.sfm_status_string.restype = ctypes.c_char_p
        L.sfm_status_string.argtypes = [_i]
        L.sfm_abi_version.restype = _i
        L.sfm_abi_version.argtypes = []
        L.sfm_last_cuda_error.restype = ctypes.c_char_p
        L.sfm_last_cuda_error.argtypes = []
        L.sfm_aux_init.argtypes = [_vp, _vp, _i, _i, _i, _i, _vp]
        L.sfm_aux_swap.argtypes = [_vp, _i, _i, _i, _i, _vp]
        L.sfm_fold_conv1d.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp]
        L.sfm_selective_scan_fold.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.sfm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ctypes.c_size_t)]
        L.sfm_selective_scan_fold_bwd.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanGrads), _vp,
                                                  ctypes.c_size_t, _vp]
        L.sfm_choose_b1.argtypes = [_i, _i, _i, _i, ctypes.POINTER(_i)]
        L.sfm_choose_variant.argtypes = [_i, _i, _i, _i, ctypes.POINTER(Variant)]
        L.sfm_get_device_error.argtypes = [_vp, _i, ctypes.POINTER(_i)]
        L.sfm_selective_scan_fold_bwd_noalloc.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanGrads), _vp]
        L.sfm_selective_scan_fold_varlen.argtypes = [ctypes.POINTER(ScanArgs), _vp, _vp]
        L.sfm_proj_gemm.argtypes = [ctypes.POINTER(ProjArgs), _vp]
        L.sfm_conv1d_tokens.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        L.sfm_selftest_wait_timeout.argtypes = [_i, _vp]
        L.sfm_mixer_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ctypes.c_size_t)]
        L.sfm_mixer_bwd.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(MixerGrads), _vp, ctypes.c_size_t, _vp]
        for name in ENTRY_POINTS:
            if name not in ("sfm_status_string", "sfm_abi_version", "sfm_last_cuda_error"):
                getattr(L, name).restype = _i
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().sfm_status_string(int(code)).decode()


class SfmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        msg = "%s: %s" % (where, status_string(code))
        if self.code == SFM_ERR_CUDA:
            msg += " (%s)" % lib().sfm_last_cuda_error().decode()
        super().__init__(msg)


def check(code: int, where: str) -> None:
    if code != SFM_OK:
        raise SfmError(code, where)
