"""The C ABI without a GPU: the library loads, exports every entry point the header
declares, validates arguments synchronously (no CUDA call is made on those paths), and
the host-side fault hook forces the CUDA-error path without launching anything."""
import ctypes
import os
import re

import pytest

from selective_scan_sfm_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def header_entry_points():
    src = open(os.path.join(ROOT, "include", "sfm.h")).read()
    return sorted(set(re.findall(r"SFM_API\s+[\w\s\*]*?\b(sfm_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    declared = header_entry_points()
    assert len(declared) >= 15
    assert sorted(_abi.ENTRY_POINTS) == declared
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert L.sfm_abi_version() == 4
    for code in range(6):
        assert _abi.status_string(code).startswith("SFM_")
    assert _abi.status_string(99) == "SFM_ERR_UNKNOWN"


FAKE = 0x7F0000000000  # never dereferenced: validation returns before any CUDA call


def good_args(**kw):
    a = _abi.ScanArgs()
    a.size = ctypes.sizeof(_abi.ScanArgs)
    B, D, L_, N = 4, 16, 51, 8
    ptrs = dict(x=FAKE, dt=FAKE + (1 << 24), z=FAKE + (2 << 24), Bm=FAKE + (3 << 24), Cm=FAKE + (4 << 24),
                A=FAKE + (5 << 24), Dskip=FAKE + (6 << 24), dt_bias=FAKE + (7 << 24), conv_w=FAKE + (8 << 24),
                conv_b=FAKE + (9 << 24), y=FAKE + (10 << 24), final_state=None)
    for k, v in ptrs.items():
        setattr(a, k, v)
    a.B, a.D, a.L, a.N, a.K, a.pad_left, a.B1, a.reset_period = B, D, L_, N, 4, 1, 1, L_
    a.dt_softplus, a.aux_init, a.swap_out = 1, 1, 0
    a.in_dtype = a.out_dtype = _abi.SFM_F32
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def call(L, a):
    return L.sfm_selective_scan_fold(ctypes.byref(a), None)


@pytest.fixture
def inject(monkeypatch):
    monkeypatch.setenv("SFM_FAULT_INJECT", "launch")


def test_valid_args_reach_the_launch_path(L, inject):
    # passing validation (struct size included) is proven by the injected CUDA error
    assert call(L, good_args()) == _abi.SFM_ERR_CUDA
    assert call(L, good_args(B1=0)) == _abi.SFM_ERR_CUDA
    assert call(L, good_args(in_dtype=_abi.SFM_BF16, out_dtype=_abi.SFM_F32)) == _abi.SFM_ERR_CUDA


@pytest.mark.parametrize("field,value,code", [
    ("size", 8, _abi.SFM_ERR_INVALID_ARG),
    ("x", None, _abi.SFM_ERR_INVALID_ARG),
    ("dt", None, _abi.SFM_ERR_INVALID_ARG),
    ("Bm", None, _abi.SFM_ERR_INVALID_ARG),
    ("A", None, _abi.SFM_ERR_INVALID_ARG),
    ("y", None, _abi.SFM_ERR_INVALID_ARG),
    ("B", 0, _abi.SFM_ERR_INVALID_ARG),
    ("D", -1, _abi.SFM_ERR_INVALID_ARG),
    ("N", 0, _abi.SFM_ERR_INVALID_ARG),
    ("N", 65, _abi.SFM_ERR_UNSUPPORTED),
    ("L", 2, _abi.SFM_ERR_INVALID_ARG),          # aux init needs at least one patch token
    ("L", 20000, _abi.SFM_ERR_UNSUPPORTED),
    ("K", 5, _abi.SFM_ERR_INVALID_ARG),
    ("K", 0, _abi.SFM_ERR_INVALID_ARG),
    ("pad_left", 4, _abi.SFM_ERR_INVALID_ARG),
    ("pad_left", -1, _abi.SFM_ERR_INVALID_ARG),
    ("B1", 3, _abi.SFM_ERR_INVALID_ARG),          # does not divide B = 4
    ("B1", -1, _abi.SFM_ERR_INVALID_ARG),
    ("reset_period", 17, _abi.SFM_ERR_UNSUPPORTED),
    ("dt_softplus", 2, _abi.SFM_ERR_INVALID_ARG),
    ("in_dtype", 7, _abi.SFM_ERR_INVALID_ARG),
    ("out_dtype", _abi.SFM_BF16, _abi.SFM_ERR_UNSUPPORTED),  # f32 in, bf16 out
    ("d_tile", 129, _abi.SFM_ERR_UNSUPPORTED),
    ("chunk", 12, _abi.SFM_ERR_UNSUPPORTED),
    ("lanes", 64, _abi.SFM_ERR_UNSUPPORTED),
    ("x", FAKE + 2, _abi.SFM_ERR_MISALIGNED),
    ("y", FAKE + (10 << 24) + 8, _abi.SFM_ERR_MISALIGNED),
    ("y", FAKE + (1 << 24), _abi.SFM_ERR_INVALID_ARG),   # output aliases dt
])
def test_scan_validation(L, inject, field, value, code):
    assert call(L, good_args(**{field: value})) == code


def test_scan_null_args_pointer(L):
    assert L.sfm_selective_scan_fold(None, None) == _abi.SFM_ERR_INVALID_ARG


def test_small_entry_points_validate(L, inject):
    assert L.sfm_aux_init(FAKE, FAKE + (1 << 24), 2, 3, 5, _abi.SFM_BF16, None) == _abi.SFM_ERR_CUDA
    assert L.sfm_aux_init(None, FAKE, 2, 3, 5, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG
    assert L.sfm_aux_init(FAKE, FAKE + 4, 2, 3, 5, _abi.SFM_BF16, None) == _abi.SFM_ERR_MISALIGNED
    assert L.sfm_aux_init(FAKE, FAKE + 16, 2, 3, 5, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG  # overlap
    assert L.sfm_aux_swap(FAKE, 2, 3, 5, _abi.SFM_F32, None) == _abi.SFM_ERR_CUDA
    assert L.sfm_aux_swap(FAKE, 2, 3, 1, _abi.SFM_F32, None) == _abi.SFM_ERR_INVALID_ARG
    conv = L.sfm_fold_conv1d
    assert conv(FAKE, FAKE + (1 << 24), None, FAKE + (2 << 24), 4, 3, 9, 4, 1, 2, 1, _abi.SFM_F32, None) == _abi.SFM_ERR_CUDA
    assert conv(FAKE, FAKE + (1 << 24), None, FAKE + (2 << 24), 4, 3, 9, 4, 1, 3, 1, _abi.SFM_F32, None) == _abi.SFM_ERR_INVALID_ARG
    assert conv(FAKE, FAKE + (1 << 24), None, FAKE + (2 << 24), 4, 3, 9, 4, 4, 1, 1, _abi.SFM_F32, None) == _abi.SFM_ERR_INVALID_ARG
    assert conv(FAKE, None, None, FAKE + (2 << 24), 4, 3, 9, 4, 1, 1, 1, _abi.SFM_F32, None) == _abi.SFM_ERR_INVALID_ARG


def test_chooser_properties(L):
    for B in (1, 2, 3, 4, 7, 16, 64, 128, 256, 1000, 4096):
        for T in (1, 49, 196, 784, 3000):
            for D, N in ((16, 8), (320, 16), (1280, 16)):
                out = ctypes.c_int(-1)
                assert L.sfm_choose_b1(B, T, D, N, ctypes.byref(out)) == _abi.SFM_OK
                assert 1 <= out.value <= B and B % out.value == 0
                v = _abi.Variant()
                assert L.sfm_choose_variant(B, T, D, N, ctypes.byref(v)) == _abi.SFM_OK
                assert v.B1 == out.value and v.lanes >= 1
                assert 1 <= v.d_tile <= 128 and v.chunk % 8 == 0 and v.chunk >= 8
    assert L.sfm_choose_b1(0, 49, 16, 8, ctypes.byref(ctypes.c_int())) == _abi.SFM_ERR_INVALID_ARG
    assert L.sfm_choose_b1(4, 49, 16, 8, None) == _abi.SFM_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        _abi.lib()


def good_grads(**kw):
    g = _abi.ScanGrads()
    g.size = ctypes.sizeof(_abi.ScanGrads)
    base = FAKE + (16 << 24)
    for i, k in enumerate(("dout", "du", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC")):
        setattr(g, k, base + (i << 24))
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def bwd_args(**kw):
    kw.setdefault("conv_w", None)
    kw.setdefault("conv_b", None)
    kw.setdefault("aux_init", 0)
    return good_args(**kw)


def test_backward_workspace_query_and_validation(L, inject):
    need = ctypes.c_size_t(0)
    assert L.sfm_scan_bwd_workspace_size(ctypes.byref(bwd_args()), ctypes.byref(need)) == _abi.SFM_OK
    assert need.value >= 3 * 4 * 16 * 51 * 4
    assert L.sfm_scan_bwd_workspace_size(ctypes.byref(good_args()), ctypes.byref(need)) == _abi.SFM_ERR_UNSUPPORTED
    ws = FAKE + (40 << 24)
    call = lambda a, g, w=ws, n=need.value: L.sfm_selective_scan_fold_bwd(ctypes.byref(a), ctypes.byref(g), w, n, None)
    assert call(bwd_args(), good_grads()) == _abi.SFM_ERR_CUDA           # valid: reaches the launch path
    assert call(bwd_args(), good_grads(), n=need.value - 1) == _abi.SFM_ERR_INVALID_ARG
    assert call(bwd_args(), good_grads(), w=ws + 16) == _abi.SFM_ERR_MISALIGNED
    assert call(bwd_args(), good_grads(), w=None) == _abi.SFM_ERR_INVALID_ARG
    assert call(bwd_args(swap_out=1), good_grads()) == _abi.SFM_ERR_UNSUPPORTED
    assert call(bwd_args(), good_grads(dz=None)) == _abi.SFM_ERR_INVALID_ARG  # z given, dz missing
    assert call(bwd_args(), good_grads(du=FAKE + (1 << 24))) == _abi.SFM_ERR_INVALID_ARG  # du aliases dt
    assert call(bwd_args(), good_grads(size=4)) == _abi.SFM_ERR_INVALID_ARG
    assert call(bwd_args(), good_grads(dA=FAKE + (20 << 24) + 2)) == _abi.SFM_ERR_MISALIGNED


def test_mixer_backward_validation(L, inject):
    need = ctypes.c_size_t(0)
    assert L.sfm_mixer_bwd_workspace_size(ctypes.byref(good_args(swap_out=1)), ctypes.byref(need)) == _abi.SFM_OK
    g = _abi.MixerGrads()
    g.size = ctypes.sizeof(_abi.MixerGrads)
    base = FAKE + (16 << 24)
    for i, k in enumerate(("dout", "dx", "dconv_w", "dconv_b", "ddt", "dz", "dA", "dDskip", "ddt_bias", "dB", "dC")):
        setattr(g, k, base + (i << 24))
    ws = FAKE + (40 << 24)
    call = lambda a, gg, n=need.value: L.sfm_mixer_bwd(ctypes.byref(a), ctypes.byref(gg), ws, n, None)
    assert call(good_args(swap_out=1), g) == _abi.SFM_ERR_CUDA       # valid: reaches the launch path
    assert call(good_args(), g, need.value - 1) == _abi.SFM_ERR_INVALID_ARG
    g.dconv_w = None
    assert call(good_args(), g) == _abi.SFM_ERR_INVALID_ARG          # conv given, no dconv_w
    g.dconv_w = FAKE + (1 << 24)                                      # aliases dt
    assert call(good_args(), g) == _abi.SFM_ERR_INVALID_ARG


# ------------------------------------------------------------------ ragged folding, projections

def varlen_args(**kw):
    # 5 samples packed into 60 positions (>= 3 per sample with aux tokens)
    return good_args(**dict(dict(B=5, L=60, B1=0, reset_period=0), **kw))


CU = FAKE + (11 << 24)


def test_varlen_validation(L, inject):
    v = L.sfm_selective_scan_fold_varlen
    assert v(ctypes.byref(varlen_args()), CU, None) == _abi.SFM_ERR_CUDA
    assert v(ctypes.byref(varlen_args(L=20000)), CU, None) == _abi.SFM_ERR_CUDA  # no per-sample cap on the total
    assert v(ctypes.byref(varlen_args()), None, None) == _abi.SFM_ERR_INVALID_ARG
    assert v(ctypes.byref(varlen_args()), CU + 2, None) == _abi.SFM_ERR_MISALIGNED
    assert v(ctypes.byref(varlen_args(reset_period=60)), CU, None) == _abi.SFM_ERR_UNSUPPORTED
    assert v(ctypes.byref(varlen_args(lanes=2)), CU, None) == _abi.SFM_ERR_UNSUPPORTED
    assert v(ctypes.byref(varlen_args(N=17)), CU, None) == _abi.SFM_ERR_UNSUPPORTED
    assert v(ctypes.byref(varlen_args(L=14)), CU, None) == _abi.SFM_ERR_INVALID_ARG   # < 3 tokens per sample
    assert v(ctypes.byref(varlen_args(B1=2)), CU, None) == _abi.SFM_ERR_INVALID_ARG   # does not divide 5
    assert v(ctypes.byref(varlen_args(y=CU)), CU, None) == _abi.SFM_ERR_INVALID_ARG  # output aliases the offsets


def proj_args(**kw):
    a = _abi.ProjArgs()
    a.size = ctypes.sizeof(_abi.ProjArgs)
    a.W, a.X, a.out0, a.out1 = FAKE, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24)
    a.M, a.K, a.Ntok, a.M0, a.L = 256, 64, 4 * 51, 128, 51
    a.token_major, a.out_dtype, a.tile_n = 0, _abi.SFM_BF16, 0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,code", [
    ("size", 8, _abi.SFM_ERR_INVALID_ARG),
    ("W", None, _abi.SFM_ERR_INVALID_ARG),
    ("out0", None, _abi.SFM_ERR_INVALID_ARG),
    ("K", 60, _abi.SFM_ERR_UNSUPPORTED),            # rows not a multiple of 16 bytes
    ("Ntok", 4 * 51 + 1, _abi.SFM_ERR_INVALID_ARG),  # not whole samples
    ("M0", 300, _abi.SFM_ERR_INVALID_ARG),
    ("out1", None, _abi.SFM_ERR_INVALID_ARG),       # M0 < M needs the second output
    ("token_major", 1, _abi.SFM_ERR_INVALID_ARG),   # token-major writes one output of all M rows
    ("tile_n", 64, _abi.SFM_ERR_UNSUPPORTED),
    ("schedule", 3, _abi.SFM_ERR_INVALID_ARG),
    ("out_dtype", 5, _abi.SFM_ERR_INVALID_ARG),
    ("X", FAKE + (1 << 24) + 8, _abi.SFM_ERR_MISALIGNED),
    ("out0", FAKE + (1 << 24), _abi.SFM_ERR_INVALID_ARG),  # output aliases X
])
def test_proj_validation(L, inject, field, value, code):
    assert L.sfm_proj_gemm(ctypes.byref(proj_args(**{field: value})), None) == code


def test_proj_valid_args_reach_the_launch_path(L, inject):
    assert L.sfm_proj_gemm(ctypes.byref(proj_args()), None) == _abi.SFM_ERR_CUDA
    assert L.sfm_proj_gemm(ctypes.byref(proj_args(token_major=1, M0=256, out1=None)), None) == _abi.SFM_ERR_CUDA
    assert L.sfm_proj_gemm(ctypes.byref(proj_args(M0=256, out1=None, tile_n=256, out_dtype=_abi.SFM_F32)),
                           None) == _abi.SFM_ERR_CUDA
    assert L.sfm_proj_gemm(ctypes.byref(proj_args(schedule=2)), None) == _abi.SFM_ERR_CUDA


def test_conv1d_tokens_validation(L, inject):
    c = L.sfm_conv1d_tokens
    W, U = FAKE + (1 << 24), FAKE + (2 << 24)
    assert c(FAKE, W, None, U, 2, 64, 51, 4, 1, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_CUDA
    assert c(FAKE, W, None, U, 0, 64, 51, 4, 1, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG
    assert c(FAKE, W, None, U, 2, 64, 51, 4, 4, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG
    assert c(FAKE, None, None, U, 2, 64, 51, 4, 1, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG
    assert c(FAKE, W, None, U + 2, 2, 64, 51, 4, 1, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_MISALIGNED
    assert c(FAKE, W, None, FAKE + 16, 2, 64, 51, 4, 1, 1, _abi.SFM_BF16, None) == _abi.SFM_ERR_INVALID_ARG


def test_selftest_wait_validation(L, inject):
    assert L.sfm_selftest_wait_timeout(0, None) == _abi.SFM_ERR_INVALID_ARG
    assert L.sfm_selftest_wait_timeout(2000000, None) == _abi.SFM_ERR_INVALID_ARG
    assert L.sfm_selftest_wait_timeout(100, None) == _abi.SFM_ERR_CUDA  # reached the launch path
