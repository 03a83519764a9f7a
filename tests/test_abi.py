"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument checks reject bad calls before any device work (CPU only)."""

import ctypes
import os
import re

import pytest

import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import build as dgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dgb200.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"DG_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    dgbuild.build()
    return ctypes.CDLL(dgbuild.LIB)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("fp8_gemm_nt", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked",
              "pack_ue8m0", "pack_ue8m0_validate", "dgb200_init", "dgb200_last_device_error",
              "dgb200_device_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.dgb200_status_string.restype = ctypes.c_char_p
    assert lib.dgb200_status_string(0) == b"DG_OK"
    assert lib.dgb200_status_string(1) == b"DG_ERR_INVALID_ARG"
    assert lib.dgb200_status_string(5) == b"DG_ERR_CUDA"


def test_host_argument_checks_fail_before_device_work(lib):
    vp = ctypes.c_void_p
    f = lib.fp8_gemm_nt
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    good = vp(0x10000)
    assert f(None, good, good, good, good, 128, 128, 128, None) == 1          # null pointer
    assert f(good, good, good, good, good, 128, 128, 100, None) == 1          # K % 128
    assert f(good, good, good, good, good, 128, 12, 128, None) == 1           # N % 8
    assert f(good, good, good, good, good, 0, 128, 128, None) == 1            # M <= 0
    assert f(vp(0x10004), good, good, good, good, 128, 128, 128, None) == 2   # A alignment
    m = lib.m_grouped_fp8_gemm_nt_masked
    m.restype = ctypes.c_int
    m.argtypes = [vp] * 6 + [ctypes.c_int] * 4 + [vp]
    assert m(good, good, good, good, good, None, 4, 64, 128, 128, None) == 1  # null masked_m
    assert m(good, good, good, good, good, good, 2048, 64, 128, 128, None) == 3  # too many groups
    p = lib.pack_ue8m0
    p.restype = ctypes.c_int
    p.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int, vp]
    assert p(None, good, 4, 4, None) == 1
    assert p(good, good, 0, 4, None) == 1
    assert p(vp(0x10002), good, 4, 4, None) == 2


def test_sfb_granularity_is_checked_on_the_host(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    good = vp(0x10000)
    f = lib.fp8_gemm_nt_sfb_gran
    f.restype = i
    f.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, i, vp]
    for gran in (0, 2, 64, 127, 256, -1):
        assert f(good, good, good, good, gran, None, good, 128, 128, 128, 0, None) == 1, gran
    assert f(good, good, good, good, 1, None, good, 128, 128, 100, 0, None) == 1      # K % 128
    assert f(good, good, good, good, 1, None, good, 128, 128, 128, 2, None) == 1      # out_f32 not 0 / 1
    c = lib.m_grouped_fp8_gemm_nt_contiguous_sfb_gran
    c.restype = i
    c.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, i, vp]
    assert c(good, good, good, good, 64, good, good, 128, 128, 128, 2, None) == 1
    assert c(good, good, good, good, 1, good, None, 128, 128, 128, 2, None) == 1      # null m_indices
    m = lib.m_grouped_fp8_gemm_nt_masked_sfb_gran
    m.restype = i
    m.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, i, vp]
    assert m(good, good, good, good, 3, good, good, 4, 64, 128, 128, None) == 1
    assert m(good, good, good, good, 1, good, good, 2048, 64, 128, 128, None) == 3    # too many groups
    ps = lib.m_grouped_fp8_gemm_nt_psum
    ps.restype = i
    ps.argtypes = [vp] * 6 + [i] * 4 + [vp]
    assert ps(good, good, good, good, good, None, 128, 128, 128, 2, None) == 1       # null psum_m
    assert ps(good, good, good, good, good, good, 0, 128, 128, 2, None) == 1         # M_total <= 0
    assert ps(good, good, good, good, good, good, 128, 128, 128, 0, None) == 1       # G <= 0
    assert ps(good, good, good, good, good, good, 128, 128, 128, 2048, None) == 3    # too many groups
    assert ps(good, good, good, good, good, vp(0x10002), 128, 128, 128, 2, None) == 2  # psum_m alignment
    import torch
    x = torch.zeros((128, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):  # the binding checks the scale-row count for the granularity
        dg.fp8_gemm_nt_sfb_gran(x, torch.zeros((128, 1), dtype=torch.int32), x,
                                torch.zeros((1, 1), dtype=torch.int32), torch.zeros((128, 128), dtype=torch.bfloat16), 1)


def test_binding_fails_loudly_without_cuda():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    a = torch.zeros((128, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        dg.fp8_gemm_nt(a, torch.zeros((128, 1), dtype=torch.int32), a,
                       torch.zeros((1, 1), dtype=torch.int32), torch.zeros((128, 128), dtype=torch.bfloat16))


def test_init_and_error_word_arguments(lib):
    """dgb200_init takes a device ordinal and dgb200_last_device_error an output
    pointer; bad arguments are refused on the host (no device needed)."""
    lib.dgb200_init.restype = ctypes.c_int
    lib.dgb200_init.argtypes = [ctypes.c_int]
    assert lib.dgb200_init(-1) in (1, 4)          # invalid ordinal (or no usable driver here)
    lib.dgb200_last_device_error.restype = ctypes.c_int
    lib.dgb200_last_device_error.argtypes = [ctypes.c_void_p]
    assert lib.dgb200_last_device_error(None) == 1


def test_tuning_switch_ranges(lib):
    """The process-wide tuning switches reject values outside their ranges and
    need no device to do so (0 restores the heuristic in each)."""
    for name, good, bad in (("dgb200_set_block_n", (0, 64, 224, 256), (-1, 100, 512)),
                            ("dgb200_set_cta_group", (0, 1, 2), (-1, 3)),
                            ("dgb200_set_splits", (0, 1, 2, 8), (-1, 9, 17))):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_int]
        for v in good:
            assert f(v) == 0, (name, v)
        for v in bad:
            assert f(v) == 3, (name, v)   # DG_ERR_UNSUPPORTED
        assert f(0) == 0
