"""FP8 block-scaled GEMMs (dense, contiguous and masked M-grouped) and the UE8M0
pack for B200, as a thin Python binding over libdgb200.so.

Every function here only checks shapes/dtypes/devices on the host and passes
raw pointers to the C ABI declared in ``include/dgb200.h``; all arithmetic runs
in the library's CUDA kernels. There is no fallback: if the shared library is
missing or cannot run on the current device, calls raise.

Tensors are torch tensors used as device memory; work is queued on torch's
current CUDA stream. No call synchronises or allocates (except the
convenience allocations of ``pack_ue8m0`` / ``empty_*`` when no output is
given), so the calls of the method can be captured in a CUDA Graph (no claim
is made for ``fp8_gemm_nt_noalloc``).
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "BLOCK", "lib_path", "load", "init", "device_error", "last_device_error", "set_block_n", "block_n_supported",
    "fp8_gemm_nt", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked",
    "pack_ue8m0", "pack_ue8m0_validate", "DgError", "set_test_hooks", "set_cta_group", "set_splits",
    "fp8_gemm_nt_noalloc", "m_grouped_bf16_gemm_nt_masked", "fp8_gemm_nt_acc", "quantize_fp8_1x128",
    "fp8_gemm_nn", "fp8_gemm_tn", "fp8_gemm_tt",
    "fp8_gemm_nt_sfb_gran", "m_grouped_fp8_gemm_nt_contiguous_sfb_gran", "m_grouped_fp8_gemm_nt_masked_sfb_gran",
    "m_grouped_fp8_gemm_nt_psum",
    "DEVERR_TIMEOUT", "DEVERR_MIXED_EXPERT_BLOCK",
]

BLOCK = 128
DEVERR_TIMEOUT = 1
DEVERR_MIXED_EXPERT_BLOCK = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libdgb200.so"
_lib = None
_lock = threading.Lock()

_STATUS = {
    0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_ALIGNMENT", 3: "DG_ERR_UNSUPPORTED",
    4: "DG_ERR_NOT_INITIALIZED", 5: "DG_ERR_CUDA", 6: "DG_ERR_SCRATCH_TOO_SMALL",
}


class DgError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")


def lib_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load():
    """Load libdgb200.so (built in-tree) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m moe_grouped_gemm_tcgen05_b200.build`")
        L = ctypes.CDLL(path)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.dgb200_status_string.restype = ctypes.c_char_p
        L.dgb200_status_string.argtypes = [i32]
        L.dgb200_init.restype = i32
        L.dgb200_init.argtypes = [i32]
        L.dgb200_last_device_error.restype = i32
        L.dgb200_last_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.dgb200_device_error.restype = i32
        L.dgb200_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        L.dgb200_set_block_n.restype = i32
        L.dgb200_set_block_n.argtypes = [i32]
        L.dgb200_block_n_supported.restype = i32
        L.dgb200_block_n_supported.argtypes = [i32]
        L.dgb200_set_cta_group.restype = i32
        L.dgb200_set_cta_group.argtypes = [i32]
        L.dgb200_set_splits.restype = i32
        L.dgb200_set_splits.argtypes = [i32]
        L.dgb200_set_test_hooks.restype = i32
        L.dgb200_set_test_hooks.argtypes = [i32, i32]
        L.fp8_gemm_nt.restype = i32
        L.fp8_gemm_nt.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp]
        L.m_grouped_bf16_gemm_nt_masked.restype = i32
        L.m_grouped_bf16_gemm_nt_masked.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.quantize_fp8_1x128.restype = i32
        L.quantize_fp8_1x128.argtypes = [vp, i32, vp, vp, vp, ctypes.c_int64, i32, vp]
        for name in ("fp8_gemm_nn", "fp8_gemm_tn", "fp8_gemm_tt"):
            getattr(L, name).restype = i32
            getattr(L, name).argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp]
        L.fp8_gemm_nt_acc.restype = i32
        L.fp8_gemm_nt_acc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.fp8_gemm_nt_noalloc.restype = i32
        L.fp8_gemm_nt_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.m_grouped_fp8_gemm_nt_contiguous.restype = i32
        L.m_grouped_fp8_gemm_nt_contiguous.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.m_grouped_fp8_gemm_nt_masked.restype = i32
        L.m_grouped_fp8_gemm_nt_masked.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.m_grouped_fp8_gemm_nt_psum.restype = i32
        L.m_grouped_fp8_gemm_nt_psum.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.fp8_gemm_nt_sfb_gran.restype = i32
        L.fp8_gemm_nt_sfb_gran.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, vp]
        L.m_grouped_fp8_gemm_nt_contiguous_sfb_gran.restype = i32
        L.m_grouped_fp8_gemm_nt_contiguous_sfb_gran.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, vp]
        L.m_grouped_fp8_gemm_nt_masked_sfb_gran.restype = i32
        L.m_grouped_fp8_gemm_nt_masked_sfb_gran.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, vp]
        L.pack_ue8m0.restype = i32
        L.pack_ue8m0.argtypes = [vp, vp, i64, i32, vp]
        L.pack_ue8m0_validate.restype = i32
        L.pack_ue8m0_validate.argtypes = [vp, i64, i32, vp, vp]
        _lib = L
        return L


def _check(fn: str, status: int):
    if status != 0:
        raise DgError(fn, status)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtypes, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


_FP8 = (torch.float8_e4m3fn, torch.uint8)
_I32 = (torch.int32,)
_BF16 = (torch.bfloat16,)


def init(device=None):
    """Configure the kernels for a CUDA device (default: torch's current one);
    do it before graph capture."""
    if device is None:
        device = torch.cuda.current_device()
    elif isinstance(device, torch.device):
        device = device.index if device.index is not None else torch.cuda.current_device()
    _check("dgb200_init", load().dgb200_init(int(device)))


def last_device_error() -> int:
    """Device status bits (DEVERR_*) of the current device, then reset to 0;
    synchronises the device."""
    v = ctypes.c_int(0)
    _check("dgb200_last_device_error", load().dgb200_last_device_error(ctypes.byref(v)))
    return int(v.value)


def device_error(clear: bool = True) -> int:
    """Device status bits (DEVERR_*); synchronises the device."""
    v = ctypes.c_uint32(0)
    _check("dgb200_device_error", load().dgb200_device_error(ctypes.byref(v), 1 if clear else 0))
    return int(v.value)


def set_block_n(block_n: int):
    """Force the N tile width (0 = heuristic). For tests and tuning."""
    _check("dgb200_set_block_n", load().dgb200_set_block_n(int(block_n)))


def set_cta_group(cta_group: int):
    """Force single CTAs (1) or CTA pairs (2) for the dense GEMM (0 = heuristic)."""
    _check("dgb200_set_cta_group", load().dgb200_set_cta_group(int(cta_group)))


def set_splits(splits: int):
    """Split-K for the dense GEMM: 0 = heuristic, 1 = never, s >= 2 = s ranges of K."""
    _check("dgb200_set_splits", load().dgb200_set_splits(int(splits)))


def set_test_hooks(mode: int = 0, wait_limit_ms: int = 0):
    """Failure-path test hook: mode 1 makes CTA 0 withhold the arrive of its
    first group of scale words so that a bounded wait runs out (see
    include/dgb200.h). mode 0 = normal."""
    _check("dgb200_set_test_hooks", load().dgb200_set_test_hooks(int(mode), int(wait_limit_ms)))


def block_n_supported(block_n: int) -> bool:
    return bool(load().dgb200_block_n_supported(int(block_n)))


def _kp(K: int) -> int:
    return (K // BLOCK + 3) // 4


def fp8_gemm_nt(a, sfa, b, sfb, d):
    """d[M, N] (bf16) = (a . sfa) @ (b . sfb)^T for E4M3 a [M, K], b [N, K]."""
    _need(a, "a", _FP8)
    M, K = a.shape
    _need(b, "b", _FP8)
    N = b.shape[0]
    _need(b, "b", _FP8, (N, K))
    _need(sfa, "sfa", _I32, (M, _kp(K)))
    _need(sfb, "sfb", _I32, ((N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (M, N))
    _check("fp8_gemm_nt", load().fp8_gemm_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream()))
    return d


def _fp8_gemm_layout(name, a, sfa, b, sfb, d, a_mk: bool, b_nk: bool):
    _need(a, "a", _FP8)
    _need(b, "b", _FP8)
    if a_mk:
        M, K = a.shape
    else:
        K, M = a.shape
    N = b.shape[0] if b_nk else b.shape[1]
    _need(a, "a", _FP8, (M, K) if a_mk else (K, M))
    _need(b, "b", _FP8, (N, K) if b_nk else (K, N))
    _need(sfa, "sfa", _I32, (M, _kp(K)))
    _need(sfb, "sfb", _I32, ((N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (M, N))
    _check(name, getattr(load(), name)(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream()))
    return d


def fp8_gemm_nn(a, sfa, b, sfb, d):
    """d[M, N] = (a . sfa) @ (b . sfb) for E4M3 a [M, K], b [K, N]."""
    return _fp8_gemm_layout("fp8_gemm_nn", a, sfa, b, sfb, d, True, False)


def fp8_gemm_tn(a, sfa, b, sfb, d):
    """d[M, N] = (a . sfa)^T @ (b . sfb) for E4M3 a [K, M], b [K, N]."""
    return _fp8_gemm_layout("fp8_gemm_tn", a, sfa, b, sfb, d, False, False)


def fp8_gemm_tt(a, sfa, b, sfb, d):
    """d[M, N] = (a . sfa)^T @ (b . sfb)^T for E4M3 a [K, M], b [N, K]."""
    return _fp8_gemm_layout("fp8_gemm_tt", a, sfa, b, sfb, d, False, True)


def fp8_gemm_nt_acc(a, sfa, b, sfb, d, c=None):
    """d[M, N] = c + (a . sfa) @ (b . sfb)^T; d is bf16 or fp32, c (optional) has d's
    dtype and may be d itself (in-place accumulation)."""
    _need(a, "a", _FP8)
    M, K = a.shape
    _need(b, "b", _FP8)
    N = b.shape[0]
    _need(b, "b", _FP8, (N, K))
    _need(sfa, "sfa", _I32, (M, _kp(K)))
    _need(sfb, "sfb", _I32, ((N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", (torch.bfloat16, torch.float32), (M, N))
    if c is not None:
        _need(c, "c", (d.dtype,), (M, N))
    _check("fp8_gemm_nt_acc", load().fp8_gemm_nt_acc(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb),
                                                     None if c is None else _ptr(c), _ptr(d), M, N, K,
                                                     1 if d.dtype == torch.float32 else 0, _stream()))
    return d


def fp8_gemm_nt_noalloc(a, sfa, b, sfb, d, splits: int = 0):
    """fp8_gemm_nt that allocates no device memory: split-K scratch comes from
    static arrays of the library (8 MiB of partials, 1024 tiles). splits: 0 =
    model's choice within that scratch, 1 = none, s >= 2 = exactly s. Calls that
    overlap in time on one device race on the scratch (see include/dgb200.h)."""
    _need(a, "a", _FP8)
    M, K = a.shape
    _need(b, "b", _FP8)
    N = b.shape[0]
    _need(b, "b", _FP8, (N, K))
    _need(sfa, "sfa", _I32, (M, _kp(K)))
    _need(sfb, "sfb", _I32, ((N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (M, N))
    _check("fp8_gemm_nt_noalloc", load().fp8_gemm_nt_noalloc(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K,
                                                             int(splits), _stream()))
    return d


def m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, m_indices):
    """Contiguous M-grouped GEMM; rows tagged by expert in m_indices (-1 = padding)."""
    _need(a, "a", _FP8)
    M_total, K = a.shape
    _need(b, "b", _FP8)
    G, N = b.shape[0], b.shape[1]
    _need(b, "b", _FP8, (G, N, K))
    _need(sfa, "sfa", _I32, (M_total, _kp(K)))
    _need(sfb, "sfb", _I32, (G, (N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (M_total, N))
    _need(m_indices, "m_indices", _I32, (M_total,))
    _check("m_grouped_fp8_gemm_nt_contiguous",
           load().m_grouped_fp8_gemm_nt_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(m_indices),
                                                   M_total, N, K, G, _stream()))
    return d


def m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, masked_m, max_m=None):
    """Masked M-grouped GEMM; group g uses its first masked_m[g] rows (device tensor)."""
    _need(a, "a", _FP8)
    G, mm, K = a.shape
    if max_m is None:
        max_m = mm
    if max_m != mm:
        raise ValueError(f"max_m={max_m} does not match a.shape[1]={mm}")
    _need(b, "b", _FP8)
    N = b.shape[1]
    _need(b, "b", _FP8, (G, N, K))
    _need(sfa, "sfa", _I32, (G, max_m, _kp(K)))
    _need(sfb, "sfb", _I32, (G, (N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (G, max_m, N))
    _need(masked_m, "masked_m", _I32, (G,))
    _check("m_grouped_fp8_gemm_nt_masked",
           load().m_grouped_fp8_gemm_nt_masked(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(masked_m),
                                               G, max_m, N, K, _stream()))
    return d


def m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, d, psum_m):
    """M-grouped GEMM with groups given by psum_m (device int32 [G]): group g owns
    rows [psum_m[g-1], psum_m[g]) of a [M_total, K]; rows in no group are not written."""
    _need(a, "a", _FP8)
    M_total, K = a.shape
    _need(b, "b", _FP8)
    G, N = b.shape[0], b.shape[1]
    _need(b, "b", _FP8, (G, N, K))
    _need(sfa, "sfa", _I32, (M_total, _kp(K)))
    _need(sfb, "sfb", _I32, (G, (N + BLOCK - 1) // BLOCK, _kp(K)))
    _need(d, "d", _BF16, (M_total, N))
    _need(psum_m, "psum_m", _I32, (G,))
    _check("m_grouped_fp8_gemm_nt_psum",
           load().m_grouped_fp8_gemm_nt_psum(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(psum_m),
                                             M_total, N, K, G, _stream()))
    return d


def _sfb_rows(N: int, sfb_gran_n: int) -> int:
    if sfb_gran_n not in (1, BLOCK):
        raise ValueError(f"sfb_gran_n={sfb_gran_n}: B scale rows cover 1 or {BLOCK} rows of B")
    return N if sfb_gran_n == 1 else (N + BLOCK - 1) // BLOCK


def fp8_gemm_nt_sfb_gran(a, sfa, b, sfb, d, sfb_gran_n: int, c=None):
    """fp8_gemm_nt_acc with the B-scale granularity given: sfb [N, KP] (sfb_gran_n=1,
    one scale row per row of b) or [ceil(N/128), KP] (sfb_gran_n=128)."""
    _need(a, "a", _FP8)
    M, K = a.shape
    _need(b, "b", _FP8)
    N = b.shape[0]
    _need(b, "b", _FP8, (N, K))
    _need(sfa, "sfa", _I32, (M, _kp(K)))
    _need(sfb, "sfb", _I32, (_sfb_rows(N, sfb_gran_n), _kp(K)))
    _need(d, "d", (torch.bfloat16, torch.float32), (M, N))
    if c is not None:
        _need(c, "c", (d.dtype,), (M, N))
    _check("fp8_gemm_nt_sfb_gran",
           load().fp8_gemm_nt_sfb_gran(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), int(sfb_gran_n),
                                       None if c is None else _ptr(c), _ptr(d), M, N, K,
                                       1 if d.dtype == torch.float32 else 0, _stream()))
    return d


def m_grouped_fp8_gemm_nt_contiguous_sfb_gran(a, sfa, b, sfb, d, m_indices, sfb_gran_n: int):
    """m_grouped_fp8_gemm_nt_contiguous with sfb [G, N, KP] (sfb_gran_n=1) or
    [G, ceil(N/128), KP] (sfb_gran_n=128)."""
    _need(a, "a", _FP8)
    M_total, K = a.shape
    _need(b, "b", _FP8)
    G, N = b.shape[0], b.shape[1]
    _need(b, "b", _FP8, (G, N, K))
    _need(sfa, "sfa", _I32, (M_total, _kp(K)))
    _need(sfb, "sfb", _I32, (G, _sfb_rows(N, sfb_gran_n), _kp(K)))
    _need(d, "d", _BF16, (M_total, N))
    _need(m_indices, "m_indices", _I32, (M_total,))
    _check("m_grouped_fp8_gemm_nt_contiguous_sfb_gran",
           load().m_grouped_fp8_gemm_nt_contiguous_sfb_gran(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), int(sfb_gran_n),
                                                            _ptr(d), _ptr(m_indices), M_total, N, K, G, _stream()))
    return d


def m_grouped_fp8_gemm_nt_masked_sfb_gran(a, sfa, b, sfb, d, masked_m, sfb_gran_n: int):
    """m_grouped_fp8_gemm_nt_masked with sfb [G, N, KP] (sfb_gran_n=1) or
    [G, ceil(N/128), KP] (sfb_gran_n=128)."""
    _need(a, "a", _FP8)
    G, max_m, K = a.shape
    _need(b, "b", _FP8)
    N = b.shape[1]
    _need(b, "b", _FP8, (G, N, K))
    _need(sfa, "sfa", _I32, (G, max_m, _kp(K)))
    _need(sfb, "sfb", _I32, (G, _sfb_rows(N, sfb_gran_n), _kp(K)))
    _need(d, "d", _BF16, (G, max_m, N))
    _need(masked_m, "masked_m", _I32, (G,))
    _check("m_grouped_fp8_gemm_nt_masked_sfb_gran",
           load().m_grouped_fp8_gemm_nt_masked_sfb_gran(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), int(sfb_gran_n),
                                                        _ptr(d), _ptr(masked_m), G, max_m, N, K, _stream()))
    return d


_BF16_OPERAND = (torch.bfloat16, torch.int16, torch.uint16)  # bf16 values or their bit patterns


def m_grouped_bf16_gemm_nt_masked(a, b, d, masked_m):
    """Masked M-grouped BF16 GEMM: d[g, :m_g] = a[g, :m_g] @ b[g]^T, m_g = masked_m[g] (device)."""
    _need(a, "a", _BF16_OPERAND)
    G, max_m, K = a.shape
    _need(b, "b", _BF16_OPERAND)
    N = b.shape[1]
    _need(b, "b", _BF16_OPERAND, (G, N, K))
    _need(d, "d", _BF16, (G, max_m, N))
    _need(masked_m, "masked_m", _I32, (G,))
    _check("m_grouped_bf16_gemm_nt_masked",
           load().m_grouped_bf16_gemm_nt_masked(_ptr(a), _ptr(b), _ptr(d), _ptr(masked_m), G, max_m, N, K,
                                                _stream()))
    return d


def pack_ue8m0(sf, out=None):
    """Pack fp32 scales [..., cols] into int32 [..., ceil(cols/4)] (UE8M0, 4 per word)."""
    _need(sf, "sf", (torch.float32,))
    if sf.dim() < 1:
        raise ValueError("sf must have at least one dimension")
    cols = sf.shape[-1]
    rows = sf.numel() // cols if cols else 0
    kp = (cols + 3) // 4
    if out is None:
        out = torch.empty((*sf.shape[:-1], kp), dtype=torch.int32, device=sf.device)
    _need(out, "out", _I32, (*sf.shape[:-1], kp))
    _check("pack_ue8m0", load().pack_ue8m0(_ptr(sf), _ptr(out), rows, cols, _stream()))
    return out


def quantize_fp8_1x128(x, q=None, sf_packed=None, sf_f32=None):
    """x [rows, K] bf16/fp32 -> (q E4M3 as uint8 [rows, K], packed UE8M0 scales
    int32 [rows, ceil(K/512)], fp32 scales [rows, K/128] or None)."""
    _need(x, "x", (torch.bfloat16, torch.float32))
    rows, K = x.shape
    if q is None:
        q = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    if sf_packed is None:
        sf_packed = torch.empty((rows, _kp(K)), dtype=torch.int32, device=x.device)
    _need(q, "q", _FP8, (rows, K))
    _need(sf_packed, "sf_packed", _I32, (rows, _kp(K)))
    if sf_f32 is not None:
        _need(sf_f32, "sf_f32", (torch.float32,), (rows, K // BLOCK))
    _check("quantize_fp8_1x128",
           load().quantize_fp8_1x128(_ptr(x), 1 if x.dtype == torch.float32 else 0, _ptr(q), _ptr(sf_packed),
                                     None if sf_f32 is None else _ptr(sf_f32), rows, K, _stream()))
    return q, sf_packed, sf_f32


def pack_ue8m0_validate(sf, bad_count):
    """Write to bad_count (device int32 [1]) the number of scales with sign set or mantissa != 0."""
    _need(sf, "sf", (torch.float32,))
    _need(bad_count, "bad_count", _I32, (1,))
    cols = sf.shape[-1]
    rows = sf.numel() // cols if cols else 0
    _check("pack_ue8m0_validate", load().pack_ue8m0_validate(_ptr(sf), rows, cols, _ptr(bad_count), _stream()))
    return bad_count
