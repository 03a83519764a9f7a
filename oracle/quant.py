"""Per-token FP8 quantiser with UE8M0 block scales (oracle; test infrastructure only).

"DeepInside DeepGEMM", §5 Production Gotchas: the activations' FP8 cast and
the packing of their scales belong in a dedicated kernel before the GEMM
(four UE8M0 scales per int32 on SM100). What that kernel computes, per 1x128
block of a row of activations x (the reading used throughout, the same recipe
that builds the test inputs):

    amax = max(max |x| over the block, 1e-4 as fp32)
    e    = ceil(log2(amax / 448))         (the scale is s = 2^e, a UE8M0 byte 127 + e)
    q    = E4M3 code of x / s, rounded to nearest, ties to the even code

Because s is a power of two, x / s is exact. The exponent is an integer
decision; writing amax = m * 2^E with m in [1, 2) and 448 = 1.75 * 2^8,
ceil(log2(amax / 448)) = E - 8 + (1 if m > 1.75 else 0), which is what is
computed here (exactly, from frexp) and what the CUDA kernel computes from the
fp32 bits of amax.
"""

import numpy as np

from .fp8 import e4m3_to_f64
from .ue8m0 import pack_ue8m0

BLOCK = 128
AMAX_FLOOR = float(np.float32(1e-4))

# non-negative finite E4M3 values by code 0..126 (increasing with the code)
_POS_CODES = np.arange(127, dtype=np.uint8)
_POS_VALS = e4m3_to_f64(_POS_CODES)


def e4m3_encode_rne(v) -> np.ndarray:
    """Nearest finite E4M3 code of each value (ties to the even code, i.e. the
    one whose lowest mantissa bit is 0); magnitudes above 448 give 448. The
    sign of the input is kept (a negative value that rounds to 0 gives -0)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), _POS_VALS[-1])
    hi = np.clip(np.searchsorted(_POS_VALS, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _POS_VALS[lo]
    d_hi = _POS_VALS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def scale_exponent(amax) -> np.ndarray:
    """e = ceil(log2(max(amax, 1e-4 as fp32) / 448)) for fp32 amax values, exactly."""
    a = np.maximum(np.asarray(amax, dtype=np.float64), AMAX_FLOOR)
    m2, e2 = np.frexp(a)          # a = m2 * 2^e2, m2 in [0.5, 1)
    E, m = e2 - 1, 2.0 * m2       # a = m * 2^E, m in [1, 2)
    return (E - 8 + (m > 1.75)).astype(np.int64)


def quantize_fp8_1x128(x):
    """x: float array [R, K] of fp32-representable values, K % 128 == 0.
    Returns (q uint8 [R, K] E4M3 codes, packed int32 [R, ceil(K/512)] UE8M0
    scales four per word, sf float32 [R, K/128] the scales 2^e)."""
    x = np.asarray(x, dtype=np.float64)
    R, K = x.shape
    if K % BLOCK:
        raise ValueError(f"K={K} is not a multiple of {BLOCK}")
    xb = x.reshape(R, K // BLOCK, BLOCK)
    e = scale_exponent(np.abs(xb).max(axis=2))
    q = e4m3_encode_rne(xb * np.ldexp(1.0, -e)[:, :, None]).reshape(R, K)
    sf = np.ldexp(1.0, e).astype(np.float32)
    return q, pack_ue8m0(sf), sf
