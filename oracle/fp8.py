"""OCP E4M3 decode table (oracle; test infrastructure only).

The operands of every GEMM here are ``torch.float8_e4m3fn`` bytes ("DeepInside
DeepGEMM", §4 Hands-on Geek Guide: A and B are cast to float8_e4m3fn). The
format is the OCP 8-bit floating point E4M3 encoding:

    bit 7      sign s
    bits 6..3  exponent e, bias 7
    bits 2..0  mantissa m

    e == 0            : (-1)^s * (m / 8) * 2^(1 - 7)        (subnormal, incl. +-0)
    1 <= e <= 15      : (-1)^s * (1 + m / 8) * 2^(e - 7)
    e == 15 and m == 7: NaN (the only NaN pattern; there is no infinity)

so the largest finite magnitude is 1.75 * 2^8 = 448.

The table is built from that definition, one code at a time, with no library
float8 routine involved (the tests pin it against torch's own float8 decode).
"""

import numpy as np

E4M3_MAX = 448.0


def _decode_one(code: int) -> float:
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    sign = -1.0 if s else 1.0
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_TABLE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)


def e4m3_to_f64(codes) -> np.ndarray:
    """Decode E4M3 bytes (any integer array, values 0..255) to float64."""
    codes = np.asarray(codes)
    return _TABLE[codes.astype(np.uint8)]
