"""UE8M0 scale bytes and their four-per-int32 packing (oracle; test infrastructure only).

Sources
-------
* "DeepInside DeepGEMM", §2 Core Architecture and Data Flow Analysis, and §5
  Pitfall Warning [Input Tensor Layout and Type Mismatch]: on SM100 the scaling
  factors are UE8M0, four of them packed into one ``torch.int``.
* "[GH-ISSUE #414] pack_ue8m0_to_int is not CUDA Graph capture safe", Summary
  and Expected behavior: the packing is
  ``(x.view(torch.int) >> 23).to(torch.uint8).view(torch.int)``, and the value
  checks of the original helper are ``x_int >= 0`` and ``x_int & 0x7FFFFF == 0``
  (sign clear, mantissa zero), which the issue asks to keep only on an eager
  validation path.

Readings where the pages are silent (each also listed in the design notes):
* ``.to(torch.uint8)`` of the shifted int32 keeps its low 8 bits, i.e. the
  byte is ``(bits >> 23) & 0xFF`` (arithmetic shift; for sign-clear inputs this
  is the biased exponent field).
* ``.view(torch.int)`` of the uint8 tensor groups four consecutive bytes of
  the last dimension, little-endian: byte j of int32 word i is scale column
  ``4*i + j``. When the column count is not a multiple of four the last word
  is completed with zero bytes.
* A UE8M0 byte e stands for 2^(e - 127); 0xFF is NaN.
"""

import numpy as np


def ue8m0_to_f64(e) -> np.ndarray:
    """Value of UE8M0 bytes: 2^(e-127), NaN for 0xFF."""
    e = np.asarray(e).astype(np.int64)
    out = np.ldexp(np.ones(e.shape, dtype=np.float64), e - 127)
    return np.where(e == 255, np.nan, out)


def pack_ue8m0(sf) -> np.ndarray:
    """Pack fp32 scales [rows, cols] into int32 [rows, ceil(cols/4)].

    Follows the issue's formula step by step: reinterpret the float32 bits as
    int32, shift right by 23, keep the low byte, then view each run of four
    bytes along the last dimension as one little-endian int32.
    """
    sf = np.ascontiguousarray(np.asarray(sf, dtype=np.float32))
    if sf.ndim != 2:
        raise ValueError("pack_ue8m0 expects a 2-D [rows, cols] array")
    rows, cols = sf.shape
    bits = sf.view(np.int32)
    byte = ((bits >> 23) & 0xFF).astype(np.uint8)
    kp = (cols + 3) // 4
    padded = np.zeros((rows, 4 * kp), dtype=np.uint8)
    padded[:, :cols] = byte
    # little-endian int32 view of four consecutive bytes
    return padded.view("<i4").reshape(rows, kp).astype(np.int32)


def unpack_ue8m0(packed, cols: int) -> np.ndarray:
    """Inverse view of :func:`pack_ue8m0`: int32 [rows, KP] -> uint8 [rows, cols].

    Byte j (bits 8j..8j+7) of word i is column 4*i + j.
    """
    packed = np.asarray(packed, dtype=np.int64) & 0xFFFFFFFF
    rows, kp = packed.shape
    if cols > 4 * kp:
        raise ValueError("cols exceeds the packed width")
    out = np.empty((rows, 4 * kp), dtype=np.uint8)
    for j in range(4):
        out[:, j::4] = ((packed >> (8 * j)) & 0xFF).astype(np.uint8)
    return out[:, :cols]


def pack_ue8m0_validate(sf) -> int:
    """Number of scales that fail the issue's checks (sign set or mantissa != 0)."""
    bits = np.ascontiguousarray(np.asarray(sf, dtype=np.float32)).view(np.int32)
    bad = (bits < 0) | ((bits & 0x7FFFFF) != 0)
    return int(bad.sum())
