"""BF16 operand values (oracle; test infrastructure only).

bfloat16 is the upper half of an IEEE-754 binary32: sign, the same 8-bit
exponent with bias 127, and the top 7 bits of the fraction. Its value is the
binary32 whose bit pattern is the 16 bits followed by 16 zero bits, so decoding
is exact in float64. The BF16 masked grouped GEMM of "DeepGEMM CUDA Graph
Compatibility for Masked Grouped GEMMs" (Core Components: the BF16 masked
grouped GEMM kernel) takes its operands in this format.
"""

import numpy as np


def bf16_to_f64(bits) -> np.ndarray:
    """Decode uint16 bf16 bit patterns to float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # signalling-NaN codes widen to NaN
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
