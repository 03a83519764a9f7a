"""CPU oracle for the FP8 block-scaled GEMM path (test infrastructure only).

This package is the plain, slow, obviously-correct statement of what the
library computes. It is used only by ``tests/``, by ``__graft_entry__.smoke()``
and by ``bench.py``'s CPU-baseline / reference leg. The product path (the
CUDA library and its Python binding) never imports it, and it never imports
the product path: the two share no code, no tables and no helpers.

Everything is numpy in float64.

Modules
-------
fp8    -- the OCP E4M3 value table (``e4m3_to_f64``)
bf16   -- bf16 operand values (``bf16_to_f64``)
quant  -- the per-token FP8 quantiser with UE8M0 block scales
ue8m0  -- UE8M0 scale bytes: decode, the capture-safe pack of fp32 scales
          into four bytes per int32, the matching unpack, and the optional
          eager validator
gemm   -- dequantise-and-multiply references for the dense NT GEMM and the
          contiguous / masked / psum_m-driven M-grouped GEMMs, and the BF16
          masked grouped GEMM

Sources (web pages about DeepGEMM):
  [P1] "DeepGEMM CUDA Graph Compatibility for Masked Grouped GEMMs:
       Implementation Guide" (instagit how-to)
  [P2] "DeepInside DeepGEMM: Unpacking DeepSeek's Unified Tensor Core Library
       for SM90 and SM100" (musen-ai)
  [P3] "[GH-ISSUE #414] [Bug] pack_ue8m0_to_int is not CUDA Graph capture
       safe" (issue mirror)
Every function names the section it follows.
"""

from .fp8 import e4m3_to_f64, E4M3_MAX  # noqa: F401
from .bf16 import bf16_to_f64  # noqa: F401
from .quant import e4m3_encode_rne, scale_exponent, quantize_fp8_1x128  # noqa: F401
from .ue8m0 import (  # noqa: F401
    ue8m0_to_f64,
    pack_ue8m0,
    unpack_ue8m0,
    pack_ue8m0_validate,
)
from .gemm import (  # noqa: F401
    dequant_rows,
    dequant_weights,
    fp8_gemm_nt,
    fp8_gemm,
    fp8_gemm_nt_acc,
    fp8_gemm_nt_sampled,
    fp8_gemm_nt_points,
    m_grouped_fp8_gemm_nt_contiguous,
    m_grouped_fp8_gemm_nt_contiguous_sampled,
    m_grouped_fp8_gemm_nt_masked,
    m_grouped_fp8_gemm_nt_masked_sampled,
    masked_valid_rows,
    psum_group_rows,
    m_grouped_fp8_gemm_nt_psum,
    m_grouped_bf16_gemm_nt_masked,
    m_grouped_bf16_gemm_nt_masked_sampled,
)
