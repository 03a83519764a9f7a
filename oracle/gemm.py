"""Dequantise-and-multiply references for the three GEMM forms (oracle; test infrastructure only).

What is computed
----------------
All three forms compute D = A . B^T with A row-major [rows, K] and B row-major
[N, K] ("NT"): "DeepInside DeepGEMM", §4 Hands-on Geek Guide, where the
standard non-grouped FP8 NT GEMM computes D = C + A @ B.T (C is absent here,
i.e. zero) and returns bf16.

Operands are E4M3 bytes with power-of-two scales stored as packed UE8M0
(§2 of the same page): activations carry one scale per 1x128 block along K,
weights one per 128x128 block. The dequantised operands are

    A^[m, k] = e4m3(a[m, k]) * 2^(ea[m, k // 128] - 127)
    B^[n, k] = e4m3(b[n, k]) * 2^(eb[n // 128, k // 128] - 127)

where ea / eb are the bytes of the packed int32 scale rows (byte j of word i is
K-block 4*i + j). The reference result is A^ . B^^T in float64.

The same page's minimal FP8 GEMM example gives B one scale row per row of B
(``b_sf`` of shape [n, k // 128]), i.e. 1x128 blocks for the weights as well.
Every dense and grouped function below takes ``sfb_gran_n``: the number of
rows of B that share one scale row, 128 (the 128x128 blocks above, sfb
[ceil(N/128), KP]) or 1 (sfb [N, KP], B^[n, k] scaled by eb[n, k // 128]).

Grouped forms (readings; the pages name them but print no definition beyond
the call shape):
* contiguous: rows of A are concatenated by expert; ``m_indices[r]`` gives the
  expert of row r. Rows with an index outside [0, G) (-1 marks padding) are
  not computed and their output is left as it was.
* psum_m-driven (same page, Tensor-Based Metadata Arguments; reading in
  psum_group_rows): A is [M_total, K] with the groups' rows end to end, group
  g owning rows [psum_m[g-1], psum_m[g]); rows in no group are left as they were.
* masked ("DeepGEMM CUDA Graph Compatibility for Masked Grouped GEMMs",
  Tensor-Based Metadata Arguments and the FAQ on dynamic shapes): A is
  [G, max_m, K] and D is [G, max_m, N]; only the first masked_m[g] rows of group
  g are valid (masked_m clamped to [0, max_m]); every other row of D is left as
  it was.

Each grouped reference returns (values, valid) where ``valid`` marks the rows
whose output is defined; rows outside it must keep their previous bits.
"""

import numpy as np

from .bf16 import bf16_to_f64
from .fp8 import e4m3_to_f64
from .ue8m0 import ue8m0_to_f64, unpack_ue8m0

BLOCK = 128  # scale granularity along K (and along N for the weights)


def _kb(K: int) -> int:
    if K % BLOCK != 0:
        raise ValueError(f"K={K} is not a multiple of {BLOCK}")
    return K // BLOCK


def dequant_rows(a, sfa) -> np.ndarray:
    """A^ for activation rows: a uint8 [R, K], sfa int32 [R, KP] -> float64 [R, K]."""
    a = np.asarray(a, dtype=np.uint8)
    R, K = a.shape
    KB = _kb(K)
    scale = ue8m0_to_f64(unpack_ue8m0(sfa, KB))  # [R, KB], one per 1x128 block
    vals = e4m3_to_f64(a).reshape(R, KB, BLOCK)
    return (vals * scale[:, :, None]).reshape(R, K)


def _gran(sfb_gran_n) -> int:
    if sfb_gran_n not in (1, BLOCK):
        raise ValueError(f"sfb_gran_n={sfb_gran_n}: B scale rows cover 1 or {BLOCK} rows of B")
    return int(sfb_gran_n)


def dequant_weights(b, sfb, cols=None, sfb_gran_n=BLOCK) -> np.ndarray:
    """B^ for weight rows: b uint8 [N, K], sfb int32 [ceil(N/gran), KP] -> float64.

    ``cols`` (optional) selects which rows n of B to dequantise, so that sampled
    checks need not expand the whole weight. Row n of B takes scale row
    n // sfb_gran_n (128x128 blocks for 128, one scale row per row of B for 1).
    """
    gran = _gran(sfb_gran_n)
    b = np.asarray(b, dtype=np.uint8)
    N, K = b.shape
    KB = _kb(K)
    if np.asarray(sfb).shape[0] != -(-N // gran):
        raise ValueError(f"sfb has {np.asarray(sfb).shape[0]} scale rows; N={N} at granularity {gran} needs {-(-N // gran)}")
    n = np.arange(N) if cols is None else np.asarray(cols, dtype=np.int64)
    row_scale = ue8m0_to_f64(unpack_ue8m0(sfb, KB))  # [ceil(N/gran), KB]
    scale = row_scale[n // gran]
    vals = e4m3_to_f64(b[n]).reshape(len(n), KB, BLOCK)
    return (vals * scale[:, :, None]).reshape(len(n), K)


def fp8_gemm_nt(a, sfa, b, sfb, sfb_gran_n=BLOCK) -> np.ndarray:
    """Dense D[M, N] = A^ . B^^T in float64."""
    return dequant_rows(a, sfa) @ dequant_weights(b, sfb, sfb_gran_n=sfb_gran_n).T


def fp8_gemm_nt_sampled(a, sfa, b, sfb, rows, cols, sfb_gran_n=BLOCK) -> np.ndarray:
    """D[rows[i], cols[i]] of the dense GEMM, one output at a time (float64)."""
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    ur, ri = np.unique(rows, return_inverse=True)
    uc, ci = np.unique(cols, return_inverse=True)
    ah = dequant_rows(np.asarray(a)[ur], np.asarray(sfa)[ur])
    bh = dequant_weights(b, sfb, cols=uc, sfb_gran_n=sfb_gran_n)
    return np.einsum("ik,ik->i", ah[ri], bh[ci])


def m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_indices, sfb_gran_n=BLOCK):
    """Contiguous M-grouped GEMM.

    a uint8 [M_total, K], sfa int32 [M_total, KP], b uint8 [G, N, K],
    sfb int32 [G, ceil(N/gran), KP], m_indices int32 [M_total].
    Returns (D float64 [M_total, N] with NaN on undefined rows, valid bool [M_total]).
    """
    b = np.asarray(b, dtype=np.uint8)
    G, N, _ = b.shape
    m_indices = np.asarray(m_indices, dtype=np.int64)
    M_total = m_indices.shape[0]
    out = np.full((M_total, N), np.nan, dtype=np.float64)
    valid = (m_indices >= 0) & (m_indices < G)
    for g in range(G):
        r = np.nonzero(m_indices == g)[0]
        if r.size == 0:
            continue
        out[r] = (dequant_rows(np.asarray(a)[r], np.asarray(sfa)[r])
                  @ dequant_weights(b[g], np.asarray(sfb)[g], sfb_gran_n=sfb_gran_n).T)
    return out, valid


def m_grouped_fp8_gemm_nt_contiguous_sampled(a, sfa, b, sfb, m_indices, rows, cols, sfb_gran_n=BLOCK):
    """Sampled outputs of the contiguous GEMM; rows must have a valid expert."""
    m_indices = np.asarray(m_indices, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    out = np.empty(rows.shape[0], dtype=np.float64)
    g_of = m_indices[rows]
    if np.any((g_of < 0) | (g_of >= np.asarray(b).shape[0])):
        raise ValueError("sampled rows must belong to an expert")
    for g in np.unique(g_of):
        sel = np.nonzero(g_of == g)[0]
        out[sel] = fp8_gemm_nt_sampled(a, sfa, np.asarray(b)[g], np.asarray(sfb)[g], rows[sel], cols[sel],
                                       sfb_gran_n=sfb_gran_n)
    return out


def psum_group_rows(psum_m, M_total: int):
    """Row range [start_g, end_g) of every group of the psum_m-driven grouped GEMM.

    Reading ("DeepGEMM CUDA Graph Compatibility for Masked Grouped GEMMs",
    Tensor-Based Metadata Arguments, names psum_m as device metadata of the
    grouped GEMMs without defining it): psum_m[g] is the inclusive prefix sum
    of the groups' row counts, so group g owns rows [psum_m[g-1], psum_m[g])
    of an unpadded A [M_total, K] (psum_m[-1] = 0). Malformed values are made
    harmless: end_g = min(max(0, psum_m[0], ..., psum_m[g]), M_total) and
    start_g = end_{g-1}, start_0 = 0, so a decreasing entry gives an empty
    group and no row belongs to two groups.
    """
    psum_m = np.asarray(psum_m, dtype=np.int64)
    ends = np.minimum(np.maximum.accumulate(np.maximum(psum_m, 0)), M_total)
    starts = np.concatenate([[0], ends[:-1]]).astype(np.int64)
    return starts, ends


def m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, psum_m, sfb_gran_n=BLOCK):
    """Grouped GEMM whose groups are given by prefix sums of their row counts.

    a uint8 [M_total, K], sfa int32 [M_total, KP], b uint8 [G, N, K],
    sfb int32 [G, ceil(N/gran), KP], psum_m int32 [G]. Rows of group g (see
    psum_group_rows) use B[g]; D[r] = A^[r] . B^[g]^T. Rows in no group are
    left as they were. Returns (D float64 [M_total, N] with NaN on rows in no
    group, valid bool [M_total]).
    """
    a = np.asarray(a, dtype=np.uint8)
    b = np.asarray(b, dtype=np.uint8)
    M_total = a.shape[0]
    G, N, _ = b.shape
    starts, ends = psum_group_rows(psum_m, M_total)
    out = np.full((M_total, N), np.nan, dtype=np.float64)
    valid = np.zeros(M_total, dtype=bool)
    for g in range(G):
        r0, r1 = int(starts[g]), int(ends[g])
        if r1 <= r0:
            continue
        out[r0:r1] = fp8_gemm_nt(a[r0:r1], np.asarray(sfa)[r0:r1], b[g], np.asarray(sfb)[g], sfb_gran_n=sfb_gran_n)
        valid[r0:r1] = True
    return out, valid


def masked_valid_rows(masked_m, G: int, max_m: int) -> np.ndarray:
    """valid[g, r] = r < clamp(masked_m[g], 0, max_m)."""
    mm = np.clip(np.asarray(masked_m, dtype=np.int64), 0, max_m)
    return np.arange(max_m)[None, :] < mm[:G, None]


def m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, masked_m, sfb_gran_n=BLOCK):
    """Masked M-grouped GEMM.

    a uint8 [G, max_m, K], sfa int32 [G, max_m, KP], b uint8 [G, N, K],
    sfb int32 [G, ceil(N/gran), KP], masked_m int32 [G].
    Returns (D float64 [G, max_m, N] with NaN on undefined rows, valid bool [G, max_m]).
    """
    a = np.asarray(a, dtype=np.uint8)
    G, max_m, _ = a.shape
    N = np.asarray(b).shape[1]
    valid = masked_valid_rows(masked_m, G, max_m)
    out = np.full((G, max_m, N), np.nan, dtype=np.float64)
    for g in range(G):
        m = int(valid[g].sum())
        if m == 0:
            continue
        out[g, :m] = fp8_gemm_nt(a[g, :m], np.asarray(sfa)[g, :m], np.asarray(b)[g], np.asarray(sfb)[g],
                                 sfb_gran_n=sfb_gran_n)
    return out, valid


def m_grouped_fp8_gemm_nt_masked_sampled(a, sfa, b, sfb, groups, rows, cols, sfb_gran_n=BLOCK):
    """Sampled outputs D[groups[i], rows[i], cols[i]] of the masked GEMM (valid rows only)."""
    groups = np.asarray(groups, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    out = np.empty(groups.shape[0], dtype=np.float64)
    for g in np.unique(groups):
        sel = np.nonzero(groups == g)[0]
        out[sel] = fp8_gemm_nt_sampled(np.asarray(a)[g], np.asarray(sfa)[g], np.asarray(b)[g],
                                       np.asarray(sfb)[g], rows[sel], cols[sel], sfb_gran_n=sfb_gran_n)
    return out


def fp8_gemm_nt_points(a_rows, sfa_rows, b_rows, n_idx, sfb, sfb_gran_n=BLOCK) -> np.ndarray:
    """Outputs one at a time: out[i] = sum_k A^_i[k] * B^[n_idx[i], k].

    a_rows / sfa_rows: the A rows of the sampled outputs and their packed scale
    rows; b_rows: row n_idx[i] of B for each output; sfb: the full packed scale
    matrix of that B ([ceil(N/gran), KP]), indexed here by n_idx // gran.
    """
    gran = _gran(sfb_gran_n)
    A = dequant_rows(a_rows, sfa_rows)
    b_rows = np.asarray(b_rows, dtype=np.uint8)
    P, K = b_rows.shape
    KB = _kb(K)
    n_idx = np.asarray(n_idx, dtype=np.int64)
    scale = ue8m0_to_f64(unpack_ue8m0(sfb, KB))[n_idx // gran]
    B = (e4m3_to_f64(b_rows).reshape(P, KB, BLOCK) * scale[:, :, None]).reshape(P, K)
    return np.einsum("ik,ik->i", A, B)


# ---- dense GEMM with other operand layouts --------------------------------------

def fp8_gemm(a, sfa, b, sfb, layout: str) -> np.ndarray:
    """Dense FP8 GEMM D[m, n] = sum_k A^[m, k] B^[n, k] for the operand layouts
    that "DeepInside DeepGEMM" §2 lists for SM100 (NT, TN, NN, TT). The first
    letter is A's storage: "n" = [M, K] (K contiguous), "t" = [K, M]; the second
    is B's: "t" = [N, K] (K contiguous), "n" = [K, N]. The scales do not depend
    on the storage: sfa is [M, KP] (one per row and 128-K block), sfb is
    [ceil(N/128), KP]. Reading: the letters follow the NT GEMM of §4 (A as
    given, B transposed); the pages name the layouts without defining them."""
    layout = layout.lower()
    if layout not in ("nt", "tn", "nn", "tt"):
        raise ValueError(f"unknown layout {layout!r}")
    A = np.asarray(a, dtype=np.uint8)
    B = np.asarray(b, dtype=np.uint8)
    A_mk = A if layout[0] == "n" else A.T
    B_nk = B if layout[1] == "t" else B.T
    return fp8_gemm_nt(np.ascontiguousarray(A_mk), sfa, np.ascontiguousarray(B_nk), sfb)


# ---- dense GEMM with an accumulation matrix ------------------------------------

def fp8_gemm_nt_acc(a, sfa, b, sfb, c=None, sfb_gran_n=BLOCK) -> np.ndarray:
    """D = C + A^ . B^^T in float64 ("DeepInside DeepGEMM", §4 Hands-on Geek
    Guide: the standard non-grouped FP8 NT GEMM computes D = C + A @ B.T; the
    example passes C as a bf16 [M, N] tensor and the output dtype).

    c: None (C = 0) or the values of C as a float array [M, N] (decoded from
    D's storage type by the caller). Readings: C has D's storage type (bf16 or
    fp32) and is added to the fp32 accumulation before the final conversion,
    so the reference is the exact sum C + A^.B^^T. sfb_gran_n as fp8_gemm_nt."""
    d = fp8_gemm_nt(a, sfa, b, sfb, sfb_gran_n=sfb_gran_n)
    if c is None:
        return d
    c = np.asarray(c, dtype=np.float64)
    if c.shape != d.shape:
        raise ValueError(f"C has shape {c.shape}, D has {d.shape}")
    return c + d


# ---- BF16 masked grouped GEMM ------------------------------------------------

def m_grouped_bf16_gemm_nt_masked(a, b, masked_m):
    """BF16 masked M-grouped GEMM ("DeepGEMM CUDA Graph Compatibility for Masked
    Grouped GEMMs", Core Components and Tensor-Based Metadata Arguments).

    a: uint16 bf16 bits [G, max_m, K]; b: uint16 bf16 bits [G, N, K];
    masked_m: int [G]. For every group g, D[g, :m_g] = A[g, :m_g] . B[g]^T with
    m_g = clamp(masked_m[g], 0, max_m), in float64 (no scales: the operands are
    plain bf16 values). Returns (D with NaN on rows outside the valid region,
    valid [G, max_m])."""
    a = np.asarray(a, dtype=np.uint16)
    b = np.asarray(b, dtype=np.uint16)
    G, max_m, K = a.shape
    N = b.shape[1]
    mm = np.clip(np.asarray(masked_m, dtype=np.int64), 0, max_m)
    out = np.full((G, max_m, N), np.nan)
    for g in range(G):
        m = int(mm[g])
        if m:
            out[g, :m] = bf16_to_f64(a[g, :m]) @ bf16_to_f64(b[g]).T
    valid = np.arange(max_m)[None, :] < mm[:, None]
    return out, valid


def m_grouped_bf16_gemm_nt_masked_sampled(a, b, masked_m, groups, rows, cols):
    """Sampled outputs D[groups[i], rows[i], cols[i]] of the BF16 masked GEMM,
    one at a time; every sampled row must be inside its group's valid rows."""
    a = np.asarray(a, dtype=np.uint16)
    b = np.asarray(b, dtype=np.uint16)
    mm = np.clip(np.asarray(masked_m, dtype=np.int64), 0, a.shape[1])
    groups = np.asarray(groups, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    if np.any(rows >= mm[groups]):
        raise ValueError("sampled rows must be valid rows of their group")
    return np.einsum("ik,ik->i", bf16_to_f64(a[groups, rows]), bf16_to_f64(b[groups, cols]))
