"""Seeded synthetic inputs shaped like DeepSeek-style dense and MoE layers.

This module only draws random numbers and quantises them to the operand format
(E4M3 bytes with one power-of-two fp32 scale per block). It holds none of the
library's arithmetic: it does not pack scales, decode E4M3 or multiply, and it
never calls the CUDA library. Tests and the benchmark feed the same arrays to
the CUDA path and to the CPU oracle.

Quantisation recipe (input preparation only): for every block (1x128 along K
for activations, 128x128 for weights) the scale is
s = 2^ceil(log2(max(amax, 1e-4) / 448)) and the stored byte is
``float8_e4m3fn(x / s)`` (round to nearest even, |x / s| <= 448 so nothing
saturates). Scales are returned as fp32 powers of two, i.e. valid UE8M0
inputs to the pack step.

Weights scaled per row (``sfb_gran_n=1``: one scale per 1x128 block of each row
of B, scales [N, K/128]) are quantised like activations; before quantisation
each row of B is multiplied by 2^u, u uniform on {-3..3}, so that neighbouring
scale rows differ as per-channel weight scales do.

Workloads (seed = 1000 + workload number, numpy PCG64):
  0  dense M=128, N=256, K=512
  1  dense M in {64, 4096} x (N, K) in {(2112,7168), (24576,1536), (7168,16384), (4096,7168)}
  2  contiguous, 8 experts, rows per expert U{3072..5120} padded to 128, N=4096, K=7168
  3  masked, 32 groups, max_m=256, masked_m U{67..124}; up (4096,7168), down (7168,2048)
  4  masked, 256 groups, max_m=512, masked_m ~ Zipf(1.1) on {0..512}, (7168,2048)
BF16 masked problems (masked_bf16 / masked_bf16_t) use workload 3's shapes and
masked_m with plain bf16 operands.
"""

from __future__ import annotations

import numpy as np
import torch

BLOCK = 128
E4M3_MAX = 448.0
AMAX_FLOOR = 1e-4
NAN_BYTE = 0x7F  # an E4M3 NaN pattern, used to fill rows that must not be read

DENSE_NK = [(2112, 7168), (24576, 1536), (7168, 16384), (4096, 7168)]
DENSE_M = [64, 4096]


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _pow2_ceil_ratio(amax: np.ndarray) -> np.ndarray:
    """2^ceil(log2(max(amax, floor) / 448)) computed exactly with frexp."""
    v = np.maximum(amax.astype(np.float64), AMAX_FLOOR) / E4M3_MAX
    mant, exp = np.frexp(v)  # v = mant * 2^exp, mant in [0.5, 1)
    e = np.where(mant == 0.5, exp - 1, exp)
    return np.ldexp(1.0, e).astype(np.float32)


def _to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quantise_rows(x: np.ndarray):
    """x float32 [R, K] -> (bytes uint8 [R, K], scales float32 [R, K/128])."""
    R, K = x.shape
    assert K % BLOCK == 0
    xb = x.reshape(R, K // BLOCK, BLOCK)
    s = _pow2_ceil_ratio(np.abs(xb).max(axis=2))
    q = _to_e4m3_bytes(xb / s[:, :, None]).reshape(R, K)
    return q, s


def quantise_blocks(w: np.ndarray):
    """w float32 [N, K] -> (bytes uint8 [N, K], scales float32 [ceil(N/128), K/128])."""
    N, K = w.shape
    assert K % BLOCK == 0
    NB = (N + BLOCK - 1) // BLOCK
    pad = np.zeros((NB * BLOCK, K), dtype=np.float32)
    pad[:N] = w
    wb = pad.reshape(NB, BLOCK, K // BLOCK, BLOCK)
    s = _pow2_ceil_ratio(np.abs(wb).max(axis=(1, 3)))
    q = _to_e4m3_bytes(wb / s[:, None, :, None]).reshape(NB * BLOCK, K)[:N]
    return np.ascontiguousarray(q), s


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def quantise_weights(rng, N: int, K: int, sfb_gran_n: int = BLOCK):
    """Random weights [N, K] quantised per 128x128 block (sfb_gran_n=128) or per
    1x128 block of each row (sfb_gran_n=1, with the per-row spread above)."""
    w = _normal(rng, (N, K))
    if sfb_gran_n == BLOCK:
        return quantise_blocks(w)
    if sfb_gran_n != 1:
        raise ValueError(f"sfb_gran_n={sfb_gran_n}")
    spread = np.ldexp(1.0, rng.integers(-3, 4, size=N)).astype(np.float32)
    return quantise_rows(w * spread[:, None])


def dense(M: int, N: int, K: int, seed: int, sfb_gran_n: int = BLOCK):
    """Dense NT problem: a [M,K], sfa_f32 [M,K/128], b [N,K], sfb_f32 [ceil(N/gran),K/128]."""
    rng = rng_for(seed)
    a, sfa = quantise_rows(_normal(rng, (M, K)))
    b, sfb = quantise_weights(rng, N, K, sfb_gran_n)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, M=M, N=N, K=K)


def grouped_weights(rng, G: int, N: int, K: int, sfb_gran_n: int = BLOCK):
    bs, sfbs = [], []
    for _ in range(G):
        b, sfb = quantise_weights(rng, N, K, sfb_gran_n)
        bs.append(b)
        sfbs.append(sfb)
    return np.stack(bs), np.stack(sfbs)


def contiguous(counts, N: int, K: int, seed: int, align: int = BLOCK, tail_blocks: int = 0,
               sfb_gran_n: int = BLOCK):
    """Contiguous M-grouped problem.

    Expert g owns ``counts[g]`` real rows, padded with -1 rows up to a multiple
    of ``align``; ``tail_blocks`` extra all-padding blocks are appended. Padding
    rows of A hold NaN bytes.
    """
    rng = rng_for(seed)
    G = len(counts)
    seg = [((c + align - 1) // align) * align for c in counts]
    M_total = int(sum(seg)) + tail_blocks * align
    m_indices = np.full(M_total, -1, dtype=np.int32)
    off = 0
    for g, (c, s) in enumerate(zip(counts, seg)):
        m_indices[off:off + c] = g
        off += s
    a = np.full((M_total, K), NAN_BYTE, dtype=np.uint8)
    sfa = np.ones((M_total, K // BLOCK), dtype=np.float32)
    valid = m_indices >= 0
    qa, qs = quantise_rows(_normal(rng, (int(valid.sum()), K)))
    a[valid] = qa
    sfa[valid] = qs
    b, sfb = grouped_weights(rng, G, N, K, sfb_gran_n)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, m_indices=m_indices,
                M_total=M_total, N=N, K=K, G=G)


def psum(counts, M_total: int, N: int, K: int, seed: int, sfb_gran_n: int = BLOCK):
    """Grouped problem with the groups given by psum_m: group g owns counts[g]
    rows, the groups' rows end to end from row 0 without padding; psum_m is
    the running total of counts. Rows past sum(counts) (up to M_total) belong
    to no group and hold NaN bytes."""
    rng = rng_for(seed)
    counts = np.asarray(counts, dtype=np.int64)
    G = counts.shape[0]
    used = int(counts.sum())
    assert used <= M_total
    a = np.full((M_total, K), NAN_BYTE, dtype=np.uint8)
    sfa = np.ones((M_total, K // BLOCK), dtype=np.float32)
    qa, qs = quantise_rows(_normal(rng, (used, K)))
    a[:used] = qa
    sfa[:used] = qs
    b, sfb = grouped_weights(rng, G, N, K, sfb_gran_n)
    psum_m = np.cumsum(counts).astype(np.int32)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, psum_m=psum_m, M_total=M_total, N=N, K=K, G=G)


def masked(masked_m, max_m: int, N: int, K: int, seed: int, fill_invalid_nan: bool = True,
           sfb_gran_n: int = BLOCK):
    """Masked M-grouped problem: a [G,max_m,K], b [G,N,K]; rows >= masked_m hold NaN bytes."""
    rng = rng_for(seed)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = masked_m.shape[0]
    x = _normal(rng, (G * max_m, K))
    a, sfa = quantise_rows(x)
    a = a.reshape(G, max_m, K)
    sfa = sfa.reshape(G, max_m, K // BLOCK)
    if fill_invalid_nan:
        rows = np.arange(max_m)[None, :] >= np.clip(masked_m, 0, max_m)[:, None]
        a[rows] = NAN_BYTE
    b, sfb = grouped_weights(rng, G, N, K, sfb_gran_n)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, masked_m=masked_m,
                G=G, max_m=max_m, N=N, K=K)


# ---- the five workloads -------------------------------------------------

def workload0():
    return dense(128, 256, 512, seed=1000)


def workload1(M: int, N: int, K: int):
    return dense(M, N, K, seed=1001)


def contiguous_counts(seed: int = 1002, G: int = 8, lo: int = 3072, hi: int = 5120):
    return rng_for(seed).integers(lo, hi + 1, size=G)


def workload2():
    counts = contiguous_counts()
    return contiguous(counts, 4096, 7168, seed=1002)


def masked_m_uniform(rng, G: int = 32, expected: int = 96):
    lo, hi = int(np.floor(0.7 * expected)), int(np.floor(1.3 * expected))
    return rng.integers(lo, hi + 1, size=G).astype(np.int32)


def workload3(proj: str):
    N, K = (4096, 7168) if proj == "up" else (7168, 2048)
    mm = masked_m_uniform(rng_for(1003))
    return masked(mm, 256, N, K, seed=1003)


def zipf_masked_m(rng, G: int = 256, max_m: int = 512, a: float = 1.1):
    """masked_m drawn with p(m) proportional to (m+1)^-a on {0..max_m}."""
    m = np.arange(max_m + 1)
    p = (m + 1.0) ** (-a)
    p /= p.sum()
    return rng.choice(m, size=G, p=p).astype(np.int32)


def workload4():
    mm = zipf_masked_m(rng_for(1004))
    return masked(mm, 512, 7168, 2048, seed=1004, fill_invalid_nan=False)


# ---- BF16 masked problems ---------------------------------------------------
#
# Operands of the BF16 masked grouped GEMM are plain bf16 values (no scales):
# N(0,1) draws rounded to bf16 (round to nearest even on the fp32 bit
# pattern), stored as uint16 bit patterns. Rows past masked_m hold a NaN
# pattern so that a kernel that reads them would be caught.

BF16_NAN = 0x7FC1


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def masked_bf16(masked_m, max_m: int, N: int, K: int, seed: int, fill_invalid_nan: bool = True):
    """BF16 masked M-grouped problem: a [G,max_m,K], b [G,N,K] as uint16 bf16 bits."""
    rng = rng_for(seed)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = masked_m.shape[0]
    a = _to_bf16_bits(_normal(rng, (G, max_m, K)))
    if fill_invalid_nan:
        rows = np.arange(max_m)[None, :] >= np.clip(masked_m, 0, max_m)[:, None]
        a[rows] = BF16_NAN
    b = _to_bf16_bits(_normal(rng, (G, N, K)))
    return dict(a=a, b=b, masked_m=masked_m, G=G, max_m=max_m, N=N, K=K)


# ---- device-side generation for full-size workloads ------------------------
#
# Same recipe as above (N(0,1) draws, power-of-two block scales from the block
# amax, E4M3 round-to-nearest-even), drawn with torch's seeded generator on the
# target device so that multi-GB weights are produced in milliseconds. The
# random stream differs from numpy's; tests that use these inputs copy them to
# the host for the oracle.

def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _pow2_scale_t(amax: torch.Tensor) -> torch.Tensor:
    v = amax.to(torch.float64).clamp_min(AMAX_FLOOR) / E4M3_MAX
    mant, exp = torch.frexp(v)
    e = torch.where(mant == 0.5, exp - 1, exp)
    return torch.ldexp(torch.ones_like(v), e).to(torch.float32)


def quantise_rows_t(x: torch.Tensor):
    """x float32 [R, K] (any device) -> (uint8 [R, K], float32 [R, K/128])."""
    R, K = x.shape
    xb = x.view(R, K // BLOCK, BLOCK)
    s = _pow2_scale_t(xb.abs().amax(dim=2))
    q = (xb / s[:, :, None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(R, K)
    return q, s


def quantise_blocks_t(w: torch.Tensor):
    """w float32 [N, K] -> (uint8 [N, K], float32 [ceil(N/128), K/128])."""
    N, K = w.shape
    NB = (N + BLOCK - 1) // BLOCK
    if NB * BLOCK != N:
        w = torch.cat([w, torch.zeros((NB * BLOCK - N, K), dtype=w.dtype, device=w.device)])
    wb = w.view(NB, BLOCK, K // BLOCK, BLOCK)
    s = _pow2_scale_t(wb.abs().amax(dim=(1, 3)))
    q = (wb / s[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(NB * BLOCK, K)[:N]
    return q.contiguous(), s


def dense_t(M: int, N: int, K: int, seed: int, device="cuda"):
    g = _gen(device, seed)
    a, sfa = quantise_rows_t(torch.randn((M, K), generator=g, device=device))
    b, sfb = quantise_blocks_t(torch.randn((N, K), generator=g, device=device))
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, M=M, N=N, K=K)


def grouped_weights_t(g, G: int, N: int, K: int, device):
    NB = (N + BLOCK - 1) // BLOCK
    b = torch.empty((G, N, K), dtype=torch.uint8, device=device)
    sfb = torch.empty((G, NB, K // BLOCK), dtype=torch.float32, device=device)
    for i in range(G):
        b[i], sfb[i] = quantise_blocks_t(torch.randn((N, K), generator=g, device=device))
    return b, sfb


def contiguous_t(counts, N: int, K: int, seed: int, align: int = BLOCK, device="cuda"):
    G = len(counts)
    seg = [((int(c) + align - 1) // align) * align for c in counts]
    M_total = int(sum(seg))
    mi = np.full(M_total, -1, dtype=np.int32)
    off = 0
    for e, (c, s) in enumerate(zip(counts, seg)):
        mi[off:off + int(c)] = e
        off += s
    g = _gen(device, seed)
    a, sfa = quantise_rows_t(torch.randn((M_total, K), generator=g, device=device))
    b, sfb = grouped_weights_t(g, G, N, K, device)
    m_indices = torch.from_numpy(mi).to(device)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, m_indices=m_indices, M_total=M_total, N=N, K=K, G=G)


def psum_t(counts, N: int, K: int, seed: int, device="cuda"):
    """psum on the device: the groups' rows end to end (M_total = sum(counts))."""
    G = len(counts)
    M_total = int(sum(int(c) for c in counts))
    g = _gen(device, seed)
    a, sfa = quantise_rows_t(torch.randn((M_total, K), generator=g, device=device))
    b, sfb = grouped_weights_t(g, G, N, K, device)
    psum_m = torch.from_numpy(np.cumsum(np.asarray(counts, dtype=np.int64)).astype(np.int32)).to(device)
    return dict(a=a, sfa_f32=sfa, b=b, sfb_f32=sfb, psum_m=psum_m, M_total=M_total, N=N, K=K, G=G)


def masked_t(masked_m, max_m: int, N: int, K: int, seed: int, device="cuda"):
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = masked_m.shape[0]
    g = _gen(device, seed)
    a, sfa = quantise_rows_t(torch.randn((G * max_m, K), generator=g, device=device))
    b, sfb = grouped_weights_t(g, G, N, K, device)
    return dict(a=a.view(G, max_m, K), sfa_f32=sfa.view(G, max_m, K // BLOCK), b=b, sfb_f32=sfb,
                masked_m=torch.from_numpy(masked_m).to(device), masked_m_host=masked_m,
                G=G, max_m=max_m, N=N, K=K)


def masked_bf16_t(masked_m, max_m: int, N: int, K: int, seed: int, device="cuda"):
    """BF16 masked problem drawn on the device (torch bfloat16 tensors)."""
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = masked_m.shape[0]
    g = _gen(device, seed)
    a = torch.randn((G, max_m, K), generator=g, device=device).to(torch.bfloat16)
    b = torch.randn((G, N, K), generator=g, device=device).to(torch.bfloat16)
    return dict(a=a, b=b, masked_m=torch.from_numpy(masked_m).to(device), masked_m_host=masked_m,
                G=G, max_m=max_m, N=N, K=K)


def workload1_t(M: int, N: int, K: int, device="cuda"):
    return dense_t(M, N, K, seed=1001 + 7 * M + N, device=device)


def workload2_t(device="cuda"):
    return contiguous_t(contiguous_counts(), 4096, 7168, seed=1002, device=device)


def workload3_t(proj: str, device="cuda"):
    N, K = (4096, 7168) if proj == "up" else (7168, 2048)
    return masked_t(masked_m_uniform(rng_for(1003)), 256, N, K, seed=1003, device=device)


def workload4_t(device="cuda"):
    return masked_t(zipf_masked_m(rng_for(1004)), 512, 7168, 2048, seed=1004, device=device)
