"""Guard bands around D: no GEMM form writes outside its output.

D is a contiguous slice of a larger buffer whose every element starts as a
sentinel bit pattern: GUARD rows above D and GUARD rows below it. After the
call the bands must hold the sentinel bit for bit. M and N are chosen with
tails (M not a multiple of the 128/256-row tile, N not a multiple of the tile
width), so the stores the bands police are the edge cases: TMA stores clipped
at M and N, the predicated 16-byte stores of partial chunks (masked, psum_m,
contiguous forms), the fp32 epilogue's direct stores, split-K reductions and
CTA pairs whose second CTA lies past M. D is row-major with row pitch N, so a
store past column N of the last row lands in the lower band too; inside D such
a store would land in the next row, which the sentinel rows of the grouped
forms (rows past masked_m, padding rows, rows in no psum_m group) and the
oracle comparison of the valid rows police. The valid region is compared
with the oracle at the library's tolerance."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import SENTINEL_BITS, bf16_to_f64, check_fp

pytestmark = pytest.mark.gpu

GUARD = 3            # guard rows on each side of D
SENT16 = np.int16(np.uint16(SENTINEL_BITS).astype(np.int16))
SENT32 = np.int32(np.uint32(0xFFC1FFC1).astype(np.int32))   # an fp32 NaN pattern no epilogue writes


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.device_error(clear=True)
    yield
    dg.set_block_n(0)
    dg.set_cta_group(0)
    dg.set_splits(0)
    assert dg.device_error(clear=True) & dg.DEVERR_TIMEOUT == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _pack_dev(sf_f32):
    return dg.pack_ue8m0(_dev(sf_f32))


def _oracle_pack(sf_f32):
    return oracle.pack_ue8m0(sf_f32.reshape(-1, sf_f32.shape[-1])).reshape(*sf_f32.shape[:-1], -1)


class Guarded:
    """An output of `rows` x `n` elements between two bands of GUARD rows, all sentinel."""

    def __init__(self, rows, n, dtype=torch.bfloat16):
        self.rows, self.n, self.dtype = rows, n, dtype
        self.buf = torch.empty((rows + 2 * GUARD, n), dtype=dtype, device="cuda")
        self.ibuf = self.buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32)
        self.ibuf.fill_(SENT16 if dtype == torch.bfloat16 else SENT32)
        self.d = self.buf[GUARD:GUARD + rows]
        assert self.d.is_contiguous() and self.d.data_ptr() % 16 == 0

    def view(self, *shape):
        return self.d.view(*shape)

    def check_bands(self, what):
        torch.cuda.synchronize()
        sent = SENT16 if self.dtype == torch.bfloat16 else SENT32
        top = self.ibuf[:GUARD]
        bottom = self.ibuf[GUARD + self.rows:]
        assert (top == sent).all().item(), f"{what}: a store landed in the band above D"
        assert (bottom == sent).all().item(), f"{what}: a store landed in the band below D"

    def sentinel_mask(self):
        sent = SENT16 if self.dtype == torch.bfloat16 else SENT32
        return (self.ibuf[GUARD:GUARD + self.rows] == sent).cpu().numpy()


def _ref_dense(p):
    return oracle.fp8_gemm_nt(p["a"], _oracle_pack(p["sfa_f32"]), p["b"], _oracle_pack(p["sfb_f32"]))


# (M, N, K), tile width, CTA group, split count: M and N tails on single CTAs,
# pairs whose odd CTA is partly or wholly past M, and split-K
DENSE_CASES = [((200, 776, 2560), 128, 1, 1), ((200, 776, 2560), 256, 1, 1), ((77, 264, 1024), 96, 1, 1),
               ((300, 400, 1024), 160, 2, 1), ((129, 520, 1536), 256, 2, 1), ((1, 136, 1024), 224, 1, 1),
               ((300, 776, 1024), 240, 2, 1), ((257, 496, 1024), 240, 2, 1),
               ((64, 776, 4096), 128, 1, 4), ((200, 264, 2560), 64, 1, 3), ((130, 1000, 3200), 256, 1, 2)]


@pytest.mark.parametrize("mnk,bn,cg,splits", DENSE_CASES)
def test_dense_stays_inside_d(mnk, bn, cg, splits):
    M, N, K = mnk
    p = W.dense(M, N, K, seed=M + 3 * N)
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    out = Guarded(M, N)
    dg.fp8_gemm_nt(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]), out.d)
    out.check_bands(f"dense {mnk} bn={bn} cg={cg} splits={splits}")
    check_fp(bf16_to_f64(out.d), _ref_dense(p), f"dense {mnk}")


@pytest.mark.parametrize("out_f32", [False, True])
@pytest.mark.parametrize("mnk,bn,cg,splits", [((200, 776, 2560), 128, 1, 1), ((300, 400, 1024), 192, 2, 1),
                                             ((300, 776, 1024), 240, 2, 1),
                                             ((64, 520, 4096), 128, 1, 4)])
def test_accumulate_epilogue_stays_inside_d(mnk, bn, cg, splits, out_f32):
    M, N, K = mnk
    p = W.dense(M, N, K, seed=2 * M + N)
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    dtype = torch.float32 if out_f32 else torch.bfloat16
    out = Guarded(M, N, dtype)
    c = torch.from_numpy(np.random.default_rng(M).standard_normal((M, N)).astype(np.float32)).to(dtype).cuda()
    out.d.copy_(c)
    c_host = c.to(torch.float64).cpu().numpy()
    dg.fp8_gemm_nt_acc(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]), out.d, c=out.d)
    out.check_bands(f"acc {mnk} f32={out_f32}")
    check_fp(out.d.to(torch.float64).cpu().numpy(), c_host + _ref_dense(p), f"acc {mnk}")


@pytest.mark.parametrize("cg", [1, 2])
@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_operand_layouts_stay_inside_d(layout, cg):
    M, N, K = 208, 400, 1024
    p = W.dense(M, N, K, seed=9)
    dg.set_cta_group(cg)
    a = p["a"] if layout[0] == "n" else np.ascontiguousarray(p["a"].T)
    b = p["b"] if layout[1] == "t" else np.ascontiguousarray(p["b"].T)
    out = Guarded(M, N)
    getattr(dg, f"fp8_gemm_{layout}")(_dev(a), _pack_dev(p["sfa_f32"]), _dev(b), _pack_dev(p["sfb_f32"]), out.d)
    out.check_bands(f"layout {layout} cg={cg}")
    check_fp(bf16_to_f64(out.d), _ref_dense(p), f"layout {layout}")


@pytest.mark.parametrize("bn", [64, 160, 256])
def test_masked_stays_inside_d(bn):
    masked_m = np.array([0, 5, 128, 131, 200, 256, -3, 300], dtype=np.int32)
    G, max_m, N, K = 8, 256, 520, 1024
    p = W.masked(masked_m, max_m, N, K, seed=bn)
    dg.set_block_n(bn)
    out = Guarded(G * max_m, N)
    d = out.view(G, max_m, N)
    dg.m_grouped_fp8_gemm_nt_masked(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]),
                                    d, _dev(masked_m))
    out.check_bands(f"masked bn={bn}")
    ref, valid = oracle.m_grouped_fp8_gemm_nt_masked(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                     _oracle_pack(p["sfb_f32"]), masked_m)
    sent = out.sentinel_mask().reshape(G, max_m, N)
    assert sent[~valid].all(), "a row past masked_m was written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], f"masked bn={bn}")


@pytest.mark.parametrize("bn", [96, 256])
def test_bf16_masked_stays_inside_d(bn):
    masked_m = np.array([3, 0, 130, 256], dtype=np.int32)
    G, max_m, N, K = 4, 256, 264, 512
    p = W.masked_bf16(masked_m, max_m, N, K, seed=bn)
    dg.set_block_n(bn)
    out = Guarded(G * max_m, N)
    d = out.view(G, max_m, N)
    dg.m_grouped_bf16_gemm_nt_masked(_dev(p["a"]), _dev(p["b"]), d, _dev(masked_m))
    out.check_bands(f"bf16 masked bn={bn}")
    ref, valid = oracle.m_grouped_bf16_gemm_nt_masked(p["a"], p["b"], masked_m)
    sent = out.sentinel_mask().reshape(G, max_m, N)
    assert sent[~valid].all(), "a row past masked_m was written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], f"bf16 masked bn={bn}")


@pytest.mark.parametrize("bn", [64, 224])
def test_psum_stays_inside_d(bn):
    counts = np.array([70, 0, 129, 1, 200], dtype=np.int64)
    M_total, N, K = 440, 392, 1024          # rows 400..439 belong to no group
    p = W.psum(counts, M_total, N, K, seed=bn)
    dg.set_block_n(bn)
    out = Guarded(M_total, N)
    dg.m_grouped_fp8_gemm_nt_psum(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]),
                                  out.d, _dev(p["psum_m"]))
    out.check_bands(f"psum bn={bn}")
    ref, valid = oracle.m_grouped_fp8_gemm_nt_psum(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                   _oracle_pack(p["sfb_f32"]), p["psum_m"])
    sent = out.sentinel_mask()
    assert sent[~valid].all(), "a row in no group was written"
    check_fp(bf16_to_f64(out.d)[valid], ref[valid], f"psum bn={bn}")


@pytest.mark.parametrize("bn,cg", [(128, 1), (192, 1), (256, 2)])
def test_contiguous_stays_inside_d(bn, cg):
    counts = [100, 0, 300, 17]
    p = W.contiguous(counts, 392, 1024, seed=bn + cg, tail_blocks=1)
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    out = Guarded(p["M_total"], p["N"])
    dg.m_grouped_fp8_gemm_nt_contiguous(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]),
                                        _pack_dev(p["sfb_f32"]), out.d, _dev(p["m_indices"]))
    out.check_bands(f"contiguous bn={bn} cg={cg}")
    ref, valid = oracle.m_grouped_fp8_gemm_nt_contiguous(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                         _oracle_pack(p["sfb_f32"]), p["m_indices"])
    sent = out.sentinel_mask()
    assert sent[~valid].all(), "a padding row was written"
    check_fp(bf16_to_f64(out.d)[valid], ref[valid], f"contiguous bn={bn} cg={cg}")


@pytest.mark.parametrize("splits", [1, 4])
def test_noalloc_stays_inside_d(splits):
    M, N, K = 64, 776, 4096
    p = W.dense(M, N, K, seed=splits)
    dg.set_block_n(128)
    out = Guarded(M, N)
    dg.fp8_gemm_nt_noalloc(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]), out.d,
                           splits=splits)
    out.check_bands(f"noalloc splits={splits}")
    check_fp(bf16_to_f64(out.d), _ref_dense(p), f"noalloc splits={splits}")
