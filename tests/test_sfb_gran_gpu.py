"""Weights with one scale row per row of B (sfb_gran_n = 1) on the GPU vs the
CPU oracle ("DeepInside DeepGEMM", section 4: the minimal FP8 GEMM example
gives B a scale tensor [n, k / 128]). Dense (every tile width, CTA pairs,
split-K, C and fp32 output), masked and contiguous forms; exact one-hot cases;
granularity 128 through the same calls equals the plain calls bit for bit.
All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp, fill_sentinel, is_sentinel

pytestmark = pytest.mark.gpu

BLOCK_NS = [64, 96, 128, 160, 192, 224, 256]
PAIR_BLOCK_NS = [128, 160, 192, 224, 256]
DENSE_PAIR_BLOCK_NS = PAIR_BLOCK_NS + [240]   # 240: dense pairs only


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.device_error(clear=True)
    yield
    dg.set_block_n(0)
    dg.set_cta_group(0)
    dg.set_splits(0)
    assert dg.device_error(clear=True) == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _opack(sf_f32):
    return oracle.pack_ue8m0(sf_f32.reshape(-1, sf_f32.shape[-1])).reshape(*sf_f32.shape[:-1], -1)


def _dense(p, bn=0, cg=0, splits=0, c=None, out=torch.bfloat16):
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    d = torch.empty((p["M"], p["N"]), dtype=out, device="cuda")
    if out == torch.bfloat16:
        fill_sentinel(d)
    dg.fp8_gemm_nt_sfb_gran(_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]),
                            dg.pack_ue8m0(_dev(p["sfb_f32"])), d, 1, c=c)
    torch.cuda.synchronize()
    return d


def _ref(p, c=None):
    return oracle.fp8_gemm_nt_acc(p["a"], _opack(p["sfa_f32"]), p["b"], _opack(p["sfb_f32"]), c=c, sfb_gran_n=1)


@pytest.mark.parametrize("bn", BLOCK_NS)
@pytest.mark.parametrize("mnk", [(300, 400, 1024), (257, 264, 640)])
def test_dense_every_tile_width(bn, mnk):
    p = W.dense(*mnk, seed=11 * sum(mnk), sfb_gran_n=1)
    assert p["sfb_f32"].shape == (mnk[1], mnk[2] // 128)
    d = _dense(p, bn)
    assert not is_sentinel(d).any()
    check_fp(bf16_to_f64(d), _ref(p), f"per-row B scales {mnk} bn={bn}")


@pytest.mark.parametrize("bn", DENSE_PAIR_BLOCK_NS)
def test_dense_cta_pairs(bn):
    p = W.dense(300, 520, 1024, seed=bn, sfb_gran_n=1)
    d = _dense(p, bn, cg=2)
    check_fp(bf16_to_f64(d), _ref(p), f"per-row B scales, pairs bn={bn}")


@pytest.mark.parametrize("splits", [2, 3, 5])
def test_dense_split_k(splits):
    p = W.dense(64, 400, 4096, seed=50 + splits, sfb_gran_n=1)  # 8 groups of 4 K-blocks
    d = _dense(p, 64, cg=1, splits=splits)
    check_fp(bf16_to_f64(d), _ref(p), f"per-row B scales, {splits} splits")


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_dense_with_c(out):
    p = W.dense(200, 264, 768, seed=60, sfb_gran_n=1)
    c_host = np.random.default_rng(61).standard_normal((200, 264)).astype(np.float32)
    c = torch.from_numpy(c_host).to(out).cuda()
    c_vals = c.cpu().to(torch.float64).numpy()
    d = _dense(p, c=c, out=out)
    got = d.cpu().to(torch.float64).numpy()
    check_fp(got, _ref(p, c=c_vals), f"per-row B scales, C, {out}")


@pytest.mark.parametrize("bn,cg", [(b, 1) for b in BLOCK_NS] + [(b, 2) for b in DENSE_PAIR_BLOCK_NS])
def test_one_hot_rows_are_bit_exact(bn, cg):
    # one-hot A rows, power-of-two scales, a different scale row for every row
    # of B: each output is one product e4m3 * 2^a * 2^b, exact in bf16
    rng = np.random.default_rng(100 + bn + cg)
    M, N, K = 300, 304, 1152
    KB = K // 128
    ks = rng.integers(0, K, size=M)
    a = np.zeros((M, K), dtype=np.uint8)
    a[np.arange(M), ks] = 0x38
    ea = rng.integers(120, 134, size=(M, KB)).astype(np.uint8)
    eb = rng.integers(118, 137, size=(N, KB)).astype(np.uint8)
    s = rng.integers(0, 2, size=(N, K))
    e = rng.integers(4, 12, size=(N, K))
    m = rng.integers(0, 8, size=(N, K))
    b = ((s << 7) | (e << 3) | m).astype(np.uint8)
    sfa = oracle.pack_ue8m0(np.ldexp(1.0, ea.astype(np.int64) - 127).astype(np.float32))
    sfb = oracle.pack_ue8m0(np.ldexp(1.0, eb.astype(np.int64) - 127).astype(np.float32))
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt_sfb_gran(_dev(a), _dev(sfa), _dev(b), _dev(sfb), d, 1)
    want = oracle.fp8_gemm_nt(a, sfa, b, sfb, sfb_gran_n=1)
    want_bf16 = torch.from_numpy(want).to(torch.bfloat16)
    assert np.array_equal(want_bf16.to(torch.float64).numpy(), want), "not exact in bf16"
    assert torch.equal(d.cpu().view(torch.int16), want_bf16.view(torch.int16))


def test_granularity_128_equals_the_plain_calls():
    p = W.dense(257, 400, 1024, seed=70)
    a, b = _dev(p["a"]), _dev(p["b"])
    sfa, sfb = dg.pack_ue8m0(_dev(p["sfa_f32"])), dg.pack_ue8m0(_dev(p["sfb_f32"]))
    d0 = torch.empty((257, 400), dtype=torch.bfloat16, device="cuda")
    d1 = torch.empty_like(d0)
    dg.fp8_gemm_nt(a, sfa, b, sfb, d0)
    dg.fp8_gemm_nt_sfb_gran(a, sfa, b, sfb, d1, 128)
    torch.cuda.synchronize()
    assert torch.equal(d0.view(torch.int16), d1.view(torch.int16))
    q = W.masked(np.array([30, 0, 129], np.int32), 160, 256, 512, seed=71)
    args = (_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]), dg.pack_ue8m0(_dev(q["sfb_f32"])))
    m0 = fill_sentinel(torch.empty((3, 160, 256), dtype=torch.bfloat16, device="cuda"))
    m1 = fill_sentinel(torch.empty_like(m0))
    mm = _dev(q["masked_m"])
    dg.m_grouped_fp8_gemm_nt_masked(*args, m0, mm)
    dg.m_grouped_fp8_gemm_nt_masked_sfb_gran(*args, m1, mm, 128)
    torch.cuda.synchronize()
    assert torch.equal(m0.view(torch.int16), m1.view(torch.int16))


@pytest.mark.parametrize("bn", [0, 64, 128, 256])
def test_masked_parity_and_sentinel(bn):
    mm = np.array([1, 0, 129, 256, 67, 300, -5], dtype=np.int32)  # empty, ragged, full, clamped
    q = W.masked(mm, 256, 384, 768, seed=80 + bn, sfb_gran_n=1)
    assert q["sfb_f32"].shape == (7, 384, 6)
    dg.set_block_n(bn)
    d = fill_sentinel(torch.empty((7, 256, 384), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_masked_sfb_gran(_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]),
                                             dg.pack_ue8m0(_dev(q["sfb_f32"])), d, _dev(mm), 1)
    torch.cuda.synchronize()
    ref, valid = oracle.m_grouped_fp8_gemm_nt_masked(q["a"], _opack(q["sfa_f32"]), q["b"], _opack(q["sfb_f32"]), mm,
                                                     sfb_gran_n=1)
    sent = is_sentinel(d)
    assert sent[~valid].all(), "rows outside masked_m were written"
    assert not sent[valid].any()
    check_fp(bf16_to_f64(d)[valid], ref[valid], f"masked, per-row B scales, bn={bn}")


@pytest.mark.parametrize("cg", [1, 2])
def test_contiguous_parity_and_padding(cg):
    q = W.contiguous([130, 0, 300, 5], 264, 640, seed=90 + cg, tail_blocks=1, sfb_gran_n=1)
    dg.set_cta_group(cg)
    d = fill_sentinel(torch.empty((q["M_total"], q["N"]), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_contiguous_sfb_gran(_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]),
                                                 dg.pack_ue8m0(_dev(q["sfb_f32"])), d, _dev(q["m_indices"]), 1)
    torch.cuda.synchronize()
    ref, valid = oracle.m_grouped_fp8_gemm_nt_contiguous(q["a"], _opack(q["sfa_f32"]), q["b"], _opack(q["sfb_f32"]),
                                                         q["m_indices"], sfb_gran_n=1)
    sent = is_sentinel(d)
    assert sent[~valid].all(), "padding rows were written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], f"contiguous, per-row B scales, cg={cg}")


# ---- 16-byte scale-row reads vs one-word reads ----------------------------------
# With B scaled per row, packed scale rows of a multiple of four words on 16-byte
# aligned bases are read four K groups at a time; the same scales at a 4-byte
# offset take the one-word path. Both must give identical bits (granularity 128
# compares the one-word path with itself at two alignments).

def _offset_copy(t):
    """The same values in a buffer that starts 4 bytes past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 16 == 4
    return v


@pytest.mark.parametrize("gran,bn,cg,splits", [(128, 0, 0, 0), (1, 0, 0, 0), (128, 128, 2, 0), (1, 224, 2, 0),
                                               (128, 64, 1, 5), (1, 96, 1, 5), (1, 256, 1, 3)])
def test_vector_scale_reads_equal_word_reads_dense(gran, bn, cg, splits):
    # K = 6144: 12 packed words per row; 5 split ranges start at groups 0, 2, 4, 7, 9
    M, N, K = 300 if splits == 0 else 64, 392, 6144
    p = W.dense(M, N, K, seed=200 + bn + splits + gran, sfb_gran_n=gran)
    a, b = _dev(p["a"]), _dev(p["b"])
    sfa, sfb = dg.pack_ue8m0(_dev(p["sfa_f32"])), dg.pack_ue8m0(_dev(p["sfb_f32"]))
    assert sfa.data_ptr() % 16 == 0 and sfb.data_ptr() % 16 == 0 and sfa.shape[1] % 4 == 0
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    d0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    d1 = torch.empty_like(d0)
    dg.fp8_gemm_nt_sfb_gran(a, sfa, b, sfb, d0, gran)
    dg.fp8_gemm_nt_sfb_gran(a, _offset_copy(sfa), b, _offset_copy(sfb), d1, gran)
    torch.cuda.synchronize()
    assert torch.equal(d0.view(torch.int16), d1.view(torch.int16))
    check_fp(bf16_to_f64(d0), _ref(p) if gran == 1 else
             oracle.fp8_gemm_nt(p["a"], _opack(p["sfa_f32"]), p["b"], _opack(p["sfb_f32"])), "16-byte scale reads")


@pytest.mark.parametrize("gran", [128, 1])
def test_vector_scale_reads_equal_word_reads_grouped(gran):
    mm = np.array([1, 0, 129, 256, 67], dtype=np.int32)
    q = W.masked(mm, 256, 264, 2048, seed=210 + gran, sfb_gran_n=gran)
    args = [_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]), dg.pack_ue8m0(_dev(q["sfb_f32"]))]
    m0 = fill_sentinel(torch.empty((5, 256, 264), dtype=torch.bfloat16, device="cuda"))
    m1 = fill_sentinel(torch.empty_like(m0))
    mmd = _dev(mm)
    dg.m_grouped_fp8_gemm_nt_masked_sfb_gran(*args, m0, mmd, gran)
    dg.m_grouped_fp8_gemm_nt_masked_sfb_gran(args[0], _offset_copy(args[1]), args[2], _offset_copy(args[3]), m1, mmd,
                                             gran)
    torch.cuda.synchronize()
    assert torch.equal(m0.view(torch.int16), m1.view(torch.int16))
    ref, valid = oracle.m_grouped_fp8_gemm_nt_masked(q["a"], _opack(q["sfa_f32"]), q["b"], _opack(q["sfb_f32"]), mm,
                                                     sfb_gran_n=gran)
    check_fp(bf16_to_f64(m0)[valid], ref[valid], "masked, 16-byte scale reads")
    for cg in (1, 2):
        c = W.contiguous([130, 0, 300], 264, 4096, seed=220 + gran + cg, sfb_gran_n=gran)
        args = [_dev(c["a"]), dg.pack_ue8m0(_dev(c["sfa_f32"])), _dev(c["b"]), dg.pack_ue8m0(_dev(c["sfb_f32"]))]
        dg.set_cta_group(cg)
        c0 = fill_sentinel(torch.empty((c["M_total"], 264), dtype=torch.bfloat16, device="cuda"))
        c1 = fill_sentinel(torch.empty_like(c0))
        idx = _dev(c["m_indices"])
        dg.m_grouped_fp8_gemm_nt_contiguous_sfb_gran(*args, c0, idx, gran)
        dg.m_grouped_fp8_gemm_nt_contiguous_sfb_gran(args[0], _offset_copy(args[1]), args[2], _offset_copy(args[3]),
                                                     c1, idx, gran)
        torch.cuda.synchronize()
        assert torch.equal(c0.view(torch.int16), c1.view(torch.int16)), cg
