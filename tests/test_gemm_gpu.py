"""GEMM parity on the GPU vs the CPU oracle at sizes the oracle finishes in
seconds: several tiles, ragged M/N/K tails, every tile width, exact one-hot
cases, masked and contiguous forms with sentinel-checked untouched rows, and
CUDA Graph replay with new masked_m. All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp, fill_sentinel, is_sentinel

pytestmark = pytest.mark.gpu

BLOCK_NS = [64, 96, 128, 160, 192, 224, 256]


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.device_error(clear=True)
    yield
    dg.set_block_n(0)
    dg.set_cta_group(0)
    assert dg.device_error(clear=True) & dg.DEVERR_TIMEOUT == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _pack_dev(sf_f32):
    return dg.pack_ue8m0(_dev(sf_f32))


def _oracle_pack(sf_f32):
    return oracle.pack_ue8m0(sf_f32.reshape(-1, sf_f32.shape[-1])).reshape(*sf_f32.shape[:-1], -1)


def run_dense(p, bn=0, cg=0):
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    d = torch.empty((p["M"], p["N"]), dtype=torch.bfloat16, device="cuda")
    fill_sentinel(d)
    dg.fp8_gemm_nt(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]), d)
    torch.cuda.synchronize()
    return d


def ref_dense(p):
    return oracle.fp8_gemm_nt(p["a"], _oracle_pack(p["sfa_f32"]), p["b"], _oracle_pack(p["sfb_f32"]))


@pytest.mark.parametrize("bn", BLOCK_NS)
@pytest.mark.parametrize("mnk", [(128, 256, 512), (300, 400, 1024), (257, 264, 640),
                                 (64, 264, 1024), (17, 400, 640)])   # M <= 64: 64-row A stages
def test_dense_parity_every_tile_width(bn, mnk):
    p = W.dense(*mnk, seed=sum(mnk))
    d = run_dense(p, bn)
    assert not is_sentinel(d).any()
    check_fp(bf16_to_f64(d), ref_dense(p), f"dense {mnk} bn={bn}")


PAIR_BLOCK_NS = [128, 160, 192, 224, 256]
DENSE_PAIR_BLOCK_NS = PAIR_BLOCK_NS + [240]   # 240: a 16-column tail chunk, dense pairs only


@pytest.mark.parametrize("bn", DENSE_PAIR_BLOCK_NS)
@pytest.mark.parametrize("mnk", [(300, 400, 1024), (512, 256, 512), (257, 264, 640), (1024, 1000, 2048),
                                 (512, 776, 1024)])
def test_dense_parity_cta_pairs(bn, mnk):
    # 256-row tiles on CTA pairs; M not a multiple of 256 leaves the odd CTA
    # of the last pair partly or wholly past M
    p = W.dense(*mnk, seed=3 * sum(mnk))
    d = run_dense(p, bn, cg=2)
    assert not is_sentinel(d).any()
    check_fp(bf16_to_f64(d), ref_dense(p), f"dense pairs {mnk} bn={bn}")


@pytest.mark.parametrize("mnk", [(1, 16, 128), (64, 2112, 896), (128, 8, 128), (513, 1000, 2048)])
def test_dense_parity_edge_shapes(mnk):
    p = W.dense(*mnk, seed=7)
    d = run_dense(p)
    check_fp(bf16_to_f64(d), ref_dense(p), f"dense {mnk}")


def test_dense_workload0():
    p = W.workload0()
    check_fp(bf16_to_f64(run_dense(p)), ref_dense(p), "workload 0")


def _codes(rng, shape):
    s = rng.integers(0, 2, size=shape)
    e = rng.integers(4, 12, size=shape)
    m = rng.integers(0, 8, size=shape)
    return ((s << 7) | (e << 3) | m).astype(np.uint8)


def _pack_bytes_host(byts):
    rows, cols = byts.shape
    kp = (cols + 3) // 4
    w = np.zeros((rows, kp), dtype=np.int64)
    for c in range(cols):
        w[:, c // 4] |= byts[:, c].astype(np.int64) << (8 * (c % 4))
    return w.astype(np.uint32).view(np.int32)


@pytest.mark.parametrize("bn,cg", [(b, 1) for b in BLOCK_NS] + [(b, 2) for b in DENSE_PAIR_BLOCK_NS])
def test_one_hot_rows_are_bit_exact(bn, cg):
    # one-hot A rows with power-of-two scales: every output is a single product
    # e4m3 * 2^a * 2^b, exactly representable in bf16
    rng = np.random.default_rng(bn)
    M, N, K = 300, 304, 1152
    KB = K // 128
    ks = rng.integers(0, K, size=M)
    a = np.zeros((M, K), dtype=np.uint8)
    a[np.arange(M), ks] = 0x38
    ea = rng.integers(120, 134, size=(M, KB)).astype(np.uint8)
    eb = rng.integers(120, 134, size=(3, KB)).astype(np.uint8)
    b = _codes(rng, (N, K))
    sfa, sfb = _pack_bytes_host(ea), _pack_bytes_host(eb)
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt(_dev(a), _dev(sfa), _dev(b), _dev(sfb), d)
    want = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    want_bf16 = torch.from_numpy(want).to(torch.bfloat16)
    assert torch.equal(torch.from_numpy(want_bf16.to(torch.float64).numpy()), torch.from_numpy(want)), "not exact in bf16"
    assert torch.equal(d.cpu().view(torch.int16), want_bf16.view(torch.int16))


# ------------------------------------------------------------------ masked --

def run_masked(p, masked_m=None, bn=0):
    dg.set_block_n(bn)
    G, max_m, N = p["G"], p["max_m"], p["N"]
    d = fill_sentinel(torch.empty((G, max_m, N), dtype=torch.bfloat16, device="cuda"))
    mm = p["masked_m"] if masked_m is None else masked_m
    dg.m_grouped_fp8_gemm_nt_masked(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]), _pack_dev(p["sfb_f32"]),
                                    d, _dev(np.asarray(mm, dtype=np.int32)))
    torch.cuda.synchronize()
    return d


def check_masked(p, d, masked_m=None, what="masked"):
    mm = p["masked_m"] if masked_m is None else masked_m
    ref, valid = oracle.m_grouped_fp8_gemm_nt_masked(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                     _oracle_pack(p["sfb_f32"]), mm)
    sent = is_sentinel(d)
    assert sent[~valid].all(), f"{what}: a row past masked_m was written"
    assert not sent[valid].any(), f"{what}: a valid row was not written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], what)


@pytest.mark.parametrize("bn", [64, 96, 160, 256])
def test_masked_parity_and_sentinel(bn):
    mm = np.array([0, 1, 128, 200, 77, -3, 500], dtype=np.int32)
    p = W.masked(mm, 200, 272, 384, seed=11)
    d = run_masked(p, bn=bn)
    check_masked(p, d, what=f"masked bn={bn}")


def test_masked_all_empty_writes_nothing():
    p = W.masked(np.zeros(4, dtype=np.int32), 64, 128, 256, seed=12)
    d = run_masked(p)
    assert is_sentinel(d).all()


def test_masked_graph_replay_with_new_masked_m():
    G, max_m, N, K = 6, 256, 384, 512
    p = W.masked(np.full(G, max_m, dtype=np.int32), max_m, N, K, seed=13, fill_invalid_nan=False)
    a, b = _dev(p["a"]), _dev(p["b"])
    sfa, sfb = _pack_dev(p["sfa_f32"]), _pack_dev(p["sfb_f32"])
    mm_dev = torch.zeros(G, dtype=torch.int32, device="cuda")
    d = torch.empty((G, max_m, N), dtype=torch.bfloat16, device="cuda")
    dg.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, mm_dev)  # warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dg.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, mm_dev)
    rng = np.random.default_rng(5)
    for it in range(3):
        new = rng.integers(0, max_m + 1, size=G).astype(np.int32)
        new[it] = 0
        mm_dev.copy_(torch.from_numpy(new))
        fill_sentinel(d)
        g.replay()
        torch.cuda.synchronize()
        check_masked(p, d, masked_m=new, what=f"replay {it}")
    del g


# -------------------------------------------------------------- contiguous --

def run_contig(p, m_indices=None, bn=0):
    dg.set_block_n(bn)
    mi = p["m_indices"] if m_indices is None else m_indices
    d = fill_sentinel(torch.empty((p["M_total"], p["N"]), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_contiguous(_dev(p["a"]), _pack_dev(p["sfa_f32"]), _dev(p["b"]),
                                        _pack_dev(p["sfb_f32"]), d, _dev(mi))
    torch.cuda.synchronize()
    return d


def check_contig(p, d, m_indices=None, what="contiguous"):
    mi = p["m_indices"] if m_indices is None else m_indices
    ref, valid = oracle.m_grouped_fp8_gemm_nt_contiguous(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                         _oracle_pack(p["sfb_f32"]), mi)
    sent = is_sentinel(d)
    assert sent[~valid].all(), f"{what}: a padding row was written"
    assert not sent[valid].any(), f"{what}: a valid row was not written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], what)


@pytest.mark.parametrize("bn", [64, 192, 224, 256])
def test_contiguous_parity_and_padding(bn):
    p = W.contiguous([5, 0, 130, 128, 1], 264, 512, seed=21, tail_blocks=1)
    d = run_contig(p, bn=bn)
    check_contig(p, d, what=f"contiguous bn={bn}")
    assert dg.device_error(clear=True) == 0


CONTIG_PAIR_LAYOUTS = {
    # experts' 128-row block counts 1, 0, 2, 1, 1 and a padding block: pairs
    # (0,1) and (2,3) hold two experts each, pair (4,5) one expert and padding
    "boundaries": dict(counts=[5, 0, 130, 128, 1], tail_blocks=1),
    # odd block counts everywhere, some experts empty
    "odd": dict(counts=[300, 0, 129, 640, 1, 0, 257], tail_blocks=0),
    # an odd number of blocks in total: the last pair's second block is past M
    "odd_total": dict(counts=[200, 130], tail_blocks=0),
}


@pytest.mark.parametrize("bn", PAIR_BLOCK_NS)
@pytest.mark.parametrize("layout", sorted(CONTIG_PAIR_LAYOUTS))
def test_contiguous_parity_cta_pairs(bn, layout):
    # 256-row pair tiles over 128-row aligned experts: a pair whose blocks
    # belong to two experts is computed in two passes, one per expert
    lay = CONTIG_PAIR_LAYOUTS[layout]
    p = W.contiguous(lay["counts"], 264, 640, seed=17 + bn, tail_blocks=lay["tail_blocks"])
    dg.set_cta_group(2)
    d = run_contig(p, bn=bn)
    check_contig(p, d, what=f"contiguous pairs {layout} bn={bn}")
    assert dg.device_error(clear=True) == 0


@pytest.mark.parametrize("cg", [1, 2])
def test_contiguous_beyond_the_block_table(cg):
    # more 128-row blocks than the kernel keeps experts for in shared memory
    # (1024): the tile walk reads m_indices directly; sampled outputs and the
    # sentinel rows are checked
    counts = [128 * 300 + 5, 128 * 200, 128 * 410 + 77, 128 * 120 + 128]   # 1033 blocks
    p = W.contiguous(counts, 256, 256, seed=29, tail_blocks=2)
    assert p["M_total"] // 128 > 1024
    dg.set_cta_group(cg)
    d = run_contig(p)
    assert dg.device_error(clear=True) == 0
    mi = p["m_indices"]
    sent = is_sentinel(d)
    assert sent[mi < 0].all() and not sent[mi >= 0].any()
    rng = np.random.default_rng(5)
    rows = rng.choice(np.nonzero(mi >= 0)[0], 256, replace=False)
    cols = rng.integers(0, p["N"], 256)
    ref = oracle.m_grouped_fp8_gemm_nt_contiguous_sampled(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                          _oracle_pack(p["sfb_f32"]), mi, rows, cols)
    got = bf16_to_f64(d)[rows, cols]
    check_fp(got, ref, f"contiguous, {p['M_total'] // 128} blocks, cg={cg}")


def test_contiguous_pairs_leading_padding_block():
    p = W.contiguous([128, 300], 256, 512, seed=23)
    mi = p["m_indices"].copy()
    mi[0:128] = -1            # the first pair's first block holds padding only
    dg.set_cta_group(2)
    d = run_contig(p, m_indices=mi)
    check_contig(p, d, m_indices=mi, what="contiguous pairs, leading padding block")
    assert dg.device_error(clear=True) == 0


@pytest.mark.parametrize("cg", [1, 2])
def test_contiguous_mixed_block_is_flagged(cg):
    p = W.contiguous([100, 100], 128, 256, seed=22)
    mi = p["m_indices"].copy()
    mi[40:60] = 1  # expert 1 inside expert 0's first block
    dg.set_cta_group(cg)
    d = run_contig(p, m_indices=mi)
    assert dg.device_error(clear=True) & dg.DEVERR_MIXED_EXPERT_BLOCK
    # the block's rows of the larger index are computed, the others untouched
    sent = is_sentinel(d)
    assert sent[0:40].all() and sent[60:128].all()
    ref, _ = oracle.m_grouped_fp8_gemm_nt_contiguous(p["a"], _oracle_pack(p["sfa_f32"]), p["b"],
                                                     _oracle_pack(p["sfb_f32"]), mi)
    check_fp(bf16_to_f64(d)[40:60], ref[40:60], "mixed block rows")
    ok = np.nonzero(mi[128:] >= 0)[0] + 128
    check_fp(bf16_to_f64(d)[ok], ref[ok], "clean blocks")
