"""Grouped FP8 GEMM with the groups given by psum_m, on the GPU vs the CPU
oracle. Reading of "DeepGEMM CUDA Graph Compatibility for Masked Grouped
GEMMs", Tensor-Based Metadata Arguments: psum_m[g] is the inclusive prefix sum
of the groups' row counts; group g owns rows [psum_m[g-1], psum_m[g]) of an
unpadded A. Groups start at any row (tiles straddle group boundaries), empty
groups, rows in no group (sentinel must survive), malformed psum_m (negative,
decreasing, past M_total), every tile width, exact one-hot cases, and CUDA
Graph replay with new psum_m. All calls go through the C ABI."""

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
    assert dg.device_error(clear=True) == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _opack(sf_f32):
    return oracle.pack_ue8m0(sf_f32.reshape(-1, sf_f32.shape[-1])).reshape(*sf_f32.shape[:-1], -1)


def _run(q, psum_m=None, bn=0):
    dg.set_block_n(bn)
    d = fill_sentinel(torch.empty((q["M_total"], q["N"]), dtype=torch.bfloat16, device="cuda"))
    ps = q["psum_m"] if psum_m is None else np.asarray(psum_m, dtype=np.int32)
    dg.m_grouped_fp8_gemm_nt_psum(_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]),
                                  dg.pack_ue8m0(_dev(q["sfb_f32"])), d, _dev(ps))
    torch.cuda.synchronize()
    return d, ps


def _check(q, d, ps, what):
    ref, valid = oracle.m_grouped_fp8_gemm_nt_psum(q["a"], _opack(q["sfa_f32"]), q["b"], _opack(q["sfb_f32"]), ps)
    sent = is_sentinel(d)
    assert sent[~valid].all(), f"{what}: rows in no group were written"
    assert not sent[valid].any(), f"{what}: rows of a group were not written"
    if valid.any():
        check_fp(bf16_to_f64(d)[valid], ref[valid], what)


@pytest.mark.parametrize("bn", BLOCK_NS)
def test_psum_parity_every_tile_width(bn):
    # boundaries inside 128-row blocks, an empty group, a 1-row group, 37 rows in no group
    counts = [37, 0, 200, 1, 129, 96]
    q = W.psum(counts, sum(counts) + 37, 264, 640, seed=300 + bn)
    d, ps = _run(q, bn=bn)
    _check(q, d, ps, f"psum bn={bn}")


@pytest.mark.parametrize("psum_m", [[-3, 50, 20, 300, 900], [0, 0, 0, 0, 0], [400, 400, 400, 400, 400],
                                    [130, 129, 260, 391, 392]])
def test_psum_malformed_and_degenerate(psum_m):
    q = W.psum([100, 100, 100, 100], 400, 136, 512, seed=310)
    q["b"] = np.concatenate([q["b"], q["b"][:1]])          # five groups of weights
    q["sfb_f32"] = np.concatenate([q["sfb_f32"], q["sfb_f32"][:1]])
    d, ps = _run(q, psum_m=psum_m)
    _check(q, d, ps, f"psum {psum_m}")


def test_psum_one_hot_rows_are_bit_exact():
    rng = np.random.default_rng(320)
    M, N, K, G = 300, 200, 1152, 3
    KB = K // 128
    ks = rng.integers(0, K, size=M)
    a = np.zeros((M, K), dtype=np.uint8)
    a[np.arange(M), ks] = 0x38
    ea = rng.integers(120, 134, size=(M, KB)).astype(np.uint8)
    eb = rng.integers(120, 134, size=(G, 2, KB)).astype(np.uint8)
    s = rng.integers(0, 2, size=(G, N, K))
    e = rng.integers(4, 12, size=(G, N, K))
    m = rng.integers(0, 8, size=(G, N, K))
    b = ((s << 7) | (e << 3) | m).astype(np.uint8)
    sfa = oracle.pack_ue8m0(np.ldexp(1.0, ea.astype(np.int64) - 127).astype(np.float32))
    sfb = oracle.pack_ue8m0(np.ldexp(1.0, eb.reshape(G * 2, KB).astype(np.int64) - 127).astype(np.float32))
    sfb = sfb.reshape(G, 2, -1)
    psum_m = np.array([77, 77, 290], dtype=np.int32)
    d = fill_sentinel(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_psum(_dev(a), _dev(sfa), _dev(b), _dev(sfb), d, _dev(psum_m))
    ref, valid = oracle.m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, psum_m)
    want = torch.from_numpy(ref[valid]).to(torch.bfloat16)
    assert np.array_equal(want.to(torch.float64).numpy(), ref[valid]), "not exact in bf16"
    assert torch.equal(d.cpu()[torch.from_numpy(valid)].view(torch.int16), want.view(torch.int16))
    assert is_sentinel(d)[~valid].all()


def test_psum_graph_replay_with_new_psum_m():
    q = W.psum([150, 150, 150, 150], 600, 264, 512, seed=330)
    a, b = _dev(q["a"]), _dev(q["b"])
    sfa, sfb = dg.pack_ue8m0(_dev(q["sfa_f32"])), dg.pack_ue8m0(_dev(q["sfb_f32"]))
    d = torch.empty((600, 264), dtype=torch.bfloat16, device="cuda")
    ps = _dev(q["psum_m"])
    dg.m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, d, ps)   # eager first call before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            dg.m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, d, ps)
    for new in ([150, 300, 450, 600], [0, 5, 300, 301], [600, 600, 600, 600], [10, 10, 10, 10]):
        ps.copy_(torch.tensor(new, dtype=torch.int32))
        fill_sentinel(d)
        g.replay()
        torch.cuda.synchronize()
        _check(q, d, np.array(new, dtype=np.int32), f"replay {new}")
    del g


def test_psum_matches_contiguous_on_aligned_groups():
    # groups whose segments are 128-row aligned: the psum form and the
    # contiguous form (rows tagged per row) write identical bits
    counts = [128, 256, 0, 384]
    q = W.psum(counts, 768, 264, 1024, seed=340)
    d, ps = _run(q, bn=128)
    dg.set_block_n(128)
    m_indices = np.concatenate([np.full(c, g, np.int32) for g, c in enumerate(counts)])
    dc = fill_sentinel(torch.empty_like(d))
    dg.m_grouped_fp8_gemm_nt_contiguous(_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]),
                                        dg.pack_ue8m0(_dev(q["sfb_f32"])), dc, _dev(m_indices))
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), dc.view(torch.int16))
