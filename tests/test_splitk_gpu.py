"""Split-K of the dense GEMM on the GPU vs the CPU oracle: forced split
counts over ragged shapes (uneven K ranges, several m-blocks, N tails),
bit-identical results on repeated calls (partials are added in split order,
whichever unit finishes last), and CUDA Graph replay (the per-tile counters
return to zero by themselves). All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp, fill_sentinel, is_sentinel

pytestmark = pytest.mark.gpu


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


def _ref(p):
    return oracle.fp8_gemm_nt(p["a"], oracle.pack_ue8m0(p["sfa_f32"]), p["b"], oracle.pack_ue8m0(p["sfb_f32"]))


def _inputs(p):
    return (_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]), dg.pack_ue8m0(_dev(p["sfb_f32"])))


# (M, N, K): K groups of four 128-K blocks = K / 512 (rounded up)
SHAPES = [(64, 512, 4096),     # 8 groups, one m-block
          (200, 776, 2560),    # 5 groups, two m-blocks, N tail
          (1, 264, 1024),      # 2 groups, a single row
          (130, 1024, 3200)]   # 7 groups (last one partial: 25 K-blocks), M tail


@pytest.mark.parametrize("splits", [2, 3, 5, 8])
@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("mnk", SHAPES)
def test_split_k_parity(mnk, bn, splits):
    M, N, K = mnk
    groups = (K // 128 + 3) // 4
    if splits > groups:
        pytest.skip("more ranges than K groups")
    p = W.dense(M, N, K, seed=11 * M + N + K)
    dg.set_block_n(bn)
    dg.set_splits(splits)
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fill_sentinel(d)
    dg.fp8_gemm_nt(*_inputs(p), d)
    torch.cuda.synchronize()
    assert not is_sentinel(d).any()
    check_fp(bf16_to_f64(d), _ref(p), f"split-K {mnk} bn={bn} splits={splits}")


def test_split_k_more_ranges_than_groups_is_refused():
    p = W.dense(64, 256, 1024, seed=5)   # 2 K groups
    dg.set_splits(3)
    d = torch.empty((64, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dg.DgError):
        dg.fp8_gemm_nt(*_inputs(p), d)


def test_split_k_is_deterministic_and_counters_reset():
    p = W.dense(200, 1024, 8192, seed=21)
    dg.set_splits(6)
    args = _inputs(p)
    outs = []
    for _ in range(5):
        d = torch.empty((200, 1024), dtype=torch.bfloat16, device="cuda")
        dg.fp8_gemm_nt(*args, d)
        outs.append(d)
    torch.cuda.synchronize()
    for d in outs[1:]:
        assert torch.equal(d.view(torch.int16), outs[0].view(torch.int16))
    check_fp(bf16_to_f64(outs[0]), _ref(p), "split-K repeated")


def test_split_k_matches_unsplit_within_tolerance_and_heuristic_small_m():
    # the heuristic splits a small-M problem with a long K; compare with a
    # forced unsplit run and the oracle
    p = W.dense(64, 2112, 7168, seed=22)
    args = _inputs(p)
    d0 = torch.empty((64, 2112), dtype=torch.bfloat16, device="cuda")
    d1 = torch.empty_like(d0)
    dg.set_splits(0)
    dg.fp8_gemm_nt(*args, d0)
    dg.set_splits(1)
    dg.fp8_gemm_nt(*args, d1)
    torch.cuda.synchronize()
    ref = _ref(p)
    check_fp(bf16_to_f64(d0), ref, "heuristic")
    check_fp(bf16_to_f64(d1), ref, "unsplit")


def test_split_k_graph_replay_with_new_inputs():
    M, N, K = 64, 768, 4096
    ps = [W.dense(M, N, K, seed=40 + i) for i in range(3)]
    dg.set_splits(4)
    a, sfa, b, sfb = _inputs(ps[0])
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt(a, sfa, b, sfb, d)          # eager warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            dg.fp8_gemm_nt(a, sfa, b, sfb, d)
    for p in ps:
        na, nsfa, nb, nsfb = _inputs(p)
        a.copy_(na)
        sfa.copy_(nsfa)
        b.copy_(nb)
        sfb.copy_(nsfb)
        g.replay()
        torch.cuda.synchronize()
        check_fp(bf16_to_f64(d), _ref(p), "split-K graph replay")
    del g
