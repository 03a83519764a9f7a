"""Split-K of the dense GEMM on the GPU vs the CPU oracle: forced split
counts over ragged shapes (uneven K ranges, several m-blocks, N tails),
bit-identical results on repeated calls (partials are added in split order),
CUDA Graph replay, splitting calls running at the same time on two streams
(the units of a tile meet inside their cluster, so calls share no scratch),
and no device allocation by the library after its module is loaded. All
calls go through the C ABI."""

import os
import subprocess
import sys
import textwrap

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


@pytest.mark.parametrize("splits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("bn", [64, 96, 128, 256])
@pytest.mark.parametrize("mnk", SHAPES)
def test_split_k_parity(mnk, bn, splits):
    # every cluster size (2..8 CTAs) at several tile widths: pieces of 8
    # columns dealt unevenly among the CTAs, 64-row A stages for M <= 64
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


def test_split_k_calls_run_concurrently_on_two_streams():
    # Many small splitting calls on two streams at once, each stream with its
    # own inputs and outputs: every result must match the oracle (a shared
    # workspace would mix the partials of the two streams' tiles).
    M, N, K = 64, 512, 7168
    ps = [W.dense(M, N, K, seed=60 + i) for i in range(2)]
    args = [_inputs(p) for p in ps]
    dg.set_block_n(128)
    dg.set_splits(4)
    streams = [torch.cuda.Stream() for _ in range(2)]
    outs = [[torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(40)] for _ in range(2)]
    torch.cuda.synchronize()
    for i in range(40):
        for j in range(2):
            with torch.cuda.stream(streams[j]):
                dg.fp8_gemm_nt(*args[j], outs[j][i])
    torch.cuda.synchronize()
    for j in range(2):
        check_fp(bf16_to_f64(outs[j][0]), _ref(ps[j]), f"stream {j}")
        for d in outs[j][1:]:
            assert torch.equal(d.view(torch.int16), outs[j][0].view(torch.int16)), f"stream {j}"


_PROBE = textwrap.dedent("""
    import sys, numpy as np, torch
    sys.path.insert(0, {root!r})
    import moe_grouped_gemm_tcgen05_b200 as dg
    from moe_grouped_gemm_tcgen05_b200 import workloads as W
    torch.cuda.set_device(0)
    p = W.dense_t(64, 2112, 7168, seed=5)
    sfa, sfb = [torch.zeros((r, 14), dtype=torch.int32, device="cuda") for r in (64, 17)]
    sfa.fill_(0x7f7f7f7f)
    sfb.fill_(0x7f7f7f7f)
    d = torch.empty((64, 2112), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    dg.init()                                    # loads the module, sets up the device
    dg.set_splits(4)
    dg.fp8_gemm_nt(p["a"], sfa, p["b"], sfb, d)   # the first launch of this kernel
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        dg.fp8_gemm_nt(p["a"], sfa, p["b"], sfb, d)
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info()[0]
    print(free0 - free1, free1 - free2)
""")


def test_library_allocates_nothing_in_a_fresh_process():
    # Setting up the device and the first launch load the module (its code
    # and static arrays); after that, splitting calls leave the device's free
    # memory exactly unchanged, and the load itself stays far below the 40 MB
    # a split-K workspace would take.
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _PROBE.format(root=root)], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    load_bytes, calls_bytes = (int(x) for x in out.stdout.split()[-2:])
    assert calls_bytes == 0, (load_bytes, calls_bytes)
    assert load_bytes < 32 << 20, (load_bytes, calls_bytes)
