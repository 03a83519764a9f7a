"""Every compute entry point of the method is CUDA-Graph capture safe
("DeepGEMM CUDA Graph Compatibility for Masked Grouped GEMMs", Stateless
Kernel Architecture: no allocation, no host synchronisation, launch
configuration fixed by the dimensions): each call is captured in global
capture mode, where a hidden synchronisation or allocation makes the capture
fail, and one replay must reproduce the eager result bit for bit. All calls
go through the C ABI. fp8_gemm_nt_noalloc, an addition of this library with
no counterpart in the method, is not covered here: no claim is made about
capturing it."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import fill_sentinel

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


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def eager_equals_replay(call, outs, reset):
    """Run `call` eagerly, then capture it (global mode) and replay once; `reset`
    restores every output (and in-place input) before each run."""
    reset()
    call()
    torch.cuda.synchronize()
    want = [_bits(o).clone() for o in outs]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s, capture_error_mode="global"):
            call()
    torch.cuda.current_stream().wait_stream(s)
    reset()
    g.replay()
    torch.cuda.synchronize()
    for o, w in zip(outs, want):
        assert torch.equal(_bits(o), w)
    del g


def _dense_ops(M, N, K, seed, gran=128):
    p = W.dense(M, N, K, seed=seed, sfb_gran_n=gran)
    return (_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]), dg.pack_ue8m0(_dev(p["sfb_f32"]))), p


@pytest.mark.parametrize("M,cg,splits", [(300, 1, 0), (512, 2, 0), (64, 1, 3)])
def test_fp8_gemm_nt(M, cg, splits):
    (a, sfa, b, sfb), p = _dense_ops(M, 400, 2048, seed=400 + M)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    d = torch.empty((M, 400), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.fp8_gemm_nt(a, sfa, b, sfb, d), [d], lambda: fill_sentinel(d))


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_fp8_gemm_nt_acc_in_place(out):
    (a, sfa, b, sfb), p = _dense_ops(200, 264, 1024, seed=410)
    c0 = torch.randn((200, 264), device="cuda").to(out)
    d = torch.empty_like(c0)
    eager_equals_replay(lambda: dg.fp8_gemm_nt_acc(a, sfa, b, sfb, d, c=d), [d], lambda: d.copy_(c0))


@pytest.mark.parametrize("name", ["fp8_gemm_nn", "fp8_gemm_tn", "fp8_gemm_tt"])
def test_layouts(name):
    (a, sfa, b, sfb), p = _dense_ops(256, 256, 1024, seed=420)
    a_op = a if name == "fp8_gemm_nn" else a.t().contiguous()
    b_op = b if name == "fp8_gemm_tt" else b.t().contiguous()
    d = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    fn = getattr(dg, name)
    eager_equals_replay(lambda: fn(a_op, sfa, b_op, sfb, d), [d], lambda: fill_sentinel(d))


def test_per_row_weight_scales():
    (a, sfa, b, sfb), p = _dense_ops(300, 264, 4096, seed=430, gran=1)
    d = torch.empty((300, 264), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.fp8_gemm_nt_sfb_gran(a, sfa, b, sfb, d, 1), [d], lambda: fill_sentinel(d))


@pytest.mark.parametrize("cg", [1, 2])
def test_contiguous(cg):
    q = W.contiguous([130, 0, 300], 264, 1024, seed=440 + cg, tail_blocks=1)
    args = (_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]), dg.pack_ue8m0(_dev(q["sfb_f32"])))
    idx = _dev(q["m_indices"])
    dg.set_cta_group(cg)
    d = torch.empty((q["M_total"], 264), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.m_grouped_fp8_gemm_nt_contiguous(*args, d, idx), [d], lambda: fill_sentinel(d))


def test_masked_and_psum():
    q = W.masked(np.array([1, 0, 129, 256], np.int32), 256, 264, 1024, seed=450)
    args = (_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]), dg.pack_ue8m0(_dev(q["sfb_f32"])))
    mm = _dev(q["masked_m"])
    d = torch.empty((4, 256, 264), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.m_grouped_fp8_gemm_nt_masked(*args, d, mm), [d], lambda: fill_sentinel(d))
    r = W.psum([37, 0, 200, 129], 400, 264, 1024, seed=451)
    args = (_dev(r["a"]), dg.pack_ue8m0(_dev(r["sfa_f32"])), _dev(r["b"]), dg.pack_ue8m0(_dev(r["sfb_f32"])))
    ps = _dev(r["psum_m"])
    e = torch.empty((400, 264), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.m_grouped_fp8_gemm_nt_psum(*args, e, ps), [e], lambda: fill_sentinel(e))


def test_bf16_masked_and_quantiser():
    q = W.masked_bf16(np.array([3, 70, 0], np.int32), 128, 256, 512, seed=460)
    bits = lambda t: torch.from_numpy(np.ascontiguousarray(t).view(np.int16)).cuda().view(torch.bfloat16)
    a, b, mm = bits(q["a"]), bits(q["b"]), _dev(q["masked_m"])
    d = torch.empty((3, 128, 256), dtype=torch.bfloat16, device="cuda")
    eager_equals_replay(lambda: dg.m_grouped_bf16_gemm_nt_masked(a, b, d, mm), [d], lambda: fill_sentinel(d))
    x = torch.randn((300, 1024), device="cuda").to(torch.bfloat16)
    qx = torch.empty((300, 1024), dtype=torch.uint8, device="cuda")
    sp = torch.empty((300, 2), dtype=torch.int32, device="cuda")
    sf = torch.empty((300, 8), dtype=torch.float32, device="cuda")

    def reset():
        qx.fill_(0xAA)
        sp.fill_(-1)
        sf.fill_(-1.0)

    eager_equals_replay(lambda: dg.quantize_fp8_1x128(x, qx, sp, sf), [qx.view(torch.int16), sp, sf], reset)
