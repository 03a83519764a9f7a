"""Dense FP8 GEMM in the TN/NN/TT operand layouts on the GPU: parity with the
CPU oracle, and bit-identical results to fp8_gemm_nt on transposed copies of
the operands (same tile width: the MMAs accumulate in the same order), with M
and N tails. All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp, fill_sentinel, is_sentinel

pytestmark = pytest.mark.gpu

FN = {"nn": dg.fp8_gemm_nn, "tn": dg.fp8_gemm_tn, "tt": dg.fp8_gemm_tt}


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


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("bn,cg", [(128, 1), (256, 1), (256, 2)])
@pytest.mark.parametrize("mnk", [(128, 256, 512), (272, 400, 1024), (512, 768, 2048), (400, 528, 640)])
def test_layout_parity_and_equal_to_nt(layout, bn, cg, mnk):
    M, N, K = mnk
    p = W.dense(M, N, K, seed=M + 5 * N + K + bn)
    a_mk, b_nk = p["a"], p["b"]
    a = a_mk if layout[0] == "n" else np.ascontiguousarray(a_mk.T)
    b = b_nk if layout[1] == "t" else np.ascontiguousarray(b_nk.T)
    sfa = dg.pack_ue8m0(_dev(p["sfa_f32"]))
    sfb = dg.pack_ue8m0(_dev(p["sfb_f32"]))
    dg.set_block_n(bn)
    dg.set_cta_group(cg)   # 2: CTA pairs, a 256-row tile with one 128-byte atom of A and of B per CTA
    d = fill_sentinel(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    FN[layout](_dev(a), sfa, _dev(b), sfb, d)
    d_nt = torch.empty_like(d)
    dg.set_splits(1)   # the layouts run unsplit; compare with the unsplit NT kernel
    dg.fp8_gemm_nt(_dev(a_mk), sfa, _dev(b_nk), sfb, d_nt)
    torch.cuda.synchronize()
    assert not is_sentinel(d).any()
    ref = oracle.fp8_gemm(a, oracle.pack_ue8m0(p["sfa_f32"]), b, oracle.pack_ue8m0(p["sfb_f32"]), layout)
    check_fp(bf16_to_f64(d), ref, f"{layout} {mnk} bn={bn} cg={cg}")
    assert torch.equal(d.view(torch.int16), d_nt.view(torch.int16)), f"{layout} differs from nt"


def test_layout_host_checks():
    M, N, K = 120, 256, 512          # A stored [K, M] needs M % 16 == 0
    a = torch.zeros((K, M), dtype=torch.uint8, device="cuda")
    b = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((M, 1), dtype=torch.int32, device="cuda")
    sfb = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dg.DgError, match="DG_ERR_INVALID_ARG"):
        dg.fp8_gemm_tt(a, sfa, b, sfb, d)
