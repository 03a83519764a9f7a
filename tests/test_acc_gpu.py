"""Dense GEMM with an accumulation matrix, D = C + A.B^T, on the GPU vs the
CPU oracle: bf16 and fp32 outputs, with and without C, in place (C = D),
on single CTAs, CTA pairs and split-K. All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp

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


def _inputs(p):
    return (_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]), dg.pack_ue8m0(_dev(p["sfb_f32"])))


def _ref(p, c):
    return oracle.fp8_gemm_nt_acc(p["a"], oracle.pack_ue8m0(p["sfa_f32"]), p["b"], oracle.pack_ue8m0(p["sfb_f32"]),
                                  None if c is None else c.detach().cpu().to(torch.float64).numpy())


def _check_f32(got, ref, what):
    # fp32 output: no bf16 rounding, only the fp32 accumulation order
    got = got.detach().cpu().to(torch.float64).numpy()
    assert np.isfinite(got).all(), what
    rms = float(np.sqrt(np.mean(ref * ref)))
    bad = np.abs(got - ref) > 2e-4 * np.abs(ref) + 2e-4 * rms
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off"
    check_fp(got, ref, what)


CONFIGS = [  # (M, N, K, bn, cg, splits)
    (300, 400, 1024, 0, 0, 0),
    (257, 264, 640, 128, 1, 1),
    (512, 1000, 2048, 224, 2, 1),    # CTA pairs
    (300, 776, 1024, 240, 2, 1),     # CTA pairs, 240-wide tiles (16-column tail chunk)
    (64, 2112, 4096, 64, 1, 4),      # split-K (8 K groups)
    (1, 520, 512, 0, 0, 0),
]


@pytest.mark.parametrize("cfg", CONFIGS)
@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("mode", ["c", "none", "inplace"])
def test_acc_parity(cfg, out, mode):
    M, N, K, bn, cg, splits = cfg
    p = W.dense(M, N, K, seed=M + 3 * N + K)
    args = _inputs(p)
    dg.set_block_n(bn)
    dg.set_cta_group(cg)
    dg.set_splits(splits)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    g = torch.Generator().manual_seed(M + N)
    c = (torch.randn((M, N), generator=g) * 4).to(dt).cuda() if mode != "none" else None
    if mode == "inplace":
        d = c.clone()
        dg.fp8_gemm_nt_acc(*args, d, c=d)
    else:
        d = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
        dg.fp8_gemm_nt_acc(*args, d, c=c)
    torch.cuda.synchronize()
    ref = _ref(p, c)
    what = f"acc {cfg} {out} {mode}"
    if out == "bf16":
        check_fp(bf16_to_f64(d), ref, what)
    else:
        _check_f32(d, ref, what)


def test_acc_without_c_bf16_equals_fp8_gemm_nt():
    p = W.dense(384, 768, 2048, seed=5)
    args = _inputs(p)
    d0 = torch.empty((384, 768), dtype=torch.bfloat16, device="cuda")
    d1 = torch.empty_like(d0)
    dg.fp8_gemm_nt(*args, d0)
    dg.fp8_gemm_nt_acc(*args, d1)
    torch.cuda.synchronize()
    assert torch.equal(d0.view(torch.int16), d1.view(torch.int16))
