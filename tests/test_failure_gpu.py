"""Failure path on the GPU without a fault: a test hook makes CTA 0 withhold one
pipeline arrive, so a bounded wait inside the kernel runs out (short limit).
The kernel must record DG_DEVERR_TIMEOUT and return; the context must stay
usable and the next call must be correct."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp

pytestmark = pytest.mark.gpu


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _dense(p):
    d = torch.empty((p["M"], p["N"]), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt(_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]),
                   dg.pack_ue8m0(_dev(p["sfb_f32"])), d)
    return d


def _masked(q):
    d = torch.zeros((q["G"], q["max_m"], q["N"]), dtype=torch.bfloat16, device="cuda")
    dg.m_grouped_fp8_gemm_nt_masked(_dev(q["a"]), dg.pack_ue8m0(_dev(q["sfa_f32"])), _dev(q["b"]),
                                    dg.pack_ue8m0(_dev(q["sfb_f32"])), d, _dev(q["masked_m"]))
    return d


@pytest.mark.parametrize("form", ["dense", "dense_pairs", "masked"])
def test_timeout_is_reported_and_context_survives(form):
    dg.init()
    dg.device_error(clear=True)
    dg.set_cta_group(2 if form == "dense_pairs" else 0)
    p = W.dense(384, 512, 1024, seed=31)
    q = W.masked(np.array([100, 0, 256], dtype=np.int32), 256, 256, 512, seed=32)
    try:
        dg.set_test_hooks(1, 200)
        _masked(q) if form == "masked" else _dense(p)
        torch.cuda.synchronize()
        assert dg.device_error(clear=True) & dg.DEVERR_TIMEOUT
    finally:
        dg.set_test_hooks(0, 0)
    # same process, same context: the next calls are correct and clean
    d = _dense(p)
    torch.cuda.synchronize()
    ref = oracle.fp8_gemm_nt(p["a"], oracle.pack_ue8m0(p["sfa_f32"]), p["b"], oracle.pack_ue8m0(p["sfb_f32"]))
    check_fp(bf16_to_f64(d), ref, "after timeout")
    dm = _masked(q)
    torch.cuda.synchronize()
    refm, valid = oracle.m_grouped_fp8_gemm_nt_masked(
        q["a"], oracle.pack_ue8m0(q["sfa_f32"].reshape(-1, 4)).reshape(3, 256, 1), q["b"],
        oracle.pack_ue8m0(q["sfb_f32"].reshape(-1, 4)).reshape(3, 2, 1), q["masked_m"])
    check_fp(bf16_to_f64(dm)[valid], refm[valid], "masked after timeout")
    assert dg.device_error(clear=True) == 0
    dg.set_cta_group(0)


def test_timeout_under_split_k_then_counters_are_zeroed():
    """A split-K launch that gives up leaves per-tile counters part-way;
    clearing the status word zeroes them, so the next split-K calls are right."""
    dg.init()
    dg.device_error(clear=True)
    dg.set_splits(4)
    p = W.dense(200, 512, 4096, seed=33)
    try:
        dg.set_test_hooks(1, 200)
        _dense(p)
        torch.cuda.synchronize()
        assert dg.device_error(clear=True) & dg.DEVERR_TIMEOUT
    finally:
        dg.set_test_hooks(0, 0)
    ref = oracle.fp8_gemm_nt(p["a"], oracle.pack_ue8m0(p["sfa_f32"]), p["b"], oracle.pack_ue8m0(p["sfb_f32"]))
    try:
        for _ in range(3):
            d = _dense(p)
            torch.cuda.synchronize()
            check_fp(bf16_to_f64(d), ref, "split-K after timeout")
        assert dg.device_error(clear=True) == 0
    finally:
        dg.set_splits(0)
