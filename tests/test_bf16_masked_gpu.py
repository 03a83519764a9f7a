"""BF16 masked grouped GEMM on the GPU vs the CPU oracle: every tile width
with ragged and out-of-range masked_m, rows past masked_m left bit-identical
(sentinel), CUDA Graph replay with new masked_m, and the decode-sized
workload (32 groups, max_m = 256, up and down projections) on sampled
outputs. All calls go through the C ABI."""

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


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _run(q, bn=0, masked_m=None):
    dg.set_block_n(bn)
    mm = q["masked_m"] if masked_m is None else masked_m
    d = fill_sentinel(torch.empty((q["G"], q["max_m"], q["N"]), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_bf16_gemm_nt_masked(_dev_bf16(q["a"]), _dev_bf16(q["b"]), d,
                                     torch.from_numpy(np.asarray(mm, dtype=np.int32)).cuda())
    torch.cuda.synchronize()
    return d


def _check(q, d, masked_m=None, what="bf16 masked"):
    mm = q["masked_m"] if masked_m is None else masked_m
    ref, valid = oracle.m_grouped_bf16_gemm_nt_masked(q["a"], q["b"], mm)
    sent = is_sentinel(d)
    assert sent[~valid].all(), f"{what}: a row past masked_m was written"
    assert not sent[valid].any(), f"{what}: a valid row was not written"
    check_fp(bf16_to_f64(d)[valid], ref[valid], what)


@pytest.mark.parametrize("bn", BLOCK_NS)
def test_bf16_masked_parity_every_tile_width(bn):
    # ragged counts, an empty group, one clamped from above and one negative;
    # N tail (264) and 10 K-blocks of 64
    q = W.masked_bf16(np.array([1, 0, 200, 300, 129, -4], dtype=np.int32), 256, 264, 640, seed=40 + bn)
    d = _run(q, bn)
    _check(q, d, what=f"bf16 masked bn={bn}")


@pytest.mark.parametrize("mnk", [(64, 8, 64), (130, 1000, 192), (256, 256, 4096)])
def test_bf16_masked_shapes(mnk):
    max_m, N, K = mnk
    q = W.masked_bf16(np.array([max_m, max_m // 2, 3], dtype=np.int32), max_m, N, K, seed=sum(mnk))
    _check(q, _run(q), what=f"bf16 masked {mnk}")


def test_bf16_masked_graph_replay_with_new_masked_m():
    # rows beyond the first masked_m become valid in later replays: no NaN fill
    q = W.masked_bf16(np.array([100, 50, 0, 256], dtype=np.int32), 256, 512, 1024, seed=51, fill_invalid_nan=False)
    a, b = _dev_bf16(q["a"]), _dev_bf16(q["b"])
    mm_dev = torch.from_numpy(q["masked_m"]).cuda()
    d = torch.empty((q["G"], q["max_m"], q["N"]), dtype=torch.bfloat16, device="cuda")
    dg.m_grouped_bf16_gemm_nt_masked(a, b, d, mm_dev)   # eager warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            dg.m_grouped_bf16_gemm_nt_masked(a, b, d, mm_dev)
    for mm in ([7, 256, 0, 1], [0, 0, 0, 0], [256, 255, 128, 64]):
        mm = np.array(mm, dtype=np.int32)
        fill_sentinel(d)
        mm_dev.copy_(torch.from_numpy(mm))
        g.replay()
        torch.cuda.synchronize()
        _check(q, d, masked_m=mm, what=f"bf16 masked replay {mm.tolist()}")
    del g


@pytest.mark.parametrize("proj", ["up", "down"])
def test_bf16_masked_decode_workload_sampled(proj):
    # 32 groups, max_m = 256, masked_m U{67..124}: the decode shapes in bf16
    N, K = (4096, 7168) if proj == "up" else (7168, 2048)
    mm = W.masked_m_uniform(W.rng_for(1003))
    q = W.masked_bf16_t(mm, 256, N, K, seed=1003)
    d = fill_sentinel(torch.empty((q["G"], 256, N), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_bf16_gemm_nt_masked(q["a"], q["b"], d, q["masked_m"])
    torch.cuda.synchronize()
    valid = np.arange(256)[None, :] < mm[:, None]
    sent = is_sentinel(d)
    assert sent[~valid].all() and not sent[valid].any()
    rng = np.random.default_rng(7)
    gs = rng.integers(0, q["G"], 2048)
    rs = (rng.random(2048) * mm[gs]).astype(np.int64)
    cs = rng.integers(0, N, 2048)
    a_bits = q["a"].view(torch.int16).cpu().numpy().view(np.uint16)
    b_bits = q["b"].view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.m_grouped_bf16_gemm_nt_masked_sampled(a_bits, b_bits, mm, gs, rs, cs)
    got = bf16_to_f64(d)[gs, rs, cs]
    check_fp(got, ref, f"bf16 masked decode {proj}")


def test_bf16_masked_host_checks():
    q = W.masked_bf16(np.array([4], dtype=np.int32), 8, 16, 96, seed=3)   # K = 96: not a multiple of 64
    with pytest.raises(dg.DgError, match="DG_ERR_INVALID_ARG"):
        _run(q)
