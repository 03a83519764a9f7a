"""Per-token FP8 quantiser on the GPU vs the CPU oracle, bit for bit: E4M3
codes, packed UE8M0 scales (with the zero padding bytes of each row's last
word) and fp32 scales, for bf16 and fp32 inputs over widely varying block
magnitudes, zero blocks, amax exactly 448 * 2^k and the next float up,
values that round to zero; graph replay; and quantise -> GEMM end to end.
All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import bf16_to_f64, check_fp

pytestmark = pytest.mark.gpu


def _inputs(rows, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, K)) * np.power(10.0, rng.uniform(-6, 6, size=(rows, K // 128))).repeat(128, axis=1)
    x = x.astype(np.float32)
    if rows > 2:
        x[1, :128] = 0.0                                        # a zero block
        x[2, 128:256] = 0.0
        x[2, 130] = np.float32(448.0 * 2.0 ** -3)              # amax exactly 448 * 2^k
        if K >= 384:
            x[2, 256:384] = 1e-30                               # codes round to zero
            x[2, 300] = np.nextafter(np.float32(448.0 * 4), np.float32(np.inf))   # just above 448 * 2^k
    return x


def _check_exact(x64, q, packed, sf32):
    q_ref, p_ref, s_ref = oracle.quantize_fp8_1x128(x64)
    got_q = q.cpu().numpy()
    bad = np.nonzero(got_q != q_ref)
    assert bad[0].size == 0, f"{bad[0].size} codes differ, first at {bad[0][0]},{bad[1][0]}: {got_q[bad][0]:#x} vs {q_ref[bad][0]:#x}"
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    if sf32 is not None:
        assert np.array_equal(sf32.cpu().numpy(), s_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,K", [(1, 128), (300, 640), (77, 7168), (1024, 1536)])
def test_quantiser_bit_exact(dtype, rows, K):
    x = _inputs(rows, K, seed=rows + K)
    xt = torch.from_numpy(x)
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)
    x64 = xt.to(torch.float64).numpy()        # the exact values the kernel sees
    xd = xt.cuda()
    sf32 = torch.empty((rows, K // 128), dtype=torch.float32, device="cuda")
    packed = torch.full((rows, (K // 128 + 3) // 4), -1, dtype=torch.int32, device="cuda")  # padding must be zeroed
    q, packed, sf32 = dg.quantize_fp8_1x128(xd, sf_packed=packed, sf_f32=sf32)
    torch.cuda.synchronize()
    _check_exact(x64, q, packed, sf32)


def test_quantiser_graph_replay_with_new_inputs():
    rows, K = 256, 2048
    xd = torch.empty((rows, K), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    packed = torch.empty((rows, K // 512), dtype=torch.int32, device="cuda")
    xd.copy_(torch.from_numpy(_inputs(rows, K, 1)).to(torch.bfloat16))
    dg.quantize_fp8_1x128(xd, q, packed)       # eager warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            dg.quantize_fp8_1x128(xd, q, packed)
    for seed in (2, 3):
        xt = torch.from_numpy(_inputs(rows, K, seed)).to(torch.bfloat16)
        xd.copy_(xt)
        g.replay()
        torch.cuda.synchronize()
        _check_exact(xt.to(torch.float64).numpy(), q, packed, None)
    del g


def test_quantise_then_gemm_end_to_end():
    # activations quantised on the GPU feed the GEMM; the oracle multiplies
    # its own quantisation of the same values (bit-identical, checked above)
    M, N, K = 200, 512, 2048
    rng = np.random.default_rng(4)
    xt = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    p = W.dense(M, N, K, seed=9)          # B and its scales
    q, packed, _ = dg.quantize_fp8_1x128(xt.cuda())
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    b = torch.from_numpy(p["b"]).cuda()
    sfb = dg.pack_ue8m0(torch.from_numpy(p["sfb_f32"]).cuda())
    dg.fp8_gemm_nt(q, packed, b, sfb, d)
    torch.cuda.synchronize()
    q_ref, p_ref, _ = oracle.quantize_fp8_1x128(xt.to(torch.float64).numpy())
    ref = oracle.fp8_gemm_nt(q_ref, p_ref, p["b"], oracle.pack_ue8m0(p["sfb_f32"]))
    check_fp(bf16_to_f64(d), ref, "quantise -> GEMM")


def test_quantiser_host_checks():
    # the library's own checks, through the C ABI (the binding checks shapes first)
    lib = dg.load()
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((4, 256), dtype=torch.uint8, device="cuda")
    sfp = torch.empty((4, 1), dtype=torch.int32, device="cuda")
    args = lambda K, xf=0: (x.data_ptr(), xf, q.data_ptr(), sfp.data_ptr(), None, 4, K, None)
    assert lib.quantize_fp8_1x128(*args(100)) == 1       # K % 128
    assert lib.quantize_fp8_1x128(*args(256, 2)) == 1    # x_f32 not 0/1
    assert lib.quantize_fp8_1x128(x.data_ptr() + 2, 0, q.data_ptr(), sfp.data_ptr(), None, 4, 128, None) == 2
