"""fp8_gemm_nt_noalloc (the dense GEMM whose split-K scratch is a static
array of the library instead of an allocation) against the existing entry
point fp8_gemm_nt: bit-identical results on two calls in a row, a clear
refusal when the request needs more scratch than the static arrays hold, and
no device allocation by the call (checked in a fresh process). Collected last
on purpose; it also passes on its own."""

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

from helpers import bf16_to_f64, check_fp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.device_error(clear=True)
    yield
    dg.set_block_n(0)
    dg.set_splits(0)
    assert dg.device_error(clear=True) == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _inputs(p):
    return (_dev(p["a"]), dg.pack_ue8m0(_dev(p["sfa_f32"])), _dev(p["b"]), dg.pack_ue8m0(_dev(p["sfb_f32"])))


def _ref(p):
    return oracle.fp8_gemm_nt(p["a"], oracle.pack_ue8m0(p["sfa_f32"]), p["b"], oracle.pack_ue8m0(p["sfb_f32"]))


@pytest.mark.parametrize("mnk,bn,splits", [((64, 2112, 7168), 64, 4),     # split-K through the static scratch
                                          ((200, 776, 2560), 128, 3),    # two m-blocks, N tail, uneven ranges
                                          ((300, 512, 1024), 256, 1)])   # no split
def test_matches_existing_entry_point_on_two_calls_in_a_row(mnk, bn, splits):
    M, N, K = mnk
    p = W.dense(M, N, K, seed=7 * M + N)
    args = _inputs(p)
    dg.set_block_n(bn)
    dg.set_splits(splits)
    want = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt(*args, want)
    got = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    for d in got:
        dg.fp8_gemm_nt_noalloc(*args, d, splits=splits)
    torch.cuda.synchronize()
    for d in got:
        assert torch.equal(d.view(torch.int16), want.view(torch.int16))
    check_fp(bf16_to_f64(got[1]), _ref(p), f"noalloc {mnk} splits={splits}")


def test_auto_split_within_static_scratch():
    p = W.dense(64, 4096, 7168, seed=3)
    args = _inputs(p)
    d = torch.empty((64, 4096), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        dg.fp8_gemm_nt_noalloc(*args, d)
        torch.cuda.synchronize()
        check_fp(bf16_to_f64(d), _ref(p), "noalloc auto")


def test_request_beyond_static_scratch_is_refused():
    # 8 m-blocks x 16 n-tiles x 8 splits of 128 x 256 fp32 partials: 128 MiB > 8 MiB
    M, N, K = 1024, 4096, 4096
    a = torch.zeros((M, K), dtype=torch.float8_e4m3fn, device="cuda")
    b = torch.zeros((N, K), dtype=torch.float8_e4m3fn, device="cuda")
    sfa = torch.zeros((M, K // 512), dtype=torch.int32, device="cuda")
    sfb = torch.zeros((N // 128, K // 512), dtype=torch.int32, device="cuda")
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.set_block_n(256)
    with pytest.raises(dg.DgError, match="DG_ERR_SCRATCH_TOO_SMALL"):
        dg.fp8_gemm_nt_noalloc(a, sfa, b, sfb, d, splits=8)
    with pytest.raises(dg.DgError, match="DG_ERR_UNSUPPORTED"):
        dg.fp8_gemm_nt_noalloc(a, sfa, b, sfb, d, splits=17)


_PROBE = textwrap.dedent("""
    import sys, numpy as np, torch
    sys.path.insert(0, {root!r})
    import oracle
    import moe_grouped_gemm_tcgen05_b200 as dg
    from moe_grouped_gemm_tcgen05_b200 import workloads as W
    torch.cuda.set_device(0)
    # inputs prepared without calling the library
    p = W.dense(64, 2112, 7168, seed=5)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    p = dict(a=dev(p["a"]), b=dev(p["b"]), sfa=oracle.pack_ue8m0(p["sfa_f32"]), sfb=oracle.pack_ue8m0(p["sfb_f32"]))
    sfa, sfb = dev(p["sfa"]), dev(p["sfb"])
    d = torch.empty((64, 2112), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    # the first call loads the library's module: its code and static arrays
    dg.fp8_gemm_nt_noalloc(p["a"], sfa, p["b"], sfb, d, splits=4)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        dg.fp8_gemm_nt_noalloc(p["a"], sfa, p["b"], sfb, d, splits=4)
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info()[0]
    # a deliberate 16 MiB allocation shows that the measurement sees one
    x = torch.empty(16 << 20, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    free3 = torch.cuda.mem_get_info()[0]
    print(free0 - free1, free1 - free2, free2 - free3)
""")


def test_no_device_allocation_in_a_fresh_process():
    # The first call loads the library's module (its code and the static
    # arrays, about 8 MiB of them). After it, further calls must leave the
    # device's free memory exactly unchanged; a 16 MiB allocation made on
    # purpose afterwards shows that the measurement sees one of that size.
    out = subprocess.run([sys.executable, "-c", _PROBE.format(root=ROOT)], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    load_bytes, calls_bytes, probe_bytes = (int(x) for x in out.stdout.split()[-3:])
    assert probe_bytes >= 16 << 20, (load_bytes, calls_bytes, probe_bytes)
    assert calls_bytes == 0, (load_bytes, calls_bytes, probe_bytes)
    assert load_bytes < 32 << 20, (load_bytes, calls_bytes, probe_bytes)
