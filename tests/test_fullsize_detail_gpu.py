"""Parity at full size for the workloads the benchmark times beside the
headline, each in the launch configuration the benchmark uses (the built-in
tile choice, no forced widths, CTA pairs or split counts):

  - psum_m groups: the 8 experts of the contiguous workload, unpadded
    (34,332 rows), N = 4096, K = 7168
  - the NN / TN / TT operand layouts at 4096 x 7168 x 16384
  - one weight scale row per row of B (sfb_gran_n = 1) at 4096 x 7168 x 16384,
    with scales that differ from row to row
  - D = C + A.B^T with fp32 C and D, in place, at 4096 x 7168 x 16384

At these sizes the kernels run many waves of persistent tiles with K up to
16384, which the small parity tests do not reach. Each case checks 2048
seeded outputs that the oracle computes one by one, plus finiteness of the
whole output."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import check_fp, fill_sentinel

pytestmark = pytest.mark.gpu

SAMPLES = 2048
BIG = (4096, 7168, 16384)


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.set_block_n(0)
    dg.set_cta_group(0)
    dg.set_splits(0)
    dg.device_error(clear=True)
    yield
    assert dg.device_error(clear=True) == 0


def _host(t):
    return t.detach().cpu().numpy()


def _pack_host(sf):
    sf = _host(sf)
    return oracle.pack_ue8m0(sf.reshape(-1, sf.shape[-1])).reshape(*sf.shape[:-1], -1)


def _points(a, sfa_f32, b, sfb_f32, rows, cols, sfb_gran_n=128):
    """Oracle outputs at (rows[i], cols[i]); only the sampled rows of A and B leave the device."""
    r = torch.from_numpy(rows).to(a.device)
    c = torch.from_numpy(cols).to(b.device)
    return oracle.fp8_gemm_nt_points(_host(a[r]), _pack_host(sfa_f32[r]), _host(b[c]), cols, _pack_host(sfb_f32),
                                     sfb_gran_n=sfb_gran_n)


def _got(d, rows, cols):
    r = torch.from_numpy(rows).to(d.device)
    c = torch.from_numpy(cols).to(d.device)
    return d[r, c].to(torch.float64).cpu().numpy()


def _samples(M, N, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(0, M, SAMPLES), rng.integers(0, N, SAMPLES)


@pytest.fixture(scope="module")
def big():
    M, N, K = BIG
    p = W.workload1_t(M, N, K)
    p["sfa"] = dg.pack_ue8m0(p["sfa_f32"])
    p["sfb"] = dg.pack_ue8m0(p["sfb_f32"])
    rows, cols = _samples(M, N, 17)
    p["rows"], p["cols"] = rows, cols
    p["ref"] = _points(p["a"], p["sfa_f32"], p["b"], p["sfb_f32"], rows, cols)
    yield p
    del p


def test_psum_groups_full_size():
    counts = W.contiguous_counts()
    p = W.psum_t(counts, 4096, 7168, seed=1002)
    sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
    d = fill_sentinel(torch.empty((p["M_total"], p["N"]), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_psum(p["a"], sfa, p["b"], sfb, d, p["psum_m"])
    torch.cuda.synchronize()
    assert torch.isfinite(d).all().item(), "a row of some group was not written"
    ends = np.cumsum(np.asarray(counts, dtype=np.int64))
    rows, cols = _samples(p["M_total"], p["N"], 5)
    grp = np.searchsorted(ends, rows, side="right")   # group g owns rows [ends[g-1], ends[g])
    ref = np.empty(SAMPLES)
    for g in np.unique(grp):
        sel = np.nonzero(grp == g)[0]
        ref[sel] = _points(p["a"], p["sfa_f32"], p["b"][g], p["sfb_f32"][g], rows[sel], cols[sel])
    check_fp(_got(d, rows, cols), ref, "psum_m 8 groups x 4096 x 7168")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_operand_layouts_full_size(big, layout):
    M, N, K = BIG
    a = big["a"] if layout[0] == "n" else big["a"].t().contiguous()
    b = big["b"] if layout[1] == "t" else big["b"].t().contiguous()
    d = fill_sentinel(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    getattr(dg, f"fp8_gemm_{layout}")(a, big["sfa"], b, big["sfb"], d)
    torch.cuda.synchronize()
    assert torch.isfinite(d).all().item()
    check_fp(_got(d, big["rows"], big["cols"]), big["ref"], f"{layout} {M}x{N}x{K}")


def test_per_row_weight_scales_full_size(big):
    M, N, K = BIG
    # one scale row per row of B: the 128x128 block scale times 2^j, j in [-2, 2]
    # drawn per row and K block, so neighbouring rows really differ
    g = torch.Generator(device="cuda")
    g.manual_seed(31)
    shift = torch.randint(-2, 3, (N, K // 128), generator=g, device="cuda").to(torch.float32)
    sfb_rows_f32 = (big["sfb_f32"].repeat_interleave(128, dim=0)[:N] * torch.exp2(shift)).contiguous()
    sfb_rows = dg.pack_ue8m0(sfb_rows_f32)
    d = fill_sentinel(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    dg.fp8_gemm_nt_sfb_gran(big["a"], big["sfa"], big["b"], sfb_rows, d, 1)
    torch.cuda.synchronize()
    assert torch.isfinite(d).all().item()
    ref = _points(big["a"], big["sfa_f32"], big["b"], sfb_rows_f32, big["rows"], big["cols"], sfb_gran_n=1)
    check_fp(_got(d, big["rows"], big["cols"]), ref, f"per-row B scales {M}x{N}x{K}")


def test_accumulate_fp32_in_place_full_size(big):
    M, N, K = BIG
    g = torch.Generator(device="cuda")
    g.manual_seed(32)
    d = torch.randn((M, N), generator=g, device="cuda", dtype=torch.float32)
    c_at = _got(d, big["rows"], big["cols"])
    dg.fp8_gemm_nt_acc(big["a"], big["sfa"], big["b"], big["sfb"], d, c=d)
    torch.cuda.synchronize()
    assert torch.isfinite(d).all().item()
    check_fp(_got(d, big["rows"], big["cols"]), c_at + big["ref"], f"D = C + A.B^T fp32 in place {M}x{N}x{K}")
