"""Parity at the full workload sizes, in the launch configuration the benchmark
times (built-in tile heuristic, CUDA Graph replay for the grouped forms).
Outputs are checked on seeded samples that the oracle computes one by one;
rows that must stay untouched are checked exhaustively against a sentinel."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W

from helpers import SENTINEL_BITS, check_fp, fill_sentinel

pytestmark = pytest.mark.gpu

SAMPLES = 2048
SENT = np.int16(np.uint16(SENTINEL_BITS).astype(np.int16))


@pytest.fixture(autouse=True)
def _reset():
    dg.init()
    dg.set_block_n(0)
    dg.device_error(clear=True)
    yield
    assert dg.device_error(clear=True) == 0


def _host(t):
    return t.detach().cpu().numpy()


def _pack_host(sf):
    sf = _host(sf)
    return oracle.pack_ue8m0(sf.reshape(-1, sf.shape[-1])).reshape(*sf.shape[:-1], -1)


def _points(a, sfa_f32, b, sfb_f32, rows, cols):
    """Oracle values at (rows[i], cols[i]); a/b may be device tensors, only the sampled rows move."""
    r = torch.from_numpy(rows).to(a.device)
    c = torch.from_numpy(cols).to(b.device)
    return oracle.fp8_gemm_nt_points(_host(a[r]), _pack_host(sfa_f32[r]), _host(b[c]), cols, _pack_host(sfb_f32))


def _got(d, idx):
    return d[tuple(torch.from_numpy(i).to(d.device) for i in idx)].to(torch.float64).cpu().numpy()


@pytest.mark.parametrize("M", W.DENSE_M)
@pytest.mark.parametrize("NK", W.DENSE_NK)
def test_dense_full_size(M, NK):
    N, K = NK
    p = W.workload1_t(M, N, K)
    sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
    d = fill_sentinel(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    dg.fp8_gemm_nt(p["a"], sfa, p["b"], sfb, d)
    torch.cuda.synchronize()
    assert torch.isfinite(d).all().item(), "non-finite output (or an unwritten sentinel)"
    rng = np.random.default_rng(M + N + K)
    rows = rng.integers(0, M, SAMPLES)
    cols = rng.integers(0, N, SAMPLES)
    ref = _points(p["a"], p["sfa_f32"], p["b"], p["sfb_f32"], rows, cols)
    check_fp(_got(d, (rows, cols)), ref, f"dense {M}x{N}x{K}")


def test_contiguous_full_size():
    p = W.workload2_t()
    sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
    d = fill_sentinel(torch.empty((p["M_total"], p["N"]), dtype=torch.bfloat16, device="cuda"))
    dg.m_grouped_fp8_gemm_nt_contiguous(p["a"], sfa, p["b"], sfb, d, p["m_indices"])
    torch.cuda.synchronize()
    mi = _host(p["m_indices"])
    pad = torch.from_numpy(mi < 0).cuda()
    assert (d.view(torch.int16)[pad] == SENT).all().item(), "a padding row was written"
    assert torch.isfinite(d[~pad]).all().item()
    rng = np.random.default_rng(2)
    valid_rows = np.nonzero(mi >= 0)[0]
    rows = rng.choice(valid_rows, SAMPLES)
    cols = rng.integers(0, p["N"], SAMPLES)
    got = _got(d, (rows, cols))
    ref = np.empty(SAMPLES)
    for e in np.unique(mi[rows]):
        sel = np.nonzero(mi[rows] == e)[0]
        ref[sel] = _points(p["a"], p["sfa_f32"], p["b"][e], p["sfb_f32"][e], rows[sel], cols[sel])
    check_fp(got, ref, "contiguous 8x4096x7168")


def _masked_replays(p, with_pack, draws, what):
    G, max_m, N, K = p["G"], p["max_m"], p["N"], p["K"]
    kp = (K // 128 + 3) // 4
    sfb = dg.pack_ue8m0(p["sfb_f32"])
    sfa = torch.empty((G, max_m, kp), dtype=torch.int32, device="cuda")
    dg.pack_ue8m0(p["sfa_f32"], sfa)
    d = torch.empty((G, max_m, N), dtype=torch.bfloat16, device="cuda")
    mm = p["masked_m"]

    def call():
        if with_pack:
            dg.pack_ue8m0(p["sfa_f32"], sfa)
        dg.m_grouped_fp8_gemm_nt_masked(p["a"], sfa, p["b"], sfb, d, mm)

    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    if with_pack:
        assert np.array_equal(_host(sfa), _pack_host(p["sfa_f32"])), "packed activation scales differ"
    for it, m_draw in enumerate(draws):
        mm.copy_(torch.from_numpy(m_draw.astype(np.int32)))
        if with_pack and it > 0:
            # a fresh quantisation of the activations, copied into the captured
            # buffers; the graph's pack kernel packs its scales
            gen = torch.Generator(device="cuda")
            gen.manual_seed(900 + it)
            qa, qs = W.quantise_rows_t(torch.randn((G * max_m, K), generator=gen, device="cuda"))
            p["a"].copy_(qa.view(G, max_m, K))
            p["sfa_f32"].copy_(qs.view(G, max_m, K // 128))
            del qa, qs
        fill_sentinel(d)
        g.replay()
        torch.cuda.synchronize()
        if with_pack:
            assert np.array_equal(_host(sfa), _pack_host(p["sfa_f32"])), f"{what} replay {it}: packed scales differ"
        m_clamped = np.clip(m_draw, 0, max_m)
        invalid = torch.from_numpy(np.arange(max_m)[None, :] >= m_clamped[:, None]).cuda()
        assert (d.view(torch.int16)[invalid] == SENT).all().item(), f"{what}: a row past masked_m was written"
        assert torch.isfinite(d[~invalid]).all().item(), f"{what}: a valid row was not written"
        rng = np.random.default_rng(100 + it)
        nz = np.nonzero(m_clamped > 0)[0]
        grp = rng.choice(nz, SAMPLES)
        rows = (rng.random(SAMPLES) * m_clamped[grp]).astype(np.int64)
        cols = rng.integers(0, N, SAMPLES)
        got = _got(d, (grp, rows, cols))
        ref = np.empty(SAMPLES)
        for gi in np.unique(grp):
            sel = np.nonzero(grp == gi)[0]
            ref[sel] = _points(p["a"][gi], p["sfa_f32"][gi], p["b"][gi], p["sfb_f32"][gi], rows[sel], cols[sel])
        check_fp(got, ref, f"{what} replay {it}")
    del g


@pytest.mark.parametrize("proj", ["up", "down"])
def test_masked_decode_full_size_graph_replay(proj):
    p = W.workload3_t(proj)
    draws = [p["masked_m_host"], W.masked_m_uniform(W.rng_for(77)), W.masked_m_uniform(W.rng_for(78))]
    _masked_replays(p, False, draws, f"masked decode {proj}")


def test_masked_zipf_full_size_pack_and_gemm_graph():
    # replays with fresh masked_m and, from the second on, fresh activations and scales
    p = W.workload4_t()
    draws = [p["masked_m_host"], W.zipf_masked_m(W.rng_for(79)), W.zipf_masked_m(W.rng_for(80))]
    _masked_replays(p, True, draws, "masked zipf")
