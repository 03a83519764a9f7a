"""The seeded input generator produces valid operands (CPU only)."""

import numpy as np
import torch

from moe_grouped_gemm_tcgen05_b200 import workloads as W


def _decode(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _is_pow2(s):
    bits = np.asarray(s, dtype=np.float32).view(np.int32)
    return ((bits & 0x7FFFFF) == 0) & (bits > 0)


def test_dense_quantisation_is_valid_and_close():
    p = W.dense(70, 200, 384, seed=1)
    assert p["a"].dtype == np.uint8 and p["a"].shape == (70, 384)
    assert p["sfa_f32"].shape == (70, 3) and p["sfb_f32"].shape == (2, 3)
    assert _is_pow2(p["sfa_f32"]).all() and _is_pow2(p["sfb_f32"]).all()
    # regenerate the fp32 source and check the quantised value is within E4M3 precision
    rng = W.rng_for(1)
    x = rng.standard_normal(size=(70, 384), dtype=np.float32)
    xa = _decode(p["a"]) * np.repeat(p["sfa_f32"].astype(np.float64), 128, axis=1)
    assert np.all(np.abs(xa - x) <= 2.0 ** -4 * np.abs(x) + np.repeat(p["sfa_f32"], 128, axis=1) * 2.0 ** -9)
    assert np.all(np.abs(_decode(p["a"])) <= 448)


def test_same_seed_same_bytes():
    p1 = W.dense(8, 16, 128, seed=5)
    p2 = W.dense(8, 16, 128, seed=5)
    assert np.array_equal(p1["a"], p2["a"]) and np.array_equal(p1["sfb_f32"], p2["sfb_f32"])


def test_contiguous_layout():
    p = W.contiguous([5, 0, 130], 64, 256, seed=2, tail_blocks=1)
    mi = p["m_indices"]
    assert p["M_total"] == 128 + 0 + 256 + 128
    assert (mi[:5] == 0).all() and (mi[5:128] == -1).all()
    assert (mi[128:258] == 2).all() and (mi[258:] == -1).all()
    assert (p["a"][mi < 0] == W.NAN_BYTE).all()


def test_masked_distributions():
    mm = W.masked_m_uniform(W.rng_for(1003))
    assert mm.min() >= 67 and mm.max() <= 124 and mm.size == 32
    z = W.zipf_masked_m(W.rng_for(1004))
    assert z.size == 256 and z.min() >= 0 and z.max() <= 512
    m = np.arange(513)
    p = (m + 1.0) ** -1.1
    p /= p.sum()
    # closed-form mean / P(0) of the truncated Zipf(1.1) on {0..512}
    assert abs(float((m * p).sum()) - 57.4) < 0.5 and abs(p[0] - 0.191) < 0.002
    assert 30 < z.mean() < 90 and 25 < (z == 0).sum() < 75


def test_per_row_weight_scales():
    # one scale per 1x128 block of each row of B; rows carry a power-of-two spread
    p = W.dense(16, 300, 512, seed=4, sfb_gran_n=1)
    assert p["sfb_f32"].shape == (300, 4) and _is_pow2(p["sfb_f32"]).all()
    assert np.all(np.abs(_decode(p["b"])) <= 448)
    assert len(np.unique(p["sfb_f32"][:128, 0])) > 1  # rows of one 128-block differ
    q = W.masked(np.array([3, 0], np.int32), 8, 136, 256, seed=5, sfb_gran_n=1)
    assert q["sfb_f32"].shape == (2, 136, 2)


def test_psum_layout():
    p = W.psum([70, 0, 100], 200, 256, 512, seed=6)
    assert list(p["psum_m"]) == [70, 70, 170] and p["psum_m"].dtype == np.int32
    assert p["a"].shape == (200, 512) and p["b"].shape == (3, 256, 512) and p["sfb_f32"].shape == (3, 2, 4)
    assert np.all(p["a"][170:] == W.NAN_BYTE)             # rows in no group
    assert not np.any(p["a"][:170] == W.NAN_BYTE)
    assert _is_pow2(p["sfa_f32"]).all()
