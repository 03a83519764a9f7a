"""UE8M0 pack on the GPU vs the oracle: bit-exact, eager and under CUDA Graph
replay ("[GH-ISSUE #414] pack_ue8m0_to_int is not CUDA Graph capture safe",
Suggested validation: compare eager and captured/replayed output, cover valid
positive zero-mantissa inputs, keep eager validation of malformed values)."""

import numpy as np
import pytest
import torch

import oracle
import moe_grouped_gemm_tcgen05_b200 as dg

pytestmark = pytest.mark.gpu


def _pow2_scales(rng, shape, lo=-40, hi=40):
    return np.ldexp(np.float32(1.0), rng.integers(lo, hi + 1, size=shape)).astype(np.float32)


def _check_pack(sf_np, sf_dev=None):
    sf_dev = torch.from_numpy(sf_np).cuda() if sf_dev is None else sf_dev
    got = dg.pack_ue8m0(sf_dev)
    torch.cuda.synchronize()
    want = oracle.pack_ue8m0(sf_np.reshape(-1, sf_np.shape[-1])).reshape(*sf_np.shape[:-1], -1)
    assert np.array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("shape", [(1, 1), (3, 4), (7, 56), (129, 14), (1000, 57), (2, 5, 16), (4, 3, 7)])
def test_pack_powers_of_two_bit_exact(shape):
    rng = np.random.default_rng(sum(shape))
    _check_pack(_pow2_scales(rng, shape))


def test_pack_every_finite_power_of_two():
    sf = np.ldexp(np.float32(1.0), np.arange(-126, 128)).astype(np.float32).reshape(127, 2)
    _check_pack(sf)
    _check_pack(np.ascontiguousarray(sf.reshape(-1, 254)[:, :252]))


def test_pack_special_values_follow_the_formula():
    vals = np.array([0.0, -0.0, 1.5, 3.0, -2.0, np.inf, -np.inf, np.nan, 1e-45, 2.0 ** -149,
                     np.float32(3.4e38), 0.3, -7.0, 2.0 ** 127, 2.0 ** -126, 1.0], dtype=np.float32)
    _check_pack(vals.reshape(4, 4))
    _check_pack(vals.reshape(2, 8))
    _check_pack(vals[:15].reshape(3, 5))


def test_pack_unaligned_input_uses_general_path():
    rng = np.random.default_rng(1)
    base = torch.from_numpy(_pow2_scales(rng, (65 * 8 + 1,))).cuda()
    view = base[1:].view(65, 8)  # 4-byte aligned, not 16-byte aligned
    _check_pack(view.cpu().numpy(), view)


def test_pack_graph_replay_matches_eager():
    rng = np.random.default_rng(2)
    rows, cols = 512, 56
    sf = torch.from_numpy(_pow2_scales(rng, (rows, cols))).cuda()
    out = torch.empty((rows, 14), dtype=torch.int32, device="cuda")
    dg.pack_ue8m0(sf, out)  # eager warm-up
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dg.pack_ue8m0(sf, out)
    for it in range(3):
        new = _pow2_scales(np.random.default_rng(10 + it), (rows, cols))
        sf.copy_(torch.from_numpy(new))
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), oracle.pack_ue8m0(new))
        if it == 0:
            dg.pack_ue8m0(sf, eager)
            torch.cuda.synchronize()
            assert torch.equal(eager, out)
    del g


def test_validate_counts_like_the_oracle():
    rng = np.random.default_rng(3)
    sf = _pow2_scales(rng, (300, 16))
    sf[5, 3] = 3.0
    sf[7, 0] = -1.0
    sf[299, 15] = 1.25
    sf[100, 1] = -0.0
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.pack_ue8m0_validate(torch.from_numpy(sf).cuda(), bad)
    torch.cuda.synchronize()
    assert int(bad.item()) == oracle.pack_ue8m0_validate(sf) == 4
