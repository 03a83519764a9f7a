"""Pins for the CPU oracle, independent of the oracle itself (CPU only).

Each pin checks the oracle against something it does not compute itself:
worked examples derived by hand from the pack formula in "[GH-ISSUE #414]
pack_ue8m0_to_int is not CUDA Graph capture safe", the OCP E4M3 definition
(spot values, and torch's own float8 decode for all 256 codes), closed forms
(one-hot operands, powers of two), exact rational brute force on tiny shapes,
and special cases that reduce to a library matmul. The last tests plant
mistakes in a copy of the oracle and check that the pins catch them.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import gemm as og

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_e4m3(codes):
    """torch's float8_e4m3fn decode of byte codes, as float64 (library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(codes, dtype=np.uint8)))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


# ---------------------------------------------------------------- E4M3 ----

def test_e4m3_spot_values_from_ocp_definition():
    spots = {
        0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
        0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0,
        0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0,
    }
    for code, want in spots.items():
        got = oracle.e4m3_to_f64(np.array([code]))[0]
        assert got == want and math.copysign(1, got) == math.copysign(1, want), hex(code)
    assert np.isnan(oracle.e4m3_to_f64(np.array([0x7F, 0xFF]))).all()
    assert oracle.E4M3_MAX == 448.0


def test_e4m3_table_matches_torch_float8_decode():
    codes = np.arange(256)
    mine = oracle.e4m3_to_f64(codes)
    ref = torch_e4m3(codes)
    same = (mine == ref) | (np.isnan(mine) & np.isnan(ref))
    assert same.all(), codes[~same]


# --------------------------------------------------------------- UE8M0 ----

def test_ue8m0_decode_closed_form():
    v = oracle.ue8m0_to_f64(np.array([0, 1, 126, 127, 128, 254, 255]))
    assert v[0] == 2.0 ** -127 and v[1] == 2.0 ** -126
    assert v[2] == 0.5 and v[3] == 1.0 and v[4] == 2.0 and v[5] == 2.0 ** 127
    assert np.isnan(v[6])


def _read_pack_golden():
    cases = []
    with open(os.path.join(GOLDEN, "pack_ue8m0_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            scales, byts, word = [p.strip() for p in line.split("|")]
            cases.append(([float(s) for s in scales.split()],
                          [int(x, 16) for x in byts.split()], int(word, 16)))
    return cases


def test_pack_matches_hand_worked_examples():
    cases = _read_pack_golden()
    assert len(cases) >= 4
    for scales, byts, word in cases:
        got = oracle.pack_ue8m0(np.array([scales], dtype=np.float32))
        assert got.shape == (1, 1)
        assert (int(got[0, 0]) & 0xFFFFFFFF) == word, (scales, hex(int(got[0, 0]) & 0xFFFFFFFF))
        assert list(oracle.unpack_ue8m0(got, 4)[0]) == byts


def test_pack_every_finite_positive_power_of_two():
    # all 254 normal powers of two 2^-126 .. 2^127: byte = e + 127, and it decodes back exactly
    e = np.arange(-126, 128)
    sf = np.ldexp(np.float32(1.0), e).astype(np.float32)
    n = sf.size
    cols = 4 * ((n + 3) // 4)
    grid = np.ones(cols, dtype=np.float32)
    grid[:n] = sf
    packed = oracle.pack_ue8m0(grid.reshape(1, cols))
    byts = oracle.unpack_ue8m0(packed, cols)[0, :n]
    assert (byts.astype(np.int64) == e + 127).all()
    assert (oracle.ue8m0_to_f64(byts) == sf.astype(np.float64)).all()
    assert oracle.pack_ue8m0_validate(grid.reshape(1, cols)) == 0


def test_pack_ragged_columns_pad_with_zero_bytes():
    sf = np.array([[2.0, 4.0, 8.0, 16.0, 0.5, 0.25]], dtype=np.float32)
    p = oracle.pack_ue8m0(sf)
    assert p.shape == (1, 2)
    assert (int(p[0, 1]) & 0xFFFFFFFF) == 0x00007D7E  # bytes 7E 7D 00 00
    assert (int(p[0, 0]) & 0xFFFFFFFF) == 0x83828180


def test_validator_counts_issue_conditions():
    sf = np.array([[1.0, -1.0, 3.0, 0.0, float("inf"), 1.5, -0.0, 2.0 ** -20]], dtype=np.float32)
    # sign set: -1.0, -0.0 ; mantissa != 0: 3.0, 1.5
    assert oracle.pack_ue8m0_validate(sf) == 4


# ---------------------------------------------------------------- GEMM ----

def _rand_codes(rng, shape, lo_exp=4, hi_exp=11):
    """E4M3 codes with exponent field in [lo_exp, hi_exp] and random sign/mantissa."""
    s = rng.integers(0, 2, size=shape)
    e = rng.integers(lo_exp, hi_exp + 1, size=shape)
    m = rng.integers(0, 8, size=shape)
    return ((s << 7) | (e << 3) | m).astype(np.uint8)


def _pack_bytes(byts):
    """Pack a uint8 [rows, cols] array of UE8M0 bytes into int32 words (test-side, little-endian)."""
    rows, cols = byts.shape
    kp = (cols + 3) // 4
    w = np.zeros((rows, kp), dtype=np.int64)
    for c in range(cols):
        w[:, c // 4] |= byts[:, c].astype(np.int64) << (8 * (c % 4))
    return w.astype(np.uint32).view(np.int32)


def _exact_gemm(a, ea, b, eb, gran=128):
    """Exact rational D = A^ B^^T with explicit block loops (no shared code with the oracle).
    Row n of B takes scale row n // gran (128x128 blocks, or one row per row of B)."""
    M, K = a.shape
    N = b.shape[0]
    av = torch_e4m3(a)
    bv = torch_e4m3(b)
    out = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for kb in range(K // 128):
                sa = Fraction(2) ** (int(ea[m, kb]) - 127)
                sb = Fraction(2) ** (int(eb[n // gran, kb]) - 127)
                part = Fraction(0)
                for kk in range(128):
                    k = kb * 128 + kk
                    part += Fraction(av[m, k]) * Fraction(bv[n, k])
                acc += part * sa * sb
            out[m][n] = acc
    return out


@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 128, 1), (8, 7, 256, 2), (1, 8, 256, 3)])
def test_dense_equals_exact_rational_brute_force(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    ea = rng.integers(124, 131, size=(M, K // 128)).astype(np.uint8)
    eb = rng.integers(124, 131, size=((N + 127) // 128, K // 128)).astype(np.uint8)
    got = oracle.fp8_gemm_nt(a, _pack_bytes(ea), b, _pack_bytes(eb))
    exact = _exact_gemm(a, ea, b, eb)
    for m in range(M):
        for n in range(N):
            assert Fraction(got[m, n]) == exact[m][n], (m, n)


def test_dense_multi_block_n_exact():
    # N spans two 128-row weight blocks with different scales; checks the n // 128 index
    rng = np.random.default_rng(7)
    M, N, K = 2, 130, 256
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    ea = rng.integers(125, 130, size=(M, 2)).astype(np.uint8)
    eb = np.array([[126, 129], [131, 123]], dtype=np.uint8)
    got = oracle.fp8_gemm_nt(a, _pack_bytes(ea), b, _pack_bytes(eb))
    exact = _exact_gemm(a, ea, b, eb)
    for m in range(M):
        for n in (0, 1, 126, 127, 128, 129):
            assert Fraction(got[m, n]) == exact[m][n], (m, n)


def one_hot_check(gemm_fn, gran=128) -> bool:
    """D of one-hot A rows must be exactly 2^pa * b[n, k_m] * 2^pb(n // gran, k_m // 128)."""
    rng = np.random.default_rng(11)
    M, N, K = 6, 300, 640  # 5 K-blocks (ragged packing), 3 N-blocks
    KB, NB = K // 128, -(-N // gran)
    ks = np.array([0, 127, 128, 300, 511, 639])
    a = np.zeros((M, K), dtype=np.uint8)
    a[np.arange(M), ks] = 0x38  # 1.0
    ea = np.full((M, KB), 127, dtype=np.uint8)
    pa = np.array([0, 3, -2, 5, 1, -4])
    ea[np.arange(M), ks // 128] = 127 + pa
    b = _rand_codes(rng, (N, K))
    eb = rng.integers(120, 135, size=(NB, KB)).astype(np.uint8)
    got = gemm_fn(a, _pack_bytes(ea), b, _pack_bytes(eb))
    bv = torch_e4m3(b)
    n = np.arange(N)
    for m in range(M):
        want = (2.0 ** pa[m]) * bv[n, ks[m]] * np.ldexp(1.0, eb[n // gran, ks[m] // 128].astype(np.int64) - 127)
        if got.shape != (M, N) or not np.array_equal(got[m], want):
            return False
    return True


def test_one_hot_rows_exact():
    assert one_hot_check(oracle.fp8_gemm_nt)


def test_identity_times_b_is_b_scaled():
    # A = I (128x128, one 1x128 block per row), unit A scales -> D = B^ exactly
    rng = np.random.default_rng(5)
    N, K = 200, 128
    a = np.where(np.eye(K, dtype=bool), 0x38, 0x00).astype(np.uint8)
    b = _rand_codes(rng, (N, K))
    eb = np.array([[129], [125]], dtype=np.uint8)
    d = oracle.fp8_gemm_nt(a, _pack_bytes(np.full((K, 1), 127, np.uint8)), b, _pack_bytes(eb))
    want = (torch_e4m3(b) * np.ldexp(1.0, eb[np.arange(N) // 128, 0].astype(np.int64) - 127)[:, None]).T
    assert np.array_equal(d, want)


def test_unit_scales_reduce_to_plain_matmul():
    rng = np.random.default_rng(9)
    M, N, K = 37, 150, 384
    a = _rand_codes(rng, (M, K), 0, 14)
    b = _rand_codes(rng, (N, K), 0, 14)
    ones_a = _pack_bytes(np.full((M, 3), 127, np.uint8))
    ones_b = _pack_bytes(np.full((2, 3), 127, np.uint8))
    got = oracle.fp8_gemm_nt(a, ones_a, b, ones_b)
    ref = (torch.from_numpy(torch_e4m3(a)) @ torch.from_numpy(torch_e4m3(b)).T).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-9)


def test_sampled_matches_full():
    rng = np.random.default_rng(3)
    M, N, K = 20, 260, 512
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    sfa = _pack_bytes(rng.integers(120, 135, size=(M, 4)).astype(np.uint8))
    sfb = _pack_bytes(rng.integers(120, 135, size=(3, 4)).astype(np.uint8))
    full = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    r = rng.integers(0, M, size=50)
    c = rng.integers(0, N, size=50)
    assert np.array_equal(oracle.fp8_gemm_nt_sampled(a, sfa, b, sfb, r, c), full[r, c])


def test_masked_rows_and_clamp():
    rng = np.random.default_rng(4)
    G, max_m, N, K = 4, 9, 130, 256
    a = _rand_codes(rng, (G, max_m, K))
    b = _rand_codes(rng, (G, N, K))
    sfa = _pack_bytes(rng.integers(120, 135, size=(G * max_m, 2)).astype(np.uint8)).reshape(G, max_m, 1)
    sfb = _pack_bytes(rng.integers(120, 135, size=(G * 2, 2)).astype(np.uint8)).reshape(G, 2, 1)
    masked_m = np.array([3, -5, 100, 0], dtype=np.int32)
    d, valid = oracle.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, masked_m)
    assert valid.sum(axis=1).tolist() == [3, 0, max_m, 0]
    assert np.isnan(d[~valid]).all()
    for g in range(G):
        m = int(valid[g].sum())
        if m:
            assert np.array_equal(d[g, :m], oracle.fp8_gemm_nt(a[g, :m], sfa[g, :m], b[g], sfb[g]))
    # a single full group is exactly the dense GEMM
    d1, _ = oracle.m_grouped_fp8_gemm_nt_masked(a[2:3], sfa[2:3], b[2:3], sfb[2:3], np.array([max_m]))
    assert np.array_equal(d1[0], oracle.fp8_gemm_nt(a[2], sfa[2], b[2], sfb[2]))


def test_contiguous_rows_follow_their_expert():
    rng = np.random.default_rng(6)
    G, N, K = 3, 140, 256
    m_indices = np.array([0] * 5 + [-1] * 3 + [2] * 4 + [1] * 2 + [-1] * 2, dtype=np.int32)
    Mt = m_indices.size
    a = _rand_codes(rng, (Mt, K))
    b = _rand_codes(rng, (G, N, K))
    sfa = _pack_bytes(rng.integers(120, 135, size=(Mt, 2)).astype(np.uint8))
    sfb = _pack_bytes(rng.integers(120, 135, size=(G * 2, 2)).astype(np.uint8)).reshape(G, 2, 1)
    d, valid = oracle.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_indices)
    assert np.array_equal(valid, m_indices >= 0)
    assert np.isnan(d[~valid]).all()
    for r in np.nonzero(valid)[0]:
        g = m_indices[r]
        assert np.array_equal(d[r], oracle.fp8_gemm_nt(a[r:r + 1], sfa[r:r + 1], b[g], sfb[g])[0])
    rows = np.nonzero(valid)[0]
    cols = rng.integers(0, N, size=rows.size)
    s = oracle.m_grouped_fp8_gemm_nt_contiguous_sampled(a, sfa, b, sfb, m_indices, rows, cols)
    assert np.array_equal(s, d[rows, cols])


# ----------------------------------------------------- planted mistakes ----

def _planted(kind):
    """A copy of the dense oracle with one plausible mistake planted (CPU only)."""
    def fn(a, sfa, b, sfb):
        A = og.dequant_rows(a, sfa)
        if kind == "weight_scale_per_row":
            # B scale indexed by n instead of n // 128
            N, K = b.shape
            KB = K // 128
            s = oracle.ue8m0_to_f64(oracle.unpack_ue8m0(sfb, KB))
            idx = np.minimum(np.arange(N), s.shape[0] - 1)
            B = (oracle.e4m3_to_f64(b).reshape(N, KB, 128) * s[idx][:, :, None]).reshape(N, K)
        else:
            B = og.dequant_weights(b, sfb)
        if kind == "byte_order_reversed":
            M, K = A.shape
            KB = K // 128
            rev = oracle.unpack_ue8m0(sfa, 4 * sfa.shape[1]).reshape(M, -1, 4)[:, :, ::-1].reshape(M, -1)[:, :KB]
            A = (oracle.e4m3_to_f64(a).reshape(M, KB, 128) * oracle.ue8m0_to_f64(rev)[:, :, None]).reshape(M, K)
        if kind == "transposed_b":
            return A @ B[:, : A.shape[1]].T if B.shape[1] != A.shape[1] else (A @ B.T)[:, ::-1]
        if kind == "dropped_last_block":
            A = A.copy()
            A[:, -128:] = 0
        return A @ B.T
    return fn


@pytest.mark.parametrize("kind", ["weight_scale_per_row", "byte_order_reversed", "transposed_b", "dropped_last_block"])
def test_pins_catch_planted_mistakes(kind):
    assert not one_hot_check(_planted(kind)), kind


def test_points_match_full():
    rng = np.random.default_rng(8)
    M, N, K = 9, 300, 640
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    sfa = _pack_bytes(rng.integers(120, 135, size=(M, 5)).astype(np.uint8))
    sfb = _pack_bytes(rng.integers(120, 135, size=(3, 5)).astype(np.uint8))
    full = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    r = rng.integers(0, M, size=40)
    c = rng.integers(0, N, size=40)
    pts = oracle.fp8_gemm_nt_points(a[r], sfa[r], b[c], c, sfb)
    np.testing.assert_allclose(pts, full[r, c], rtol=1e-13, atol=0)


# ------------------------------------------------------ BF16 masked GEMM ----

def torch_bf16(bits):
    """torch's bfloat16 decode of uint16 bit patterns, as float64 (library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def test_bf16_spot_values_from_binary32_layout():
    # sign | 8-bit exponent (bias 127) | 7-bit fraction
    cases = {0x3F80: 1.0, 0xC000: -2.0, 0x3FC0: 1.5, 0x4049: 3.140625, 0x0000: 0.0,
             0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126, 0x7F7F: (2 - 2.0 ** -7) * 2.0 ** 127}
    got = oracle.bf16_to_f64(np.array(list(cases), dtype=np.uint16))
    assert got.tolist() == list(cases.values())
    assert np.isinf(oracle.bf16_to_f64(np.array([0x7F80], np.uint16)))[0]
    assert np.isnan(oracle.bf16_to_f64(np.array([0x7FC0], np.uint16)))[0]


def test_bf16_decode_matches_torch_for_every_code():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine, ref = oracle.bf16_to_f64(codes), torch_bf16(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def _bf16_bits_of(vals):
    """Exact bf16 bit patterns of values that bf16 represents (a test helper)."""
    u = np.asarray(vals, dtype=np.float32).view(np.uint32)
    assert (u & 0xFFFF == 0).all()
    return (u >> 16).astype(np.uint16)


def test_bf16_masked_equals_exact_rational_brute_force():
    rng = np.random.default_rng(12)
    G, max_m, N, K = 3, 5, 4, 16
    # values m * 2^e with 8-bit m and a narrow exponent range: every product
    # and partial sum is exact in float64, so the oracle must equal the
    # rational sum exactly
    def draw(shape):
        m = rng.integers(-255, 256, size=shape)
        e = rng.integers(-8, 0, size=shape)
        return _bf16_bits_of((m * np.ldexp(1.0, e)).astype(np.float32))
    a, b = draw((G, max_m, K)), draw((G, N, K))
    masked_m = np.array([5, 2, 0], dtype=np.int32)
    d, valid = oracle.m_grouped_bf16_gemm_nt_masked(a, b, masked_m)
    av, bv = torch_bf16(a), torch_bf16(b)
    for g in range(G):
        for m in range(max_m):
            for n in range(N):
                if m < masked_m[g]:
                    exact = sum(Fraction(float(av[g, m, k])) * Fraction(float(bv[g, n, k])) for k in range(K))
                    assert Fraction(d[g, m, n]) == exact
                else:
                    assert not valid[g, m] and np.isnan(d[g, m, n])


def bf16_one_hot_check(fn) -> bool:
    """One-hot A rows pick one column of B exactly: D[g, m, n] = B[g, n, k_m]."""
    rng = np.random.default_rng(13)
    G, max_m, N, K = 2, 6, 40, 192
    ks = np.array([0, 63, 64, 100, 150, 191])
    a = np.zeros((G, max_m, K), dtype=np.uint16)
    a[:, np.arange(max_m), ks] = 0x3F80
    b = rng.integers(0, 0x7F00, size=(G, N, K)).astype(np.uint16) | (rng.integers(0, 2, size=(G, N, K)) << 15).astype(np.uint16)
    masked_m = np.array([6, 4], dtype=np.int32)
    d, valid = fn(a, b, masked_m)
    bv = torch_bf16(b)
    for g in range(G):
        for m in range(int(masked_m[g])):
            if not np.array_equal(d[g, m], bv[g, :, ks[m]]):
                return False
    return bool(valid[1, :4].all() and not valid[1, 4:].any())


def test_bf16_masked_one_hot_exact():
    assert bf16_one_hot_check(oracle.m_grouped_bf16_gemm_nt_masked)


def test_bf16_masked_clamp_and_sampled():
    rng = np.random.default_rng(14)
    G, max_m, N, K = 4, 7, 30, 64
    a = rng.integers(0x3C00, 0x4000, size=(G, max_m, K)).astype(np.uint16)
    b = rng.integers(0x3C00, 0x4000, size=(G, N, K)).astype(np.uint16)
    masked_m = np.array([3, -2, 50, 0], dtype=np.int32)
    d, valid = oracle.m_grouped_bf16_gemm_nt_masked(a, b, masked_m)
    assert valid.sum(axis=1).tolist() == [3, 0, max_m, 0]
    # the whole valid region is a plain library matmul of the decoded values
    for g in range(G):
        m = int(valid[g].sum())
        if m:
            ref = (torch.from_numpy(torch_bf16(a[g, :m])) @ torch.from_numpy(torch_bf16(b[g])).T).numpy()
            np.testing.assert_allclose(d[g, :m], ref, rtol=1e-13, atol=0)
    gs = np.array([0, 0, 2, 2]); rs = np.array([0, 2, 6, 1]); cs = np.array([5, 29, 0, 17])
    assert np.array_equal(oracle.m_grouped_bf16_gemm_nt_masked_sampled(a, b, masked_m, gs, rs, cs), d[gs, rs, cs])


def _planted_bf16(kind):
    """A copy of the BF16 masked oracle with one plausible mistake planted (CPU only)."""
    def fn(a, b, masked_m):
        G, max_m, K = a.shape
        mm = np.clip(masked_m, 0, max_m)
        if kind == "rows_off_by_one":
            mm = np.clip(masked_m + 1, 0, max_m)
        out = np.full((G, max_m, b.shape[1]), np.nan)
        for g in range(G):
            m = int(mm[g])
            A = oracle.bf16_to_f64(a[g, :m])
            B = oracle.bf16_to_f64(b[g])
            if kind == "half_swapped":   # low and high bytes of each code swapped
                B = oracle.bf16_to_f64(((b[g] >> 8) | (b[g] << 8)).astype(np.uint16))
            if kind == "wrong_group":
                B = oracle.bf16_to_f64(b[(g + 1) % G])
            out[g, :m] = A @ B.T
        valid = np.arange(max_m)[None, :] < mm[:, None]
        return out, valid
    return fn


@pytest.mark.parametrize("kind", ["rows_off_by_one", "half_swapped", "wrong_group"])
def test_bf16_pins_catch_planted_mistakes(kind):
    assert not bf16_one_hot_check(_planted_bf16(kind)), kind


# ------------------------------------------- dense GEMM with a C matrix ----

def test_acc_with_zero_or_absent_c_is_the_plain_gemm():
    rng = np.random.default_rng(21)
    M, N, K = 17, 140, 384
    a, b = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    sfa = _pack_bytes(rng.integers(120, 135, size=(M, 3)).astype(np.uint8))
    sfb = _pack_bytes(rng.integers(120, 135, size=(2, 3)).astype(np.uint8))
    plain = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    assert np.array_equal(oracle.fp8_gemm_nt_acc(a, sfa, b, sfb), plain)
    assert np.array_equal(oracle.fp8_gemm_nt_acc(a, sfa, b, sfb, np.zeros((M, N))), plain)


def test_acc_with_zero_a_returns_c_exactly():
    rng = np.random.default_rng(22)
    M, N, K = 9, 64, 256
    a = np.zeros((M, K), dtype=np.uint8)
    b = _rand_codes(rng, (N, K))
    c = rng.standard_normal((M, N)).astype(np.float32).astype(np.float64)
    sfa = _pack_bytes(np.full((M, 2), 127, np.uint8))
    sfb = _pack_bytes(np.full((1, 2), 127, np.uint8))
    assert np.array_equal(oracle.fp8_gemm_nt_acc(a, sfa, b, sfb, c), c)


def test_acc_one_hot_plus_c_exact():
    # one-hot A rows select one (scaled) column of B; adding a C of small
    # integers keeps every sum exact in float64
    rng = np.random.default_rng(23)
    M, N, K = 4, 130, 256
    ks = np.array([0, 100, 128, 255])
    a = np.zeros((M, K), dtype=np.uint8)
    a[np.arange(M), ks] = 0x38
    b = _rand_codes(rng, (N, K))
    sfa = _pack_bytes(np.full((M, 2), 127, np.uint8))
    sfb = _pack_bytes(np.full((2, 2), 127, np.uint8))
    c = rng.integers(-8, 9, size=(M, N)).astype(np.float64)
    got = oracle.fp8_gemm_nt_acc(a, sfa, b, sfb, c)
    bv = torch_e4m3(b)
    for m in range(M):
        assert np.array_equal(got[m], c[m] + bv[:, ks[m]])


# ------------------------------------------------ per-token quantiser ----

def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes)
    got = oracle.e4m3_encode_rne(vals)
    # +0 and -0 keep their sign; every other value maps back to its own code
    assert np.array_equal(got, codes)


def test_e4m3_encode_ties_go_to_the_even_code():
    pos = oracle.e4m3_to_f64(np.arange(127, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2          # exact in float64
    got = oracle.e4m3_encode_rne(mids)
    lo = np.arange(126)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode_rne(-mids), (want | 0x80).astype(np.uint8))


def test_e4m3_encode_matches_torch_float8_cast():
    rng = np.random.default_rng(31)
    v = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(5000) * 0.01,
                        rng.uniform(-448, 448, 5000)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode_rne(v.astype(np.float64)), ref)


def test_scale_exponent_brackets_amax():
    rng = np.random.default_rng(32)
    amax = np.concatenate([
        np.abs(rng.standard_normal(5000)).astype(np.float32),
        (448.0 * np.ldexp(1.0, rng.integers(-30, 30, 200))).astype(np.float32),         # exactly 448 * 2^k
        np.nextafter((448.0 * np.ldexp(1.0, rng.integers(-30, 30, 200))).astype(np.float32),
                     np.float32(np.inf)),                                               # just above
        np.array([0.0, 1e-9, 9.99e-5], dtype=np.float32)])                              # below the floor
    e = oracle.scale_exponent(amax)
    a = np.maximum(amax.astype(np.float64), float(np.float32(1e-4)))
    assert (448.0 * np.ldexp(1.0, e) >= a).all()
    assert (448.0 * np.ldexp(1.0, e - 1) < a).all()


def test_quantiser_matches_the_input_generator():
    # two independent routes to the same recipe: the oracle (exact integer
    # exponent, its own E4M3 encoder) and the input generator (float64 ratio,
    # torch's float8 cast)
    from moe_grouped_gemm_tcgen05_b200 import workloads as W
    rng = np.random.default_rng(33)
    x = (rng.standard_normal((37, 640)) * rng.uniform(0.01, 100, size=(37, 1))).astype(np.float32)
    q_ref, sf_ref = W.quantise_rows(x)
    q, packed, sf = oracle.quantize_fp8_1x128(x.astype(np.float64))
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sf, sf_ref)
    assert np.array_equal(packed, oracle.pack_ue8m0(sf_ref))


def _planted_quant(kind):
    """A copy of the quantiser's exponent rule / encoder with one mistake (CPU only)."""
    def scale_exp(amax):
        a = np.maximum(np.asarray(amax, dtype=np.float64), float(np.float32(1e-4)))
        m2, e2 = np.frexp(a)
        E, m = e2 - 1, 2.0 * m2
        if kind == "threshold_inclusive":
            return (E - 8 + (m >= 1.75)).astype(np.int64)
        if kind == "floor_not_ceil":
            return (E - 8).astype(np.int64)
        return (E - 8 + (m > 1.75)).astype(np.int64)
    return scale_exp


@pytest.mark.parametrize("kind", ["threshold_inclusive", "floor_not_ceil"])
def test_quantiser_pins_catch_planted_mistakes(kind):
    amax = (448.0 * np.ldexp(1.0, np.arange(-10, 10))).astype(np.float32)
    amax = np.concatenate([amax, np.nextafter(amax, np.float32(np.inf)), np.float32([3.0, 0.3])])
    e = _planted_quant(kind)(amax)
    a = amax.astype(np.float64)
    ok = (448.0 * np.ldexp(1.0, e) >= a).all() and (448.0 * np.ldexp(1.0, e - 1) < a).all()
    assert not ok, kind


def test_encoder_pin_catches_ties_away_from_zero():
    pos = oracle.e4m3_to_f64(np.arange(127, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    away = np.arange(1, 127).astype(np.uint8)              # always the upper neighbour
    assert not np.array_equal(away, oracle.e4m3_encode_rne(mids))


# ------------------------------------------- other operand layouts ----

@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_layouts_equal_exact_rational_brute_force(layout):
    # D[m, n] = sum_k A[m, k] B[n, k] with each operand read from its own
    # storage order, computed with exact rationals straight from the codes
    rng = np.random.default_rng(41)
    M, N, K = 3, 5, 256
    a_mk = _rand_codes(rng, (M, K))
    b_nk = _rand_codes(rng, (N, K))
    ea = rng.integers(120, 135, size=(M, 2)).astype(np.uint8)
    eb = rng.integers(120, 135, size=(1, 2)).astype(np.uint8)
    a = a_mk if layout[0] == "n" else np.ascontiguousarray(a_mk.T)
    b = b_nk if layout[1] == "t" else np.ascontiguousarray(b_nk.T)
    got = oracle.fp8_gemm(a, _pack_bytes(ea), b, _pack_bytes(eb), layout)
    av, bv = torch_e4m3(a), torch_e4m3(b)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                x = av[m, k] if layout[0] == "n" else av[k, m]
                y = bv[n, k] if layout[1] == "t" else bv[k, n]
                acc += (Fraction(float(x)) * Fraction(2) ** (int(ea[m, k // 128]) - 127) *
                        Fraction(float(y)) * Fraction(2) ** (int(eb[0, k // 128]) - 127))
            assert Fraction(got[m, n]) == acc, (layout, m, n)


def test_layout_pin_catches_an_unswapped_operand():
    rng = np.random.default_rng(42)
    M, K = 128, 128
    a = _rand_codes(rng, (M, K))
    ones = _pack_bytes(np.full((M, 1), 127, np.uint8))
    ones_b = _pack_bytes(np.full((1, 1), 127, np.uint8))  # one 128x128 block of B
    # reading a [K, M] A as if it were [M, K] changes the result
    assert not np.array_equal(oracle.fp8_gemm(a, ones, a, ones_b, "tt"), oracle.fp8_gemm(a, ones, a, ones_b, "nt"))


# ------------------------------------ weights with one scale row per row ----
# "DeepInside DeepGEMM", section 4: the minimal FP8 GEMM example gives B a scale
# tensor of shape [n, k // 128], one scale per 1x128 block of each row of B.

def _gemm_rows(a, sfa, b, sfb):
    return oracle.fp8_gemm_nt(a, sfa, b, sfb, sfb_gran_n=1)


@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 128, 21), (8, 7, 256, 22), (2, 3, 384, 23)])
def test_per_row_weight_scales_equal_exact_rational_brute_force(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    ea = rng.integers(124, 131, size=(M, K // 128)).astype(np.uint8)
    eb = rng.integers(120, 136, size=(N, K // 128)).astype(np.uint8)
    got = _gemm_rows(a, _pack_bytes(ea), b, _pack_bytes(eb))
    exact = _exact_gemm(a, ea, b, eb, gran=1)
    for m in range(M):
        for n in range(N):
            assert Fraction(got[m, n]) == exact[m][n], (m, n)


def test_per_row_one_hot_rows_exact():
    assert one_hot_check(_gemm_rows, gran=1)


def test_per_row_scales_repeated_over_blocks_equal_block_scales():
    # scale rows that repeat each 128x128 block row reduce to the block form
    rng = np.random.default_rng(24)
    M, N, K = 5, 300, 512
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    sfa = _pack_bytes(rng.integers(122, 133, size=(M, K // 128)).astype(np.uint8))
    eb = rng.integers(120, 136, size=(3, K // 128)).astype(np.uint8)
    block = oracle.fp8_gemm_nt(a, sfa, b, _pack_bytes(eb))
    rows = _gemm_rows(a, sfa, b, _pack_bytes(np.repeat(eb, 128, axis=0)[:N]))
    assert np.array_equal(block, rows)


def test_per_row_scale_moves_only_its_own_column():
    # raising the scale bytes of row n0 of B by 3 multiplies column n0 of D by 8
    # exactly (powers of two) and leaves every other column, including the
    # rest of n0's 128-row block, unchanged
    rng = np.random.default_rng(25)
    M, N, K, n0 = 4, 260, 384, 131
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (N, K))
    sfa = _pack_bytes(rng.integers(122, 133, size=(M, K // 128)).astype(np.uint8))
    eb = rng.integers(120, 130, size=(N, K // 128)).astype(np.uint8)
    d0 = _gemm_rows(a, sfa, b, _pack_bytes(eb))
    eb2 = eb.copy()
    eb2[n0] += 3
    d1 = _gemm_rows(a, sfa, b, _pack_bytes(eb2))
    others = np.arange(N) != n0
    assert np.array_equal(d1[:, others], d0[:, others])
    assert np.array_equal(d1[:, n0], 8.0 * d0[:, n0])


def test_per_row_grouped_forms_follow_the_dense_one():
    rng = np.random.default_rng(26)
    G, max_m, N, K = 3, 20, 140, 256
    a = _rand_codes(rng, (G, max_m, K))
    b = _rand_codes(rng, (G, N, K))
    sfa = _pack_bytes(rng.integers(122, 133, size=(G * max_m, K // 128)).astype(np.uint8)).reshape(G, max_m, -1)
    eb = rng.integers(120, 136, size=(G, N, K // 128)).astype(np.uint8)
    sfb = _pack_bytes(eb.reshape(G * N, -1)).reshape(G, N, -1)
    mm = np.array([7, 0, 20], dtype=np.int32)
    d, valid = oracle.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, mm, sfb_gran_n=1)
    for g in range(G):
        m = int(mm[g])
        assert np.array_equal(d[g, :m], _gemm_rows(a[g, :m], sfa[g, :m], b[g], sfb[g]))
        assert np.all(np.isnan(d[g, m:])) and valid[g].sum() == m
    # contiguous: the same rows laid end to end, padding rows marked -1
    idx = np.concatenate([np.full(7, 0), np.full(3, -1), np.full(20, 2)]).astype(np.int32)
    ac = np.concatenate([a[0, :7], a[1, :3], a[2]])
    sc = np.concatenate([sfa[0, :7], sfa[1, :3], sfa[2]])
    dc, vc = oracle.m_grouped_fp8_gemm_nt_contiguous(ac, sc, b, sfb, idx, sfb_gran_n=1)
    assert np.array_equal(dc[:7], d[0, :7]) and np.array_equal(dc[10:], d[2, :20]) and not vc[7:10].any()
    pts = oracle.m_grouped_fp8_gemm_nt_masked_sampled(a, sfa, b, sfb, [0, 2, 2], [6, 0, 19], [0, 139, 77],
                                                      sfb_gran_n=1)
    assert np.array_equal(pts, [d[0, 6, 0], d[2, 0, 139], d[2, 19, 77]])


def test_per_row_granularity_is_checked():
    a = np.zeros((1, 128), np.uint8)
    b = np.zeros((130, 128), np.uint8)
    with pytest.raises(ValueError):
        oracle.fp8_gemm_nt(a, np.zeros((1, 1), np.int32), b, np.zeros((130, 1), np.int32), sfb_gran_n=64)
    with pytest.raises(ValueError):  # 2 scale rows cover 130 rows only at granularity 128
        oracle.fp8_gemm_nt(a, np.zeros((1, 1), np.int32), b, np.zeros((2, 1), np.int32), sfb_gran_n=1)


def _planted_rows(kind):
    """A copy of the per-row oracle with one plausible mistake planted (CPU only)."""
    def fn(a, sfa, b, sfb):
        N, K = b.shape
        KB = K // 128
        s = oracle.ue8m0_to_f64(oracle.unpack_ue8m0(sfb, KB))
        n = np.arange(N)
        idx = {"block_index": n // 128, "next_row": np.minimum(n + 1, N - 1), "first_row": n * 0}[kind]
        B = (oracle.e4m3_to_f64(b).reshape(N, KB, 128) * s[idx][:, :, None]).reshape(N, K)
        return og.dequant_rows(a, sfa) @ B.T
    return fn


@pytest.mark.parametrize("kind", ["block_index", "next_row", "first_row"])
def test_per_row_pins_catch_planted_mistakes(kind):
    assert not one_hot_check(_planted_rows(kind), gran=1), kind


# ------------------------------------------- groups given by psum_m ----
# Reading of "DeepGEMM CUDA Graph Compatibility for Masked Grouped GEMMs",
# Tensor-Based Metadata Arguments: psum_m[g] is the inclusive prefix sum of the
# groups' row counts; group g owns rows [psum_m[g-1], psum_m[g]) of A.

def test_psum_rows_hand_worked():
    # well formed: counts 2, 0, 4 over 7 rows (row 6 in no group)
    s, e = oracle.psum_group_rows([2, 2, 6], 7)
    assert list(s) == [0, 2, 2] and list(e) == [2, 2, 6]
    # malformed entries: negative, decreasing, past M_total
    s, e = oracle.psum_group_rows([-3, 5, 2, 9, 100], 8)
    assert list(s) == [0, 0, 5, 5, 8] and list(e) == [0, 5, 5, 8, 8]


def _psum_exact(a, ea, b, eb, owner):
    """Exact rational D for rows with an owning group (owner[r] = g or -1), 128x128 B blocks."""
    M, K = a.shape
    N = b.shape[1]
    av, bv = torch_e4m3(a), [torch_e4m3(b[g]) for g in range(b.shape[0])]
    out = {}
    for r in range(M):
        g = owner[r]
        if g < 0:
            continue
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += (Fraction(av[r, k]) * Fraction(2) ** (int(ea[r, k // 128]) - 127) *
                        Fraction(bv[g][n, k]) * Fraction(2) ** (int(eb[g, n // 128, k // 128]) - 127))
            out[(r, n)] = acc
    return out


def test_psum_equals_exact_rational_brute_force():
    rng = np.random.default_rng(31)
    M, N, K, G = 7, 3, 256, 3
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (G, N, K))
    ea = rng.integers(124, 131, size=(M, 2)).astype(np.uint8)
    eb = rng.integers(124, 131, size=(G, 1, 2)).astype(np.uint8)
    psum = [2, 2, 6]
    owner = [0, 0, 2, 2, 2, 2, -1]  # written out by hand from the reading
    d, valid = oracle.m_grouped_fp8_gemm_nt_psum(a, _pack_bytes(ea), b,
                                                 _pack_bytes(eb.reshape(G, 2)).reshape(G, 1, 1), psum)
    exact = _psum_exact(a, ea, b, eb, owner)
    assert list(valid) == [o >= 0 for o in owner]
    assert np.all(np.isnan(d[6]))
    for (r, n), v in exact.items():
        assert Fraction(d[r, n]) == v, (r, n)


def test_psum_reduces_to_the_contiguous_form():
    # the same rows tagged per row with their group (m_indices) give the same D
    rng = np.random.default_rng(32)
    M, N, K, G = 300, 140, 384, 4
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (G, N, K))
    sfa = _pack_bytes(rng.integers(122, 133, size=(M, K // 128)).astype(np.uint8))
    sfb = _pack_bytes(rng.integers(120, 136, size=(G * 2, K // 128)).astype(np.uint8)).reshape(G, 2, -1)
    counts = [37, 0, 150, 90]  # 277 rows in groups, 23 in none
    psum = np.cumsum(counts)
    m_indices = np.concatenate([np.full(c, g) for g, c in enumerate(counts)] + [np.full(M - psum[-1], -1)])
    d, valid = oracle.m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, psum)
    dc, vc = oracle.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_indices.astype(np.int32))
    assert np.array_equal(valid, vc)
    assert np.array_equal(d[valid], dc[vc])


def _planted_psum(kind):
    """A copy of the psum oracle with one plausible mistake planted (CPU only)."""
    def fn(a, sfa, b, sfb, psum_m):
        M = a.shape[0]
        ps = np.asarray(psum_m, dtype=np.int64)
        if kind == "exclusive_read":       # psum_m taken as the groups' first rows
            starts, ends = ps, np.concatenate([ps[1:], [M]])
        elif kind == "no_running_max":     # decreasing entries not clamped
            ends = np.minimum(np.maximum(ps, 0), M)
            starts = np.concatenate([[0], ends[:-1]])
        else:                              # "expert_off_by_one": group g uses B[g + 1]
            starts, ends = oracle.psum_group_rows(ps, M)
        out = np.full((M, b.shape[1]), np.nan)
        for g in range(b.shape[0]):
            if ends[g] > starts[g]:
                gb = min(g + 1, b.shape[0] - 1) if kind == "expert_off_by_one" else g
                out[starts[g]:ends[g]] = oracle.fp8_gemm_nt(a[starts[g]:ends[g]], sfa[starts[g]:ends[g]], b[gb], sfb[gb])
        return out
    return fn


@pytest.mark.parametrize("kind", ["exclusive_read", "no_running_max", "expert_off_by_one"])
def test_psum_pins_catch_planted_mistakes(kind):
    rng = np.random.default_rng(33)
    M, N, K, G = 40, 16, 128, 4
    a = _rand_codes(rng, (M, K))
    b = _rand_codes(rng, (G, N, K))
    sfa = _pack_bytes(np.full((M, 1), 127, np.uint8))
    sfb = _pack_bytes(np.full((G, 1), 127, np.uint8)).reshape(G, 1, 1)
    psum = np.array([10, 25, 20, 38])  # one decreasing entry: group 2 is empty
    want, _ = oracle.m_grouped_fp8_gemm_nt_psum(a, sfa, b, sfb, psum)
    got = _planted_psum(kind)(a, sfa, b, sfb, psum)
    assert not np.array_equal(np.nan_to_num(got, nan=1e300), np.nan_to_num(want, nan=1e300)), kind
