"""Pins for the CPU oracle: facts fixed by the pages, closed forms, published
known-answer vectors and brute force, independent of the oracle's own code.
CPU only."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import brute
import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.strip()
    return out


def bf16(vals, shape=None):
    a = np.asarray(vals, dtype=np.float32)
    if shape is not None:
        a = a.reshape(shape)
    return W.f32_to_bf16_bits(a)


# ------------------------------------------------------------------ E2M1 grid
def test_e2m1_values_match_pages(orc):
    g = golden("e2m1_values.txt")
    vals = [orc.e2m1_decode(c) for c in range(16)]
    assert len(vals) == int(g["n_codes"])
    assert max(abs(v) for v in vals) == float(g["max_magnitude"])
    assert min(vals) == -float(g["max_magnitude"])
    for v in g["present"].split():
        assert float(v) in vals and -float(v) in vals
    for v in g["absent"].split():
        assert float(v) not in vals and -float(v) not in vals
    # agrees with the bit-field definition enumerated independently
    np.testing.assert_array_equal(np.array(vals), brute.e2m1_grid())
    # 16 distinct codes, 15 distinct values (+0 and -0 coincide)
    assert len(set(vals)) == 15


def test_five_not_representable(orc):
    assert orc.e2m1_decode(orc.e2m1_rne(5.0)) == 4.0     # tie between 4 and 6 -> even mantissa
    assert orc.e2m1_decode(orc.e2m1_rne(-5.0)) == -4.0
    ups = sum(orc.e2m1_sr(5.0, u) == 7 for u in range(0, 65536, 1))
    assert ups == 32768                                  # P(6) = P(4) = 1/2 under SR


def test_e2m1_rne_brute_force(orc):
    rng = np.random.default_rng(11)
    grid = brute.e2m1_grid()[:8]
    mids = (grid[1:] + grid[:-1]) / 2
    ys = np.concatenate([
        grid, -grid, mids, -mids,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        [0.0, -0.0, 6.0, 6.5, 7.0, 100.0, -1e30, 1e-30, -1e-30],
        rng.uniform(-8, 8, 4000).astype(np.float32),
        rng.standard_normal(2000).astype(np.float32) * 0.3,
    ]).astype(np.float32)
    expect = brute.e2m1_rne(ys.astype(np.float64))
    got = np.array([orc.e2m1_rne(float(y)) for y in ys], dtype=np.uint8)
    np.testing.assert_array_equal(got, expect)


# ------------------------------------------------------------------ E4M3 grid
def test_e4m3_decode_matches_definition(orc):
    grid = brute.e4m3_grid()
    got = np.array([orc.e4m3_decode(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(grid))
    ok = ~np.isnan(grid)
    np.testing.assert_array_equal(got[ok], grid[ok])
    assert np.nanmax(got) == 448.0
    assert orc.e4m3_decode(0x51) == 9.0


def test_e4m3_rne_brute_force(orc):
    rng = np.random.default_rng(12)
    grid = brute.e4m3_grid()[:0x7F]
    mids = (grid[1:] + grid[:-1]) / 2
    ys = np.concatenate([
        grid, mids,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)).astype(np.float64),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)).astype(np.float64),
        [0.0, 448.0, 449.0, 464.0, 465.0, 480.0, 1e9, 2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11],
        np.exp(rng.uniform(-12, 7, 4000)),
    ])
    expect = brute.e4m3_rne_sat(ys)
    got = np.array([orc.e4m3_rne_sat(float(y)) for y in ys], dtype=np.uint8)
    np.testing.assert_array_equal(got, expect)


# ------------------------------------------------------------------ stochastic rounding
def test_sr_exact_probabilities(orc):
    g = golden("sr_example.txt")
    x = float(g["value"])
    lo, hi = float(g["low"]), float(g["high"])
    codes = [orc.e2m1_sr(x, u) for u in range(65536)]
    vals = np.array([orc.e2m1_decode(c) for c in codes])
    assert set(vals.tolist()) == {lo, hi}
    assert np.mean(vals == hi) == float(g["p_high"])
    assert np.mean(vals) == float(g["mean"])             # exactly, over all 2^16 draws


def test_sr_unbiased_on_grid_and_between(orc):
    # SR of any value lies on one of its two neighbours; on the grid it is exact.
    grid = brute.e2m1_grid()[:8]
    for v in grid:
        assert all(orc.e2m1_decode(orc.e2m1_sr(float(v), u)) == v for u in (0, 1, 12345, 65535))
    rng = np.random.default_rng(13)
    for y in rng.uniform(0, 6, 200):
        y = float(np.float32(y))
        i = np.searchsorted(grid, y, side="right") - 1
        lo, hi = grid[i], grid[min(i + 1, 7)]
        us = np.arange(0, 65536, 7)
        vals = np.array([orc.e2m1_decode(orc.e2m1_sr(y, int(u))) for u in us])
        assert set(np.unique(vals)) <= {lo, hi}
        # P(up) = floor(f * 2^16) / 2^16 within the sampling grid of u
        f = (y - lo) / (hi - lo) if hi > lo else 0.0
        assert abs(np.mean(vals == hi) - f) <= 2.0 / 65536 * 7 + 1e-12


def test_sr_2p25_philox_1e6_draws(orc):
    """10^6 Philox draws of SR(2.25) through the tensor quantiser: the frequency of 3
    and the mean sit within 3 sigma of 1/4 and 2.25."""
    g = golden("sr_example.txt")
    rows, cols = 1024, 1088
    x = np.full((rows, cols), 2.25, dtype=np.float32)
    x[:, ::16] = 6.0            # each block's max is 6 -> block scale exactly 1 with S = 1
    xb = bf16(x)
    q, sf, gsc = orc.nvfp4_quantize(xb, 0, rounding=1, seed=1234, amax=(2688.0, 2688.0))
    assert gsc == 1.0 and np.all(sf == 0x38)            # E4M3 0x38 == 1.0
    codes = brute.unpack_nibbles(q)
    vals = np.array([orc.e2m1_decode(c) for c in range(16)])[codes]
    v = vals[x == 2.25]
    n = v.size
    assert n >= int(g["draws"])
    p_hi = float(g["p_high"])
    sigma_p = math.sqrt(p_hi * (1 - p_hi) / n)
    assert abs(np.mean(v == 3.0) - p_hi) <= 3 * sigma_p
    assert set(np.unique(v)) == {2.0, 3.0}
    sigma_mean = math.sqrt(0.1875 / n)                     # var of {2 w.p. 3/4, 3 w.p. 1/4}
    assert abs(np.mean(v) - float(g["mean"])) <= 3 * sigma_mean


def test_sr_tensor_unbiased_over_seeds(orc):
    """E[dequant(SR(x))] = x: average over many seeds converges to the input."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    xb = bf16(x)
    xf = W.bf16_bits_to_f32(xb).astype(np.float64)
    acc = np.zeros_like(xf)
    n = 400
    for s in range(n):
        q, sf, g = orc.nvfp4_quantize(xb, 0, rounding=1, seed=1000 + s)
        acc += orc.nvfp4_dequant(q, sf, g)
    mean = acc / n
    _, sf, g = orc.nvfp4_quantize(xb, 0, rounding=0)
    dg = np.repeat(np.array([orc.e4m3_decode(b) for b in sf.reshape(-1)]).reshape(sf.shape),
                   16, axis=1) * g
    step = dg * 2.0                                  # largest grid gap (2) times block scale
    # elements whose scaled value exceeds 6 (the block scale rounded down) saturate: SR is
    # only unbiased inside the grid's range
    inside = np.abs(xf) / dg < 6.0
    assert inside.mean() > 0.9
    # per-element standard error <= step/2/sqrt(n); allow 5 sigma
    err = np.abs(mean - xf)
    assert np.all(err[inside] <= 5 * step[inside] / 2 / math.sqrt(n) + 1e-12)
    assert abs(np.mean((mean - xf)[inside])) < 1e-3


# ------------------------------------------------------------------ block scale example
def _block_example():
    g = golden("block_scale_example.txt")
    rng = np.random.default_rng(5)
    bs = int(g["block_size"])
    blk = rng.uniform(-50, 50, (16, bs)).astype(np.float32)
    blk[0, 3] = float(g["block_max"])
    return g, blk


def test_minus54_becomes_minus6_times_9_no_global_scale(orc):
    g, blk = _block_example()
    q, sf, gsc = orc.nvfp4_quantize(bf16(blk), 0, amax=(2688.0, 2688.0))   # S = g = 1
    assert gsc == 1.0
    assert sf[0, 0] == 0x51 and orc.e4m3_decode(int(sf[0, 0])) == float(g["multiplier"])
    codes = brute.unpack_nibbles(q)
    assert orc.e2m1_decode(int(codes[0, 3])) == float(g["element"])
    assert codes[0, 3] == 0xF


def test_minus54_with_computed_global_scale(orc):
    g, blk = _block_example()
    q, sf, gsc = orc.nvfp4_quantize(bf16(blk), 0)
    codes = brute.unpack_nibbles(q)
    assert orc.e2m1_decode(int(codes[0, 3])) == float(g["element"])
    mult = orc.e4m3_decode(int(sf[0, 0])) * gsc
    assert abs(mult - float(g["multiplier"])) <= 9.0 * 2.0 ** -20


# ------------------------------------------------------------------ 2D scaling
def test_2d_scale_transpose_invariant(orc):
    rng = np.random.default_rng(6)
    w = bf16(rng.standard_normal((64, 48)).astype(np.float32) * 0.02)
    qr, sr_, gr = orc.nvfp4_quantize(w, 0, scaling=1)
    qc, sc_, gc = orc.nvfp4_quantize(w, 1, scaling=1)
    assert gr == gc
    # scale of element (r, c): rowwise sr_[r, c//16]; columnwise sc_[c, r//16]
    R, C = 64, 48
    rr, cc = np.meshgrid(np.arange(R), np.arange(C), indexing="ij")
    np.testing.assert_array_equal(sr_[rr, cc // 16], sc_[cc, rr // 16])
    np.testing.assert_array_equal(brute.unpack_nibbles(qr), brute.unpack_nibbles(qc).T)
    # quantising W^T rowwise gives the transposed scales as well
    wt = np.ascontiguousarray(w.T)
    qt, st, gt = orc.nvfp4_quantize(wt, 0, scaling=1)
    np.testing.assert_array_equal(st, sc_)
    np.testing.assert_array_equal(qt, qc)
    # 1D scales are NOT transpose invariant on generic data
    _, s1r, _ = orc.nvfp4_quantize(w, 0, scaling=0)
    _, s1c, _ = orc.nvfp4_quantize(w, 1, scaling=0)
    assert not np.array_equal(s1r[rr, cc // 16], s1c[cc, rr // 16])


def test_2d_outlier_zeroes_the_tile(orc):
    """One large value in a 16x16 tile lifts the shared multiplier so that the other
    values round to zero (iitak, "How it works"); 1D blocks keep more of them."""
    rng = np.random.default_rng(7)
    w = rng.standard_normal((16, 16)).astype(np.float32) * 0.02
    w[5, 9] = 100 * np.abs(w).max()
    wb = bf16(w)
    q2, _, _ = orc.nvfp4_quantize(wb, 0, scaling=1)
    q1, _, _ = orc.nvfp4_quantize(wb, 0, scaling=0)
    z2 = np.mean((brute.unpack_nibbles(q2) & 7) == 0)
    z1 = np.mean((brute.unpack_nibbles(q1) & 7) == 0)
    assert z2 > 0.9 and z2 > z1


# ------------------------------------------------------------------ Hadamard
def _rht_matrix(orc, signs):
    T = np.zeros((16, 16))
    for j in range(16):
        e = np.zeros(16, dtype=np.float32)
        e[j] = 1
        T[:, j] = orc.rht16(signs, e)
    return T


def test_hadamard_closed_form(orc):
    ones = np.ones(16, dtype=np.float32)
    H = 4.0 * _rht_matrix(orc, ones)
    np.testing.assert_array_equal(H, brute.sylvester_hadamard(16))
    np.testing.assert_array_equal(H @ H.T, 16.0 * np.eye(16))


def test_rht_orthonormal_and_inverse(orc):
    signs = orc.rht_signs(99)
    assert set(np.unique(signs)) <= {-1.0, 1.0} and len(np.unique(signs)) == 2
    T = _rht_matrix(orc, signs)
    np.testing.assert_allclose(T @ T.T, np.eye(16), atol=0)
    np.testing.assert_array_equal(T, brute.sylvester_hadamard(16) @ np.diag(signs) / 4)
    rng = np.random.default_rng(8)
    for _ in range(50):
        v = rng.standard_normal(16).astype(np.float32)
        out = orc.rht16(signs, v).astype(np.float64)
        ref = T @ v.astype(np.float64)
        np.testing.assert_allclose(out, ref, rtol=0, atol=4 * np.abs(v).sum() * 2.0 ** -24)
        assert abs(np.linalg.norm(out) - np.linalg.norm(v)) <= 1e-5 * np.linalg.norm(v)


def test_rht_cancels_in_product(orc):
    """With one sign draw for both operands, sum_k (Ta)_k (Tb)_k = a.b."""
    signs = orc.rht_signs(5)
    rng = np.random.default_rng(9)
    a = rng.standard_normal(16).astype(np.float32)
    b = rng.standard_normal(16).astype(np.float32)
    ta, tb = orc.rht16(signs, a).astype(np.float64), orc.rht16(signs, b).astype(np.float64)
    assert abs(ta @ tb - a.astype(np.float64) @ b) < 1e-5


# ------------------------------------------------------------------ Philox
def test_philox_known_answers(orc):
    with open(os.path.join(GOLDEN, "philox_kat.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(t, 16) for t in r]
        assert orc.philox4x32_10(v[0:4], v[4:6]) == tuple(v[6:10])


def test_sr_bits_mapping(orc):
    # MXFP8 stream: idx -> counter idx/8, word (idx%8)/2, half idx%2
    seed, off = 0x1234_5678_9ABC_DEF0, 77
    for idx in [0, 1, 7, 8, 9, 1000003, 2 ** 40 + 5]:
        j = idx >> 3
        w = orc.philox4x32_10([j & 0xFFFFFFFF, j >> 32, 2, off], [seed & 0xFFFFFFFF, seed >> 32])
        word = w[(idx & 7) >> 1]
        expect = (word >> 16) if idx & 1 else word & 0xFFFF
        assert orc.sr_bits(seed, off, 2, idx) == expect


def test_sr_bits_nvfp4_mapping(orc):
    """NVFP4 streams: one 32-bit word per 4 elements (word (idx/4)%4 of the Philox call
    for idx/16); element k takes v = (hi byte, lo byte) = (B2,B0), (rev B0, rev B2),
    (B3,B1), (rev B1, rev B3) and u = 65535 - v."""
    rev = lambda b: int(f"{b:08b}"[::-1], 2)
    seed, off = 0xDEADBEEF_0BADF00D, 3
    for idx in [0, 1, 2, 3, 4, 15, 16, 17, 999999, 2 ** 36 + 13]:
        j = idx >> 4
        w = orc.philox4x32_10([j & 0xFFFFFFFF, j >> 32, 0, off], [seed & 0xFFFFFFFF, seed >> 32])
        word = w[(idx >> 2) & 3]
        B = [(word >> (8 * i)) & 0xFF for i in range(4)]
        hi, lo = [(B[2], B[0]), (rev(B[0]), rev(B[2])), (B[3], B[1]), (rev(B[1]), rev(B[3]))][idx & 3]
        assert orc.sr_bits_nvfp4(seed, off, 0, idx) == 65535 - ((hi << 8) | lo)
    # every element's draw is uniform: over many groups each bit is set about half the time
    us = np.array([orc.sr_bits_nvfp4(7, 0, 1, i) for i in range(40000)])
    for k in range(4):
        bits = (us[k::4][:, None] >> np.arange(16)) & 1
        assert np.all(np.abs(bits.mean(axis=0) - 0.5) < 0.03)


# Largest |P(up_2k and up_2k+1) - P(up_2k) P(up_2k+1)| over every pair of thresholds,
# found by exact enumeration (attained at t = 21845 = 65535/3 for both elements).
SR_PAIR_MAX_COV = 5.444 / 65536


def test_sr_bits_nvfp4_joint_law(orc):
    """Exact joint law of the two draws that share a byte pair.  Over all 2^16 values
    of (B0, B2) -- the two bytes elements 0 and 1 of a 4-group read -- each element's u
    takes every 16-bit value exactly once (uniform marginals, so every element rounds up
    with probability exactly floor(f 2^16)/2^16), and the two rounding decisions are
    nearly but not exactly independent: the covariance of 'u0 < t0' and 'u1 < t1' never
    exceeds SR_PAIR_MAX_COV (correlation <= 3.8e-4 at P(up) = 1/3).  Elements 0 and 2
    (disjoint bytes) are exactly independent.  The oracle's stream obeys this law."""
    rev = np.array([int(f"{b:08b}"[::-1], 2) for b in range(256)])
    B0, B2 = np.meshgrid(np.arange(256), np.arange(256), indexing="ij")
    u0 = (65535 - ((B2 << 8) | B0)).ravel()
    u1 = (65535 - ((rev[B0] << 8) | rev[B2])).ravel()
    np.testing.assert_array_equal(np.sort(u0), np.arange(65536))
    np.testing.assert_array_equal(np.sort(u1), np.arange(65536))
    # the oracle's draws for elements 4g and 4g+1 (and 4g+2, 4g+3) are pairs of this law
    pair_of = np.empty(65536, dtype=np.int64)
    pair_of[u0] = u1
    for idx0 in range(0, 4 * 3000, 4):
        d = [orc.sr_bits_nvfp4(99, 5, 0, idx0 + k) for k in range(4)]
        assert pair_of[d[0]] == d[1] and pair_of[d[2]] == d[3]

    def cov(t0, t1):
        return np.mean((u0 < t0) & (u1 < t1)) - (t0 / 65536) * (t1 / 65536)

    worst = cov(21845, 21845)
    assert abs(worst - SR_PAIR_MAX_COV) < 1e-3 / 65536
    rng = np.random.default_rng(21)
    ts = np.concatenate([rng.integers(0, 65537, (3000, 2)),
                         [[t, t] for t in (1, 255, 256, 4096, 16384, 32768, 49152, 65535)]])
    for t0, t1 in ts:
        assert abs(cov(t0, t1)) <= SR_PAIR_MAX_COV + 1e-12


def test_e4m3_sr_sat_enumerated(orc):
    """Stochastic rounding onto the E4M3 grid (MXFP8 with stochastic rounding), over
    all 2^16 draws u for a value inside every kind of E4M3 interval: the subnormal
    steps of 2^-9, the interval starting at the smallest normal 2^-6, ordinary binades
    and the top interval below 448.  Grid neighbours come from the bit-field
    enumeration in brute.py: only the two neighbours occur, exactly the draws
    u < floor(f 2^16) round up (f = exact rational position between them), the rule
    is sign-symmetric, grid values never move and everything >= 448 saturates."""
    grid = brute.e4m3_grid()[:0x7F]            # magnitudes of codes 0x00 .. 0x7E
    us = np.arange(65536)
    sub = 2.0 ** -9
    ys = [0.3 * sub, sub + 0.3 * sub, 3 * sub + 0.71 * sub, 7 * sub + 0.5 * sub + sub / 1024,
          2.0 ** -6 + 0.3 * sub, 2.0 ** -6 * 1.875 + 0.41 * 2.0 ** -9,
          1.03, 2.25 + 0.0421, 9.7, 250.3, 270.0, 440.0, 447.9]
    for y in ys:
        c = int(np.searchsorted(grid, y, side="right") - 1)
        lo, hi = Fraction(float(grid[c])), Fraction(float(grid[c + 1]))
        t = int((Fraction(y) - lo) / (hi - lo) * 65536)      # floor: the value is positive
        assert 0 < t < 65536
        codes = np.array([orc.e4m3_sr_sat(y, int(u)) for u in us])
        expect = np.where(us < t, c + 1, c)
        np.testing.assert_array_equal(codes, expect)
        neg = np.array([orc.e4m3_sr_sat(-y, int(u)) for u in us[::97]])
        np.testing.assert_array_equal(neg, expect[::97] | 0x80)
    for c in range(0x7F):                       # grid values stay put for every u
        for u in (0, 1, 0x7FFF, 0xFFFF):
            assert orc.e4m3_sr_sat(float(grid[c]), u) == c
            assert orc.e4m3_sr_sat(-float(grid[c]), u) == 0x80 | c
    for y in (448.0, 448.5, 464.0, 1e6):        # satfinite: 448 = code 0x7E
        for u in (0, 0x8000, 0xFFFF):
            assert orc.e4m3_sr_sat(y, u) == 0x7E
            assert orc.e4m3_sr_sat(-y, u) == 0xFE
    # the mean over all draws is the value itself, up to the 2^-16 resolution
    for y in ys:
        c = int(np.searchsorted(grid, y, side="right") - 1)
        vals = grid[[orc.e4m3_sr_sat(y, int(u)) for u in us[::1]]]
        assert abs(vals.mean() - y) <= (grid[c + 1] - grid[c]) / 65536


# ------------------------------------------------------------------ global scale
def test_global_scale(orc):
    assert orc.global_scale(0.0) == (1.0, 1.0)
    S, g = orc.global_scale(2688.0)
    assert S == 1.0 and g == 1.0
    for amax in [1e-3, 0.5, 3.0, 54.0, 1e6]:
        S, g = orc.global_scale(amax)
        assert abs(S * amax / 2688.0 - 1) < 2 ** -22 and abs(g / amax * 2688.0 - 1) < 2 ** -22
    S, g = orc.global_scale(1e-38)
    assert S == 2.0 ** 118 and g == 2.0 ** -118


# ------------------------------------------------------------------ tensor-level properties
@pytest.mark.parametrize("scaling", [0, 1])
@pytest.mark.parametrize("direction", [0, 1])
def test_quantize_elements_are_nearest_codes(orc, scaling, direction):
    """Every RNE code is the brute-force nearest code of y = x * (S/d); every scale byte
    is the brute-force nearest E4M3 of (amax_b / 6) * S."""
    x, _ = W.tiny_linear(0, M=32, N=16, K=64)
    q, sf, g = orc.nvfp4_quantize(x, direction, scaling=scaling)
    xf = W.bf16_bits_to_f32(x)
    v = xf.T if direction else xf
    amax = np.float32(np.abs(v).max())
    S = np.float32(2688.0) / amax
    assert np.float32(g) == amax / np.float32(2688.0)
    nr, nc = v.shape
    blocks = np.abs(v).reshape(nr, nc // 16, 16).max(axis=2)
    if scaling:
        t = blocks.reshape(nr // 16, 16, nc // 16).max(axis=1)
        blocks = np.repeat(t, 16, axis=0)
    s = (blocks.astype(np.float32) / np.float32(6.0)) * S
    np.testing.assert_array_equal(sf, brute.e4m3_rne_sat(s.astype(np.float64)))
    d = brute.e4m3_grid()[sf].astype(np.float32)
    r = np.where(d != 0, S / np.where(d != 0, d, 1), 0).astype(np.float32)
    y = (v * np.repeat(r, 16, axis=1)).astype(np.float32)
    codes = brute.unpack_nibbles(q)
    np.testing.assert_array_equal(codes, brute.e2m1_rne(y.astype(np.float64)))


def test_quantize_colwise_rht_matches_transform_then_rowwise(orc):
    """Columnwise+RHT equals: transpose, transform every 16-vector with the closed-form
    matrix (1/4) H D, then the plain rowwise nearest-code rule on the result."""
    rng = np.random.default_rng(10)
    x = W.f32_to_bf16_bits(W.student_t(rng, (48, 32), 3.0, 1e-3))
    seed = 77
    q, sf, g = orc.nvfp4_quantize(x, 1, rht=1, seed=seed)
    T = brute.sylvester_hadamard(16) @ np.diag(orc.rht_signs(seed)) / 4
    v = W.bf16_bits_to_f32(x).T.astype(np.float64)
    tv = (v.reshape(v.shape[0], -1, 16) @ T.T).reshape(v.shape)
    amax = np.abs(tv).max()
    assert abs(g * 2688.0 / amax - 1) < 1e-6
    dq = orc.nvfp4_dequant(q, sf, g)
    # dequantised error bounded by half the largest grid gap times the block scale
    blocks = np.abs(tv).reshape(tv.shape[0], -1, 16).max(axis=2)
    bound = np.repeat(blocks, 16, axis=1) / 6.0 * 1.07 + 1e-12
    assert np.all(np.abs(dq - tv) <= bound)


def test_quantize_zero_and_sign(orc):
    x = np.zeros((16, 32), dtype=np.float32)
    x[0, :16] = -0.0
    x[1, 16] = -1.0
    x[1, 17] = 1e-6
    x[1, 18] = -1e-6
    q, sf, g = orc.nvfp4_quantize(bf16(x), 0)
    codes = brute.unpack_nibbles(q)
    assert np.all(codes[0, :16] == 8)            # -0 keeps its sign
    assert sf[0, 0] == 0 and sf[2, 1] == 0       # all-zero blocks have scale 0
    assert codes[1, 16] == 0xF                   # the block max maps to -6
    assert codes[1, 17] == 0 and codes[1, 18] == 8
    qz, sfz, gz = orc.nvfp4_quantize(bf16(np.zeros((16, 16))), 0)
    assert gz == 1.0 and np.all(qz == 0) and np.all(sfz == 0)


# ------------------------------------------------------------------ MXFP8
def test_mxfp8_scale_rule_and_elements(orc):
    rng = np.random.default_rng(15)
    x = W.f32_to_bf16_bits(W.student_t(rng, (64, 96), 3.0, 1e-3))
    for direction in (0, 1):
        q, e8 = orc.mxfp8_quantize(x, direction)
        v = W.bf16_bits_to_f32(x).astype(np.float64)
        v = v.T if direction else v
        e = e8.astype(np.int64) - 127
        amax = np.abs(v).reshape(v.shape[0], -1, 32).max(axis=2)
        scaled = amax * 2.0 ** (-e)
        ok = amax > 0
        assert np.all((scaled[ok] >= 256) & (scaled[ok] < 512))       # OCP floor rule
        y = v * np.repeat(2.0 ** (-e), 32, axis=1)
        np.testing.assert_array_equal(q, brute.e4m3_rne_sat(y))


def test_mxfp8_worked_values(orc):
    x = np.zeros((32, 32), dtype=np.float32)
    x[0, 0] = 1.0
    x[0, 1] = -0.5
    q, e8 = orc.mxfp8_quantize(bf16(x), 0)
    assert e8[0, 0] == 127 - 8                       # floor(log2 1) - 8 = -8
    assert q[0, 0] == 0x78                           # 256 = 2^8: exponent field 15, mantissa 0
    assert q[0, 1] == 0xF0                           # -128
    assert e8[1, 0] == 0                             # all-zero block: e = -127


def test_storage_accounting(orc):
    g = golden("storage_bits.txt")
    x = W.heavy_tailed(1, 64, 128)
    q, sf, _ = orc.nvfp4_quantize(x, 0)
    bits = 8 * (q.size + sf.size) + 32
    per_elem = bits / x.size
    assert abs(per_elem - 4.5) < 0.01
    assert round(16 / 4.5, 1) == pytest.approx(float(g["bf16_over_nvfp4"]), abs=0.05)
    q8, e8 = orc.mxfp8_quantize(x, 1)
    assert 8 * (q8.size + e8.size) / x.size == float(g["mxfp8_bits_per_number"])


# ------------------------------------------------------------------ dequant + GEMM
def test_dequant_f32_is_rounded_f64(orc):
    x, w = W.tiny_linear(0, 32, 16, 64)
    q, sf, g = orc.nvfp4_quantize(x, 0)
    d64 = orc.nvfp4_dequant(q, sf, g, f64=True)
    d32 = orc.nvfp4_dequant(q, sf, g, f64=False)
    np.testing.assert_array_equal(d32, d64.astype(np.float32))
    # exact definition: code value * scale * g
    codes = brute.unpack_nibbles(q)
    ref = brute.e2m1_grid()[codes] * np.repeat(brute.e4m3_grid()[sf], 16, axis=1) * g
    np.testing.assert_array_equal(d64, ref)


def test_gemm_oracle_exact_small(orc):
    """FP64 GEMM vs exact rational arithmetic on a small non-square case."""
    x, w = W.tiny_linear(3, M=5, N=3, K=48)
    x = np.tile(x, (4, 1))[:16]
    w = np.tile(w, (6, 1))[:16]
    qa, sa, ga = orc.nvfp4_quantize(x, 0)
    qb, sb, gb = orc.nvfp4_quantize(w, 0)
    D, A = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    ah = orc.nvfp4_dequant(qa, sa, ga)
    bh = orc.nvfp4_dequant(qb, sb, gb)
    for i in (0, 3, 15):
        for j in (0, 2, 7, 15):
            exact = sum(Fraction(float(ah[i, k])) * Fraction(float(bh[j, k])) for k in range(48))
            assert abs(Fraction(D[i, j]) - exact) <= Fraction(1, 10 ** 12) * (
                1 + abs(Fraction(A[i, j])))
            absx = sum(abs(Fraction(float(ah[i, k])) * Fraction(float(bh[j, k])))
                       for k in range(48))
            assert abs(Fraction(A[i, j]) - absx) <= Fraction(1, 10 ** 12) * (1 + absx)


def test_gemm_oracle_vs_numpy(orc):
    x, w = W.tiny_linear(0)
    qa, sa, ga = orc.nvfp4_quantize(x, 0)
    qb, sb, gb = orc.nvfp4_quantize(w, 0)
    D, A = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    ah = orc.nvfp4_dequant(qa, sa, ga)
    bh = orc.nvfp4_dequant(qb, sb, gb)
    np.testing.assert_allclose(D, ah @ bh.T, rtol=0, atol=1e-12 * (1 + np.abs(ah) @ np.abs(bh).T).max())
    np.testing.assert_allclose(A, np.abs(ah) @ np.abs(bh).T, rtol=1e-12)
    sel = np.array([5, 0, 127])
    Ds, _ = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=sel)
    np.testing.assert_array_equal(Ds, D[sel])
    # the quantised GEMM approximates the bf16 GEMM
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    wf = W.bf16_bits_to_f32(w).astype(np.float64)
    rel = np.linalg.norm(D - xf @ wf.T) / np.linalg.norm(xf @ wf.T)
    assert rel < 0.2


def _mx_hat(q, e8):
    """MXFP8 values from the bit-field grid of brute.py: E4M3 value x 2^(byte - 127)."""
    grid = brute.e4m3_grid()
    return grid[q] * np.repeat(2.0 ** (e8.astype(np.int64) - 127), 32, axis=1)


def test_mxfp8_gemm_oracle_closed_form(orc):
    """Hand-built MXFP8 operands whose product is known in closed form: every A
    element is +-1.0 (E4M3 0x38 / 0xB8) and every B element 2.0 (0x40); block b of
    A row i has scale 2^(i-b) and block b of B row j has 2^(j+b-1), so
    D[i][j] = sum over blocks of 32 * s * 2^(i+j), s the block's sign."""
    M, N, K = 3, 4, 128
    signs = np.array([1, -1, 1, 1])
    qa = np.repeat(np.where(signs > 0, 0x38, 0xB8), 32)[None, :].repeat(M, 0).astype(np.uint8)
    e8a = np.array([[127 + i - b for b in range(4)] for i in range(M)], dtype=np.uint8)
    qb = np.full((N, K), 0x40, dtype=np.uint8)
    e8b = np.array([[127 + j + b - 1 for b in range(4)] for j in range(N)], dtype=np.uint8)
    D, A = orc.mxfp8_gemm_rows(qa, e8a, qb, e8b)
    for i in range(M):
        for j in range(N):
            assert D[i, j] == 32 * signs.sum() * 2.0 ** (i + j)
            assert A[i, j] == 32 * 4 * 2.0 ** (i + j)
    np.testing.assert_array_equal(orc.mxfp8_dequant(qa, e8a), _mx_hat(qa, e8a))


def test_mxfp8_gemm_oracle_exact_and_numpy(orc):
    """The MXFP8 GEMM reference on quantised heavy-tailed data: against exact rational
    sums for sampled entries and against numpy on the brute-force dequantisation."""
    rng = np.random.default_rng(31)
    x = W.f32_to_bf16_bits(W.student_t(rng, (16, 96), 3.0))
    w = W.f32_to_bf16_bits(W.normal(rng, (24, 96), 0.02))
    qa, ea = orc.mxfp8_quantize(x, 0)
    qb, eb = orc.mxfp8_quantize(w, 0)
    D, A = orc.mxfp8_gemm_rows(qa, ea, qb, eb)
    ah, bh = _mx_hat(qa, ea), _mx_hat(qb, eb)
    for i in (0, 7, 15):
        for j in (0, 11, 23):
            exact = sum(Fraction(float(ah[i, k])) * Fraction(float(bh[j, k])) for k in range(96))
            assert Fraction(D[i, j]) == exact       # every partial sum here is exact in FP64
    np.testing.assert_allclose(D, ah @ bh.T, rtol=0, atol=1e-13 * A.max())
    np.testing.assert_allclose(A, np.abs(ah) @ np.abs(bh).T, rtol=1e-13)
    sel = np.array([9, 2])
    Ds, _ = orc.mxfp8_gemm_rows(qa, ea, qb, eb, rows_sel=sel)
    np.testing.assert_array_equal(Ds, D[sel])
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    wf = W.bf16_bits_to_f32(w).astype(np.float64)
    rel = np.linalg.norm(D - xf @ wf.T) / np.linalg.norm(xf @ wf.T)
    assert rel < 0.05                                # 8-bit operands track the bf16 product


def test_grouped_gemm_oracle_matches_dense(orc):
    rng = np.random.default_rng(16)
    x = W.f32_to_bf16_bits(rng.standard_normal((40, 32)).astype(np.float32))
    wts = [W.f32_to_bf16_bits(rng.standard_normal((16, 32)).astype(np.float32) * 0.02)
           for _ in range(3)]
    off = np.array([0, 8, 8, 40])
    qa, sa, ga = orc.nvfp4_quantize(np.vstack([x, np.zeros((8, 32), np.uint16)])[:48], 0)
    qbs = [orc.nvfp4_quantize(w, 0) for w in wts]
    qb = np.stack([t[0] for t in qbs])
    sb = np.stack([t[1] for t in qbs])
    gb = np.array([t[2] for t in qbs], dtype=np.float32)
    sel = np.array([0, 7, 8, 39])
    D, _ = orc.nvfp4_grouped_gemm_rows(off, qa, sa, ga, qb, sb, gb, sel)
    for s, i in enumerate(sel):
        e = 0 if i < 8 else 2
        Dd, _ = orc.nvfp4_gemm_rows(qa, sa, ga, qbs[e][0], qbs[e][1], qbs[e][2], rows_sel=[i])
        np.testing.assert_array_equal(D[s], Dd[0])


# ------------------------------------------------------------------ sampled-parity mechanism
def test_slices_with_amax_and_index_base_match_full(orc):
    """A row (or column) slice quantised with the full tensor's amax and the slice's
    element-index base reproduces that part of the full result, for SR and RHT too."""
    rng = np.random.default_rng(17)
    x = W.f32_to_bf16_bits(W.student_t(rng, (96, 64), 3.0, 1e-3))
    R, C = x.shape
    for direction, rht in ((0, 0), (1, 0), (1, 1)):
        am = (orc.amax(x, 0), orc.amax(x, 1, rht=rht, seed=3))
        qf, sff, gf = orc.nvfp4_quantize(x, direction, rounding=1, rht=rht, seed=3)
        if direction == 0:
            r0, r1 = 32, 64
            qs, sfs, gs = orc.nvfp4_quantize(x[r0:r1], 0, rounding=1, seed=3, amax=am,
                                             idx_base=r0 * C)
            np.testing.assert_array_equal(qs, qf[r0:r1])
            np.testing.assert_array_equal(sfs, sff[r0:r1])
        else:
            c0, c1 = 16, 48
            qs, sfs, gs = orc.nvfp4_quantize(np.ascontiguousarray(x[:, c0:c1]), 1, rounding=1,
                                             rht=rht, seed=3, amax=am, idx_base=c0 * R)
            np.testing.assert_array_equal(qs, qf[c0:c1])
            np.testing.assert_array_equal(sfs, sff[c0:c1])
        assert gs == gf
    q8, e8 = orc.mxfp8_quantize(x, 1, rounding=1, seed=4)
    q8s, e8s = orc.mxfp8_quantize(np.ascontiguousarray(x[:, 32:64]), 1, rounding=1, seed=4,
                                  idx_base=32 * R)
    np.testing.assert_array_equal(q8s, q8[32:64])
    np.testing.assert_array_equal(e8s, e8[32:64])
