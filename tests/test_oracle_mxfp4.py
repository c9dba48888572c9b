"""Pins for the oracle's MXFP4 (the OCP Microscaling 4-bit format the pages set
NVFP4 against: 32-element blocks, E8M0 scale, E2M1 elements), from the E2M1 grid,
the scale rule's closed form, brute force and layout invariants -- none of them
re-runs the oracle's own arithmetic.  CPU only."""
import math

import numpy as np

import workloads as W

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # E2M1 magnitudes, code = index


def bf16(vals, shape=None):
    a = np.asarray(vals, dtype=np.float32)
    if shape is not None:
        a = a.reshape(shape)
    return W.f32_to_bf16_bits(a)


def nearest_code(y):
    """Brute force: nearest E2M1 magnitude, ties to the even code, saturating at 6."""
    a = min(abs(y), 6.0)
    best = min(range(8), key=lambda m: (abs(a - GRID[m]), m & 1))
    return (8 if math.copysign(1.0, y) < 0 else 0) | best


def scale_byte(amax):
    """OCP rule: floor(log2 amax) - 2, clamped to [-127, 127], plus 127; amax 0 -> 0."""
    if amax == 0.0:
        return 0
    e = math.floor(math.log2(amax)) - 2
    return max(-127, min(127, e)) + 127


def codes_of(q):
    c = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.uint8)
    c[:, 0::2] = q & 0xF
    c[:, 1::2] = q >> 4
    return c


def test_unit_scale_block_is_exact(orc):
    vals = GRID * 4  # amax 6 -> e = 0
    q, e8 = orc.mxfp4_quantize(bf16(vals, (1, 32)), 0)
    assert e8[0, 0] == 127
    assert list(codes_of(q)[0]) == list(range(8)) * 4
    np.testing.assert_array_equal(orc.mxfp4_dequant(q, e8)[0], vals)


def test_ties_and_saturation_at_unit_scale(orc):
    # amax 7 -> floor(log2 7) = 2 -> e = 0; 7 saturates to 6; ties go to even codes
    vals = [7.0, 5.0, -5.0, 0.25, 0.75, 2.5, 1.25, -3.5] + [0.0] * 24
    q, e8 = orc.mxfp4_quantize(bf16(vals, (1, 32)), 0)
    assert e8[0, 0] == 127
    expect = [6.0, 4.0, -4.0, 0.0, 1.0, 2.0, 1.0, -4.0]
    np.testing.assert_array_equal(orc.mxfp4_dequant(q, e8)[0, :8], expect)


def test_scale_byte_closed_form(orc):
    for amax, byte in [(1.0, 125), (0.75, 124), (6.0, 127), (8.0, 128), (2.0 ** -100, 25),
                       (0.0, 0), (2.0 ** -130, 0)]:
        assert scale_byte(amax) == byte
        vals = [amax] + [0.0] * 31
        _, e8 = orc.mxfp4_quantize(bf16(vals, (1, 32)), 0)
        assert e8[0, 0] == byte, amax
    # the largest finite bf16 (just under 2^128): floor(log2) = 127 -> e = 125
    big = np.array([[0x7F7F] + [0] * 31], dtype=np.uint16)
    _, e8 = orc.mxfp4_quantize(big, 0)
    assert e8[0, 0] == 252


def test_brute_force_blocks(orc):
    rng = np.random.default_rng(11)
    for trial in range(40):
        scale = 2.0 ** rng.integers(-20, 20)
        x = bf16(rng.standard_normal((2, 64)) * scale * rng.choice([1.0, 0.01, 100.0], (2, 64)))
        xf = W.bf16_bits_to_f32(x).astype(np.float64)
        q, e8 = orc.mxfp4_quantize(x, 0)
        c = codes_of(q)
        for r in range(2):
            for b in range(2):
                blk = xf[r, 32 * b:32 * b + 32]
                byte = scale_byte(float(np.max(np.abs(blk))))
                assert e8[r, b] == byte
                e = byte - 127
                for i in range(32):
                    assert c[r, 32 * b + i] == nearest_code(blk[i] * 2.0 ** -e), (trial, r, b, i)


def test_power_of_two_equivariance(orc):
    rng = np.random.default_rng(5)
    x = bf16(rng.standard_normal((4, 64)))
    q0, e0 = orc.mxfp4_quantize(x, 0)
    for k in (-30, -3, 5, 40):
        xk = bf16(W.bf16_bits_to_f32(x) * np.float32(2.0 ** k))
        qk, ek = orc.mxfp4_quantize(xk, 0)
        np.testing.assert_array_equal(qk, q0)
        np.testing.assert_array_equal(ek.astype(int), e0.astype(int) + k)


def test_columnwise_is_rowwise_of_transpose(orc):
    rng = np.random.default_rng(9)
    x = bf16(rng.standard_normal((64, 96)))
    qc, ec = orc.mxfp4_quantize(x, 1)
    qr, er = orc.mxfp4_quantize(np.ascontiguousarray(x.T), 0)
    np.testing.assert_array_equal(qc, qr)
    np.testing.assert_array_equal(ec, er)


def test_nvfp4_error_below_mxfp4(orc):
    """The pages report NVFP4 ahead of MXFP4 (finer 16-element blocks with an E4M3
    scale and a tensor scale, against 32-element blocks with a power-of-two scale):
    on Gaussian data its squared quantisation error is clearly lower."""
    rng = np.random.default_rng(2)
    x = bf16(rng.standard_normal((128, 512)))
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    qn, sn, gn = orc.nvfp4_quantize(x, 0)
    err_nv = np.mean((orc.nvfp4_dequant(qn, sn, gn) - xf) ** 2)
    qm, em = orc.mxfp4_quantize(x, 0)
    err_mx = np.mean((orc.mxfp4_dequant(qm, em) - xf) ** 2)
    assert err_nv < 0.75 * err_mx, (err_nv, err_mx)


def test_mxfp4_gemm_oracle_closed_form(orc):
    """Hand-built MXFP4 operands with a closed-form product: A elements +-1 (code 2 /
    10), B elements 3 (code 5); block b of A row i scaled 2^(i-b), of B row j 2^(j+b);
    so D[i][j] = 3 * 32 * sum_b s_b * 2^(i+j), s_b the block's sign."""
    M, N, K = 2, 3, 128
    signs = [1, 1, -1, 1]
    codes = np.concatenate([np.full(32, 2 if s > 0 else 10, dtype=np.uint8) for s in signs])
    qa = np.tile(codes[0::2] | (codes[1::2] << 4), (M, 1))
    e8a = np.array([[127 + i - b for b in range(4)] for i in range(M)], dtype=np.uint8)
    qb = np.full((N, K // 2), 5 | (5 << 4), dtype=np.uint8)
    e8b = np.array([[127 + j + b for b in range(4)] for j in range(N)], dtype=np.uint8)
    D, A = orc.mxfp4_gemm_rows(qa, e8a, qb, e8b)
    for i in range(M):
        for j in range(N):
            assert D[i, j] == 3 * 32 * sum(signs) * 2.0 ** (i + j)
            assert A[i, j] == 3 * 32 * 4 * 2.0 ** (i + j)


def test_mxfp4_gemm_oracle_vs_numpy(orc):
    """The MXFP4 GEMM reference against numpy on the independent dequantisation of this
    file's grid (E2M1 magnitude x 2^(byte - 127)), on quantised Gaussian data; and NVFP4's
    product of the same data is closer to the bf16 product than MXFP4's."""
    rng = np.random.default_rng(33)
    x = W.f32_to_bf16_bits(W.normal(rng, (32, 256)))
    w = W.f32_to_bf16_bits(W.normal(rng, (48, 256), 0.02))
    qa, ea = orc.mxfp4_quantize(x, 0)
    qb, eb = orc.mxfp4_quantize(w, 0)
    D, A = orc.mxfp4_gemm_rows(qa, ea, qb, eb)

    def hat(q, e):
        mag = np.array(GRID + [-g for g in GRID])[codes_of(q)]
        return mag * np.repeat(2.0 ** (e.astype(np.int64) - 127), 32, axis=1)

    ah, bh = hat(qa, ea), hat(qb, eb)
    np.testing.assert_allclose(D, ah @ bh.T, rtol=0, atol=1e-13 * A.max())
    np.testing.assert_allclose(A, np.abs(ah) @ np.abs(bh).T, rtol=1e-13)
    ref = W.bf16_bits_to_f32(x).astype(np.float64) @ W.bf16_bits_to_f32(w).astype(np.float64).T
    na, sa_, ga = orc.nvfp4_quantize(x, 0)
    nb, sb_, gb = orc.nvfp4_quantize(w, 0)
    Dn, _ = orc.nvfp4_gemm_rows(na, sa_, ga, nb, sb_, gb)
    assert np.linalg.norm(Dn - ref) < np.linalg.norm(D - ref)
