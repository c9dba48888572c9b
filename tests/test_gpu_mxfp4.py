"""GPU parity of mxfp4_quantize (OCP MXFP4: 32-element blocks, E8M0 scale, E2M1
elements, RNE) against the oracle: codes and scale bytes bit for bit, both
directions from one call, on ragged tiles, padded rows, special values and the
16384 x 20480 gradient the benchmark quantises (sampled slices)."""
import numpy as np
import pytest

import workloads as W
from gpu_util import cuda_available, host, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


def _check_full(nv, orc, x, directions):
    (qr, er), (qc, ec) = nv.mxfp4(to_dev(x), directions)
    if directions & nv.NVFP4_ROWWISE:
        q, e = orc.mxfp4_quantize(x, 0)
        np.testing.assert_array_equal(host(qr), q)
        np.testing.assert_array_equal(host(er), e)
    if directions & nv.NVFP4_COLWISE:
        q, e = orc.mxfp4_quantize(x, 1)
        np.testing.assert_array_equal(host(qc), q)
        np.testing.assert_array_equal(host(ec), e)


@pytest.mark.parametrize("shape", [(32, 32), (64, 128), (96, 160), (160, 96), (256, 1024),
                                   (1056, 2080)])
@pytest.mark.parametrize("directions", [1, 2, 3])
def test_mxfp4_bitexact(nv, orc, shape, directions):
    rng = np.random.default_rng(shape[0] * 7 + shape[1] + directions)
    x = W.f32_to_bf16_bits((rng.standard_normal(shape) *
                            rng.choice([1.0, 1e-3, 40.0], shape)).astype(np.float32))
    _check_full(nv, orc, x, directions)


def test_mxfp4_special_values(nv, orc):
    """Zero blocks, bf16 subnormals, values near the bf16 maximum, signed zeros,
    exact ties and saturating blocks."""
    rng = np.random.default_rng(4)
    x = W.f32_to_bf16_bits(rng.standard_normal((128, 256)).astype(np.float32))
    x[0:32, 0:32] = 0                                    # all-zero block (both directions)
    x[32, 0:32] = 0x8000                                 # negative zeros
    x[33, 0:32] = np.arange(1, 33, dtype=np.uint16)      # bf16 subnormals
    x[34, 0:32] = 0x7F7F                                 # largest finite bf16
    x[35, 32:64] = 0xFF7F                                # and its negative
    ties = np.array([5.0, 7.0, 0.25, 0.75, 2.5, 1.25, 3.5, 6.0] * 4, dtype=np.float32)
    x[36, 64:96] = W.f32_to_bf16_bits(ties)
    x[37, 64:96] = W.f32_to_bf16_bits(-ties)
    _check_full(nv, orc, x, 3)


def test_mxfp4_padded_rows(nv, orc):
    """ld > cols: the input is a column slice of a wider tensor."""
    import torch
    rng = np.random.default_rng(8)
    full = W.f32_to_bf16_bits(rng.standard_normal((96, 200)).astype(np.float32))
    dev = to_dev(full)[:, :160]
    assert dev.stride(0) == 200
    (qr, er), (qc, ec) = nv.mxfp4(dev, 3)
    x = np.ascontiguousarray(full[:, :160])
    for d, (qg, eg) in ((0, (qr, er)), (1, (qc, ec))):
        q, e = orc.mxfp4_quantize(x, d)
        np.testing.assert_array_equal(host(qg), q)
        np.testing.assert_array_equal(host(eg), e)
    torch.cuda.synchronize()


def test_mxfp4_gradient_full_size_sampled(nv, orc):
    """The heavy-tailed 16384 x 20480 gradient (Student-t df 3) in both directions;
    sampled 32-row and 32-column slices against the oracle (blocks are local, so a
    slice quantises exactly as inside the full tensor)."""
    rng = np.random.default_rng(4)
    R, C = 16384, 20480
    x = W.f32_to_bf16_bits(W.student_t(rng, (R, C), 3.0, 1.0))
    (qr, er), (qc, ec) = nv.mxfp4(to_dev(x), 3)
    for r0 in (0, R // 2 + 32 * 13, R - 32):
        q, e = orc.mxfp4_quantize(x[r0:r0 + 32], 0)
        np.testing.assert_array_equal(host(qr[r0:r0 + 32]), q)
        np.testing.assert_array_equal(host(er[r0:r0 + 32]), e)
    for c0 in (0, C // 2 + 32 * 7, C - 32):
        q, e = orc.mxfp4_quantize(np.ascontiguousarray(x[:, c0:c0 + 32]), 1)
        np.testing.assert_array_equal(host(qc[c0:c0 + 32]), q)
        np.testing.assert_array_equal(host(ec[c0:c0 + 32]), e)


@pytest.fixture(params=["256", "128"])
def tile_n(request, monkeypatch):
    monkeypatch.setenv("NVFP4_GEMM_TILE_N", request.param)
    return int(request.param)


def test_mxfp4_tiled_scales_bitexact(nv, orc):
    """mxfp4_quantize with NVFP4_SF_MMA: the same scale bytes, placed in the tensor cores'
    128x4 atoms of 32-blocks (read back through that layout), both directions."""
    from gpu_util import sf_mma_to_rowmajor
    rng = np.random.default_rng(51)
    x = W.f32_to_bf16_bits(W.student_t(rng, (384, 640), 3.0))
    (qr, er), (qc, ec) = nv.mxfp4(to_dev(x), 3, sf_layout=nv.NVFP4_SF_MMA)
    for d, q_, e_, rows, K in ((0, qr, er, 384, 640), (1, qc, ec, 640, 384)):
        q, e = orc.mxfp4_quantize(x, d)
        np.testing.assert_array_equal(host(q_), q)
        np.testing.assert_array_equal(sf_mma_to_rowmajor(host(e_), rows, K // 2), e)


@pytest.mark.parametrize("mnk", [(256, 512, 512), (288, 416, 768), (32, 32, 256),
                                 (384, 128, 1024)])
@pytest.mark.parametrize("bf16_out", [False, True])
def test_mxfp4_gemm_shapes(nv, orc, tile_n, mnk, bf16_out):
    """The block-scaled MXFP4 GEMM (kind::mxf4) on operands the GPU quantiser wrote with
    tiled scales, every output against the oracle's FP64 GEMM of the oracle's own
    quantisation of the same bf16 inputs."""
    from gpu_util import check_gemm
    M, N, K = mnk
    rng = np.random.default_rng(M + 2 * N + K)
    x = W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0))
    w = W.f32_to_bf16_bits(W.normal(rng, (N, K), 0.02))
    (qa, sa), _ = nv.mxfp4(to_dev(x), nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
    (qb, sb), _ = nv.mxfp4(to_dev(w), nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
    D = host(nv.mx4_gemm(qa, sa, qb, sb, nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32))
    if bf16_out:
        D = W.bf16_bits_to_f32(D.view(np.uint16))
    oa, ea = orc.mxfp4_quantize(x, 0)
    ob, eb = orc.mxfp4_quantize(w, 0)
    Dr, Ar = orc.mxfp4_gemm_rows(oa, ea, ob, eb)
    check_gemm(D, Dr, Ar, bf16_out)


def test_nvfp4_more_accurate_than_mxfp4_on_gpu(nv):
    """The pages' comparison at the GEMM level (hightech page; asector page, "NVFP4 and
    Blackwell": NVFP4 ahead of the OCP's MXFP4): the same activations and weights through
    the NVFP4 GEMM and the MXFP4 GEMM on the tensor cores; NVFP4's product is closer to
    the bf16 product, on Gaussian activations and on heavy-tailed ones."""
    import torch
    rng = np.random.default_rng(52)
    M, N, K = 512, 512, 2048
    w = W.f32_to_bf16_bits(W.normal(rng, (N, K), 0.02))
    for x in (W.f32_to_bf16_bits(W.normal(rng, (M, K))),
              W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0))):
        xd, wd = to_dev(x), to_dev(w)
        ref = (xd.float() @ wd.float().T).double()
        A = nv.quantize(xd, sf_layout=nv.NVFP4_SF_MMA)["row"]
        B = nv.quantize(wd, sf_layout=nv.NVFP4_SF_MMA)["row"]
        Dn = nv.gemm(A, B, nv.NVFP4_OUT_F32).double()
        (qa, sa), _ = nv.mxfp4(xd, nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
        (qb, sb), _ = nv.mxfp4(wd, nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
        Dm = nv.mx4_gemm(qa, sa, qb, sb, nv.NVFP4_OUT_F32).double()
        en = torch.linalg.norm(Dn - ref).item() / torch.linalg.norm(ref).item()
        em = torch.linalg.norm(Dm - ref).item() / torch.linalg.norm(ref).item()
        assert en < em, (en, em)
