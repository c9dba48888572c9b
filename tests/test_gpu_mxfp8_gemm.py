"""GPU parity of the MXFP8 path of the backward pass (iitak page, "How it works": the
backward pass runs in 8-bit MXFP8): the quantiser's MXFP8 codes and E8M0 scales in the
tensor cores' tiled layout, bit for bit against the oracle, and the block-scaled MXFP8
GEMM (tcgen05 kind::mxf8f6f4) against the oracle's FP64 GEMM of the dequantised
operands: |D - D_ref| <= 1e-3 sum_k |a_hat||b_hat| (plus half a bf16 ulp of D_ref for
bf16 output), both output-tile widths."""
import numpy as np
import pytest

import workloads as W
from gpu_util import check_gemm, cuda_available, host, rowmajor_to_sf_mma, sf_mma_to_rowmajor, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


@pytest.fixture(params=["256", "128"])
def tile_n(request, monkeypatch):
    monkeypatch.setenv("NVFP4_GEMM_TILE_N", request.param)
    return int(request.param)


def mx_tiled(e8, rows, K):
    """Row-major E8M0 bytes [rows, K/32] -> the tiled layout (128x4 atoms of 32-blocks)."""
    return rowmajor_to_sf_mma(e8, rows, K // 2)


def mx_rowmajor(sf, rows, K):
    return sf_mma_to_rowmajor(sf, rows, K // 2)


def _upload(q, e8):
    import torch
    rows, K = q.shape
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(),
            torch.from_numpy(mx_tiled(e8, rows, K)).cuda())


@pytest.mark.parametrize("mnk", [(256, 512, 512), (272, 400, 768), (128, 256, 128),
                                 (384, 128, 1024), (16, 16, 128), (528, 272, 384)])
@pytest.mark.parametrize("bf16_out", [False, True])
def test_mxfp8_gemm_shapes(nv, orc, tile_n, mnk, bf16_out):
    """Operands quantised by the oracle (Student-t activations-like A, N(0, 0.02) B):
    ragged M and N tiles, K of one to eight pipeline stages, every output checked."""
    M, N, K = mnk
    rng = np.random.default_rng(M * 3 + N + K)
    x = W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0, 1.0))
    w = W.f32_to_bf16_bits(W.normal(rng, (N, K), 0.02))
    qa, ea = orc.mxfp8_quantize(x, 0)
    qb, eb = orc.mxfp8_quantize(w, 0)
    A, SA = _upload(qa, ea)
    B, SB = _upload(qb, eb)
    D = host(nv.mx_gemm(A, SA, B, SB, nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32))
    if bf16_out:
        D = W.bf16_bits_to_f32(D.view(np.uint16))
    Dr, Ar = orc.mxfp8_gemm_rows(qa, ea, qb, eb)
    check_gemm(D, Dr, Ar, bf16_out)


def test_mxfp8_quantize_tiled_scales_bitexact(nv, orc):
    """The quantiser's MXFP8 outputs with mx_sf_layout = NVFP4_SF_MMA: codes and scale
    bytes (read back through the tiled layout) equal the oracle's, both directions,
    round to nearest and stochastic rounding, next to the NVFP4 outputs of one pass."""
    rng = np.random.default_rng(41)
    x = W.f32_to_bf16_bits(W.student_t(rng, (384, 640), 3.0, 1e-3))
    for rounding in (0, 1):
        out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=rounding, rht=True,
                          seed=5, sf_layout=nv.NVFP4_SF_MMA,
                          mx_outputs=nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE, mx_rounding=rounding,
                          mx_sf_layout=nv.NVFP4_SF_MMA)
        for d, key, rows, K in ((0, "mx_row", 384, 640), (1, "mx_col", 640, 384)):
            q, e8 = orc.mxfp8_quantize(x, d, rounding, 5)
            mq, me = out[key]
            np.testing.assert_array_equal(host(mq), q)
            np.testing.assert_array_equal(mx_rowmajor(host(me), rows, K), e8)


def test_mxfp8_backward_gemms_from_gpu_quantiser(nv, orc, tile_n):
    """The two backward GEMMs of a linear layer in MXFP8, fed by the GPU quantiser as a
    training step would run them: dgrad dX = dY W (A = dY rowwise, B = W columnwise) and
    wgrad dW = dY^T X (A = dY columnwise, B = X columnwise); tokens 512, hidden 256,
    FFN 640; dY Student-t(3), X N(0,1), W N(0,0.02); every output checked."""
    rng = np.random.default_rng(44)
    T, H, F = 512, 256, 640
    x = W.f32_to_bf16_bits(W.normal(rng, (T, H)))
    w = W.f32_to_bf16_bits(W.normal(rng, (F, H), 0.02))
    dy = W.f32_to_bf16_bits(W.student_t(rng, (T, F), 3.0))
    kw = dict(rowwise=False, sf_layout=nv.NVFP4_SF_MMA, mx_sf_layout=nv.NVFP4_SF_MMA)
    both = nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE
    qdy = nv.quantize(to_dev(dy), mx_outputs=both, **kw)
    qw = nv.quantize(to_dev(w), mx_outputs=nv.NVFP4_COLWISE, **kw)["mx_col"]
    qx = nv.quantize(to_dev(x), mx_outputs=nv.NVFP4_COLWISE, **kw)["mx_col"]
    dX = W.bf16_bits_to_f32(host(nv.mx_gemm(*qdy["mx_row"], *qw)).view(np.uint16))
    dW = W.bf16_bits_to_f32(host(nv.mx_gemm(*qdy["mx_col"], *qx)).view(np.uint16))
    r_dy, e_dy = orc.mxfp8_quantize(dy, 0)
    c_dy, ce_dy = orc.mxfp8_quantize(dy, 1)
    c_w, ce_w = orc.mxfp8_quantize(w, 1)
    c_x, ce_x = orc.mxfp8_quantize(x, 1)
    Dr, Ar = orc.mxfp8_gemm_rows(r_dy, e_dy, c_w, ce_w)
    check_gemm(dX, Dr, Ar, True)
    Dr, Ar = orc.mxfp8_gemm_rows(c_dy, ce_dy, c_x, ce_x)
    check_gemm(dW, Dr, Ar, True)
    # the 8-bit backward tracks the bf16 product
    dyf = W.bf16_bits_to_f32(dy).astype(np.float64)
    wf = W.bf16_bits_to_f32(w).astype(np.float64)
    assert np.linalg.norm(dX - dyf @ wf) / np.linalg.norm(dyf @ wf) < 0.05


def test_mxfp8_gemm_amax_and_zero(nv, orc):
    """amax_out is max |D| as stored; all-zero operands (scale byte 0) give exact zeros."""
    import torch
    M, N, K = 256, 256, 256
    rng = np.random.default_rng(46)
    x = W.f32_to_bf16_bits(W.normal(rng, (M, K)))
    qa, ea = orc.mxfp8_quantize(x, 0)
    A, SA = _upload(qa, ea)
    am = torch.full((1,), 1e30, dtype=torch.float32, device="cuda")
    D = host(nv.mx_gemm(A, SA, A, SA, nv.NVFP4_OUT_F32, amax_out=am))
    assert host(am)[0] == np.max(np.abs(D)).astype(np.float32)
    z = np.zeros((M, K), dtype=np.uint16)
    qz, ez = orc.mxfp8_quantize(z, 0)
    Z, SZ = _upload(qz, ez)
    D = host(nv.mx_gemm(Z, SZ, A, SA, nv.NVFP4_OUT_F32, amax_out=am))
    assert not np.any(D) and host(am)[0] == 0.0
