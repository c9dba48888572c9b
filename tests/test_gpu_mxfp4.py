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
