"""The 12B-scale dense linear layer at full size (tokens 16384, hidden 5120, FFN 20480),
run through the same calls and switches as the benchmark step: X rowwise + columnwise
with the Hadamard (RNE), W with 16x16 2D scales both ways, dY rowwise SR + columnwise
Hadamard SR + MXFP8 columnwise, then the forward (X W^T), dgrad (dY W) and wgrad
(dY^T X) GEMMs on the GPU's own quantised operands, bf16 out.

The oracle checks sampled 16-row / 16-column slices of every quantised output bit for
bit (with the full tensors' amax), and sampled entries of every GEMM output against its
FP64 GEMM of operands it quantised itself from the bf16 inputs."""
import numpy as np
import pytest

import workloads as W
from gpu_util import check_gemm, cuda_available, host, sf_mma_to_rowmajor, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

T, H, F = 16384, 5120, 20480
SEED = 20251030  # the benchmark's seed (Hadamard signs and stochastic rounding)


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


@pytest.fixture(scope="module")
def layer(nv, orc):
    d = W.dense_linear_layer(4, T, H, F)
    x, w, dy = d["x"], d["w"], d["dy"]
    mma = nv.NVFP4_SF_MMA
    X = nv.quantize(to_dev(x), rowwise=True, colwise=True, rht=True, seed=SEED, sf_layout=mma)
    Wq = nv.quantize(to_dev(w), rowwise=True, colwise=True, scaling=nv.NVFP4_2D16x16, seed=SEED,
                     sf_layout=mma)
    D = nv.quantize(to_dev(dy), rowwise=True, colwise=True, rounding=nv.NVFP4_SR, rht=True,
                    seed=SEED, mx_outputs=nv.NVFP4_COLWISE, sf_layout=mma)
    out = dict(x=x, w=w, dy=dy, X=X, W=Wq, D=D,
               Y=nv.gemm(X["row"], Wq["row"], nv.NVFP4_OUT_BF16),
               dX=nv.gemm(D["row"], Wq["col"], nv.NVFP4_OUT_BF16),
               dW=nv.gemm(D["col"], X["col"], nv.NVFP4_OUT_BF16))
    out["am_x"] = (orc.amax(x, 0), orc.amax(x, 1, rht=1, seed=SEED))
    aw = orc.amax(w, 0)
    out["am_w"] = (aw, aw)
    out["am_d"] = (orc.amax(dy, 0), orc.amax(dy, 1, rht=1, seed=SEED))
    return out


def _rows(t, r0, n):
    """Codes and row-major scale bytes of rows r0 .. r0+n of a GPU NVFP4 tensor."""
    q = host(t.q[r0:r0 + n])
    sf = sf_mma_to_rowmajor(host(t.sf), n, t.k, padded_rows=np.arange(r0, r0 + n))
    return q, sf


# (name, input key, amax key, rounding, scaling[, rht]) of each NVFP4 output
ROWWISE = [("X", "x", "am_x", 0, 0), ("W", "w", "am_w", 0, 1), ("D", "dy", "am_d", 1, 0)]
COLWISE = [("X", "x", "am_x", 0, 0, 1), ("W", "w", "am_w", 0, 1, 0), ("D", "dy", "am_d", 1, 0, 1)]


@pytest.mark.parametrize("name,key,amk,rounding,scaling", ROWWISE)
def test_rowwise_slices_bitexact(orc, layer, name, key, amk, rounding, scaling):
    x = layer[key]
    rows, cols = x.shape
    t = layer[name]["row"]
    for r0 in (0, rows // 2 + 16 * 37, rows - 16):
        q, sf, g = orc.nvfp4_quantize(x[r0:r0 + 16], 0, rounding, scaling, 0, SEED,
                                      amax=layer[amk], idx_base=r0 * cols)
        qg, sfg = _rows(t, r0, 16)
        np.testing.assert_array_equal(qg, q)
        np.testing.assert_array_equal(sfg, sf)
        assert float(host(t.g)[0]) == g


@pytest.mark.parametrize("name,key,amk,rounding,scaling,rht", COLWISE)
def test_colwise_slices_bitexact(orc, layer, name, key, amk, rounding, scaling, rht):
    x = layer[key]
    rows, cols = x.shape
    t = layer[name]["col"]
    for c0 in (0, cols // 2 + 16 * 11, cols - 16):
        xs = np.ascontiguousarray(x[:, c0:c0 + 16])
        q, sf, g = orc.nvfp4_quantize(xs, 1, rounding, scaling, rht, SEED, amax=layer[amk],
                                      idx_base=c0 * rows)
        qg, sfg = _rows(t, c0, 16)
        np.testing.assert_array_equal(qg, q)
        np.testing.assert_array_equal(sfg, sf)
        assert float(host(t.g)[0]) == g


def test_mxfp8_columnwise_slices_bitexact(orc, layer):
    dy = layer["dy"]
    mq, me = layer["D"]["mx_col"]
    for c0 in (0, F // 2 + 32 * 5, F - 32):
        q8, e8 = orc.mxfp8_quantize(np.ascontiguousarray(dy[:, c0:c0 + 32]), 1, 0, SEED)
        np.testing.assert_array_equal(host(mq[c0:c0 + 32]), q8)
        np.testing.assert_array_equal(host(me[c0:c0 + 32]), e8)


def _oracle_rows(orc, layer, spec, i0):
    """Oracle NVFP4 rows i0 .. i0+16 of a GEMM operand.  spec = (input key, amax key,
    direction, rounding, scaling, rht): direction 1 takes columns i0.. of the input."""
    key, amk, direction, rounding, scaling, rht = spec
    x = layer[key]
    if direction == 0:
        return orc.nvfp4_quantize(x[i0:i0 + 16], 0, rounding, scaling, 0, SEED,
                                  amax=layer[amk], idx_base=i0 * x.shape[1])
    return orc.nvfp4_quantize(np.ascontiguousarray(x[:, i0:i0 + 16]), 1, rounding, scaling, rht,
                              SEED, amax=layer[amk], idx_base=i0 * x.shape[0])


# GEMM: output key, A operand spec, B operand spec, output rows, output cols
GEMMS = [
    ("Y", ("x", "am_x", 0, 0, 0, 0), ("w", "am_w", 0, 0, 1, 0), T, F),    # forward
    ("dX", ("dy", "am_d", 0, 1, 0, 0), ("w", "am_w", 1, 0, 1, 0), T, H),  # dgrad
    ("dW", ("dy", "am_d", 1, 1, 0, 1), ("x", "am_x", 1, 0, 0, 1), F, H),  # wgrad
]


@pytest.mark.parametrize("out,spec_a,spec_b,M,N", GEMMS, ids=[g[0] for g in GEMMS])
def test_gemm_sampled_entries(orc, layer, out, spec_a, spec_b, M, N):
    D = layer[out]
    for i in (0, 255, M // 2 + 129, M - 1):
        i0 = (i // 16) * 16
        qa, sa, ga = _oracle_rows(orc, layer, spec_a, i0)
        for j0 in (0, 256 * 3 + 128, N - 16):
            qb, sb, gb = _oracle_rows(orc, layer, spec_b, j0)
            Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[i - i0])
            got = W.bf16_bits_to_f32(host(D[i:i + 1, j0:j0 + 16].contiguous()))
            check_gemm(got, Dr, Ar, True)


@pytest.mark.parametrize("out,spec_a,spec_b,M,N", GEMMS, ids=[g[0] for g in GEMMS])
def test_gemm_every_output_tile(orc, layer, out, spec_a, spec_b, M, N):
    """One row x 16 columns inside every 256 x 256 output tile (the pair's tile): the row
    in M-tile mt sits at offset (37 mt + 5) % 256 and the 16 columns of N-tile nt at
    16 ((5 nt + 3) % 16), so the checks move across both CTAs of the pair, every lane
    quadrant and every epilogue warp's column range, and cover the band rasterisation
    and the persistent multi-tile loop of the full-size launch."""
    D = layer[out]
    tiles_m, tiles_n = M // 256, N // 256
    j0s = [256 * nt + 16 * ((5 * nt + 3) % 16) for nt in range(tiles_n)]
    slices = [_oracle_rows(orc, layer, spec_b, j0) for j0 in j0s]
    qb = np.concatenate([t[0] for t in slices])
    sb = np.concatenate([t[1] for t in slices])
    gb = slices[0][2]
    assert all(t[2] == gb for t in slices)
    import torch
    cols = np.concatenate([np.arange(j0, j0 + 16) for j0 in j0s])
    cols_d = torch.from_numpy(cols).to(D.device)
    worst = 0.0
    for mt in range(tiles_m):
        i = 256 * mt + (37 * mt + 5) % 256
        i0 = (i // 16) * 16
        qa, sa, ga = _oracle_rows(orc, layer, spec_a, i0)
        Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[i - i0])
        got = W.bf16_bits_to_f32(host(D[i][cols_d]))[None, :]
        worst = max(worst, check_gemm(got, Dr, Ar, True))
    assert worst <= 1.0
