"""GPU parity of the quantizer, MXFP8 and dequantisation against the CPU oracle,
through the C ABI.  Codes, scale bytes, global scales and stochastic-rounding
output must be bit-exact."""
import numpy as np
import pytest

import brute
import workloads as W
from gpu_util import cuda_available, host, sf_mma_to_rowmajor, to_dev, grouped_padded_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


def edge_tensor(rows, cols, seed):
    """Heavy-tailed values with outliers, exact zeros, negative zeros, an all-zero block,
    grid midpoints and tiny (subnormal-scale) blocks."""
    rng = np.random.default_rng(seed)
    x = W.student_t(rng, (rows, cols), 3.0, 1.0)
    x[rng.random((rows, cols)) < 0.01] *= 80.0
    x[0, :16] = 0.0
    x[1, :16] = -0.0
    if rows >= 32 and cols >= 32:
        x[2, 16:32] = np.array([6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25,
                                -5, -3.5, -2.5, -1.75, -1.25, -0.75, -0.25, -6], np.float32)
        x[3, 16:32] = rng.standard_normal(16).astype(np.float32) * 1e-30
        x[16:32, 0] = 0.0
    return W.f32_to_bf16_bits(x)


SHAPES = [(128, 256), (256, 384), (144, 80), (16, 16), (48, 1040)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("scaling", [0, 1])
@pytest.mark.parametrize("rht", [0, 1])
def test_quantize_bitexact(nv, orc, shape, rounding, scaling, rht):
    rows, cols = shape
    x = edge_tensor(rows, cols, seed=rows * 7 + cols)
    seed, offset = 1234567 + rows, 5
    out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=rounding, scaling=scaling,
                      rht=rht, seed=seed, offset=offset)
    qr, sr, gr = orc.nvfp4_quantize(x, 0, rounding, scaling, 0, seed, offset)
    qc, sc, gc = orc.nvfp4_quantize(x, 1, rounding, scaling, rht, seed, offset)
    np.testing.assert_array_equal(host(out["row"].q), qr)
    np.testing.assert_array_equal(host(out["row"].sf), sr)
    assert float(host(out["row"].g)[0]) == gr
    np.testing.assert_array_equal(host(out["col"].sf), sc)
    np.testing.assert_array_equal(host(out["col"].q), qc)
    assert float(host(out["col"].g)[0]) == gc
    assert nv.nvfp4_workspace_status(out["workspace"]) == 0


@pytest.mark.parametrize("shape", [(128, 256), (192, 320), (64, 64)])
def test_quantize_mma_layout(nv, orc, shape):
    rows, cols = shape
    x = edge_tensor(rows, cols, seed=3)
    out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=1, rht=1, seed=9,
                      sf_layout=nv.NVFP4_SF_MMA)
    qr, sr, _ = orc.nvfp4_quantize(x, 0, 1, 0, 0, 9)
    qc, sc, _ = orc.nvfp4_quantize(x, 1, 1, 0, 1, 9)
    np.testing.assert_array_equal(host(out["row"].q), qr)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["row"].sf), rows, cols), sr)
    np.testing.assert_array_equal(host(out["col"].q), qc)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["col"].sf), cols, rows), sc)


def test_quantize_worked_example(nv, orc):
    """Block max -54 -> code -6 with multiplier 9 (byte 0x51) when S = g = 1."""
    import torch
    x = np.random.default_rng(0).uniform(-50, 50, (16, 16)).astype(np.float32)
    x[0, 3] = -54.0
    xb = W.f32_to_bf16_bits(x)
    amax = torch.tensor([2688.0, 2688.0], device="cuda")
    out = nv.quantize(to_dev(xb), amax=amax)
    sf = host(out["row"].sf)
    q = brute.unpack_nibbles(host(out["row"].q))
    assert sf[0, 0] == 0x51 and q[0, 3] == 0xF
    assert float(host(out["row"].g)[0]) == 1.0


def test_sr_2p25_frequency_on_gpu(nv, orc):
    """10^6 GPU draws of SR(2.25): bit-exact with the oracle, hence the same 3-sigma check."""
    import torch
    rows, cols = 1024, 1088
    x = np.full((rows, cols), 2.25, dtype=np.float32)
    x[:, ::16] = 6.0
    xb = W.f32_to_bf16_bits(x)
    amax = torch.tensor([2688.0, 2688.0], device="cuda")
    out = nv.quantize(to_dev(xb), rounding=1, seed=1234, amax=amax)
    q, _, _ = orc.nvfp4_quantize(xb, 0, rounding=1, seed=1234, amax=(2688.0, 2688.0))
    np.testing.assert_array_equal(host(out["row"].q), q)
    codes = brute.unpack_nibbles(host(out["row"].q))[x == 2.25]
    frac3 = np.mean(codes == 5)                          # code 5 = 3.0
    assert abs(frac3 - 0.25) <= 3 * np.sqrt(0.1875 / codes.size)


@pytest.mark.parametrize("shape", [(64, 96), (128, 256), (96, 160)])
@pytest.mark.parametrize("rounding", [0, 1])
def test_mxfp8_bitexact(nv, orc, shape, rounding):
    rows, cols = shape
    x = edge_tensor(rows, cols, seed=11)
    (qr, er), (qc, ec) = nv.mxfp8(to_dev(x), nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE, rounding,
                                  seed=77, offset=3)
    oqr, oer = orc.mxfp8_quantize(x, 0, rounding, 77, 3)
    oqc, oec = orc.mxfp8_quantize(x, 1, rounding, 77, 3)
    np.testing.assert_array_equal(host(er), oer)
    np.testing.assert_array_equal(host(qr), oqr)
    np.testing.assert_array_equal(host(ec), oec)
    np.testing.assert_array_equal(host(qc), oqc)


def test_fused_gradient_recipe_small(nv, orc):
    """The gradient recipe in one pass: rowwise SR, columnwise RHT + SR, MXFP8 columnwise."""
    x = W.heavy_tailed(1, 512, 384)
    out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=1, rht=True, seed=1,
                      mx_outputs=nv.NVFP4_COLWISE, sf_layout=nv.NVFP4_SF_MMA)
    qr, sr, gr = orc.nvfp4_quantize(x, 0, 1, 0, 0, 1)
    qc, sc, gc = orc.nvfp4_quantize(x, 1, 1, 0, 1, 1)
    mq, me = orc.mxfp8_quantize(x, 1, 0, 1)
    np.testing.assert_array_equal(host(out["row"].q), qr)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["row"].sf), 512, 384), sr)
    np.testing.assert_array_equal(host(out["col"].q), qc)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["col"].sf), 384, 512), sc)
    np.testing.assert_array_equal(host(out["mx_col"][0]), mq)
    np.testing.assert_array_equal(host(out["mx_col"][1]), me)
    assert float(host(out["row"].g)[0]) == gr and float(host(out["col"].g)[0]) == gc


@pytest.mark.parametrize("bf16_out", [False, True])
@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize(nv, orc, bf16_out, layout):
    rows, cols = 128, 320
    x = edge_tensor(rows, cols, seed=5)
    out = nv.quantize(to_dev(x), sf_layout=layout)
    t = out["row"]
    d = host(nv.dequantize(t, nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32))
    q, sf, g = orc.nvfp4_quantize(x, 0)
    ref = orc.nvfp4_dequant(q, sf, g, f64=False)
    if bf16_out:
        np.testing.assert_array_equal(d.view(np.uint16), W.f32_to_bf16_bits(ref))
    else:
        np.testing.assert_array_equal(d, ref)


def test_gather_grouped_layout(nv, orc):
    """MoE act-quantize: gather rows through an index and write the grouped tiled scales."""
    import torch
    rng = np.random.default_rng(21)
    tokens, hidden = 96, 256
    x = W.f32_to_bf16_bits(rng.standard_normal((tokens, hidden)).astype(np.float32))
    counts = np.array([0, 150, 7, 0, 33, 130])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    total = int(offsets[-1])
    row_index = rng.integers(0, tokens, total).astype(np.int32)
    out = nv.quantize(to_dev(x), rows=total, row_index=torch.from_numpy(row_index).cuda(),
                      src_rows=tokens, group_offsets=torch.from_numpy(offsets).cuda(),
                      num_groups=len(counts), sf_layout=nv.NVFP4_SF_MMA)
    xg = np.ascontiguousarray(x[row_index])
    q, sf, g = orc.nvfp4_quantize(xg, 0)
    np.testing.assert_array_equal(host(out["row"].q), q)
    pr = grouped_padded_rows(offsets)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["row"].sf), total, hidden, pr), sf)
    assert float(host(out["row"].g)[0]) == g
    assert nv.nvfp4_workspace_status(out["workspace"]) == 0


def test_gather_gradient_recipe(nv, orc):
    """Gathered input (rows copied one by one into the staged tile, not TMA boxes)
    with every output of the gradient recipe: rowwise SR, columnwise Hadamard + SR and
    MXFP8 columnwise, on a ragged tile edge in both directions (320 x 320).  Each
    output equals the oracle's quantisation of the gathered matrix."""
    import torch
    rng = np.random.default_rng(71)
    tokens, cols, total = 96, 320, 320
    x = W.heavy_tailed(2, tokens, cols)
    row_index = np.concatenate([rng.permutation(tokens),
                                rng.integers(0, tokens, total - tokens)]).astype(np.int32)
    out = nv.quantize(to_dev(x), rows=total, row_index=torch.from_numpy(row_index).cuda(),
                      src_rows=tokens, rowwise=True, colwise=True, rounding=1, rht=True, seed=3,
                      mx_outputs=nv.NVFP4_COLWISE, sf_layout=nv.NVFP4_SF_MMA)
    xg = np.ascontiguousarray(x[row_index])
    qr, sr, gr = orc.nvfp4_quantize(xg, 0, 1, 0, 0, 3)
    qc, sc, gc = orc.nvfp4_quantize(xg, 1, 1, 0, 1, 3)
    mq, me = orc.mxfp8_quantize(xg, 1, 0, 3)
    np.testing.assert_array_equal(host(out["row"].q), qr)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["row"].sf), total, cols), sr)
    np.testing.assert_array_equal(host(out["col"].q), qc)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(out["col"].sf), cols, total), sc)
    np.testing.assert_array_equal(host(out["mx_col"][0]), mq)
    np.testing.assert_array_equal(host(out["mx_col"][1]), me)
    assert float(host(out["row"].g)[0]) == gr and float(host(out["col"].g)[0]) == gc
    assert nv.nvfp4_workspace_status(out["workspace"]) == 0


def test_gather_bad_index_reports(nv):
    import torch
    x = torch.zeros((32, 64), dtype=torch.bfloat16, device="cuda")
    idx = torch.tensor([0] * 15 + [99], dtype=torch.int32, device="cuda")
    out = nv.quantize(x, rows=16, row_index=idx, src_rows=32)
    assert nv.nvfp4_workspace_status(out["workspace"]) == 8     # NVFP4_ERR_INDEX


@pytest.mark.parametrize("rht", [0, 1])
def test_full_size_gradient_bitexact(nv, orc, rht):
    """The 8192 x 8192 heavy-tailed gradient (Student-t df 3, x1e-3), fused pass as the
    benchmark runs it; the oracle checks whole row and column slices at the sampled
    positions with the full tensor's amax."""
    x = W.heavy_tailed(1, 8192, 8192)
    out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=1, rht=bool(rht), seed=1,
                      mx_outputs=nv.NVFP4_COLWISE, sf_layout=nv.NVFP4_SF_MMA)
    R = C = 8192
    am = (orc.amax(x, 0), orc.amax(x, 1, rht=rht, seed=1))
    _, _, gr = orc.nvfp4_quantize(x[:16], 0, 1, 0, 0, 1, amax=am)
    assert float(host(out["row"].g)[0]) == gr
    qrow = host(out["row"].q)
    sfrow = sf_mma_to_rowmajor(host(out["row"].sf), R, C)
    for r0 in (0, 4096, 8192 - 128):
        q, sf, _ = orc.nvfp4_quantize(x[r0:r0 + 128], 0, 1, 0, 0, 1, amax=am, idx_base=r0 * C)
        np.testing.assert_array_equal(qrow[r0:r0 + 128], q)
        np.testing.assert_array_equal(sfrow[r0:r0 + 128], sf)
    qcol = host(out["col"].q)
    sfcol = sf_mma_to_rowmajor(host(out["col"].sf), C, R)
    mq, me = host(out["mx_col"][0]), host(out["mx_col"][1])
    for c0 in (0, 3000 - 3000 % 32, 8192 - 64):
        xs = np.ascontiguousarray(x[:, c0:c0 + 64])
        q, sf, g = orc.nvfp4_quantize(xs, 1, 1, 0, rht, 1, amax=am, idx_base=c0 * R)
        np.testing.assert_array_equal(qcol[c0:c0 + 64], q)
        np.testing.assert_array_equal(sfcol[c0:c0 + 64], sf)
        assert float(host(out["col"].g)[0]) == g
        q8, e8 = orc.mxfp8_quantize(xs, 1, 0, 1)
        np.testing.assert_array_equal(mq[c0:c0 + 64], q8)
        np.testing.assert_array_equal(me[c0:c0 + 64], e8)


@pytest.mark.parametrize("grouped", [False, True])
def test_gather_rows_matches_oracle(nv, orc, grouped):
    """Quantise 512 tokens once, dispatch 1008 routed rows (every token routed at least
    once, so the source amax is the routed rows' amax): the dispatched codes and scales
    equal the oracle's quantisation of the gathered rows, and the fused gather-quantize."""
    import torch
    rng = np.random.default_rng(21)
    tokens, k, E = 512, 320, 5
    x = W.f32_to_bf16_bits(W.student_t(rng, (tokens, k), 4.0, 1.0))
    row_index = np.concatenate([rng.permutation(tokens), rng.integers(0, tokens, 496)]).astype(np.int32)
    total = row_index.size
    offsets = np.array([0, 300, 300, 717, 718, total], dtype=np.int32) if grouped else None
    src = nv.quantize(to_dev(x), sf_layout=nv.NVFP4_SF_MMA)["row"]
    idx_d = torch.from_numpy(row_index).cuda()
    off_d = torch.from_numpy(offsets).cuda() if grouped else None
    got = nv.gather_rows(src, idx_d, off_d)
    xg = np.ascontiguousarray(x[row_index])
    qo, so, go = orc.nvfp4_quantize(xg, 0, amax=(orc.amax(x, 0), 0.0))
    assert np.array_equal(host(got.q), qo)
    pr = grouped_padded_rows(offsets) if grouped else None
    assert np.array_equal(sf_mma_to_rowmajor(host(got.sf), total, k, pr), so)
    assert host(got.g)[0] == np.float32(go)
    fused = nv.quantize(to_dev(x), rows=total, row_index=idx_d, src_rows=tokens,
                        group_offsets=off_d, num_groups=E if grouped else 0,
                        sf_layout=nv.NVFP4_SF_MMA)["row"]
    assert np.array_equal(host(fused.q), host(got.q))
    assert np.array_equal(host(fused.sf), host(got.sf))


def test_gather_rows_256_groups(nv, orc):
    """Dispatch into the 256-group limit: runs of more than 32 empty groups, groups of
    1, 127, 128, 129 and 256 rows, the last group non-empty after 39 empty ones.  Every
    dispatched row's codes and scale bytes equal the oracle's quantisation of the
    gathered rows; the padding rows' scale bytes are left as they were (zero here)."""
    import torch
    rng = np.random.default_rng(57)
    tokens, k, G = 704, 128, 256
    counts = np.zeros(G, dtype=np.int64)
    sizes = {0: 3, 1: 1, 2: 127, 40: 128, 41: 129, 73: 256, 74: 5, 150: 64, 215: 33}
    for e, c in sizes.items():
        counts[e] = c
    counts[255] = 134
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    total = int(offsets[-1])
    x = W.f32_to_bf16_bits(W.student_t(rng, (tokens, k), 4.0, 1.0))
    row_index = np.concatenate([rng.permutation(tokens),
                                rng.integers(0, tokens, total - tokens)]).astype(np.int32)
    src = nv.quantize(to_dev(x), sf_layout=nv.NVFP4_SF_MMA)["row"]
    got = nv.gather_rows(src, torch.from_numpy(row_index).cuda(), torch.from_numpy(offsets).cuda())
    xg = np.ascontiguousarray(x[row_index])
    qo, so, go = orc.nvfp4_quantize(xg, 0, amax=(orc.amax(x, 0), 0.0))
    assert np.array_equal(host(got.q), qo)
    pr = grouped_padded_rows(offsets)
    assert np.array_equal(sf_mma_to_rowmajor(host(got.sf), total, k, pr), so)
    sf_all = host(got.sf).reshape(-1)
    mask = np.ones(sf_all.size, dtype=bool)
    k16 = k // 16
    r = pr[:, None]
    b = np.arange(k16)[None, :]
    mask[((r // 128) * (k16 // 4) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4] = False
    assert not sf_all[mask].any()


def test_gather_rows_bad_index_reports(nv):
    import torch
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    src = nv.quantize(x, sf_layout=nv.NVFP4_SF_MMA)["row"]
    idx = torch.tensor([0, 5, 64] + [1] * 13, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    nv.gather_rows(src, idx, workspace=ws)
    assert nv.nvfp4_workspace_status(ws) == 8


@pytest.mark.parametrize("c0", [0, 64])
def test_quantize_column_slice_of_wider_tensor(nv, orc, c0):
    """ld > cols: the input is a 320-column slice (at column c0) of a 400-column tensor,
    quantised with every output of the gradient recipe in tiled and row-major layouts."""
    full = edge_tensor(192, 400, seed=31 + c0)
    xs = to_dev(full)[:, c0:c0 + 320]
    assert xs.stride(0) == 400
    x = np.ascontiguousarray(full[:, c0:c0 + 320])
    for layout in (nv.NVFP4_SF_ROWMAJOR, nv.NVFP4_SF_MMA):
        out = nv.quantize(xs, rowwise=True, colwise=True, rounding=1, rht=True, seed=9,
                          mx_outputs=nv.NVFP4_COLWISE, sf_layout=layout)
        qr, sr, gr = orc.nvfp4_quantize(x, 0, 1, 0, 0, 9)
        qc, sc, gc = orc.nvfp4_quantize(x, 1, 1, 0, 1, 9)
        mq, me = orc.mxfp8_quantize(x, 1, 0, 9)
        to_rm = (lambda sf, r, k: sf_mma_to_rowmajor(host(sf), r, k)) if layout else \
            (lambda sf, r, k: host(sf))
        np.testing.assert_array_equal(host(out["row"].q), qr)
        np.testing.assert_array_equal(to_rm(out["row"].sf, 192, 320), sr)
        np.testing.assert_array_equal(host(out["col"].q), qc)
        np.testing.assert_array_equal(to_rm(out["col"].sf, 320, 192), sc)
        assert float(host(out["row"].g)[0]) == gr and float(host(out["col"].g)[0]) == gc
        np.testing.assert_array_equal(host(out["mx_col"][0]), mq)
        np.testing.assert_array_equal(host(out["mx_col"][1]), me)
        assert nv.nvfp4_workspace_status(out["workspace"]) == 0
