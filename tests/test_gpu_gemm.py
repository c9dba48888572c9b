"""GPU parity of the tcgen05 block-scaled GEMM and the MoE grouped GEMM against the
oracle's FP64 GEMM of the dequantised operands: |D - D_ref| <= 1e-3 sum_k |a_hat||b_hat|
(plus half a bf16 ulp of D_ref for bf16 output).  Operands are quantised by the oracle
and uploaded, so these tests do not depend on the GPU quantizer."""
import numpy as np
import pytest

import workloads as W
from gpu_util import (check_gemm, cuda_available, grouped_padded_rows, host, nvfp4_operand,
                      to_dev, sf_mma_to_rowmajor)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


@pytest.fixture(params=["256", "128"])
def tile_n(request, monkeypatch):
    """Both output-tile widths of the GEMM kernel: 256 (one accumulator) and 128 (two
    accumulators in turn), forced through the library's tile override."""
    monkeypatch.setenv("NVFP4_GEMM_TILE_N", request.param)
    return int(request.param)


def _operands(orc, nv, x, w, scaling_w=0):
    qa, sa, ga = orc.nvfp4_quantize(x, 0)
    qb, sb, gb = orc.nvfp4_quantize(w, 0, scaling=scaling_w)
    A = nvfp4_operand(nv, qa, sa, ga, x.shape[0], x.shape[1])
    B = nvfp4_operand(nv, qb, sb, gb, w.shape[0], w.shape[1])
    return (qa, sa, ga), (qb, sb, gb), A, B


def test_tiny_linear_fp32(nv, orc, tile_n):
    """X 128x256 (1% outliers x50) times W^T 128x256, FP32 out, checked in full."""
    x, w = W.tiny_linear(0)
    (qa, sa, ga), (qb, sb, gb), A, B = _operands(orc, nv, x, w)
    D = host(nv.gemm(A, B, nv.NVFP4_OUT_F32))
    Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    check_gemm(D, Dr, Ar, bf16_out=False)


@pytest.mark.parametrize("mnk", [(256, 512, 512), (272, 400, 768), (128, 256, 256),
                                 (384, 128, 1024), (16, 16, 256)])
@pytest.mark.parametrize("bf16_out", [False, True])
def test_gemm_shapes(nv, orc, tile_n, mnk, bf16_out):
    M, N, K = mnk
    rng = np.random.default_rng(M + N + K)
    x = W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0, 1.0))
    w = W.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    (qa, sa, ga), (qb, sb, gb), A, B = _operands(orc, nv, x, w)
    D = host(nv.gemm(A, B, nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32))
    if bf16_out:
        D = W.bf16_bits_to_f32(D.view(np.uint16))
    Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    check_gemm(D, Dr, Ar, bf16_out)


def test_gemm_padded_ldd(nv, orc, tile_n):
    """Output with a leading dimension larger than N: the padding is left untouched."""
    import torch
    M, N, K = 128, 256, 512
    rng = np.random.default_rng(4)
    x = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    (qa, sa, ga), (qb, sb, gb), A, B = _operands(orc, nv, x, w)
    out = torch.full((M, N + 64), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    nv.nvfp4_gemm(A.q, A.sf, A.g, B.q, B.sf, B.g, M, N, K, nv.NVFP4_OUT_F32, out, N + 64, None, ws, 256)
    D = host(out)
    assert np.all(D[:, N:] == 7.0)
    Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    check_gemm(D[:, :N], Dr, Ar, False)
    assert nv.nvfp4_workspace_status(ws) == 0


def test_gemm_full_size_forward(nv, orc):
    """Weight 4096x4096 ~N(0,0.02) with 2D 16x16 scales, X 8192x4096 ~N(0,1) with 0.1%
    outlier channels x100 (1D): GEMM M=8192 N=4096 K=4096, bf16 out, the GPU quantizer
    feeding the GPU GEMM as the benchmark runs it; sampled rows against the oracle."""
    w, x, _ = W.weight_and_outlier_acts(2)
    Wq = nv.quantize(to_dev(w), scaling=nv.NVFP4_2D16x16, sf_layout=nv.NVFP4_SF_MMA)["row"]
    Xq = nv.quantize(to_dev(x), sf_layout=nv.NVFP4_SF_MMA)["row"]
    D = host(nv.gemm(Xq, Wq, nv.NVFP4_OUT_BF16))
    D = W.bf16_bits_to_f32(D.view(np.uint16))
    qb, sb, gb = orc.nvfp4_quantize(w, 0, scaling=1)
    np.testing.assert_array_equal(host(Wq.q), qb)
    np.testing.assert_array_equal(sf_mma_to_rowmajor(host(Wq.sf), 4096, 4096), sb)
    am = (orc.amax(x, 0), 0.0)
    rows = np.array([0, 1, 127, 128, 4095, 5000, 8191])
    for r in rows:
        r0 = (r // 16) * 16
        qa, sa, ga = orc.nvfp4_quantize(x[r0:r0 + 16], 0, amax=am)
        Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[r - r0])
        check_gemm(D[r:r + 1], Dr, Ar, True)


def _grouped_case(orc, nv, counts, N, K, seed):
    import torch
    rng = np.random.default_rng(seed)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    total = int(offsets[-1])
    G = len(counts)
    a = W.f32_to_bf16_bits(rng.standard_normal((total, K)).astype(np.float32))
    ws_ = [W.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
           for _ in range(G)]
    qa, sa, ga = orc.nvfp4_quantize(a, 0)
    pr = grouped_padded_rows(offsets)
    padded_total = int(sum(((c + 127) // 128) * 128 for c in counts))
    A = nvfp4_operand(nv, qa, sa, ga, total, K, pr, max(padded_total, 128))
    qbs = [orc.nvfp4_quantize(w, 0) for w in ws_]
    from gpu_util import rowmajor_to_sf_mma
    sfb = np.concatenate([rowmajor_to_sf_mma(t[1], N, K) for t in qbs])
    qb = np.stack([t[0] for t in qbs])
    gb = np.array([t[2] for t in qbs], dtype=np.float32)
    dev = dict(device="cuda")
    return (offsets, (qa, sa, ga), (qb, np.stack([t[1] for t in qbs]), gb), A,
            torch.from_numpy(qb).to(**dev), torch.from_numpy(sfb).to(**dev),
            torch.from_numpy(gb).to(**dev), torch.from_numpy(offsets.astype(np.int32)).to(**dev))


@pytest.mark.parametrize("counts", [[0, 150, 7, 0, 33, 130], [128, 256], [1, 0, 303]])
@pytest.mark.parametrize("bf16_out", [False, True])
def test_grouped_gemm(nv, orc, tile_n, counts, bf16_out):
    N, K = 256, 512
    offsets, (qa, sa, ga), (qb, sb, gb), A, qb_d, sfb_d, gb_d, off_d = _grouped_case(
        orc, nv, counts, N, K, seed=sum(counts))
    D = host(nv.grouped_gemm(off_d, A, qb_d, sfb_d, gb_d, N,
                             nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32))
    if bf16_out:
        D = W.bf16_bits_to_f32(D.view(np.uint16))
    sel = np.arange(int(offsets[-1]))
    Dr, Ar = orc.nvfp4_grouped_gemm_rows(offsets, qa, sa, ga, qb, sb, gb, sel)
    check_gemm(D, Dr, Ar, bf16_out)


def test_grouped_gemm_moe_up_sampled(nv, orc):
    """64 experts, hidden 4096 -> FFN 1536, 16384 tokens top-4 with Zipf(1.1) counts:
    the up projection on 65536 routed rows; sampled rows of several experts."""
    import torch
    rng = np.random.default_rng(3)
    tokens, hidden, ffn, E = 16384, 4096, 1536, 64
    _, row_token, offsets = W.moe_routing(rng, tokens, E, 4)
    total = int(offsets[-1])
    x = W.f32_to_bf16_bits(rng.standard_normal((tokens, hidden)).astype(np.float32))
    w_up = W.f32_to_bf16_bits(rng.standard_normal((E, ffn, hidden)).astype(np.float32) * 0.02)
    xq = nv.quantize(to_dev(x), rows=total,
                     row_index=torch.from_numpy(row_token.astype(np.int32)).cuda(),
                     src_rows=tokens, group_offsets=torch.from_numpy(offsets).cuda(),
                     num_groups=E, sf_layout=nv.NVFP4_SF_MMA)["row"]
    wq = [nv.quantize(to_dev(w_up[e]), sf_layout=nv.NVFP4_SF_MMA)["row"] for e in range(E)]
    qb_d = torch.stack([t.q for t in wq])
    sfb_d = torch.cat([t.sf for t in wq])
    gb_d = torch.cat([t.g for t in wq])
    D = host(nv.grouped_gemm(torch.from_numpy(offsets).cuda(), xq, qb_d, sfb_d, gb_d, ffn))
    D = W.bf16_bits_to_f32(D.view(np.uint16))
    am = (orc.amax(x, 0), 0.0)
    big = int(np.argmax(np.diff(offsets)))
    small = int(np.argmin(np.diff(offsets)))
    for e in (big, small, 17):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        qb, sb, gb = orc.nvfp4_quantize(w_up[e], 0)
        for r in sorted({lo, hi - 1, (lo + hi) // 2}):
            xr = np.ascontiguousarray(np.tile(x[row_token[r]], (16, 1)))
            qa, sa, ga = orc.nvfp4_quantize(xr, 0, amax=am)
            Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[0])
            check_gemm(D[r:r + 1], Dr, Ar, True)


@pytest.mark.parametrize("bf16_out", [False, True])
def test_gemm_amax_out(nv, orc, tile_n, bf16_out):
    """amax_out holds max |D| over the stored output, exactly, and replaces a stale value."""
    import torch
    M, N, K = 272, 400, 512
    rng = np.random.default_rng(11)
    x = W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0, 1.0))
    w = W.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    _, _, A, B = _operands(orc, nv, x, w)
    am = torch.full((1,), 1e30, dtype=torch.float32, device="cuda")
    D = host(nv.gemm(A, B, nv.NVFP4_OUT_BF16 if bf16_out else nv.NVFP4_OUT_F32, amax_out=am))
    if bf16_out:
        D = W.bf16_bits_to_f32(D.view(np.uint16))
    assert host(am)[0] == np.max(np.abs(D)).astype(np.float32)


def test_grouped_gemm_amax_out(nv, orc, tile_n):
    """Grouped: the max covers every group's rows and nothing from padding tiles."""
    import torch
    N, K = 256, 512
    offsets, _, _, A, qb_d, sfb_d, gb_d, off_d = _grouped_case(orc, nv, [0, 150, 7, 0, 33, 130],
                                                                N, K, seed=5)
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    D = host(nv.grouped_gemm(off_d, A, qb_d, sfb_d, gb_d, N, amax_out=am))
    D = W.bf16_bits_to_f32(D.view(np.uint16))
    assert host(am)[0] == np.max(np.abs(D)).astype(np.float32)


def test_requantize_with_gemm_amax(nv, orc):
    """Quantising the up projection's output with the GEMM's amax_out as amax_in gives the
    same bytes as the quantiser's own amax pass; and that amax_in path matches the oracle
    on an output the oracle computed itself (its FP64 grouped GEMM, rounded to bf16)."""
    import torch
    N, K = 256, 512
    counts = [0, 150, 7, 0, 33, 130]
    offsets, (qa, sa, ga), (qb, sb, gb), A, qb_d, sfb_d, gb_d, off_d = _grouped_case(
        orc, nv, counts, N, K, seed=9)
    am = torch.zeros(2, dtype=torch.float32, device="cuda")
    H = nv.grouped_gemm(off_d, A, qb_d, sfb_d, gb_d, N, amax_out=am)
    kw = dict(group_offsets=off_d, num_groups=len(counts), sf_layout=nv.NVFP4_SF_MMA)
    fused = nv.quantize(H, amax=am, **kw)["row"]
    own = nv.quantize(H, **kw)["row"]
    for f in ("q", "sf", "g"):
        assert np.array_equal(host(getattr(fused, f)), host(getattr(own, f)))
    total = int(offsets[-1])
    Dr, _ = orc.nvfp4_grouped_gemm_rows(offsets, qa, sa, ga, qb, sb, gb, np.arange(total))
    h = W.f32_to_bf16_bits(Dr.astype(np.float32))
    amax_h = float(np.max(np.abs(W.bf16_bits_to_f32(h))))
    amd = torch.tensor([amax_h, amax_h], dtype=torch.float32, device="cuda")
    got = nv.quantize(to_dev(h), amax=amd, **kw)["row"]
    q, sf, g = orc.nvfp4_quantize(h, 0, amax=(amax_h, amax_h))
    assert np.array_equal(host(got.q), q)
    assert np.array_equal(sf_mma_to_rowmajor(host(got.sf), total, N,
                                             grouped_padded_rows(offsets)), sf)
    assert float(host(got.g)[0]) == g

def test_grouped_gemm_max_groups(nv, orc, tile_n):
    """256 groups (the limit), many of them empty, ragged counts; every row checked."""
    rng = np.random.default_rng(256)
    counts = [int(c) if rng.random() > 0.3 else 0 for c in rng.integers(1, 40, 256)]
    counts[-1] += (16 - sum(counts) % 16) % 16  # the oracle quantises whole 16-row tiles
    N, K = 256, 256
    offsets, (qa, sa, ga), (qb, sb, gb), A, qb_d, sfb_d, gb_d, off_d = _grouped_case(
        orc, nv, counts, N, K, seed=256)
    D = W.bf16_bits_to_f32(host(nv.grouped_gemm(off_d, A, qb_d, sfb_d, gb_d, N)))
    Dr, Ar = orc.nvfp4_grouped_gemm_rows(offsets, qa, sa, ga, qb, sb, gb,
                                         np.arange(int(offsets[-1])))
    check_gemm(D, Dr, Ar, True)


def test_all_zero_operands(nv, orc):
    """amax 0: S = g = 1, every code and scale byte is the oracle's (zeros), and the
    GEMM of zero operands is exactly zero (with amax_out 0)."""
    import torch
    x = np.zeros((256, 512), dtype=np.uint16)
    out = nv.quantize(to_dev(x), rowwise=True, colwise=True, rounding=nv.NVFP4_SR, rht=True,
                      seed=3, sf_layout=nv.NVFP4_SF_MMA)
    for d, t in ((0, out["row"]), (1, out["col"])):
        q, sf, g = orc.nvfp4_quantize(x, d, 1, 0, d, 3)
        assert g == 1.0 and float(host(t.g)[0]) == g
        np.testing.assert_array_equal(host(t.q), q)
        np.testing.assert_array_equal(sf_mma_to_rowmajor(host(t.sf), t.rows, t.k), sf)
    am = torch.full((1,), 7.0, dtype=torch.float32, device="cuda")
    D = host(nv.gemm(out["row"], out["row"], nv.NVFP4_OUT_F32, amax_out=am))
    assert not np.any(D) and host(am)[0] == 0.0


def test_gemm_cycle_count(nv):
    """The workspace's cycle count of a GEMM call: positive, cleared by the next
    call, and divided by the call's CUDA-event time a clock between 0.5 and 2.2 GHz
    (the B200's SM clock range)."""
    import torch
    dev = torch.device("cuda")
    M, N, K = 4096, 4096, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    u8 = dict(dtype=torch.uint8, device=dev)
    qa = torch.randint(0, 256, (M, K // 2), generator=g, **u8)
    qb = torch.randint(0, 256, (N, K // 2), generator=g, **u8)
    sa = torch.randint(0x30, 0x40, (nv.nvfp4_sf_mma_bytes(M, K),), generator=g, **u8)
    sb = torch.randint(0x30, 0x40, (nv.nvfp4_sf_mma_bytes(N, K),), generator=g, **u8)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_size(M, N, K), **u8)
    for _ in range(3):
        nv.nvfp4_gemm(qa, sa, one, qb, sb, one, M, N, K, nv.NVFP4_OUT_BF16, D, N, None, ws, ws.numel())
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    nv.nvfp4_gemm(qa, sa, one, qb, sb, one, M, N, K, nv.NVFP4_OUT_BF16, D, N, None, ws, ws.numel())
    e.record()
    e.synchronize()
    cycles = nv.nvfp4_gemm_cycles(ws)
    mhz = cycles / (s.elapsed_time(e) * 1e3)
    assert nv.nvfp4_workspace_status(ws) == 0
    assert 500 < mhz < 2200, (cycles, mhz)
    # the next call restarts the count
    nv.nvfp4_gemm(qa, sa, one, qb, sb, one, 256, 256, 256, nv.NVFP4_OUT_BF16, D, N, None, ws,
                  ws.numel())
    small = nv.nvfp4_gemm_cycles(ws)
    assert 0 < small < cycles
