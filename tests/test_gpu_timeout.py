"""The device-side timeout path, exercised without faulting anything.

Every barrier wait in the quantiser and GEMM kernels gives up after a limit
(2 s), records NVFP4_ERR_TIMEOUT in the workspace status word and lets the
kernel return normally.  The test hook NVFP4_TEST_UNSIGNALLED_WAIT_NS makes the
kernels' producers issue no copy at all, so every consumer waits on a barrier
that nothing signals -- with nothing in flight -- and gives up after the given
limit (1 ms here).  Each test checks that the status word reads
NVFP4_ERR_TIMEOUT, that the call returned well within the normal 2 s limit, and
that the next normal call on the same workspace runs clean and matches the
oracle."""
import time

import numpy as np
import pytest

import workloads as W
from gpu_util import check_gemm, cuda_available, host, nvfp4_operand, sf_mma_to_rowmajor, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

HOOK = "NVFP4_TEST_UNSIGNALLED_WAIT_NS"
TIMEOUT = 6  # NVFP4_ERR_TIMEOUT


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


def test_quantize_wait_runs_out_then_recovers(nv, orc, monkeypatch):
    import torch
    x = W.heavy_tailed(21, 256, 384)
    xd = to_dev(x)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kw = dict(rowwise=True, colwise=True, rounding=nv.NVFP4_SR, rht=True, seed=3,
              mx_outputs=nv.NVFP4_COLWISE, workspace=ws)
    torch.cuda.synchronize()
    monkeypatch.setenv(HOOK, "1000000")
    t0 = time.perf_counter()
    nv.quantize(xd, **kw)                       # amax pass and fused pass, no copies
    assert nv.nvfp4_workspace_status(ws) == TIMEOUT
    assert time.perf_counter() - t0 < 1.0
    monkeypatch.delenv(HOOK)
    out = nv.quantize(xd, **kw)
    assert nv.nvfp4_workspace_status(ws) == 0
    for d, key in ((0, "row"), (1, "col")):
        q, sf, g = orc.nvfp4_quantize(x, d, 1, 0, d, 3)
        t = out[key]
        np.testing.assert_array_equal(host(t.q), q)
        np.testing.assert_array_equal(host(t.sf), sf)
        assert float(host(t.g)[0]) == g


@pytest.mark.parametrize("tile_n", ["256", "128"])
def test_gemm_wait_runs_out_then_recovers(nv, orc, monkeypatch, tile_n):
    import torch
    M, N, K = 272, 400, 512
    rng = np.random.default_rng(22)
    x = W.f32_to_bf16_bits(W.student_t(rng, (M, K), 3.0, 1.0))
    w = W.f32_to_bf16_bits(W.normal(rng, (N, K), 0.02))
    qa, sa, ga = orc.nvfp4_quantize(x, 0)
    qb, sb, gb = orc.nvfp4_quantize(w, 0)
    A = nvfp4_operand(nv, qa, sa, ga, M, K)
    B = nvfp4_operand(nv, qb, sb, gb, N, K)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("NVFP4_GEMM_TILE_N", tile_n)
    torch.cuda.synchronize()
    monkeypatch.setenv(HOOK, "1000000")
    t0 = time.perf_counter()
    nv.gemm(A, B, nv.NVFP4_OUT_F32, workspace=ws)
    assert nv.nvfp4_workspace_status(ws) == TIMEOUT
    assert time.perf_counter() - t0 < 1.0
    monkeypatch.delenv(HOOK)
    D = host(nv.gemm(A, B, nv.NVFP4_OUT_F32, workspace=ws))
    assert nv.nvfp4_workspace_status(ws) == 0
    Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb)
    check_gemm(D, Dr, Ar, False)


def test_mxfp8_gemm_wait_runs_out_then_recovers(nv, orc, monkeypatch):
    import torch
    from gpu_util import rowmajor_to_sf_mma
    M, N, K = 256, 128, 256
    rng = np.random.default_rng(23)
    x = W.f32_to_bf16_bits(W.normal(rng, (M, K)))
    w = W.f32_to_bf16_bits(W.normal(rng, (N, K), 0.02))
    qa, ea = orc.mxfp8_quantize(x, 0)
    qb, eb = orc.mxfp8_quantize(w, 0)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    A, SA = up(qa), up(rowmajor_to_sf_mma(ea, M, K // 2))
    B, SB = up(qb), up(rowmajor_to_sf_mma(eb, N, K // 2))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    monkeypatch.setenv(HOOK, "1000000")
    nv.mx_gemm(A, SA, B, SB, nv.NVFP4_OUT_F32, workspace=ws)
    assert nv.nvfp4_workspace_status(ws) == TIMEOUT
    monkeypatch.delenv(HOOK)
    D = host(nv.mx_gemm(A, SA, B, SB, nv.NVFP4_OUT_F32, workspace=ws))
    assert nv.nvfp4_workspace_status(ws) == 0
    Dr, Ar = orc.mxfp8_gemm_rows(qa, ea, qb, eb)
    check_gemm(D, Dr, Ar, False)
