"""GPU parity of the MXFP8 expert combine (iitak page, "But": expert outputs travel at
8.25 bits per number): the combine kernel against the oracle bit for bit (rows of any
count, missing slots, heavy-tailed values), and the whole return trip -- MXFP8
quantisation of the expert rows, the all-to-all, the weighted combine -- through
combine_mxfp8 on a one-rank NCCL group (every run here has one GPU; the two-rank
exchange is covered on CPU with gloo)."""
import os

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


@pytest.mark.parametrize("rows,cols,tokens,k", [(37, 96, 20, 4), (1000, 4096, 300, 4),
                                                 (5, 32, 7, 1)])
def test_combine_kernel_bitexact(nv, orc, rows, cols, tokens, k):
    import torch
    rng = np.random.default_rng(rows + cols)
    x = W.f32_to_bf16_bits(W.student_t(rng, (rows, cols), 3.0, 0.5))
    q, e8 = orc.mxfp8_quantize(x, 0)
    slot = rng.integers(-1, rows, (tokens, k)).astype(np.int32)
    w = rng.random((tokens, k)).astype(np.float32)
    dev = dict(device="cuda")
    out = torch.empty((tokens, cols), dtype=torch.bfloat16, **dev)
    ws = torch.zeros(256, dtype=torch.uint8, **dev)
    nv.mxfp8_combine(torch.from_numpy(q).to(**dev), torch.from_numpy(e8).to(**dev), rows, cols,
                     torch.from_numpy(slot).to(**dev), torch.from_numpy(w).to(**dev), tokens, k,
                     out, ws, 256)
    np.testing.assert_array_equal(host(out), orc.mxfp8_combine(q, e8, slot, w))
    assert nv.nvfp4_workspace_status(ws) == 0


def test_combine_bad_row_index_reports(nv, orc):
    import torch
    dev = dict(device="cuda")
    q = torch.zeros((4, 32), dtype=torch.uint8, **dev)
    e8 = torch.full((4, 1), 127, dtype=torch.uint8, **dev)
    slot = torch.tensor([[0, 9]], dtype=torch.int32, **dev)       # row 9 does not exist
    w = torch.ones((1, 2), dtype=torch.float32, **dev)
    out = torch.empty((1, 32), dtype=torch.bfloat16, **dev)
    ws = torch.zeros(256, dtype=torch.uint8, **dev)
    nv.mxfp8_combine(q, e8, 4, 32, slot, w, 1, 2, out, ws, 256)
    assert nv.nvfp4_workspace_status(ws) == 8                      # NVFP4_ERR_INDEX


def test_return_trip_one_rank_nccl(nv, orc):
    """combine_mxfp8 end to end on a one-rank NCCL group: 64 experts, 16384 tokens top-4
    (Zipf 1.1 routing), hidden 4096 -- the MoE workload's shape -- with the expert rows
    (65536, in arrival order) quantised on the GPU; checked against the oracle's MXFP8
    of the same rows and its combine."""
    import torch
    import torch.distributed as dist
    from nvfp4_bit_precision_b200.moe_comm import ExpertParallelPlan, combine_mxfp8, exchange_counts
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29517")
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        rng = np.random.default_rng(3)
        te, _, _ = W.moe_routing(rng, 16384, 64, 4)
        w = rng.random(te.shape).astype(np.float32)
        plan = ExpertParallelPlan(te, 64, 1)
        rows_from = exchange_counts(plan.send_counts, device="cuda")
        R = int(rows_from.sum())
        assert R == 65536
        x = W.f32_to_bf16_bits(W.student_t(np.random.default_rng(4), (R, 4096), 3.0, 0.5))
        out = combine_mxfp8(to_dev(x), rows_from, plan, w)
        torch.cuda.synchronize()
        sel = np.arange(0, 16384, 997)                       # sampled tokens, every column
        used = plan.slot_row[sel].reshape(-1)                # their rows (MXFP8 rows are
        q, e8 = orc.mxfp8_quantize(np.ascontiguousarray(x[used]), 0)  # quantised one by one)
        local = np.arange(used.size, dtype=np.int32).reshape(len(sel), -1)
        expect = orc.mxfp8_combine(q, e8, local, w[sel])
        np.testing.assert_array_equal(host(out)[sel], expect)
    finally:
        dist.destroy_process_group()
