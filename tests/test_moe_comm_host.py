"""Host side of the MXFP8 expert combine (iitak page, "But": expert outputs travel at
8.25 bits per number): the expert-parallel plan, and the whole return trip run as two
gloo ranks on CPU -- counts exchanged, the oracle's MXFP8 rows of each expert rank sent
back through exchange_rows, combined by the oracle on each token rank -- against a
single-process combine of the same rows.  CPU only."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_plan_groups_slots_by_destination():
    from nvfp4_bit_precision_b200.moe_comm import ExpertParallelPlan
    rng = np.random.default_rng(0)
    te, _, _ = W.moe_routing(rng, 300, 16, 4)
    plan = ExpertParallelPlan(te, 16, 4)
    dest = te.reshape(-1) // 4
    sent_dest = dest[plan.send_order]
    assert np.all(np.diff(sent_dest) >= 0)                     # grouped by rank, in order
    assert np.array_equal(plan.send_counts, np.bincount(dest, minlength=4))
    # slot (t, j) sits at slot_row[t, j] of the send (and the returning) order
    flat = np.arange(te.size)
    assert np.array_equal(plan.send_order[plan.slot_row.reshape(-1)], flat)
    assert np.array_equal(plan.dest_expert, te.reshape(-1)[plan.send_order])
    with pytest.raises(ValueError):
        ExpertParallelPlan(te, 15, 4)


def test_payload_is_8_25_bits_per_number():
    from nvfp4_bit_precision_b200.moe_comm import payload_bits_per_number
    assert payload_bits_per_number(4096) == 8.25             # iitak, "But"
    assert 16 / payload_bits_per_number(4096) > 1.9          # against bf16


def _expert_rows(rank, n, hidden):
    """Deterministic expert outputs of an expert rank (rows in arrival order)."""
    rng = np.random.default_rng(100 + rank)
    return W.f32_to_bf16_bits(W.student_t(rng, (n, hidden), 3.0, 0.5))


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle as orc
    from nvfp4_bit_precision_b200.moe_comm import ExpertParallelPlan, exchange_counts, exchange_rows
    E, H, T, K = 8, 96, 40, 3
    te, _, _ = W.moe_routing(np.random.default_rng(rank), T, E, K)
    weight = np.random.default_rng(50 + rank).random((T, K)).astype(np.float32)
    plan = ExpertParallelPlan(te, E, world)
    rows_from = exchange_counts(plan.send_counts)             # dispatch side: rows per source
    R = int(rows_from.sum())
    x = _expert_rows(rank, R, H)                              # this rank's expert outputs
    q, e8 = orc.mxfp8_quantize(x, 0)                          # the sender's MXFP8 rows
    q_back = exchange_rows(torch.from_numpy(q), rows_from, plan.send_counts)
    e8_back = exchange_rows(torch.from_numpy(e8), rows_from, plan.send_counts)
    got = orc.mxfp8_combine(q_back.numpy(), e8_back.numpy(), plan.slot_row, weight)
    out[rank] = (te, weight, rows_from, got)
    dist.barrier()
    dist.destroy_process_group()


def test_combine_two_gloo_ranks_matches_single_process(orc):
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    from nvfp4_bit_precision_b200.moe_comm import ExpertParallelPlan
    E, H = 8, 96
    plans = {r: ExpertParallelPlan(out[r][0], E, world) for r in range(world)}
    # expert rank d receives, from each source s in rank order, plans[s]'s rows for d
    for r in range(world):
        te, weight, rows_from, got = out[r]
        assert list(rows_from) == [int(plans[s].send_counts[r]) for s in range(world)]
    # single process: every slot's expert output row, by who computed it
    for r in range(world):
        te, weight, _, got = out[r]
        plan = plans[r]
        rows = []
        for d in range(world):
            R_d = sum(int(plans[s].send_counts[d]) for s in range(world))
            x = _expert_rows(d, R_d, H)
            start = sum(int(plans[s].send_counts[d]) for s in range(r))
            rows.append(x[start:start + int(plan.send_counts[d])])
        allx = np.concatenate(rows)                           # in this rank's send order
        q, e8 = orc.mxfp8_quantize(allx, 0)
        expect = orc.mxfp8_combine(q, e8, plan.slot_row, weight)
        np.testing.assert_array_equal(got, expect)


def test_oracle_combine_closed_form(orc):
    """The oracle's combine on hand-built rows: every element of row r is +-(1 + r/8) * 2^(r-2)
    (E4M3 code 0x38 + r with scale byte 125 + r), weights 0.5, 0.25, 0.125, a missing slot
    (-1) skipped; the weighted sums are exact in binary32, and the output is their bf16
    rounding (nearest even)."""
    H = 64
    rows = 6
    q = np.array([[0x38 + r] * H for r in range(rows)], dtype=np.uint8)
    q[:, 1::2] |= 0x80                                        # odd columns negative
    e8 = np.array([[125 + r] * (H // 32) for r in range(rows)], dtype=np.uint8)
    slot = np.array([[0, 3, -1], [5, 1, 2]], dtype=np.int32)
    w = np.array([[0.5, 0.25, 0.125], [0.5, 0.25, 0.125]], dtype=np.float32)
    got = W.bf16_bits_to_f32(orc.mxfp8_combine(q, e8, slot, w))
    val = lambda r: (1 + r / 8) * 2.0 ** (r - 2)
    for t in range(2):
        exact = sum(float(w[t, j]) * val(slot[t, j]) for j in range(3) if slot[t, j] >= 0)
        expect = W.bf16_bits_to_f32(W.f32_to_bf16_bits(np.float32([exact, -exact])))
        assert np.all(got[t, 0::2] == expect[0]) and np.all(got[t, 1::2] == expect[1])
    assert got[1, 0] == 6.8125                               # 6.796875 needs 9 bits: bf16 rounds it
