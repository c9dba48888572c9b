"""Expert-parallel combine of MoE expert outputs in MXFP8.

In expert-parallel MoE training each rank holds some of the experts; tokens go to
the ranks of their experts and the expert outputs come back.  The iitak.ru page
("Thinking Machines uskorila obuchenie Inkling 2 Small 4-bitnymi chislami",
section "But") has the outputs cross NVLink at 8.25 bits per number -- an 8-bit
element plus an 8-bit scale per 32 -- instead of 16, because compute outran the
link.  This module is that return path:

  * ``ExpertParallelPlan`` -- host bookkeeping from a rank's routing: where each
    (token, slot) goes and where its expert output lands in the receive buffer.
  * ``exchange_counts`` -- one all-to-all of the row counts, so every expert rank
    knows how many rows each source sends.
  * ``exchange_rows`` -- the all-to-all of row-major byte payloads (codes, scales).
  * ``combine_mxfp8`` -- the whole return trip on the GPU: the expert rows
    quantised to MXFP8 (``mxfp8_quantize``, OCP MX v1.0 rule), sent back in the
    order they arrived, and combined per token with the routing weights
    (``mxfp8_combine``).  Every arithmetic step runs in libnvfp4.so; torch.distributed
    (NCCL on GPUs, gloo on CPU) carries the bytes.

Experts are spread evenly: expert e lives on rank e // (num_experts // world).
"""
from __future__ import annotations

import numpy as np


class ExpertParallelPlan:
    """Send plan of one rank for its tokens' routed slots.

    token_expert: int array [tokens, k] (expert of slot j of token t).  Slots are
    sent grouped by destination rank, in (token, slot) order within a rank; the
    expert ranks return rows in the order they received them, so the combine
    finds slot (t, j) at position ``slot_row[t, j]`` of the receive buffer."""

    def __init__(self, token_expert, num_experts: int, world: int):
        te = np.asarray(token_expert, dtype=np.int64)
        if te.ndim != 2:
            raise ValueError("token_expert must be [tokens, k]")
        if world < 1 or num_experts % world:
            raise ValueError("num_experts must be a multiple of the world size")
        if te.size and (te.min() < 0 or te.max() >= num_experts):
            raise ValueError("expert id out of range")
        self.tokens, self.k = te.shape
        self.world = world
        self.experts_per_rank = num_experts // world
        dest = (te // self.experts_per_rank).reshape(-1)
        self.send_order = np.argsort(dest, kind="stable")          # flat slot ids, by rank
        self.send_counts = np.bincount(dest, minlength=world).astype(np.int64)
        pos = np.empty_like(self.send_order)
        pos[self.send_order] = np.arange(self.send_order.size)
        self.slot_row = pos.reshape(self.tokens, self.k).astype(np.int32)
        self.dest_expert = te.reshape(-1)[self.send_order]         # expert of each sent row


def exchange_counts(send_counts, group=None, device="cpu"):
    """All-to-all of the per-destination row counts: returns how many rows this rank
    receives from each source rank."""
    import torch
    import torch.distributed as dist
    send = torch.as_tensor(np.asarray(send_counts, dtype=np.int64), device=device)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.cpu().numpy()


def exchange_rows(payload, send_splits, recv_splits, group=None):
    """All-to-all of a row-major payload [rows, row_bytes] (uint8): rows are sent in
    blocks of send_splits[d] to rank d and arrive in blocks of recv_splits[s] from
    rank s.  Works on CPU tensors (gloo) and CUDA tensors (NCCL)."""
    import torch
    import torch.distributed as dist
    send_splits = [int(v) for v in send_splits]
    recv_splits = [int(v) for v in recv_splits]
    out = torch.empty((sum(recv_splits),) + tuple(payload.shape[1:]), dtype=payload.dtype,
                      device=payload.device)
    dist.all_to_all_single(out, payload.contiguous(), output_split_sizes=recv_splits,
                           input_split_sizes=send_splits, group=group)
    return out


def combine_mxfp8(expert_rows, rows_from, plan: ExpertParallelPlan, weight, group=None,
                  workspace=None):
    """Return trip of the expert outputs, compressed to MXFP8.

    expert_rows: bf16 CUDA tensor [R, H] on this (expert) rank, rows in the order they
      arrived: rows_from[0] rows from rank 0, then rows_from[1] from rank 1, ...
    plan: this rank's plan as a token owner; weight: FP32 [tokens, k] routing weights.
    Returns bf16 [tokens, H]: sum_j weight[t, j] * (the MXFP8 value of slot (t, j)'s
    expert output), FP32 accumulation in slot order."""
    import torch
    from . import mxfp8_combine as _combine
    from . import mxfp8_quantize, NVFP4_ROWWISE
    R, H = expert_rows.shape
    dev = expert_rows.device
    u8 = dict(dtype=torch.uint8, device=dev)
    q = torch.empty((R, H), **u8)
    e8 = torch.empty((R, H // 32), **u8)
    if R:
        mxfp8_quantize(expert_rows, R, H, expert_rows.stride(0), NVFP4_ROWWISE, 0, 0, 0, q, e8,
                       None, None)
    # the rows go back where they came from: rows_from[s] rows to source s, and this rank
    # gets back plan.send_counts[d] rows from each expert rank d
    q_back = exchange_rows(q, rows_from, plan.send_counts, group)
    e8_back = exchange_rows(e8, rows_from, plan.send_counts, group)
    out = torch.empty((plan.tokens, H), dtype=torch.bfloat16, device=dev)
    slot_row = torch.from_numpy(plan.slot_row).to(dev)
    w = torch.as_tensor(weight, dtype=torch.float32).to(dev).contiguous()
    ws = workspace if workspace is not None else torch.zeros(256, **u8)
    _combine(q_back, e8_back, q_back.shape[0], H, slot_row, w, plan.tokens, plan.k, out, ws,
             ws.numel())
    return out


def payload_bits_per_number(cols: int) -> float:
    """Bits a combined row costs per element on the link: 8-bit codes plus one 8-bit
    scale per 32 elements."""
    return 8.0 * (cols + cols // 32) / cols
