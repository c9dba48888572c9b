"""Benchmark of the NVFP4 training hot path on B200.

One step = one pass of every hot-path operation over one batch of synthetic input:

  dense linear layer (tokens 16384 = 2 x 8192, hidden 5120, FFN 20480):
    quantise X (rowwise RNE + columnwise Hadamard RNE), W (16x16 2D, both directions),
    forward GEMM Y = X W^T, quantise dY (rowwise SR, columnwise Hadamard + SR, MXFP8
    columnwise), dgrad dX = dY W, wgrad dW = dY^T X;
  MoE expert forward (64 experts, hidden 4096, FFN 1536, 16384 tokens, top-4 routing with
    Zipf(1.1)-skewed counts): quantise the tokens once, dispatch the quantised rows into
    the grouped layout, grouped GEMM up (its epilogue also returns max |H|), requantise
    the up output with that amax, grouped GEMM down.

value = GEMM FLOP of the step / device time of the step (TFLOP/s), over all ranks.
Multi-GPU: independent replicas (weak scaling); the only collectives are the barrier
and the max of the timings.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "NVFP4 GEMM TFLOP/s + fused-quantize HBM GB/s, % of B200 roofline"
TOKENS, HIDDEN, FFN = 16384, 5120, 20480
MOE_TOKENS, MOE_HIDDEN, MOE_FFN, EXPERTS, TOPK = 16384, 4096, 1536, 64, 4
WORKLOAD = ("dense linear layer fwd+dgrad+wgrad (tokens 16384, hidden 5120, FFN 20480) + "
            "MoE expert forward (64 experts, hidden 4096, FFN 1536, 16384 tokens, top-4, Zipf 1.1)")
DENSE_FLOP = 3 * 2 * TOKENS * FFN * HIDDEN
DENSE_FLOP_PER_GEMM = 2 * TOKENS * FFN * HIDDEN


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu --set full capture of each kernel as it stands -- the forward GEMM
# 16384x20480x5120, and the amax + fused pass on dY 16384x20480; set to None
# whenever the kernel changes.
TRAFFIC_BYTES = {"gemm_dense_fwd": 1147.3e6, "quant_dy": 2071.1e6}


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
         "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p.update({k: m[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained") if k in m})
        p["source"] = "measured"
    return p


# ----------------------------------------------------------------------------- workload
class Step:
    """Device buffers and pre-built calls of one step."""

    def __init__(self, dev, host_inputs):
        import torch
        import nvfp4_bit_precision_b200 as nv
        self.nv, self.torch, self.dev = nv, torch, dev
        h = host_inputs
        self.h = h
        u8 = dict(dtype=torch.uint8, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        T, H, F = TOKENS, HIDDEN, FFN
        # inputs (device copies; the e2e loop refreshes them from pinned host memory)
        # Two input slots, so the end-to-end loop can copy step i+1's inputs
        # while step i computes; the device-timed loop uses slot 0 only.
        self.inputs = [dict(x=torch.empty((T, H), **bf), w=torch.empty((F, H), **bf),
                            dy=torch.empty((T, F), **bf),
                            tok=torch.empty((MOE_TOKENS, MOE_HIDDEN), **bf)) for _ in range(2)]
        self.row_token = torch.from_numpy(h["row_token"].astype(np.int32)).to(dev)
        self.offsets = torch.from_numpy(h["offsets"].astype(np.int32)).to(dev)
        self.routed = int(h["offsets"][-1])
        self.upload_inputs(0)
        self.upload_inputs(1)
        sfm = nv.nvfp4_sf_mma_bytes
        mk = lambda r, k: nv.NVFP4Tensor(torch.empty((r, k // 2), **u8),
                                         torch.zeros(sfm(r, k), **u8), torch.empty(1, **f32),
                                         r, k, nv.NVFP4_SF_MMA)
        self.Xr, self.Xc = mk(T, H), mk(H, T)
        self.Wr, self.Wc = mk(F, H), mk(H, F)
        self.Dr, self.Dc = mk(T, F), mk(F, T)
        self.mx_q = torch.empty((F, T), **u8)
        self.mx_e = torch.empty((F, T // 32), **u8)
        # Two output slots, so the end-to-end loop can read step i's results back
        # while step i+1 computes; self.Y etc. are slot 0's.
        self.outs = [dict(Y=torch.empty((T, F), **bf), dX=torch.empty((T, H), **bf),
                          dW=torch.empty((F, H), **bf)) for _ in range(2)]
        self.Y, self.dX, self.dW = (self.outs[0][k] for k in ("Y", "dX", "dW"))
        self.ws = [torch.zeros(256, **u8) for _ in range(8)]
        # MoE: expert weights are quantised once (outside the step), activations every step
        R = self.routed
        gsf = nv.nvfp4_sf_mma_grouped_bytes
        self.Tq = mk(MOE_TOKENS, MOE_HIDDEN)  # tokens, quantised once before dispatch
        # the dispatched rows share the tokens' global scale
        self.A_up = nv.NVFP4Tensor(torch.empty((R, MOE_HIDDEN // 2), **u8),
                                   torch.zeros(gsf(R, EXPERTS, MOE_HIDDEN), **u8),
                                   self.Tq.g, R, MOE_HIDDEN, nv.NVFP4_SF_MMA)
        self.h_amax = torch.zeros(2, **f32)  # [0] = max |H| from the up GEMM's epilogue
        self.Hup = torch.empty((R, MOE_FFN), **bf)
        self.A_dn = nv.NVFP4Tensor(torch.empty((R, MOE_FFN // 2), **u8),
                                   torch.zeros(gsf(R, EXPERTS, MOE_FFN), **u8),
                                   torch.empty(1, **f32), R, MOE_FFN, nv.NVFP4_SF_MMA)
        for o in self.outs:
            o["Out"] = torch.empty((R, MOE_HIDDEN), **bf)
        self.Out = self.outs[0]["Out"]
        self.wup = self._quantize_experts(h["w_up"], MOE_FFN, MOE_HIDDEN)
        self.wdn = self._quantize_experts(h["w_down"], MOE_HIDDEN, MOE_FFN)
        torch.cuda.synchronize(dev)

    def _quantize_experts(self, w_host, n, k):
        torch, nv = self.torch, self.nv
        q = torch.empty((EXPERTS, n, k // 2), dtype=torch.uint8, device=self.dev)
        per = nv.nvfp4_sf_mma_bytes(n, k)
        sf = torch.zeros(EXPERTS * per, dtype=torch.uint8, device=self.dev)
        g = torch.empty(EXPERTS, dtype=torch.float32, device=self.dev)
        for e in range(EXPERTS):
            we = torch.from_numpy(w_host[e].view(np.int16)).to(self.dev).view(torch.bfloat16)
            p = nv.QuantParams()
            p.outputs, p.sf_layout = nv.NVFP4_ROWWISE, nv.NVFP4_SF_MMA
            nv.nvfp4_quantize(we, n, k, k, p, q[e], sf[e * per:].data_ptr(), g[e:].data_ptr(),
                              None, None, None, self.ws[0], 256)
        return q, sf, g

    def upload_inputs(self, slot, non_blocking=False):
        torch = self.torch
        for name, dst in self.inputs[slot].items():
            src = self.h["pinned"][name] if "pinned" in self.h else torch.from_numpy(
                self.h[name].view(np.int16))
            dst.view(torch.int16).copy_(src, non_blocking=non_blocking)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.inputs[0].values())

    def _q(self, x, rows, cols, ld, out_row, out_col, ws, rounding=0, scaling=0, rht=0,
           mx_col=None, row_index=None, src_rows=0, groups=False, amax=None):
        nv = self.nv
        p = nv.QuantParams()
        p.rounding, p.scaling, p.rht_colwise, p.sf_layout = rounding, scaling, rht, nv.NVFP4_SF_MMA
        p.outputs = (nv.NVFP4_ROWWISE if out_row is not None else 0) | (
            nv.NVFP4_COLWISE if out_col is not None else 0)
        p.seed = 20251030
        if mx_col is not None:
            p.mx_outputs = nv.NVFP4_COLWISE
            p.mx_q_col, p.mx_sf_col = mx_col[0].data_ptr(), mx_col[1].data_ptr()
        if row_index is not None:
            p.row_index, p.src_rows = row_index.data_ptr(), src_rows
        if groups:
            p.group_offsets, p.num_groups = self.offsets.data_ptr(), EXPERTS
        if amax is not None:
            p.amax_in = amax.data_ptr()
        r, c = out_row, out_col
        nv.nvfp4_quantize(x, rows, cols, ld, p, r.q if r else None, r.sf if r else None,
                          r.g if r else None, c.q if c else None, c.sf if c else None,
                          c.g if c else None, ws, 256)

    def _g(self, A, B, D, ws):
        nv = self.nv
        nv.nvfp4_gemm(A.q, A.sf, A.g, B.q, B.sf, B.g, A.rows, B.rows, A.k, nv.NVFP4_OUT_BF16, D,
                      D.stride(0), None, ws, 256)

    def run(self, ev=None, slot=0):
        """Enqueue one step on the inputs of `slot`.  ev: optional dict name -> list of
        (start, end) event pairs."""
        nv, torch = self.nv, self.torch
        T, H, F = TOKENS, HIDDEN, FFN

        def timed(name, fn):
            if ev is None:
                fn()
                return
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            ev.setdefault(name, []).append((s, e))

        ws = self.ws
        inp = self.inputs[slot]
        out = self.outs[slot]
        timed("quant_x", lambda: self._q(inp["x"], T, H, H, self.Xr, self.Xc, ws[0], rht=1))
        timed("quant_w", lambda: self._q(inp["w"], F, H, H, self.Wr, self.Wc, ws[1], scaling=1))
        timed("gemm_dense", lambda: self._g(self.Xr, self.Wr, out["Y"], ws[2]))
        timed("quant_dy", lambda: self._q(inp["dy"], T, F, F, self.Dr, self.Dc, ws[3], rounding=1,
                                          rht=1, mx_col=(self.mx_q, self.mx_e)))
        timed("gemm_dense", lambda: self._g(self.Dr, self.Wc, out["dX"], ws[4]))
        timed("gemm_dense", lambda: self._g(self.Dc, self.Xc, out["dW"], ws[5]))
        # MoE expert forward
        R = self.routed
        timed("quant_tok", lambda: self._q(inp["tok"], MOE_TOKENS, MOE_HIDDEN, MOE_HIDDEN, self.Tq,
                                           None, ws[6]))
        timed("dispatch", lambda: nv.nvfp4_gather_rows(
            self.Tq.q, self.Tq.sf, MOE_TOKENS, MOE_HIDDEN, self.row_token, R, self.offsets,
            EXPERTS, self.A_up.q, self.A_up.sf, ws[6], 256))
        qu, su, gu = self.wup
        timed("gemm_grouped", lambda: nv.nvfp4_grouped_gemm(
            EXPERTS, self.offsets, R, self.A_up.q, self.A_up.sf, self.A_up.g, qu, su, gu,
            MOE_FFN, MOE_HIDDEN, nv.NVFP4_OUT_BF16, self.Hup, self.h_amax, ws[7], 256))
        timed("quant_h", lambda: self._q(self.Hup, R, MOE_FFN, MOE_FFN, self.A_dn, None,
                                         ws[6], groups=True, amax=self.h_amax))
        qd, sd, gd = self.wdn
        timed("gemm_grouped", lambda: nv.nvfp4_grouped_gemm(
            EXPERTS, self.offsets, R, self.A_dn.q, self.A_dn.sf, self.A_dn.g, qd, sd, gd,
            MOE_HIDDEN, MOE_FFN, nv.NVFP4_OUT_BF16, out["Out"], None, ws[7], 256))

    # dense: 3 quantise calls x (amax + fused pass) + 3 GEMMs; MoE: token quantise (amax +
    # fused pass), dispatch, 2 grouped GEMMs, H quantise (fused pass only: amax from the GEMM)
    LAUNCHES_PER_STEP = 15

    def flops(self):
        return DENSE_FLOP + 2 * 2 * self.routed * MOE_FFN * MOE_HIDDEN

    def _outputs(self, slot=0):
        o = self.outs[slot]
        return [o["Y"], o["dX"], o["dW"], o["Out"]]

    def results_d2h(self, host_bufs, slot=0):
        """Copy every output of the step in output slot `slot` in full (Y, dX, dW and the
        MoE output, 1.58 GB of bf16) into pinned host buffers, asynchronously on the
        current stream; returns the bytes copied."""
        outs = self._outputs(slot)
        for h, o in zip(host_bufs, outs):
            h.copy_(o, non_blocking=True)
        return sum(o.numel() * o.element_size() for o in outs)

    def result_host_buffers(self):
        return [self.torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in self._outputs()]

    def check_status(self):
        for w in self.ws:
            s = self.nv.nvfp4_workspace_status(w)
            if s != 0:
                raise RuntimeError(f"device status {self.nv.status_string(s)}")


# The tensor pipe's own FP4 rate as ncu reports it (sm__ops_path_tensor_op_utcomma
# _src_fp4_dst_fp32: 32768 FLOP per SM per cycle, dense).  The GEMMs' roofline uses
# it at the sampled clock: 4 x the measured bf16 rate (the nominal fp4/bf16 ratio)
# is lower than what a library FP4 GEMM reaches on these shapes, so it would
# flatter the kernel.
HW_FP4_FLOP_PER_SM_CYCLE = 32768
NUM_SMS = 148


def hw_fp4_peak(clocks):
    """Dense FP4 tensor rate (TFLOP/s) at the median SM clock sampled during the timed
    region (the maximum clock when no sample was taken), and the clock used."""
    c = clocks or {}
    mhz = c.get("sm_mhz") or c.get("sm_max_mhz") or 1965
    return HW_FP4_FLOP_PER_SM_CYCLE * NUM_SMS * mhz * 1e6 / 1e12, mhz


# Measured on this machine: right after a loop of dense GEMMs, HBM-bound kernels can run
# about 20% slower for several milliseconds (the MXFP8 quantise and combine of the MoE
# output: 174 and 129 us against 142 and 108 us), and 250 ms of idle brings them back.
# The lines timed apart from the step start after such a pause, so that none inherits
# the state the GEMM loop before it left.
SETTLE_S = 0.25


def settle(torch):
    torch.cuda.synchronize()
    time.sleep(SETTLE_S)


def time_mxfp4(step, steps, warmup):
    """MXFP4 (OCP: 32-blocks, E8M0, E2M1) of the resident dY, both directions from one
    call, timed apart from the step: mean ms per launch over `steps` launches after
    `warmup`, CUDA events on the launching stream.  dY (671 MB) is larger than L2."""
    nv, torch = step.nv, step.torch
    settle(torch)
    dy = step.inputs[0]["dy"]
    R, C = dy.shape
    u8 = dict(dtype=torch.uint8, device=dy.device)
    qr, er = torch.empty((R, C // 2), **u8), torch.empty((R, C // 32), **u8)
    qc, ec = torch.empty((C, R // 2), **u8), torch.empty((C, R // 32), **u8)
    both = nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE
    run = lambda: nv.mxfp4_quantize(dy, R, C, dy.stride(0), both, qr, er, qc, ec)
    for _ in range(max(warmup, 3)):
        run()
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        run()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    n = R * C
    nbytes = 2 * n + 2 * (n // 2 + n // 32)  # one bf16 read, codes + scales both ways
    return ms, nbytes


def time_linear(step, steps, warmup):
    """The NVFP4 linear autograd op, forward + backward, on the dense layer's resident
    x [16384, 5120], W [20480, 5120] and dY [16384, 20480]: 9 launches of ours per pass
    (x, W and dY each amax + fused quantisation; the forward, dgrad and wgrad GEMMs),
    timed apart from the step with CUDA events.  Returns mean ms per pass."""
    torch = step.torch
    from nvfp4_bit_precision_b200.linear import nvfp4_linear
    inp = step.inputs[0]
    x = inp["x"].detach().requires_grad_(True)
    w = inp["w"].detach().requires_grad_(True)
    dy = inp["dy"]

    def run(i):
        x.grad = w.grad = None
        nvfp4_linear(x, w, seed=20251030, offset=i).backward(dy)

    for i in range(max(warmup, 3)):
        run(i)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(steps):
        run(i)
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


class L2Flush:
    """Reads a 256 MB buffer (twice the 126 MB L2) between timed launches, so every
    timed launch starts with its inputs out of L2.  A read leaves no dirty lines
    behind for the timed kernel to write back."""

    def __init__(self, dev):
        import torch
        self.buf = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.sum()


def time_each(fn, reps, warmup, flush):
    """Mean device time (ms) of fn() over `reps` launches, each bracketed by its own
    CUDA events on the current stream, with an L2 flush before each (not timed)."""
    import torch
    for _ in range(max(warmup, 3)):
        flush()
        fn()
    stream = torch.cuda.current_stream()
    evs = []
    for _ in range(reps):
        flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        evs.append((s, e))
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in evs) / reps


def time_configs(dev, reps, warmup, pk, fp4_peak):
    """The three smaller workloads, each timed on its own with an L2 flush before
    every launch: (1) the tiny NVFP4 linear (latency of its two quantisations and
    GEMM), (2) the fused gradient quantisation of an 8192 x 8192 Student-t tensor,
    (3) 2D weight quantisation, activation quantisation and the 8192x4096x4096 GEMM."""
    import torch
    import nvfp4_bit_precision_b200 as nv
    settle(torch)
    flush = L2Flush(dev)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(
        torch.bfloat16)
    u8 = dict(dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    sfm = nv.nvfp4_sf_mma_bytes
    mk = lambda r, k: nv.NVFP4Tensor(torch.empty((r, k // 2), **u8), torch.zeros(sfm(r, k), **u8),
                                     torch.empty(1, **f32), r, k, nv.NVFP4_SF_MMA)
    ws = [torch.zeros(256, **u8) for _ in range(4)]
    out = {}

    def q(x, rows, cols, r, c, w, **kw):
        p = nv.QuantParams()
        p.sf_layout = nv.NVFP4_SF_MMA
        p.rounding, p.scaling, p.rht_colwise = (kw.get("rounding", 0), kw.get("scaling", 0),
                                                kw.get("rht", 0))
        p.outputs = (nv.NVFP4_ROWWISE if r else 0) | (nv.NVFP4_COLWISE if c else 0)
        p.seed = 20251030
        if "mx_col" in kw:
            p.mx_outputs = nv.NVFP4_COLWISE
            p.mx_q_col, p.mx_sf_col = kw["mx_col"][0].data_ptr(), kw["mx_col"][1].data_ptr()
        nv.nvfp4_quantize(x, rows, cols, cols, p, r.q if r else None, r.sf if r else None,
                          r.g if r else None, c.q if c else None, c.sf if c else None,
                          c.g if c else None, w, 256)

    # (1) tiny linear: X 128x256, W 128x256, Y = X W^T in FP32
    x1, w1 = W.tiny_linear(0)
    x1d, w1d = bf(x1), bf(w1)
    X1, W1 = mk(128, 256), mk(128, 256)
    Y1 = torch.empty((128, 128), **f32)

    def tiny():
        q(x1d, 128, 256, X1, None, ws[0])
        q(w1d, 128, 256, W1, None, ws[1])
        nv.nvfp4_gemm(X1.q, X1.sf, X1.g, W1.q, W1.sf, W1.g, 128, 128, 256, nv.NVFP4_OUT_F32,
                      Y1, 128, None, ws[2], 256)
    ms1 = time_each(tiny, reps, warmup, flush)
    out["tiny_linear"] = {
        "workload": "X 128x256 (1% entries x50), W 128x256; 1D RNE rowwise; GEMM 128x128x256 "
                    "FP32 out", "launches": 5, "latency_us": round(ms1 * 1e3, 2),
        "bound": "launch latency", "note": "two quantisations (amax + fused pass each) and "
                                           "the GEMM, cold L2"}

    # (2) fused gradient quantisation of G 8192x8192
    n2 = 8192
    g2 = bf(W.heavy_tailed(1, n2, n2, 1e-3))
    R2, C2 = mk(n2, n2), mk(n2, n2)
    mxq, mxe = torch.empty((n2, n2), **u8), torch.empty((n2, n2 // 32), **u8)
    ms2 = time_each(lambda: q(g2, n2, n2, R2, C2, ws[0], rounding=1, rht=1, mx_col=(mxq, mxe)),
                    reps, warmup, flush)
    e2 = n2 * n2
    b2 = 2 * 2 * e2 + 2 * (e2 // 2 + e2 // 16) + e2 + e2 // 32
    gbs2 = b2 / (ms2 / 1e3) / 1e9
    out["gradient_quantize"] = {
        "workload": "G 8192x8192 Student-t(3) x 1e-3; NVFP4 rowwise SR + columnwise RHT+SR + "
                    "MXFP8 columnwise", "us": round(ms2 * 1e3, 2), "algorithmic_bytes": b2,
        "bound": "hbm", "achieved": round(gbs2, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
        "frac": round(gbs2 / pk["hbm_gbs"], 4), "target_us_at_0.70": round(
            b2 / (0.7 * pk["hbm_gbs"] * 1e9) * 1e6, 1), "peak_note": f"of {pk['source']}"}

    # (3) weight 2D + outlier activations + GEMM 8192x4096x4096
    w3, x3, _ = W.weight_and_outlier_acts(2)
    w3d, x3d = bf(w3), bf(x3)
    W3r, W3c, X3 = mk(4096, 4096), mk(4096, 4096), mk(8192, 4096)
    Y3 = torch.empty((8192, 4096), dtype=torch.bfloat16, device=dev)
    msw = time_each(lambda: q(w3d, 4096, 4096, W3r, W3c, ws[0], scaling=1), reps, warmup, flush)
    msx = time_each(lambda: q(x3d, 8192, 4096, X3, None, ws[1]), reps, warmup, flush)
    msg = time_each(lambda: nv.nvfp4_gemm(X3.q, X3.sf, X3.g, W3r.q, W3r.sf, W3r.g, 8192, 4096,
                                          4096, nv.NVFP4_OUT_BF16, Y3, 4096, None, ws[2], 256),
                    reps, warmup, flush)
    fl3 = 2 * 8192 * 4096 * 4096
    tf3 = fl3 / (msg / 1e3) / 1e12
    bw = 2 * 2 * 4096 * 4096 + 2 * (4096 * 4096 // 2 + 4096 * 4096 // 16)
    bx = 2 * 2 * 8192 * 4096 + (8192 * 4096 // 2 + 8192 * 4096 // 16)
    out["weight2d_gemm"] = {
        "workload": "W 4096x4096 2D 16x16 both directions; X 8192x4096 (0.1% channels x100) 1D "
                    "RNE rowwise; GEMM 8192x4096x4096 bf16 out",
        "gemm_us": round(msg * 1e3, 2), "gemm_tflops": round(tf3, 1),
        "gemm_frac_of_4x_bf16_burst": round(tf3 / (4.0 * pk["bf16_tflops"]), 4),
        "gemm_frac_of_hw_fp4_peak": round(tf3 / fp4_peak, 4),
        "quant_w_us": round(msw * 1e3, 2),
        "quant_w_frac_of_hbm": round(bw / (msw / 1e3) / 1e9 / pk["hbm_gbs"], 4),
        "quant_x_us": round(msx * 1e3, 2),
        "quant_x_frac_of_hbm": round(bx / (msx / 1e3) / 1e9 / pk["hbm_gbs"], 4)}
    for w in ws:
        s = nv.nvfp4_workspace_status(w)
        if s != 0:
            raise RuntimeError(f"device status {nv.status_string(s)}")
    return out


def time_mxfp8_backward(step, steps, warmup, fp8_peak, hw_fp8_peak):
    """The backward GEMMs of the dense layer in MXFP8 (the recipe on the iitak page,
    "How it works": the backward pass in 8-bit MXFP8): dgrad dX = dY W (A = dY
    rowwise, B = W columnwise) and wgrad dW = dY^T X (A = dY columnwise, B = X
    columnwise), 16384 x 5120 x 20480 and 20480 x 5120 x 16384, on operands the
    quantiser writes with tiled E8M0 scales from the resident bf16 tensors.  Each
    GEMM launch and the dY quantisation (both directions, one pass) are timed apart
    from the step with CUDA events after warm-up; inputs are larger than L2."""
    nv, torch = step.nv, step.torch
    inp = step.inputs[0]
    T, H, F = TOKENS, HIDDEN, FFN
    dev = inp["dy"].device
    u8 = dict(dtype=torch.uint8, device=dev)
    mk = lambda r, k: (torch.empty((r, k), **u8), torch.zeros(nv.mxfp8_sf_mma_bytes(r, k), **u8))
    dyr, dyc, wc, xc = mk(T, F), mk(F, T), mk(H, F), mk(H, T)

    def mxq(x, rows, cols, row, col):
        p = nv.QuantParams()
        p.mx_outputs = (nv.NVFP4_ROWWISE if row else 0) | (nv.NVFP4_COLWISE if col else 0)
        p.mx_sf_layout = nv.NVFP4_SF_MMA
        if row:
            p.mx_q_row, p.mx_sf_row = row[0].data_ptr(), row[1].data_ptr()
        if col:
            p.mx_q_col, p.mx_sf_col = col[0].data_ptr(), col[1].data_ptr()
        nv.nvfp4_quantize(x, rows, cols, cols, p, None, None, None, None, None, None,
                          step.ws[0], 256)

    mxq(inp["w"], F, H, None, wc)
    mxq(inp["x"], T, H, None, xc)
    stream = torch.cuda.current_stream()
    runs = {"quant_dy": lambda: mxq(inp["dy"], T, F, dyr, dyc),
            "dgrad": lambda: nv.mxfp8_gemm(dyr[0], dyr[1], wc[0], wc[1], T, H, F,
                                           nv.NVFP4_OUT_BF16, step.dX, H, None, step.ws[4], 256),
            "wgrad": lambda: nv.mxfp8_gemm(dyc[0], dyc[1], xc[0], xc[1], F, H, T,
                                           nv.NVFP4_OUT_BF16, step.dW, H, None, step.ws[5], 256)}
    ms, mhz = {}, {}
    for name, fn in runs.items():
        for _ in range(max(warmup, 3)):
            fn()
        evs = []
        for _ in range(steps):
            s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s_.record(stream)
            fn()
            e_.record(stream)
            evs.append((s_, e_))
        torch.cuda.synchronize()
        ms[name] = sum(a.elapsed_time(b) for a, b in evs) / steps
        if name != "quant_dy":  # the last launch's own SM clock
            ws_i = step.ws[4] if name == "dgrad" else step.ws[5]
            mhz[name] = nv.nvfp4_gemm_cycles(ws_i) / (evs[-1][0].elapsed_time(evs[-1][1]) * 1e3)
    step.check_status()
    flop = 2 * T * H * F
    tf = {k: flop / (ms[k] / 1e3) / 1e12 for k in ("dgrad", "wgrad")}
    mean_tf = 2 * flop / ((ms["dgrad"] + ms["wgrad"]) / 1e3) / 1e12
    n = T * F
    qbytes = 2 * n + 2 * (n + n // 32)
    return {"kernel": "gemm_kernel<MXFP8> (tcgen05 kind::mxf8f6f4, UE8M0 block-32 scales): dgrad "
                      "16384x5120x20480 and wgrad 20480x5120x16384, bf16 out, timed apart from "
                      "the step", "bound": "tensor",
            "dgrad_us": round(ms["dgrad"] * 1e3, 1), "wgrad_us": round(ms["wgrad"] * 1e3, 1),
            "dgrad_tflops": round(tf["dgrad"], 1), "wgrad_tflops": round(tf["wgrad"], 1),
            "achieved": round(mean_tf, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
            "frac": round(mean_tf / fp8_peak, 4),
            "peak_note": "2 x the measured bf16 burst rate (nominal fp8/bf16 ratio)",
            "frac_of_hw_fp8_peak": round(mean_tf / hw_fp8_peak, 4),
            "hw_fp8_peak": round(hw_fp8_peak, 1),
            "hw_peak_note": "dense FP8 tensor rate of the chip (16384 FLOP per SM per cycle) at the "
                            "sampled SM clock",
            "sm_mhz_in_kernel": round((mhz["dgrad"] + mhz["wgrad"]) / 2, 1),
            "quant_dy_mxfp8_both_us": round(ms["quant_dy"] * 1e3, 1),
            "quant_dy_mxfp8_both_gbs": round(qbytes / (ms["quant_dy"] / 1e3) / 1e9, 1)}


def time_mxfp4_gemm(step, steps, warmup, fp4_peak, hw_fp4):
    """The dense layer's forward GEMM (16384 x 20480 x 5120) in MXFP4 (kind::mxf4, E8M0
    scales per 32) on the resident x and W quantised by mxfp4_quantize with tiled scales,
    timed apart from the step with CUDA events after warm-up; the OCP format the pages
    set NVFP4 against."""
    nv, torch = step.nv, step.torch
    inp = step.inputs[0]
    T, H, F = TOKENS, HIDDEN, FFN
    (qa, sa), _ = nv.mxfp4(inp["x"], nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
    (qb, sb), _ = nv.mxfp4(inp["w"], nv.NVFP4_ROWWISE, sf_layout=nv.NVFP4_SF_MMA)
    run = lambda: nv.mxfp4_gemm(qa, sa, qb, sb, T, F, H, nv.NVFP4_OUT_BF16, step.Y, F, None,
                                step.ws[2], 256)
    for _ in range(max(warmup, 3)):
        run()
    stream = torch.cuda.current_stream()
    evs = []
    for _ in range(steps):
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_.record(stream)
        run()
        e_.record(stream)
        evs.append((s_, e_))
    torch.cuda.synchronize()
    step.check_status()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    tf = DENSE_FLOP_PER_GEMM / (ms / 1e3) / 1e12
    mhz = nv.nvfp4_gemm_cycles(step.ws[2]) / (evs[-1][0].elapsed_time(evs[-1][1]) * 1e3)
    return {"kernel": "gemm_kernel<MXFP4> (tcgen05 kind::mxf4, UE8M0 block-32 scales), "
                      "16384x20480x5120, bf16 out, timed apart from the step", "bound": "tensor",
            "us": round(ms * 1e3, 1), "achieved": round(tf, 1), "peak": round(fp4_peak, 1),
            "unit": "TFLOP/s", "frac": round(tf / fp4_peak, 4),
            "peak_note": "4 x the measured bf16 burst rate (nominal fp4/bf16 ratio)",
            "frac_of_hw_fp4_peak": round(tf / hw_fp4, 4),
            "sm_mhz_in_kernel": round(mhz, 1)}


def time_moe_combine(step, steps, warmup, pk):
    """The MXFP8 return trip of the MoE expert outputs without the network: the down
    projection's output Out [65536, 4096] (rows in expert order) quantised to MXFP8
    rowwise, then each token's 4 rows combined with weights 1/4 into [16384, 4096] bf16
    (mxfp8_combine).  Timed apart from the step with CUDA events; on one GPU there is no
    all-to-all to time.  Link bytes: what an expert-parallel run would send per step."""
    nv, torch = step.nv, step.torch
    dev = step.Out.device
    R, H = step.Out.shape
    te = step.h["token_expert"]
    order = np.argsort(te.reshape(-1), kind="stable")
    pos = np.empty_like(order)
    pos[order] = np.arange(order.size)
    slot = torch.from_numpy(pos.reshape(te.shape).astype(np.int32)).to(dev)
    w = torch.full(te.shape, 1.0 / TOPK, dtype=torch.float32, device=dev)
    u8 = dict(dtype=torch.uint8, device=dev)
    q, e8 = torch.empty((R, H), **u8), torch.empty((R, H // 32), **u8)
    out = torch.empty((MOE_TOKENS, H), dtype=torch.bfloat16, device=dev)

    quant = lambda: nv.mxfp8_quantize(step.Out, R, H, H, nv.NVFP4_ROWWISE, 0, 0, 0, q, e8, None, None)
    comb = lambda: nv.mxfp8_combine(q, e8, R, H, slot, w, MOE_TOKENS, TOPK, out, step.ws[6], 256)

    settle(torch)
    for _ in range(max(warmup, 3)):
        quant()
        comb()
    stream = torch.cuda.current_stream()
    evs = []
    torch.cuda.synchronize()
    for _ in range(steps):
        ev3 = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev3[0].record(stream)
        quant()
        ev3[1].record(stream)
        comb()
        ev3[2].record(stream)
        evs.append(ev3)
    torch.cuda.synchronize()
    step.check_status()
    q_ms = sum(a.elapsed_time(b) for a, b, _ in evs) / steps
    c_ms = sum(b.elapsed_time(c) for _, b, c in evs) / steps
    ms = q_ms + c_ms
    nbytes = 2 * R * H + 2 * (R * H + R * H // 32) + MOE_TOKENS * H * 2
    return {"kernel": "mxfp8_quantize (rowwise) + mxfp8_combine_kernel on the MoE output "
                      "65536x4096 -> 16384x4096 bf16, top-4 weights 1/4", "bound": "hbm",
            "us": round(ms * 1e3, 1), "quantize_us": round(q_ms * 1e3, 1),
            "combine_us": round(c_ms * 1e3, 1), "algorithmic_bytes": nbytes,
            "achieved": round(nbytes / (ms / 1e3) / 1e9, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], 4),
            "link_bytes_mxfp8": R * H + R * H // 32, "link_bytes_bf16": 2 * R * H,
            "note": "one GPU: no all-to-all is timed; link bytes are what an expert-parallel "
                    "run would send back per step; timed after a 250 ms pause that follows the "
                    "GEMM lines"}


def quant_algorithmic_bytes():
    """Bytes the dY quantisation must move: two reads of the bf16 input (amax pass and
    quantise pass), NVFP4 codes and scales in both directions, MXFP8 codes and scales."""
    n = TOKENS * FFN
    return 2 * 2 * n + 2 * (n // 2 + n // 16) + n + n // 32


def host_inputs(seed_dense=4, seed_moe=3):
    d = W.dense_linear_layer(seed_dense, TOKENS, HIDDEN, FFN)
    rng = np.random.default_rng(seed_moe)
    tok = W.f32_to_bf16_bits(W.normal(rng, (MOE_TOKENS, MOE_HIDDEN)))
    token_expert, row_token, offsets = W.moe_routing(rng, MOE_TOKENS, EXPERTS, TOPK)
    w_up = W.f32_to_bf16_bits(W.normal(rng, (EXPERTS, MOE_FFN, MOE_HIDDEN), 0.02))
    w_down = W.f32_to_bf16_bits(W.normal(rng, (EXPERTS, MOE_HIDDEN, MOE_FFN), 0.02))
    return dict(x=d["x"], w=d["w"], dy=d["dy"], tok=tok, row_token=row_token, offsets=offsets,
                w_up=w_up, w_down=w_down, token_expert=token_expert)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms by NVML (read-only queries)
    on a host thread while the timed region runs; `nvidia-smi` starts too slowly for a
    region of a few hundred milliseconds."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80))

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self.handle = None
        self.nvml = None
        self.thread = None
        self.stop = None

    def _open(self):
        import pynvml as N
        N.nvmlInit()
        self.nvml = N
        try:
            import torch
            p = torch.cuda.get_device_properties(self.device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.handle = N.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            self.handle = N.nvmlDeviceGetHandleByIndex(int(getattr(self.device, "index", 0) or 0))
        self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.handle, N.NVML_CLOCK_SM)

    def _run(self):
        N = self.nvml
        get_reasons = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(N, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self.stop.is_set():
            try:
                mhz = N.nvmlDeviceGetClockInfo(self.handle, N.NVML_CLOCK_SM)
                bits = get_reasons(self.handle) if get_reasons else 0
                self.raw.append((time.perf_counter(), mhz, bits))
                self.first.set()
            except Exception:
                pass
            self.stop.wait(0.005)

    def __enter__(self):
        # NVML is opened and the thread has taken its first sample before the
        # timed region starts; only samples taken inside the region are kept.
        import threading
        try:
            self._open()
        except Exception:
            self.handle = None
            return self
        self.raw = []
        self.stop = threading.Event()
        self.first = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        self.first.wait(timeout=2.0)
        self.t_begin = time.perf_counter()
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            t_end = time.perf_counter()
            self.stop.set()
            self.thread.join(timeout=5)
            self.samples = [(m, b) for t, m, b in self.raw if self.t_begin <= t <= t_end]
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = set()
        for smp in self.samples:
            for name, attr, default in self.REASONS:
                if smp[1] & getattr(self.nvml, attr, default):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(smp[0] for smp in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml, 5 ms"}


# ----------------------------------------------------------------------------- CPU oracle
_SAMPLE_INPUTS = {}
GEMM_SAMPLE_N = 2048


def _sample_inputs():
    """Inputs of the oracle sample, built once per process (their set-up -- including
    quantising the 20480-row B operands of the GEMM pieces -- is not timed)."""
    if _SAMPLE_INPUTS:
        return _SAMPLE_INPUTS
    import oracle as orc
    rng = np.random.default_rng(7)
    am = (1.0, 1.0)
    d = _SAMPLE_INPUTS
    d["xs"] = W.f32_to_bf16_bits(W.normal(rng, (32, HIDDEN)))
    d["ws"] = W.f32_to_bf16_bits(W.normal(rng, (32, HIDDEN), 0.02))
    d["dys"] = W.f32_to_bf16_bits(W.student_t(rng, (32, FFN), 3.0))
    d["qa"] = orc.nvfp4_quantize(d["xs"], 0, amax=am)
    # 2048 of the FFN rows of W: the GEMM piece's time scales with the rows it spans
    d["qb"] = orc.nvfp4_quantize(W.f32_to_bf16_bits(W.normal(rng, (GEMM_SAMPLE_N, HIDDEN), 0.02)),
                                 0)
    d["acts"] = W.f32_to_bf16_bits(W.normal(rng, (32, MOE_HIDDEN)))
    d["hs"] = W.f32_to_bf16_bits(W.normal(rng, (32, MOE_FFN)))
    d["qa2"] = orc.nvfp4_quantize(d["acts"], 0, amax=am)
    d["qb2"] = orc.nvfp4_quantize(
        W.f32_to_bf16_bits(W.normal(rng, (MOE_FFN, MOE_HIDDEN), 0.02)), 0)
    return d


def oracle_sample():
    """Time the CPU oracle (one thread) on a bounded sample of the step and extrapolate
    to a full step.

    Sample: every quantisation on 32-row (token) slices of its operand, and the FP64
    GEMM reference on 2 output rows of each GEMM.  Each piece's time is scaled by
    (full size / sample size); value = step GEMM FLOP / extrapolated step time."""
    import oracle as orc
    d = _sample_inputs()
    t_full = 0.0
    pieces = []

    def tq(fn, work_scale):
        nonlocal t_full
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        t_full += dt * work_scale
        pieces.append(dt)

    am = (1.0, 1.0)
    xs, ws_, dys = d["xs"], d["ws"], d["dys"]
    tq(lambda: (orc.nvfp4_quantize(xs, 0, amax=am),
                orc.nvfp4_quantize(xs, 1, rht=1, amax=am)), TOKENS / 32)
    tq(lambda: (orc.nvfp4_quantize(ws_, 0, scaling=1, amax=am),
                orc.nvfp4_quantize(ws_, 1, scaling=1, amax=am)), FFN / 32)
    tq(lambda: (orc.nvfp4_quantize(dys, 0, rounding=1, amax=am),
                orc.nvfp4_quantize(dys, 1, rounding=1, rht=1, amax=am),
                orc.mxfp8_quantize(dys, 1)), TOKENS / 32)
    # GEMM reference: 2 rows of each dense GEMM (same cost for the three shapes' K*N)
    qa, sa, ga = d["qa"]
    qb, sb, gb = d["qb"]
    tq(lambda: orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[0, 1]),
       3 * TOKENS / 2 * FFN / GEMM_SAMPLE_N)
    routed = MOE_TOKENS * TOPK
    # the tokens are quantised once, then dispatched; the up output is requantised
    tq(lambda: orc.nvfp4_quantize(d["acts"], 0, amax=am), MOE_TOKENS / 32)
    tq(lambda: orc.nvfp4_quantize(d["hs"], 0, amax=am), routed / 32)
    # grouped GEMMs: per routed row the work equals one dense row of N x K
    qa2, sa2, ga2 = d["qa2"]
    qb2, sb2, gb2 = d["qb2"]
    tq(lambda: orc.nvfp4_gemm_rows(qa2, sa2, ga2, qb2, sb2, gb2, rows_sel=[0, 1]),
       2 * routed / 2)
    flops = DENSE_FLOP + 2 * 2 * routed * MOE_FFN * MOE_HIDDEN
    return {"value": flops / t_full / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": ("each quantisation on 32-row slices, each GEMM on 2 output rows (the dense "
                       "GEMMs over 2048 of their output columns); per-piece time scaled to the "
                       "full step"),
            "sample_seconds": round(sum(pieces), 2), "extrapolated_step_s": round(t_full, 1)}


def _worker_warm(_):
    _sample_inputs()
    return os.getpid()


def _worker_sample(_):
    return oracle_sample()["sample_seconds"]


def oracle_baseline():
    """The oracle on one host core (oracle_sample) and on all of them: one spawned
    worker per core, each building its inputs first (not timed), then every worker
    runs the same sample at once; the wall time of that round gives the all-core
    rate (workers x the sample's share of a step / wall time).  The oracle itself is
    single-threaded C; the all-core figure is its rate with the step's independent
    pieces spread over the cores."""
    import concurrent.futures as cf
    import multiprocessing as mp
    one = oracle_sample()
    one = oracle_sample()  # second run: inputs built, caches warm
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    out = dict(one)
    out["single_core"] = {"value": one["value"], "cores": 1,
                          "sample_seconds": one["sample_seconds"]}
    try:
        with cf.ProcessPoolExecutor(max_workers=cores, mp_context=mp.get_context("spawn")) as ex:
            list(ex.map(_worker_warm, range(cores)))
            t0 = time.perf_counter()
            secs = list(ex.map(_worker_sample, range(cores)))
            wall = time.perf_counter() - t0
        # each worker did one sample's worth of work (one["sample_seconds"] on one core)
        out["value"] = one["value"] * cores * one["sample_seconds"] / wall
        out["cores"] = cores
        out["all_core_wall_s"] = round(wall, 2)
        out["worker_sample_seconds_median"] = round(statistics.median(secs), 2)
        out["sample"] = (f"{cores} workers at once, each timing the one-core sample (each "
                         "quantisation on 32-row slices, each GEMM on 2 output rows); rate = "
                         "workers x sample share of a step / wall time")
    except Exception as e:  # no process pool on this host: report the one-core figure
        out["all_core_error"] = str(e)[:200]
    return out


def grouped_roofline(times, steps, step, pk, fp4_peak):
    """The two grouped GEMMs of the MoE forward (launches alternate up, down) against
    their roofline: per launch max(FLOP / FP4 peak, algorithmic bytes / HBM), the bytes
    being A codes and scales, every expert's B codes and scales, and the bf16 output."""
    R = step.routed
    out = {}
    tot_ms = tot_roof = 0.0
    for name, (N, K), ts in (("up", (MOE_FFN, MOE_HIDDEN), times[0::2]),
                             ("down", (MOE_HIDDEN, MOE_FFN), times[1::2])):
        ms = sum(ts) / len(ts)
        flop = 2 * R * N * K
        nbytes = R * K // 2 + R * K // 16 + EXPERTS * N * (K // 2 + K // 16) + 2 * R * N
        roof_ms = max(flop / (fp4_peak * 1e12), nbytes / (pk["hbm_gbs"] * 1e9)) * 1e3
        out[name] = {"us": round(ms * 1e3, 1), "roofline_us": round(roof_ms * 1e3, 1),
                     "tflops": round(flop / (ms / 1e3) / 1e12, 1), "algorithmic_bytes": nbytes,
                     "frac": round(roof_ms / ms, 4)}
        tot_ms += ms
        tot_roof += roof_ms
    out["frac"] = round(tot_roof / tot_ms, 4)
    out["note"] = ("roofline time / measured time, up and down together; FP4 peak as in "
                   "`roofline`, HBM of " + pk["source"])
    return out


def bench_config(world):
    """The workload's `config`, the same on both arms.  Every token is routed to
    TOPK experts, so the routed row count is fixed."""
    return {"workload": WORKLOAD, "tokens": TOKENS, "hidden": HIDDEN, "ffn": FFN,
            "moe": {"experts": EXPERTS, "hidden": MOE_HIDDEN, "ffn": MOE_FFN,
                    "tokens": MOE_TOKENS, "top_k": TOPK, "routed_rows": MOE_TOKENS * TOPK},
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (dY 671 MB, X 168 MB, W 210 MB > 126 MB)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    vals = []
    for _ in range(args.warmup):
        oracle_sample()
    for _ in range(args.steps):
        vals.append(oracle_sample()["value"])
    info = oracle_sample()
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(world),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": info["cores"],
                             "kind": "oracle", "sample": info["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(times, world, device=None):
    """Max of each timing over all ranks (the slowest replica sets the job time)."""
    if world <= 1:
        return [float(t) for t in times]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in times], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_tflops(flops_per_step, world, steps, ms):
    """Whole-job throughput: every replica's GEMM FLOP over the slowest replica's time."""
    return flops_per_step * world * steps / (ms / 1e3) / 1e12


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    h = host_inputs()
    pinned = {k: torch.from_numpy(h[k].view(np.int16)).pin_memory()
              for k in ("x", "w", "dy", "tok")}
    h["pinned"] = pinned
    step = Step(dev, h)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        step.run()
    torch.cuda.synchronize()
    step.check_status()

    # ---------------- device-timed region
    ev = {}
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step.run(ev)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1)
    step.check_status()
    clocks = clk.summary()
    per_kernel = {k: [s.elapsed_time(e) for s, e in v] for k, v in ev.items()}
    # The SM clock the dense GEMMs of the last timed step ran at: each call's own
    # cycle count (longest CTA, entry to exit) over its CUDA-event time.  The event
    # also spans the launch gap, so this slightly underestimates the clock.
    kernel_mhz = [step.nv.nvfp4_gemm_cycles(step.ws[i]) / (s.elapsed_time(e) * 1e3)
                  for i, (s, e) in zip((2, 4, 5), ev["gemm_dense"][-3:])]
    kernel_mhz = sum(kernel_mhz) / len(kernel_mhz)

    # ---------------- end to end: pinned host inputs -> device, results -> host
    barrier()
    torch.cuda.synchronize()
    # Step i+1's inputs are copied in (from pinned host memory, on a copy stream) and
    # step i-1's results are read back (into pinned host memory, on a second copy
    # stream) while step i computes; every step copies its own inputs in and all of
    # its results out.  Inputs and outputs have two slots each.
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    copy_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    landed = [torch.cuda.Event(), torch.cuda.Event()]    # slot's inputs copied in
    consumed = [torch.cuda.Event(), torch.cuda.Event()]   # slot's step done (inputs free)
    read_back = [torch.cuda.Event(), torch.cuda.Event()]  # slot's outputs copied out
    host_out = [step.result_host_buffers() for _ in range(2)]
    e0.record(stream)
    copy_stream.wait_event(e0)
    with torch.cuda.stream(copy_stream):
        step.upload_inputs(0, non_blocking=True)
    landed[0].record(copy_stream)
    d2h = 0
    for i in range(args.steps):
        slot = i % 2
        if i + 1 < args.steps:
            nxt = 1 - slot
            if i >= 1:
                copy_stream.wait_event(consumed[nxt])
            with torch.cuda.stream(copy_stream):
                step.upload_inputs(nxt, non_blocking=True)
            landed[nxt].record(copy_stream)
        stream.wait_event(landed[slot])
        if i >= 2:
            stream.wait_event(read_back[slot])  # step i-2's results are out of this slot
        step.run(slot=slot)
        consumed[slot].record(stream)
        d2h_stream.wait_event(consumed[slot])
        with torch.cuda.stream(d2h_stream):
            d2h = step.results_d2h(host_out[slot], slot)
        read_back[slot].record(d2h_stream)
    stream.wait_stream(d2h_stream)
    stream.wait_stream(copy_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    if args.steps >= 2:
        # Both slots computed the same inputs (a fixed seed): their read-back results
        # must agree bit for bit, or the overlap of copies and kernels raced.
        for a_, b_ in zip(host_out[0], host_out[1]):
            if not torch.equal(a_, b_):
                raise RuntimeError("end-to-end results differ between the two slots")
    ms_e2e = e0.elapsed_time(e1)

    mx4_ms, mx4_bytes = time_mxfp4(step, args.steps, args.warmup)
    lin_ms = time_linear(step, args.steps, args.warmup)
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)
    value = job_tflops(step.flops(), world, args.steps, ms)
    value_e2e = job_tflops(step.flops(), world, args.steps, ms_e2e)
    pk = peaks()
    fp4_peak, fp4_mhz = hw_fp4_peak(clocks)
    derived_peak = 4.0 * pk["bf16_tflops"]
    cfgs = time_configs(dev, max(args.steps, 10), args.warmup, pk, fp4_peak)
    mx8 = time_mxfp8_backward(step, args.steps, args.warmup, derived_peak / 2, fp4_peak / 2)
    mx4g = time_mxfp4_gemm(step, args.steps, args.warmup, derived_peak, fp4_peak)
    comb = time_moe_combine(step, args.steps, args.warmup, pk)
    gd = per_kernel["gemm_dense"]
    gemm_ms = sum(gd) / len(gd)
    gemm_tflops = DENSE_FLOP_PER_GEMM / (gemm_ms / 1e3) / 1e12
    qd = per_kernel["quant_dy"]
    qdy_ms = sum(qd) / len(qd)
    qbytes = quant_algorithmic_bytes()
    qgbs = qbytes / (qdy_ms / 1e3) / 1e9
    breakdown = {k: round(sum(v) / args.steps, 4) for k, v in per_kernel.items()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp4",
            "data": "synthetic (seeded numpy: N(0,1) activations, N(0,0.02) weights, "
                    "Student-t df=3 gradients, Zipf(1.1) top-4 routing)",
            "config": bench_config(world),
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel (dense NVFP4 GEMM, "
                         "16384x20480x5120 class, mean of fwd/dgrad/wgrad launches)",
                         "achieved": round(gemm_tflops, 1), "peak": round(derived_peak, 1),
                         "unit": "TFLOP/s", "frac": round(gemm_tflops / derived_peak, 4),
                         "traffic": TRAFFIC_BYTES["gemm_dense_fwd"],
                         "traffic_note": "bytes per launch of the forward GEMM 16384x20480x5120 "
                                         "(ncu capture); algorithmic operand bytes 104 MB + "
                                         "output 671 MB",
                         "peak_note": f"4 x {pk['bf16_tflops']} TFLOP/s burst bf16 of "
                                      f"{pk['source']} (the nominal fp4/bf16 ratio; the step is "
                                      f"milliseconds long, so the burst figure)",
                         "frac_of_hw_fp4_peak": round(gemm_tflops / fp4_peak, 4),
                         "hw_fp4_peak": round(fp4_peak, 1),
                         "hw_fp4_peak_note": f"dense FP4 tensor rate of the chip (ncu: 32768 FLOP "
                                             f"per SM per cycle, 148 SMs) at the median SM clock "
                                             f"NVML reported in the timed region, {fp4_mhz} MHz; "
                                             f"the 4 x bf16 figure lies below what the kernel and "
                                             f"a library FP4 GEMM reach, so this is the stricter "
                                             f"fraction",
                         "sm_mhz_in_kernel": round(kernel_mhz, 1),
                         "frac_at_kernel_clock": round(gemm_tflops / hw_fp4_peak(
                             {"sm_mhz": kernel_mhz})[0], 4),
                         "kernel_clock_note": "the chip's FP4 rate at the SM clock counted inside "
                                              "the GEMM (clock64 of the longest CTA, "
                                              "nvfp4_gemm_cycles) over its CUDA-event time, mean of "
                                              "the last step's three launches: the clock the power "
                                              "limit holds the kernel at, which the NVML reading in "
                                              "`clocks` does not show"},
            "quantize_roofline": {"bound": "hbm", "kernel": "amax_kernel + quant_kernel on dY "
                                  "16384x20480 (row SR, col RHT+SR, MXFP8 col)",
                                  "achieved": round(qgbs, 1), "peak": pk["hbm_gbs"],
                                  "unit": "GB/s", "frac": round(qgbs / pk["hbm_gbs"], 4),
                                  "algorithmic_bytes": qbytes,
                                  "traffic": TRAFFIC_BYTES["quant_dy"],
                                  "traffic_note": "amax + fused pass, DRAM bytes of one ncu capture",
                                  "peak_note": f"of {pk['source']}"},
            "breakdown_ms_per_step": breakdown,
            "grouped_gemm_roofline": grouped_roofline(per_kernel["gemm_grouped"], args.steps,
                                                      step, pk, fp4_peak),
            "configs": cfgs,
            "next_rows": {"mxfp8_backward_gemm": mx8, "mxfp4_gemm": mx4g,
                          "moe_combine_mxfp8": comb, "mxfp4_quantize": {
                "bound": "hbm", "kernel": "mxfp4_kernel on dY 16384x20480, both directions "
                "(timed apart from the step)", "ms": round(mx4_ms, 4),
                "achieved": round(mx4_bytes / (mx4_ms / 1e3) / 1e9, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(mx4_bytes / (mx4_ms / 1e3) / 1e9 / pk["hbm_gbs"], 4),
                "algorithmic_bytes": mx4_bytes, "peak_note": f"of {pk['source']}"},
                "nvfp4_linear": {
                    "kernel": "NVFP4LinearFunction forward + backward on the dense layer "
                    "(x 16384x5120, W 20480x5120, dY 16384x20480; 9 launches per pass; timed "
                    "apart from the step)", "ms": round(lin_ms, 4),
                    "value": round(3 * DENSE_FLOP_PER_GEMM / (lin_ms / 1e3) / 1e12, 1),
                    "unit": "TFLOP/s"}},
            "e2e": {"value": round(value_e2e, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(ms_e2e / args.steps, 3),
                    "note": "every step copies all its bf16 inputs in from pinned host memory "
                            "and all its bf16 outputs out in full; copies in, kernels and "
                            "copies out of consecutive steps overlap on three streams (two "
                            "input and two output slots): PCIe bounds it"},
            "gpu_launches": Step.LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
