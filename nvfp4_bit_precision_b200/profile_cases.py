"""Single-case drivers for profiling one kernel launch under ncu.

    python -m nvfp4_bit_precision_b200.profile_cases gemm M N K [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases mxfp8-gemm M N K [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases grouped-gemm N K [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases quant-grad ROWS COLS [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases quant-act ROWS COLS [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases quant-weight ROWS COLS [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases mxfp4 ROWS COLS [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases dispatch TOKENS HIDDEN [--warm W]
    python -m nvfp4_bit_precision_b200.profile_cases combine TOKENS HIDDEN [--warm W]

Each runs W untimed launches of the case, then one more, on synthetic operands
(codes and in-range scale bytes drawn on the device; bf16 inputs ~N(0, 1e-3)),
and exits 0 when the device status word is clear.  Pair with `ncu -s W -c 1`.
"""
from __future__ import annotations

import argparse
import sys


def _gemm(nv, torch, M, N, K, warm):
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    u8 = dict(dtype=torch.uint8, device=dev)
    qa = torch.randint(0, 256, (M, K // 2), generator=g, **u8)
    qb = torch.randint(0, 256, (N, K // 2), generator=g, **u8)
    sa = torch.randint(0x30, 0x40, (nv.nvfp4_sf_mma_bytes(M, K),), generator=g, **u8)
    sb = torch.randint(0x30, 0x40, (nv.nvfp4_sf_mma_bytes(N, K),), generator=g, **u8)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, **u8)
    for _ in range(warm + 1):
        nv.nvfp4_gemm(qa, sa, one, qb, sb, one, M, N, K, nv.NVFP4_OUT_BF16, D, N, None, ws, 256)
    return ws


def _mxfp8_gemm(nv, torch, M, N, K, warm):
    """MXFP8 GEMM on random E4M3 codes (NaN codes 0x7F/0xFF mapped to 0) and E8M0
    scale bytes near 127."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    u8 = dict(dtype=torch.uint8, device=dev)
    qa = torch.randint(0, 256, (M, K), generator=g, **u8)
    qb = torch.randint(0, 256, (N, K), generator=g, **u8)
    for q in (qa, qb):
        q[(q & 0x7F) == 0x7F] = 0
    sa = torch.randint(120, 134, (nv.mxfp8_sf_mma_bytes(M, K),), generator=g, **u8)
    sb = torch.randint(120, 134, (nv.mxfp8_sf_mma_bytes(N, K),), generator=g, **u8)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, **u8)
    for _ in range(warm + 1):
        nv.mxfp8_gemm(qa, sa, qb, sb, M, N, K, nv.NVFP4_OUT_BF16, D, N, None, ws, 256)
    return ws


def _grouped(nv, torch, N, K, warm):
    import numpy as np

    import workloads as W
    dev = torch.device("cuda")
    rng = np.random.default_rng(3)
    _, _, offsets = W.moe_routing(rng, 16384, 64, 4)
    R, G = int(offsets[-1]), 64
    u8 = dict(dtype=torch.uint8, device=dev)
    qa = torch.randint(0, 256, (R, K // 2), **u8)
    sa = torch.randint(0x30, 0x40, (nv.nvfp4_sf_mma_grouped_bytes(R, G, K),), **u8)
    qb = torch.randint(0, 256, (G, N, K // 2), **u8)
    sb = torch.randint(0x30, 0x40, (G * nv.nvfp4_sf_mma_bytes(N, K),), **u8)
    ga = torch.ones(1, dtype=torch.float32, device=dev)
    gb = torch.ones(G, dtype=torch.float32, device=dev)
    off = torch.from_numpy(offsets.astype(np.int32)).to(dev)
    D = torch.empty((R, N), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, **u8)
    for _ in range(warm + 1):
        nv.nvfp4_grouped_gemm(G, off, R, qa, sa, ga, qb, sb, gb, N, K, nv.NVFP4_OUT_BF16, D, None,
                              ws, 256)
    return ws


def _quant_grad(nv, torch, rows, cols, warm):
    """The gradient recipe: rowwise SR, columnwise Hadamard + SR, MXFP8 columnwise."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    x = (torch.randn((rows, cols), generator=g, device=dev) * 1e-3).to(torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    for _ in range(warm + 1):
        nv.quantize(x, rowwise=True, colwise=True, rounding=nv.NVFP4_SR, rht=True, seed=5,
                    mx_outputs=nv.NVFP4_COLWISE, sf_layout=nv.NVFP4_SF_MMA, workspace=ws)
    return ws


def _quant_act(nv, torch, rows, cols, warm):
    """The activation recipe: rowwise and columnwise Hadamard, both RNE."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    x = torch.randn((rows, cols), generator=g, device=dev).to(torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    for _ in range(warm + 1):
        nv.quantize(x, rowwise=True, colwise=True, rht=True, sf_layout=nv.NVFP4_SF_MMA, workspace=ws)
    return ws


def _quant_weight(nv, torch, rows, cols, warm):
    """The weight recipe: 16x16 2D scales, both directions, RNE."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(4)
    x = (torch.randn((rows, cols), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    for _ in range(warm + 1):
        nv.quantize(x, rowwise=True, colwise=True, scaling=nv.NVFP4_2D16x16, sf_layout=nv.NVFP4_SF_MMA,
                    workspace=ws)
    return ws


def _mxfp4(nv, torch, rows, cols, warm):
    """MXFP4 of a bf16 ~N(0, 1) tensor, both directions."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(2)
    x = torch.randn((rows, cols), generator=g, device=dev).to(torch.bfloat16)
    for _ in range(warm + 1):
        nv.mxfp4(x, nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE)
    return None


def _dispatch(nv, torch, tokens, hidden, warm):
    """MoE dispatch of quantised token rows (top-4 Zipf(1.1) routing over 64 experts)
    into the grouped layout."""
    import numpy as np

    import workloads as W
    dev = torch.device("cuda")
    _, row_token, offsets = W.moe_routing(np.random.default_rng(3), tokens, 64, 4)
    R = int(offsets[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    x = torch.randn((tokens, hidden), generator=g, device=dev).to(torch.bfloat16)
    t = nv.quantize(x, sf_layout=nv.NVFP4_SF_MMA)["row"]
    u8 = dict(dtype=torch.uint8, device=dev)
    qd = torch.empty((R, hidden // 2), **u8)
    sd = torch.zeros(nv.nvfp4_sf_mma_grouped_bytes(R, 64, hidden), **u8)
    rt = torch.from_numpy(row_token.astype(np.int32)).to(dev)
    off = torch.from_numpy(offsets.astype(np.int32)).to(dev)
    ws = torch.zeros(256, **u8)
    for _ in range(warm + 1):
        nv.nvfp4_gather_rows(t.q, t.sf, tokens, hidden, rt, R, off, 64, qd, sd, ws, 256)
    return ws


def _combine(nv, torch, tokens, hidden, warm):
    """MXFP8 combine of top-4 expert rows (in expert order) into tokens x hidden bf16."""
    import numpy as np
    dev = torch.device("cuda")
    R, k = 4 * tokens, 4
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    out_rows = torch.randn((R, hidden), generator=g, device=dev).to(torch.bfloat16)
    u8 = dict(dtype=torch.uint8, device=dev)
    q, e8 = torch.empty((R, hidden), **u8), torch.empty((R, hidden // 32), **u8)
    nv.mxfp8_quantize(out_rows, R, hidden, hidden, nv.NVFP4_ROWWISE, 0, 0, 0, q, e8, None, None)
    slot = torch.from_numpy(np.random.default_rng(7).permutation(R).reshape(tokens, k).astype(np.int32)).to(dev)
    w = torch.full((tokens, k), 1.0 / k, dtype=torch.float32, device=dev)
    out = torch.empty((tokens, hidden), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, **u8)
    for _ in range(warm + 1):
        nv.mxfp8_combine(q, e8, R, hidden, slot, w, tokens, k, out, ws, 256)
    return ws


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["gemm", "mxfp8-gemm", "grouped-gemm", "quant-grad", "quant-act",
                                         "quant-weight", "mxfp4", "dispatch", "combine"])
    ap.add_argument("dims", type=int, nargs="+")
    ap.add_argument("--warm", type=int, default=3)
    args = ap.parse_args(argv)
    import torch

    import nvfp4_bit_precision_b200 as nv
    if args.case == "gemm":
        ws = _gemm(nv, torch, *args.dims[:3], args.warm)
    elif args.case == "mxfp8-gemm":
        ws = _mxfp8_gemm(nv, torch, *args.dims[:3], args.warm)
    elif args.case == "grouped-gemm":
        ws = _grouped(nv, torch, *args.dims[:2], args.warm)
    elif args.case == "quant-grad":
        ws = _quant_grad(nv, torch, *args.dims[:2], args.warm)
    elif args.case == "quant-act":
        ws = _quant_act(nv, torch, *args.dims[:2], args.warm)
    elif args.case == "quant-weight":
        ws = _quant_weight(nv, torch, *args.dims[:2], args.warm)
    elif args.case == "dispatch":
        ws = _dispatch(nv, torch, *args.dims[:2], args.warm)
    elif args.case == "combine":
        ws = _combine(nv, torch, *args.dims[:2], args.warm)
    else:
        ws = _mxfp4(nv, torch, *args.dims[:2], args.warm)
    torch.cuda.synchronize()
    status = nv.nvfp4_workspace_status(ws) if ws is not None else 0
    print(f"{args.case} {args.dims}: status {nv.status_string(status)}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
