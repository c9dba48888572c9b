"""Helpers for the GPU parity tests: uploads, layout conversions written from the
published 128x4 scale-atom description, and tolerance checks."""
import numpy as np

import workloads as W


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def to_dev(a_bf16_bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a_bf16_bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16)


def host(t) -> np.ndarray:
    """Device tensor -> numpy; bf16 comes back as its uint16 bit patterns."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.detach().cpu().numpy()


def sf_mma_to_rowmajor(sf_flat: np.ndarray, rows: int, k: int, padded_rows=None) -> np.ndarray:
    """Tiled scale bytes -> [rows, k/16].  Byte (r, b) sits at
    ((r//128) * (k/64) + b//4) * 512 + (r%32) * 16 + ((r%128)//32) * 4 + b%4,
    with r replaced by its padded row when a grouped layout is used."""
    k16 = k // 16
    r = np.arange(rows)[:, None] if padded_rows is None else np.asarray(padded_rows)[:, None]
    b = np.arange(k16)[None, :]
    off = ((r // 128) * (k16 // 4) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    return np.asarray(sf_flat).reshape(-1)[off]


def grouped_padded_rows(offsets: np.ndarray) -> np.ndarray:
    """Padded scale row of every output row for a grouped (MoE) layout."""
    rows = []
    pad = 0
    for e in range(len(offsets) - 1):
        cnt = offsets[e + 1] - offsets[e]
        rows.extend(range(pad, pad + cnt))
        pad += ((cnt + 127) // 128) * 128
    return np.array(rows, dtype=np.int64)


def check_gemm(D_gpu: np.ndarray, D_ref: np.ndarray, A_ref: np.ndarray, bf16_out: bool):
    """|D - D_ref| <= 1e-3 * sum_k |a_hat||b_hat| (+ half a bf16 ulp of D_ref for bf16 output).
    Returns the largest error normalised by the bound."""
    D_gpu = D_gpu.astype(np.float64)
    bound = 1e-3 * A_ref
    if bf16_out:
        bound = bound + np.abs(D_ref) * 2.0 ** -8 + 1e-30
    err = np.abs(D_gpu - D_ref)
    worst = float(np.max(err / np.maximum(bound, 1e-300)))
    assert np.all(err <= bound), f"GEMM error above tolerance: worst err/bound = {worst}"
    return worst


def bf16_bits_of_f32(a: np.ndarray) -> np.ndarray:
    return W.f32_to_bf16_bits(a)


def rowmajor_to_sf_mma(sf: np.ndarray, rows: int, k: int, padded_rows=None, total_padded=None):
    """[rows, k/16] scale bytes -> tiled layout (inverse of sf_mma_to_rowmajor)."""
    k16 = k // 16
    r = np.arange(rows)[:, None] if padded_rows is None else np.asarray(padded_rows)[:, None]
    b = np.arange(k16)[None, :]
    off = ((r // 128) * (k16 // 4) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    prow = (int(r.max()) // 128 + 1) * 128 if total_padded is None else total_padded
    out = np.zeros(prow * k16, dtype=np.uint8)
    out[off.reshape(-1)] = np.asarray(sf).reshape(-1)
    return out


def nvfp4_operand(nv, q, sf, g, rows, k, padded_rows=None, total_padded=None):
    """Device NVFP4Tensor built from oracle-side codes/scales (tiled scale layout)."""
    import torch
    sfm = rowmajor_to_sf_mma(sf, rows, k, padded_rows, total_padded)
    return nv.NVFP4Tensor(torch.from_numpy(np.ascontiguousarray(q)).cuda(),
                          torch.from_numpy(sfm).cuda(),
                          torch.tensor([g], dtype=torch.float32, device="cuda"), rows, k,
                          nv.NVFP4_SF_MMA)
