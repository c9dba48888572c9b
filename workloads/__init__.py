"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no quantisation arithmetic: it only draws random numbers
(NumPy PCG64), rounds them to bf16 bit patterns and builds MoE routing.  Both
the CPU oracle and the CUDA path consume exactly these arrays.

Stand-ins: the pages train a 12B hybrid Mamba-Transformer on 10T tokens and an
MoE model (Inkling 2 Small); neither dataset nor weights exist here, so these
generators reproduce the shapes and value distributions instead.
"""
from __future__ import annotations

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def student_t(rng: np.random.Generator, shape, df: float = 3.0, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_t(df, size=shape).astype(np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


# ----------------------------------------------------------------- workloads
def tiny_linear(seed: int = 0, M: int = 128, N: int = 128, K: int = 256):
    """X [M,K] ~ N(0,1) with 1% of entries scaled x50; W [N,K] ~ N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    x = normal(rng, (M, K))
    n_out = int(round(0.01 * M * K))
    idx = rng.choice(M * K, size=n_out, replace=False)
    x.reshape(-1)[idx] *= np.float32(50.0)
    w = normal(rng, (N, K), 0.02)
    return f32_to_bf16_bits(x), f32_to_bf16_bits(w)


def heavy_tailed(seed: int = 1, rows: int = 8192, cols: int = 8192, scale: float = 1e-3):
    """Gradient-like tensor: Student-t (df = 3) times `scale`."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(student_t(rng, (rows, cols), 3.0, scale))


def weight_and_outlier_acts(seed: int = 2, M: int = 8192, N: int = 4096, K: int = 4096,
                            outlier_frac: float = 0.001, outlier_mult: float = 100.0):
    """W [N,K] ~ N(0, 0.02); X [M,K] ~ N(0,1) with a fraction of channels (columns) x100."""
    rng = np.random.default_rng(seed)
    w = normal(rng, (N, K), 0.02)
    x = normal(rng, (M, K))
    n_ch = max(1, int(outlier_frac * K))
    ch = rng.choice(K, size=n_ch, replace=False)
    x[:, ch] *= np.float32(outlier_mult)
    return f32_to_bf16_bits(w), f32_to_bf16_bits(x), np.sort(ch)


def moe_routing(rng: np.random.Generator, tokens: int, experts: int, top_k: int,
                zipf_s: float = 1.1):
    """Top-k routing with Zipf(s)-skewed expert popularity.

    Expert popularity is proportional to rank^-s over a random permutation of the
    experts; each token draws `top_k` distinct experts without replacement in
    proportion to popularity (Gumbel top-k).  Returns (token_expert [tokens, k],
    expert order of routed rows: row_token [tokens*k], offsets [experts+1]).
    """
    ranks = np.arange(1, experts + 1, dtype=np.float64)
    pop = ranks ** (-zipf_s)
    pop /= pop.sum()
    perm = rng.permutation(experts)
    p = np.empty(experts)
    p[perm] = pop
    g = rng.gumbel(size=(tokens, experts))
    keys = np.log(p)[None, :] + g
    te = np.argsort(-keys, axis=1)[:, :top_k].astype(np.int32)
    flat_e = te.reshape(-1)
    flat_t = np.repeat(np.arange(tokens, dtype=np.int32), top_k)
    order = np.argsort(flat_e, kind="stable")
    row_token = flat_t[order]
    counts = np.bincount(flat_e, minlength=experts)
    offsets = np.zeros(experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    return te, row_token, offsets


def moe_expert_forward(seed: int = 3, tokens: int = 16384, hidden: int = 4096,
                       ffn: int = 1536, experts: int = 64, top_k: int = 4):
    """Token activations ~N(0,1), W_up [E, ffn, hidden], W_down [E, hidden, ffn] ~N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    x = normal(rng, (tokens, hidden))
    te, row_token, offsets = moe_routing(rng, tokens, experts, top_k)
    w_up = normal(rng, (experts, ffn, hidden), 0.02)
    w_down = normal(rng, (experts, hidden, ffn), 0.02)
    return dict(x=f32_to_bf16_bits(x), w_up=f32_to_bf16_bits(w_up),
                w_down=f32_to_bf16_bits(w_down), token_expert=te, row_token=row_token,
                offsets=offsets)


def dense_linear_layer(seed: int = 4, tokens: int = 16384, hidden: int = 5120,
                       ffn: int = 20480):
    """X [tokens, hidden] ~N(0,1); W [ffn, hidden] ~N(0, 0.02); dY [tokens, ffn] Student-t(3)."""
    rng = np.random.default_rng(seed)
    x = normal(rng, (tokens, hidden))
    w = normal(rng, (ffn, hidden), 0.02)
    dy = student_t(rng, (tokens, ffn), 3.0, 1.0)
    return dict(x=f32_to_bf16_bits(x), w=f32_to_bf16_bits(w), dy=f32_to_bf16_bits(dy))
