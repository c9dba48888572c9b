"""CPU oracle for the NVFP4 quantizer, MXFP8 requantizer and block-scaled GEMM.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The arithmetic
lives in ``nvfp4_oracle.c`` (plain C, single thread); this module only builds
that file with gcc and marshals numpy arrays into it.  It shares nothing with
the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c into liboracle.so (IEEE binary32/64, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class QParams(ctypes.Structure):
    _fields_ = [("rounding", ctypes.c_int), ("scaling", ctypes.c_int), ("rht", ctypes.c_int),
                ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint32),
                ("has_amax", ctypes.c_int), ("amax_row", ctypes.c_float),
                ("amax_col", ctypes.c_float), ("idx_base", ctypes.c_uint64)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, u8, u16, u32, u64 = (ctypes.c_int64, ctypes.c_uint8, ctypes.c_uint16,
                                  ctypes.c_uint32, ctypes.c_uint64)
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_sr_bits.argtypes = [u64, u32, u32, u64]
        L.orc_sr_bits.restype = u16
        L.orc_sr_bits_nvfp4.argtypes = [u64, u32, u32, u64]
        L.orc_sr_bits_nvfp4.restype = u16
        L.orc_e2m1_decode.argtypes = [u8]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_rne.argtypes = [ctypes.c_float]
        L.orc_e2m1_rne.restype = u8
        L.orc_e2m1_sr.argtypes = [ctypes.c_float, u16]
        L.orc_e2m1_sr.restype = u8
        L.orc_e4m3_decode.argtypes = [u8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_rne_sat.argtypes = [ctypes.c_double]
        L.orc_e4m3_rne_sat.restype = u8
        L.orc_e4m3_sr_sat.argtypes = [ctypes.c_double, u16]
        L.orc_e4m3_sr_sat.restype = u8
        L.orc_rht_signs.argtypes = [u64, P]
        L.orc_rht16.argtypes = [P, P, P]
        L.orc_global_scale.argtypes = [ctypes.c_float, P, P]
        L.orc_nvfp4_quantize.argtypes = [P, i64, i64, i64, ctypes.c_int, ctypes.POINTER(QParams),
                                         P, P, P]
        L.orc_nvfp4_quantize.restype = ctypes.c_int
        L.orc_mxfp8_quantize.argtypes = [P, i64, i64, i64, ctypes.c_int, ctypes.c_int, u64, u32,
                                         u64, P, P]
        L.orc_amax.argtypes = [P, i64, i64, i64, ctypes.c_int, ctypes.c_int, u64]
        L.orc_amax.restype = ctypes.c_float
        L.orc_mxfp8_quantize.restype = ctypes.c_int
        L.orc_mxfp4_quantize.argtypes = [P, i64, i64, i64, ctypes.c_int, P, P]
        L.orc_mxfp4_quantize.restype = ctypes.c_int
        L.orc_nvfp4_dequant_f64.argtypes = [P, P, ctypes.c_float, i64, i64, P]
        L.orc_nvfp4_dequant_f32.argtypes = [P, P, ctypes.c_float, i64, i64, P]
        L.orc_nvfp4_gemm_rows.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, i64, i64,
                                          i64, P, i64, P, P]
        L.orc_nvfp4_gemm_rows.restype = ctypes.c_int
        L.orc_nvfp4_grouped_gemm_rows.argtypes = [ctypes.c_int, P, P, P, ctypes.c_float, P, P, P,
                                                  i64, i64, P, i64, P, P]
        L.orc_nvfp4_grouped_gemm_rows.restype = ctypes.c_int
        L.orc_mxfp8_dequant_f64.argtypes = [P, P, i64, i64, P]
        L.orc_mxfp8_gemm_rows.argtypes = [P, P, P, P, i64, i64, i64, P, i64, P, P]
        L.orc_mxfp8_gemm_rows.restype = ctypes.c_int
        L.orc_mxfp4_dequant_f64.argtypes = [P, P, i64, i64, P]
        L.orc_mxfp4_gemm_rows.argtypes = [P, P, P, P, i64, i64, i64, P, i64, P, P]
        L.orc_mxfp4_gemm_rows.restype = ctypes.c_int
        L.orc_mxfp8_combine.argtypes = [P, P, i64, i64, P, P, i64, ctypes.c_int, P]
        L.orc_mxfp8_combine.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalar pieces
def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> Tuple[int, int, int, int]:
    c = np.array(ctr, dtype=np.uint32)
    k = np.array(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(o))
    return tuple(int(v) for v in o)


def sr_bits(seed: int, offset: int, stream: int, idx: int) -> int:
    return int(lib().orc_sr_bits(seed, offset, stream, idx))


def sr_bits_nvfp4(seed: int, offset: int, stream: int, idx: int) -> int:
    return int(lib().orc_sr_bits_nvfp4(seed, offset, stream, idx))


def e2m1_decode(code: int) -> float:
    return float(lib().orc_e2m1_decode(code))


def e2m1_rne(y: float) -> int:
    return int(lib().orc_e2m1_rne(y))


def e2m1_sr(y: float, u: int) -> int:
    return int(lib().orc_e2m1_sr(y, u))


def e4m3_decode(b: int) -> float:
    return float(lib().orc_e4m3_decode(b))


def e4m3_rne_sat(y: float) -> int:
    return int(lib().orc_e4m3_rne_sat(y))


def e4m3_sr_sat(y: float, u: int) -> int:
    return int(lib().orc_e4m3_sr_sat(y, u))


def rht_signs(seed: int) -> np.ndarray:
    s = np.zeros(16, dtype=np.float32)
    lib().orc_rht_signs(seed, _p(s))
    return s


def rht16(signs: np.ndarray, v: np.ndarray) -> np.ndarray:
    i = np.ascontiguousarray(v, dtype=np.float32)
    o = np.zeros(16, dtype=np.float32)
    lib().orc_rht16(_p(np.ascontiguousarray(signs, dtype=np.float32)), _p(i), _p(o))
    return o


def global_scale(amax: float) -> Tuple[float, float]:
    S = np.zeros(1, dtype=np.float32)
    g = np.zeros(1, dtype=np.float32)
    lib().orc_global_scale(ctypes.c_float(amax), _p(S), _p(g))
    return float(S[0]), float(g[0])


# ---------------------------------------------------------------- tensor pieces
def amax(x_bf16: np.ndarray, direction: int, rht: int = 0, seed: int = 0) -> float:
    """Tensor amax of one direction (over the Hadamard-rotated vectors when rht)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    v = float(lib().orc_amax(_p(x), rows, cols, cols, direction, rht, seed))
    if v < 0:
        raise ValueError("oracle amax: invalid arguments")
    return v


def nvfp4_quantize(x_bf16: np.ndarray, direction: int, rounding: int = 0, scaling: int = 0,
                   rht: int = 0, seed: int = 0, offset: int = 0,
                   amax: Optional[Tuple[float, float]] = None, idx_base: int = 0):
    """Quantise a bf16 matrix (given as uint16 bit patterns, [rows, cols]).

    direction 0: rowwise -> codes [rows, cols/2], scales [rows, cols/16].
    direction 1: columnwise (on x^T) -> codes [cols, rows/2], scales [cols, rows/16].
    Returns (codes u8, scale bytes u8, g float).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    nr, nc = (cols, rows) if direction else (rows, cols)
    q = np.zeros((nr, nc // 2), dtype=np.uint8)
    sf = np.zeros((nr, nc // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    p = QParams(rounding, scaling, rht, seed, offset, 1 if amax is not None else 0,
                amax[0] if amax is not None else 0.0, amax[1] if amax is not None else 0.0,
                idx_base)
    rc = lib().orc_nvfp4_quantize(_p(x), rows, cols, cols, direction, ctypes.byref(p), _p(q),
                                  _p(sf), _p(g))
    if rc != 0:
        raise ValueError("oracle nvfp4_quantize: invalid arguments")
    return q, sf, float(g[0])


def mxfp8_quantize(x_bf16: np.ndarray, direction: int, rounding: int = 0, seed: int = 0,
                   offset: int = 0, idx_base: int = 0):
    """MXFP8: codes [rows, cols] + E8M0 [rows, cols/32] (direction 0) or on x^T (1)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    nr, nc = (cols, rows) if direction else (rows, cols)
    q = np.zeros((nr, nc), dtype=np.uint8)
    e8 = np.zeros((nr, nc // 32), dtype=np.uint8)
    rc = lib().orc_mxfp8_quantize(_p(x), rows, cols, cols, direction, rounding, seed, offset,
                                  idx_base, _p(q), _p(e8))
    if rc != 0:
        raise ValueError("oracle mxfp8_quantize: invalid arguments")
    return q, e8


def mxfp4_quantize(x_bf16: np.ndarray, direction: int):
    """MXFP4 (OCP MX, E2M1 elements, E8M0 scale per 32): codes [rows, cols/2] +
    E8M0 [rows, cols/32] (direction 0) or the same on x^T (direction 1)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    nr, nc = (cols, rows) if direction else (rows, cols)
    q = np.zeros((nr, nc // 2), dtype=np.uint8)
    e8 = np.zeros((nr, nc // 32), dtype=np.uint8)
    rc = lib().orc_mxfp4_quantize(_p(x), rows, cols, cols, direction, _p(q), _p(e8))
    if rc != 0:
        raise ValueError("oracle mxfp4_quantize: invalid arguments")
    return q, e8


def mxfp4_dequant(q: np.ndarray, e8: np.ndarray) -> np.ndarray:
    """x_hat = e2m1(code) * 2^(e8 - 127), exact in binary64."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    rows, half = q.shape
    codes = np.empty((rows, half * 2), dtype=np.uint8)
    codes[:, 0::2] = q & 0xF
    codes[:, 1::2] = q >> 4
    mag = np.array([e2m1_decode(c) for c in range(16)], dtype=np.float64)
    scale = np.ldexp(1.0, np.repeat(np.asarray(e8, dtype=np.int64) - 127, 32, axis=1))
    return mag[codes] * scale


def nvfp4_dequant(q: np.ndarray, sf: np.ndarray, g: float, f64: bool = True) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, half = q.shape
    cols = half * 2
    out = np.zeros((rows, cols), dtype=np.float64 if f64 else np.float32)
    fn = lib().orc_nvfp4_dequant_f64 if f64 else lib().orc_nvfp4_dequant_f32
    fn(_p(q), _p(sf), ctypes.c_float(g), rows, cols, _p(out))
    return out


def nvfp4_gemm_rows(qa, sfa, ga, qb, sfb, gb, rows_sel=None):
    """FP64 D = A_hat B_hat^T for the selected rows of A; also sum |a_hat||b_hat|."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qb.shape[0]
    sel = np.arange(M, dtype=np.int64) if rows_sel is None else np.ascontiguousarray(
        rows_sel, dtype=np.int64)
    out = np.zeros((len(sel), N), dtype=np.float64)
    absout = np.zeros((len(sel), N), dtype=np.float64)
    rc = lib().orc_nvfp4_gemm_rows(_p(qa), _p(sfa), ctypes.c_float(ga), _p(qb), _p(sfb),
                                   ctypes.c_float(gb), M, N, K, _p(sel), len(sel), _p(out),
                                   _p(absout))
    if rc != 0:
        raise ValueError("oracle gemm: invalid arguments")
    return out, absout


def nvfp4_grouped_gemm_rows(offsets, qa, sfa, ga, qb, sfb, gb, rows_sel):
    """Grouped FP64 reference: rows [off[e], off[e+1]) of A times expert e's B."""
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    G = len(off) - 1
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    gbv = np.ascontiguousarray(gb, dtype=np.float32)
    K = qa.shape[1] * 2
    N = qb.shape[1]
    sel = np.ascontiguousarray(rows_sel, dtype=np.int64)
    out = np.zeros((len(sel), N), dtype=np.float64)
    absout = np.zeros((len(sel), N), dtype=np.float64)
    rc = lib().orc_nvfp4_grouped_gemm_rows(G, _p(off), _p(qa), _p(sfa), ctypes.c_float(ga),
                                           _p(qb), _p(sfb), _p(gbv), N, K, _p(sel), len(sel),
                                           _p(out), _p(absout))
    if rc != 0:
        raise ValueError("oracle grouped gemm: invalid arguments")
    return out, absout


def mxfp8_dequant(q: np.ndarray, e8: np.ndarray) -> np.ndarray:
    """Binary64 values of MXFP8 codes [rows, cols] with row-major E8M0 scales [rows, cols/32]."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    e8 = np.ascontiguousarray(e8, dtype=np.uint8)
    rows, cols = q.shape
    out = np.zeros((rows, cols), dtype=np.float64)
    lib().orc_mxfp8_dequant_f64(_p(q), _p(e8), rows, cols, _p(out))
    return out


def mxfp8_gemm_rows(qa, e8a, qb, e8b, rows_sel=None):
    """FP64 D = A_hat B_hat^T of MXFP8 operands for the selected rows of A; also
    sum |a_hat||b_hat|."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    e8a = np.ascontiguousarray(e8a, dtype=np.uint8)
    e8b = np.ascontiguousarray(e8b, dtype=np.uint8)
    M, K = qa.shape
    N = qb.shape[0]
    sel = np.arange(M, dtype=np.int64) if rows_sel is None else np.ascontiguousarray(
        rows_sel, dtype=np.int64)
    out = np.zeros((len(sel), N), dtype=np.float64)
    absout = np.zeros((len(sel), N), dtype=np.float64)
    rc = lib().orc_mxfp8_gemm_rows(_p(qa), _p(e8a), _p(qb), _p(e8b), M, N, K, _p(sel), len(sel),
                                   _p(out), _p(absout))
    if rc != 0:
        raise ValueError("oracle mxfp8 gemm: invalid arguments")
    return out, absout


def mxfp4_gemm_rows(qa, e8a, qb, e8b, rows_sel=None):
    """FP64 D = A_hat B_hat^T of MXFP4 operands (codes [., K/2], row-major E8M0 [., K/32])
    for the selected rows of A; also sum |a_hat||b_hat|."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    e8a = np.ascontiguousarray(e8a, dtype=np.uint8)
    e8b = np.ascontiguousarray(e8b, dtype=np.uint8)
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qb.shape[0]
    sel = np.arange(M, dtype=np.int64) if rows_sel is None else np.ascontiguousarray(
        rows_sel, dtype=np.int64)
    out = np.zeros((len(sel), N), dtype=np.float64)
    absout = np.zeros((len(sel), N), dtype=np.float64)
    rc = lib().orc_mxfp4_gemm_rows(_p(qa), _p(e8a), _p(qb), _p(e8b), M, N, K, _p(sel), len(sel),
                                   _p(out), _p(absout))
    if rc != 0:
        raise ValueError("oracle mxfp4 gemm: invalid arguments")
    return out, absout


def mxfp8_combine(q, e8, slot_row, weight):
    """bf16 bits [tokens, cols] of sum_j weight[t, j] * xhat(slot_row[t, j]) (binary32, one
    rounding per product and per sum, j in order; slot_row -1 = none)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    e8 = np.ascontiguousarray(e8, dtype=np.uint8)
    sr = np.ascontiguousarray(slot_row, dtype=np.int32)
    w = np.ascontiguousarray(weight, dtype=np.float32)
    rows, cols = q.shape
    tokens, k = sr.shape
    out = np.zeros((tokens, cols), dtype=np.uint16)
    rc = lib().orc_mxfp8_combine(_p(q), _p(e8), rows, cols, _p(sr), _p(w), tokens, k, _p(out))
    if rc != 0:
        raise ValueError("oracle mxfp8_combine: invalid arguments")
    return out
