"""Python binding of libnvfp4 -- the B200 (sm_100a) NVFP4 quantizer and
block-scaled GEMM.

The C functions keep their names (``nvfp4_quantize``, ``nvfp4_dequantize``,
``mxfp8_quantize``, ``mxfp4_quantize``, ``nvfp4_gemm``, ``nvfp4_grouped_gemm``); this module only
marshals arguments: torch tensors become device pointers and the current torch
stream becomes the ``cudaStream_t``.  Every arithmetic step runs in the CUDA
kernels of ``libnvfp4.so``.  There is no fallback: importing this package
raises if the library is missing, and every call raises ``NVFP4Error`` on a
non-zero status.

The convenience wrappers (``quantize``, ``dequantize``, ``mxfp8``, ``mxfp4``, ``gemm``,
``grouped_gemm``) allocate their outputs with torch and call the C functions.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

from . import build as _build

if _build.stale():
    try:
        _build.build()
    except Exception as exc:  # no nvcc / compile error: there is no CPU fallback
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing and could not be built: {exc}") from exc

_lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- constants
NVFP4_OK = 0
NVFP4_RNE, NVFP4_SR = 0, 1
NVFP4_1D16, NVFP4_2D16x16 = 0, 1
NVFP4_ROWWISE, NVFP4_COLWISE = 1, 2
NVFP4_SF_ROWMAJOR, NVFP4_SF_MMA = 0, 1
NVFP4_OUT_F32, NVFP4_OUT_BF16 = 0, 1

EXPORTED = [
    "nvfp4_quantize", "nvfp4_dequantize", "mxfp8_quantize", "nvfp4_gemm", "nvfp4_grouped_gemm",
    "nvfp4_quantize_workspace_size", "nvfp4_gemm_workspace_size", "nvfp4_sf_mma_bytes",
    "nvfp4_sf_mma_grouped_bytes", "nvfp4_workspace_status", "nvfp4_status_string",
    "nvfp4_version", "nvfp4_quantize_noalloc", "nvfp4_quantize_noalloc_status",
    "nvfp4_gather_rows", "mxfp4_quantize", "mxfp8_gemm", "mxfp8_sf_mma_bytes", "mxfp4_gemm",
    "mxfp8_combine", "nvfp4_gemm_cycles",
]


class QuantParams(ctypes.Structure):
    """Mirror of ``nvfp4_quant_params`` (include/nvfp4.h)."""
    _fields_ = [
        ("rounding", ctypes.c_int), ("scaling", ctypes.c_int), ("outputs", ctypes.c_int),
        ("rht_colwise", ctypes.c_int), ("sf_layout", ctypes.c_int),
        ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint32),
        ("amax_in", ctypes.c_void_p),
        ("row_index", ctypes.c_void_p), ("src_rows", ctypes.c_int64),
        ("group_offsets", ctypes.c_void_p), ("num_groups", ctypes.c_int),
        ("mx_outputs", ctypes.c_int), ("mx_rounding", ctypes.c_int),
        ("mx_q_row", ctypes.c_void_p), ("mx_sf_row", ctypes.c_void_p),
        ("mx_q_col", ctypes.c_void_p), ("mx_sf_col", ctypes.c_void_p),
        ("mx_sf_layout", ctypes.c_int),
    ]


_P, _I64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_lib.nvfp4_quantize.argtypes = [_P, _I64, _I64, _I64, ctypes.POINTER(QuantParams), _P, _P, _P,
                                _P, _P, _P, _P, _SZ, _P]
_lib.nvfp4_quantize_noalloc.argtypes = [_P, _I64, _I64, _I64, ctypes.POINTER(QuantParams), _P,
                                        _P, _P, _P, _P, _P, _P]
_lib.mxfp8_quantize.argtypes = [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                ctypes.c_uint64, ctypes.c_uint32, _P, _P, _P, _P, _P]
_lib.mxfp4_quantize.argtypes = [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                _P, _P]
_lib.mxfp4_gemm.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _I64, _P, _P, _SZ,
                            _P]
_lib.nvfp4_dequantize.argtypes = [_P, _P, _P, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _P]
_lib.nvfp4_gemm.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _I64, _P,
                            _P, _SZ, _P]
_lib.mxfp8_gemm.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _I64, _P, _P, _SZ,
                            _P]
_lib.mxfp8_combine.argtypes = [_P, _P, _I64, _I64, _P, _P, _I64, ctypes.c_int, _P, _P, _SZ, _P]
_lib.mxfp8_sf_mma_bytes.argtypes = [_I64, _I64]
_lib.mxfp8_sf_mma_bytes.restype = _SZ
_lib.nvfp4_grouped_gemm.argtypes = [ctypes.c_int, _P, _I64, _P, _P, _P, _P, _P, _P, _I64, _I64,
                                    ctypes.c_int, _P, _P, _P, _SZ, _P]
_lib.nvfp4_gather_rows.argtypes = [_P, _P, _I64, _I64, _P, _I64, _P, ctypes.c_int, _P, _P, _P,
                                   _SZ, _P]
_lib.nvfp4_quantize_workspace_size.argtypes = [_I64, _I64, ctypes.POINTER(QuantParams)]
_lib.nvfp4_quantize_workspace_size.restype = _SZ
_lib.nvfp4_gemm_workspace_size.argtypes = [_I64, _I64, _I64]
_lib.nvfp4_gemm_workspace_size.restype = _SZ
_lib.nvfp4_sf_mma_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_sf_mma_bytes.restype = _SZ
_lib.nvfp4_sf_mma_grouped_bytes.argtypes = [_I64, ctypes.c_int, _I64]
_lib.nvfp4_sf_mma_grouped_bytes.restype = _SZ
_lib.nvfp4_workspace_status.argtypes = [_P, _P]
_lib.nvfp4_gemm_cycles.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint64)]
_lib.nvfp4_quantize_noalloc_status.argtypes = [_P]
_lib.nvfp4_status_string.argtypes = [ctypes.c_int]
_lib.nvfp4_status_string.restype = ctypes.c_char_p
_lib.nvfp4_version.restype = ctypes.c_int
for _n in ("nvfp4_quantize", "nvfp4_quantize_noalloc", "mxfp8_quantize", "mxfp4_quantize",
           "nvfp4_dequantize", "nvfp4_gemm", "mxfp8_gemm", "mxfp4_gemm", "mxfp8_combine",
           "nvfp4_grouped_gemm", "nvfp4_gather_rows", "nvfp4_workspace_status",
           "nvfp4_quantize_noalloc_status", "nvfp4_gemm_cycles"):
    getattr(_lib, _n).restype = ctypes.c_int


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def status_string(s: int) -> str:
    return _lib.nvfp4_status_string(int(s)).decode()


def _check(status: int, where: str) -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------- raw C calls
def nvfp4_quantize(x, rows, cols, ld, params: QuantParams, q_row, sf_row, g_row, q_col, sf_col,
                   g_col, workspace, ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_quantize(_ptr(x), rows, cols, ld, ctypes.byref(params), _ptr(q_row),
                               _ptr(sf_row), _ptr(g_row), _ptr(q_col), _ptr(sf_col), _ptr(g_col),
                               _ptr(workspace), ws_bytes, _stream(stream)), "nvfp4_quantize")


def nvfp4_quantize_noalloc(x, rows, cols, ld, params: QuantParams, q_row, sf_row, g_row, q_col,
                           sf_col, g_col, stream=None) -> None:
    """nvfp4_quantize without a workspace, for callers that cannot allocate device
    memory; its scratch lives in an array inside the library (see include/nvfp4.h)."""
    _check(_lib.nvfp4_quantize_noalloc(_ptr(x), rows, cols, ld, ctypes.byref(params), _ptr(q_row),
                                       _ptr(sf_row), _ptr(g_row), _ptr(q_col), _ptr(sf_col),
                                       _ptr(g_col), _stream(stream)), "nvfp4_quantize_noalloc")


def mxfp8_quantize(x, rows, cols, ld, directions, rounding, seed, offset, q_row, e8_row, q_col,
                   e8_col, stream=None) -> None:
    _check(_lib.mxfp8_quantize(_ptr(x), rows, cols, ld, directions, rounding, seed, offset,
                               _ptr(q_row), _ptr(e8_row), _ptr(q_col), _ptr(e8_col),
                               _stream(stream)), "mxfp8_quantize")


def mxfp4_quantize(x, rows, cols, ld, directions, q_row, e8_row, q_col, e8_col,
                   stream=None, sf_layout=NVFP4_SF_ROWMAJOR) -> None:
    _check(_lib.mxfp4_quantize(_ptr(x), rows, cols, ld, directions, sf_layout, _ptr(q_row),
                               _ptr(e8_row), _ptr(q_col), _ptr(e8_col), _stream(stream)),
           "mxfp4_quantize")


def mxfp4_gemm(qa, sfa, qb, sfb, M, N, K, out_dtype, D, ldd, amax_out, workspace, ws_bytes,
               stream=None) -> None:
    _check(_lib.mxfp4_gemm(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), M, N, K, out_dtype, _ptr(D),
                           ldd, _ptr(amax_out), _ptr(workspace), ws_bytes, _stream(stream)),
           "mxfp4_gemm")


def nvfp4_dequantize(q, sf, g, rows, cols, sf_layout, out_dtype, out, stream=None) -> None:
    _check(_lib.nvfp4_dequantize(_ptr(q), _ptr(sf), _ptr(g), rows, cols, sf_layout, out_dtype,
                                 _ptr(out), _stream(stream)), "nvfp4_dequantize")


def nvfp4_gemm(qa, sfa, ga, qb, sfb, gb, M, N, K, out_dtype, D, ldd, amax_out, workspace,
               ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_gemm(_ptr(qa), _ptr(sfa), _ptr(ga), _ptr(qb), _ptr(sfb), _ptr(gb), M, N, K,
                           out_dtype, _ptr(D), ldd, _ptr(amax_out), _ptr(workspace), ws_bytes,
                           _stream(stream)),
           "nvfp4_gemm")


def mxfp8_gemm(qa, sfa, qb, sfb, M, N, K, out_dtype, D, ldd, amax_out, workspace, ws_bytes,
               stream=None) -> None:
    _check(_lib.mxfp8_gemm(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), M, N, K, out_dtype, _ptr(D),
                           ldd, _ptr(amax_out), _ptr(workspace), ws_bytes, _stream(stream)),
           "mxfp8_gemm")


def mxfp8_combine(q, e8, rows, cols, slot_row, weight, tokens, k, out, workspace=None,
                  ws_bytes=0, stream=None) -> None:
    _check(_lib.mxfp8_combine(_ptr(q), _ptr(e8), rows, cols, _ptr(slot_row), _ptr(weight), tokens,
                              k, _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "mxfp8_combine")


def nvfp4_grouped_gemm(G, group_offsets, total_rows, qa, sfa, ga, qb, sfb, gb, N, K, out_dtype, D,
                       amax_out, workspace, ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_grouped_gemm(G, _ptr(group_offsets), total_rows, _ptr(qa), _ptr(sfa),
                                   _ptr(ga), _ptr(qb), _ptr(sfb), _ptr(gb), N, K, out_dtype,
                                   _ptr(D), _ptr(amax_out), _ptr(workspace), ws_bytes,
                                   _stream(stream)),
           "nvfp4_grouped_gemm")


def nvfp4_gather_rows(q_src, sf_src, src_rows, k, row_index, rows, group_offsets, num_groups,
                      q_dst, sf_dst, workspace, ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_gather_rows(_ptr(q_src), _ptr(sf_src), src_rows, k, _ptr(row_index), rows,
                                  _ptr(group_offsets), num_groups, _ptr(q_dst), _ptr(sf_dst),
                                  _ptr(workspace), ws_bytes, _stream(stream)),
           "nvfp4_gather_rows")


def nvfp4_workspace_status(workspace, stream=None) -> int:
    return int(_lib.nvfp4_workspace_status(_ptr(workspace), _stream(stream)))


def nvfp4_gemm_cycles(workspace, stream=None) -> int:
    """SM cycles (entry to exit) of the longest CTA of the last GEMM call on
    `workspace`; synchronises the stream."""
    v = ctypes.c_uint64(0)
    _check(_lib.nvfp4_gemm_cycles(_ptr(workspace), _stream(stream), ctypes.byref(v)),
           "nvfp4_gemm_cycles")
    return int(v.value)


def nvfp4_quantize_noalloc_status(stream=None) -> int:
    return int(_lib.nvfp4_quantize_noalloc_status(_stream(stream)))


def nvfp4_sf_mma_bytes(rows: int, k: int) -> int:
    return int(_lib.nvfp4_sf_mma_bytes(rows, k))


def mxfp8_sf_mma_bytes(rows: int, k: int) -> int:
    return int(_lib.mxfp8_sf_mma_bytes(rows, k))


def nvfp4_sf_mma_grouped_bytes(total_rows: int, num_groups: int, k: int) -> int:
    return int(_lib.nvfp4_sf_mma_grouped_bytes(total_rows, num_groups, k))


def nvfp4_quantize_workspace_size(rows: int = 0, cols: int = 0) -> int:
    return int(_lib.nvfp4_quantize_workspace_size(rows, cols, None))


def nvfp4_gemm_workspace_size(M: int = 0, N: int = 0, K: int = 0) -> int:
    return int(_lib.nvfp4_gemm_workspace_size(M, N, K))


def nvfp4_version() -> int:
    return int(_lib.nvfp4_version())


# ----------------------------------------------------------------- convenience wrappers
@dataclass
class NVFP4Tensor:
    """Codes [rows, k/2] u8, scale bytes (row-major [rows, k/16] or tiled bytes), g [1] f32."""
    q: object
    sf: object
    g: object
    rows: int
    k: int
    sf_layout: int


def _workspace(device, nbytes: int = 256):
    import torch
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def quantize(x, *, rowwise: bool = True, colwise: bool = False, rounding: int = NVFP4_RNE,
             scaling: int = NVFP4_1D16, rht: bool = False, sf_layout: int = NVFP4_SF_ROWMAJOR,
             seed: int = 0, offset: int = 0, amax=None, mx_outputs: int = 0,
             mx_rounding: int = NVFP4_RNE, mx_sf_layout: int = NVFP4_SF_ROWMAJOR,
             row_index=None, src_rows: int = 0, group_offsets=None, num_groups: int = 0,
             rows: Optional[int] = None, workspace=None, stream=None):
    """Quantise a bf16 [rows, cols] CUDA tensor.  Returns dict with 'row', 'col'
    (NVFP4Tensor or None), 'mx_row', 'mx_col' ((codes, e8m0) or None)."""
    import torch
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    cols = x.shape[1]
    ld = x.stride(0)
    assert x.stride(1) == 1
    n_rows = rows if rows is not None else x.shape[0]
    dev = x.device
    u8 = dict(dtype=torch.uint8, device=dev)

    def sf_alloc(r, k, grouped=False):
        if sf_layout == NVFP4_SF_MMA:
            n = (nvfp4_sf_mma_grouped_bytes(r, num_groups, k) if grouped
                 else nvfp4_sf_mma_bytes(r, k))
            return torch.zeros(n, **u8)
        return torch.empty((r, k // 16), **u8)

    out = {"row": None, "col": None, "mx_row": None, "mx_col": None}
    q_row = sf_row = g_row = q_col = sf_col = g_col = None
    if rowwise:
        q_row = torch.empty((n_rows, cols // 2), **u8)
        sf_row = sf_alloc(n_rows, cols, grouped=group_offsets is not None)
        g_row = torch.empty(1, dtype=torch.float32, device=dev)
        out["row"] = NVFP4Tensor(q_row, sf_row, g_row, n_rows, cols, sf_layout)
    if colwise:
        q_col = torch.empty((cols, n_rows // 2), **u8)
        sf_col = sf_alloc(cols, n_rows)
        g_col = torch.empty(1, dtype=torch.float32, device=dev)
        out["col"] = NVFP4Tensor(q_col, sf_col, g_col, cols, n_rows, sf_layout)
    p = QuantParams()
    p.rounding, p.scaling = rounding, scaling
    p.outputs = (NVFP4_ROWWISE if rowwise else 0) | (NVFP4_COLWISE if colwise else 0)
    p.rht_colwise = 1 if rht else 0
    p.sf_layout = sf_layout
    p.seed, p.offset = seed, offset
    p.amax_in = _ptr(amax)
    p.row_index = _ptr(row_index)
    p.src_rows = src_rows if row_index is not None else 0
    p.group_offsets = _ptr(group_offsets)
    p.num_groups = num_groups
    p.mx_outputs, p.mx_rounding, p.mx_sf_layout = mx_outputs, mx_rounding, mx_sf_layout

    def mx_sf_alloc(r, k):
        if mx_sf_layout == NVFP4_SF_MMA:
            return torch.zeros(mxfp8_sf_mma_bytes(r, k), **u8)
        return torch.empty((r, k // 32), **u8)

    if mx_outputs & NVFP4_ROWWISE:
        mq, me = torch.empty((n_rows, cols), **u8), mx_sf_alloc(n_rows, cols)
        p.mx_q_row, p.mx_sf_row = mq.data_ptr(), me.data_ptr()
        out["mx_row"] = (mq, me)
    if mx_outputs & NVFP4_COLWISE:
        mq, me = torch.empty((cols, n_rows), **u8), mx_sf_alloc(cols, n_rows)
        p.mx_q_col, p.mx_sf_col = mq.data_ptr(), me.data_ptr()
        out["mx_col"] = (mq, me)
    ws = workspace if workspace is not None else _workspace(dev)
    nvfp4_quantize(x, n_rows, cols, ld, p, q_row, sf_row, g_row, q_col, sf_col, g_col, ws,
                   ws.numel(), stream)
    out["workspace"] = ws
    return out


def mxfp8(x, directions: int = NVFP4_COLWISE, rounding: int = NVFP4_RNE, seed: int = 0,
          offset: int = 0, stream=None):
    import torch
    rows, cols = x.shape
    u8 = dict(dtype=torch.uint8, device=x.device)
    qr = er = qc = ec = None
    if directions & NVFP4_ROWWISE:
        qr, er = torch.empty((rows, cols), **u8), torch.empty((rows, cols // 32), **u8)
    if directions & NVFP4_COLWISE:
        qc, ec = torch.empty((cols, rows), **u8), torch.empty((cols, rows // 32), **u8)
    mxfp8_quantize(x, rows, cols, x.stride(0), directions, rounding, seed, offset, qr, er, qc, ec,
                   stream)
    return (qr, er), (qc, ec)


def mxfp4(x, directions: int = NVFP4_ROWWISE | NVFP4_COLWISE, stream=None,
          sf_layout: int = NVFP4_SF_ROWMAJOR):
    """MXFP4 codes and E8M0 scales of a bf16 [rows, cols] tensor:
    ((q_row [rows, cols/2], e8 [rows, cols/32]) or (None, None),
     (q_col [cols, rows/2], e8 [cols, rows/32]) or (None, None)); with
    sf_layout = NVFP4_SF_MMA the scales are flat tiled buffers (mxfp4_gemm's layout)."""
    import torch
    rows, cols = x.shape
    u8 = dict(dtype=torch.uint8, device=x.device)

    def e8(r, k):
        if sf_layout == NVFP4_SF_MMA:
            return torch.zeros(mxfp8_sf_mma_bytes(r, k), **u8)
        return torch.empty((r, k // 32), **u8)

    qr = er = qc = ec = None
    if directions & NVFP4_ROWWISE:
        qr, er = torch.empty((rows, cols // 2), **u8), e8(rows, cols)
    if directions & NVFP4_COLWISE:
        qc, ec = torch.empty((cols, rows // 2), **u8), e8(cols, rows)
    mxfp4_quantize(x, rows, cols, x.stride(0), directions, qr, er, qc, ec, stream, sf_layout)
    return (qr, er), (qc, ec)


def mx4_gemm(qa, sfa, qb, sfb, out_dtype: int = NVFP4_OUT_BF16, out=None, amax_out=None,
             workspace=None, stream=None):
    """D = A_hat B_hat^T of MXFP4 operands: qa [M, K/2], qb [N, K/2] codes with E8M0 scales
    in the tiled layout (mxfp4(..., sf_layout=NVFP4_SF_MMA))."""
    import torch
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qb.shape[0]
    dt = torch.bfloat16 if out_dtype == NVFP4_OUT_BF16 else torch.float32
    D = out if out is not None else torch.empty((M, N), dtype=dt, device=qa.device)
    ws = workspace if workspace is not None else _workspace(qa.device)
    mxfp4_gemm(qa, sfa, qb, sfb, M, N, K, out_dtype, D, D.stride(0), amax_out, ws, ws.numel(),
               stream)
    return D


def dequantize(t: NVFP4Tensor, out_dtype: int = NVFP4_OUT_F32, stream=None):
    import torch
    dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
    out = torch.empty((t.rows, t.k), dtype=dt, device=t.q.device)
    nvfp4_dequantize(t.q, t.sf, t.g, t.rows, t.k, t.sf_layout, out_dtype, out, stream)
    return out


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, out_dtype: int = NVFP4_OUT_BF16, out=None,
         amax_out=None, workspace=None, stream=None):
    """D = A B^T for NVFP4 operands A [M, K] and B [N, K] (tiled scale layout).
    ``amax_out`` (optional device f32 [1]) receives max |D| as stored."""
    import torch
    assert a.k == b.k and a.sf_layout == NVFP4_SF_MMA and b.sf_layout == NVFP4_SF_MMA
    M, N, K = a.rows, b.rows, a.k
    dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=a.q.device)
    ws = workspace if workspace is not None else _workspace(a.q.device)
    nvfp4_gemm(a.q, a.sf, a.g, b.q, b.sf, b.g, M, N, K, out_dtype, out, out.stride(0), amax_out,
               ws, ws.numel(), stream)
    return out


def mx_gemm(qa, sfa, qb, sfb, out_dtype: int = NVFP4_OUT_BF16, out=None, amax_out=None,
            workspace=None, stream=None):
    """D = A_hat B_hat^T of MXFP8 operands: qa [M, K], qb [N, K] E4M3 codes with E8M0
    scales in the tiled layout (quantize(..., mx_sf_layout=NVFP4_SF_MMA))."""
    import torch
    M, K = qa.shape
    N = qb.shape[0]
    dt = torch.bfloat16 if out_dtype == NVFP4_OUT_BF16 else torch.float32
    D = out if out is not None else torch.empty((M, N), dtype=dt, device=qa.device)
    ws = workspace if workspace is not None else _workspace(qa.device)
    mxfp8_gemm(qa, sfa, qb, sfb, M, N, K, out_dtype, D, D.stride(0), amax_out, ws, ws.numel(),
               stream)
    return D


def grouped_gemm(group_offsets, a: NVFP4Tensor, qb, sfb, gb, N: int, out_dtype: int = NVFP4_OUT_BF16,
                 out=None, amax_out=None, workspace=None, stream=None):
    """MoE grouped D = A_e B_e^T; qb [G, N, K/2], sfb tiled per expert, gb [G]."""
    import torch
    G = group_offsets.numel() - 1
    dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((a.rows, N), dtype=dt, device=a.q.device)
    ws = workspace if workspace is not None else _workspace(a.q.device)
    nvfp4_grouped_gemm(G, group_offsets, a.rows, a.q, a.sf, a.g, qb, sfb, gb, N, a.k, out_dtype,
                       out, amax_out, ws, ws.numel(), stream)
    return out


def gather_rows(t: NVFP4Tensor, row_index, group_offsets=None, workspace=None, stream=None):
    """MoE dispatch of an already quantised operand: row i of the result is row
    ``row_index[i]`` of ``t`` (codes and tiled scales), laid out per expert
    group when ``group_offsets`` (device int32 [G+1]) is given."""
    import torch
    assert t.sf_layout == NVFP4_SF_MMA
    rows = row_index.numel()
    G = 0 if group_offsets is None else group_offsets.numel() - 1
    u8 = dict(dtype=torch.uint8, device=t.q.device)
    q = torch.empty((rows, t.k // 2), **u8)
    n = nvfp4_sf_mma_grouped_bytes(rows, G, t.k) if G else nvfp4_sf_mma_bytes(rows, t.k)
    sf = torch.zeros(n, **u8)
    ws = workspace if workspace is not None else _workspace(t.q.device)
    nvfp4_gather_rows(t.q, t.sf, t.rows, t.k, row_index, rows, group_offsets, G, q, sf, ws,
                      ws.numel(), stream)
    return NVFP4Tensor(q, sf, t.g, rows, t.k, NVFP4_SF_MMA)
