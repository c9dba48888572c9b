"""The C-ABI library loads, exports every function include/nvfp4.h declares, and
rejects bad arguments on the host before any device work.  CPU only: the calls
below fail validation before they would touch memory or a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(\w+)\s*\(", src)) - {"if", "sizeof", "defined"})


def test_exports_every_declared_function(nv):
    names = declared_functions()
    assert "nvfp4_quantize" in names and "nvfp4_grouped_gemm" in names
    for n in names:
        assert hasattr(nv._lib, n), n
    assert set(nv.EXPORTED) <= set(names)


def test_status_strings(nv):
    assert nv.status_string(0) == "ok"
    assert "timed out" in nv.status_string(6)
    assert nv.nvfp4_version() >= 100


def test_size_helpers(nv):
    assert nv.nvfp4_sf_mma_bytes(128, 256) == 128 * 16
    assert nv.nvfp4_sf_mma_bytes(130, 256) == 256 * 16
    assert nv.nvfp4_sf_mma_grouped_bytes(300, 4, 512) == (384 + 512) * 32
    assert nv.nvfp4_quantize_workspace_size() >= 16
    assert nv.nvfp4_gemm_workspace_size() >= 24  # status word + the call's cycle count


def test_gemm_cycles_argument_errors(nv):
    c = ctypes.c_uint64(7)
    assert nv._lib.nvfp4_gemm_cycles(None, None, ctypes.byref(c)) == 1
    assert nv._lib.nvfp4_gemm_cycles(FAKE, None, None) == 1
    assert c.value == 7


FAKE = 1 << 20  # a 16-byte aligned non-null address that validation never dereferences


def q(nv, rows, cols, ld, p, ws=FAKE, outs=(FAKE,) * 6):
    return nv._lib.nvfp4_quantize(FAKE, rows, cols, ld, ctypes.byref(p), *outs, ws, 256, None)


def test_quantize_argument_errors(nv):
    p = nv.QuantParams()
    p.outputs = nv.NVFP4_ROWWISE
    assert nv._lib.nvfp4_quantize(None, 16, 16, 16, ctypes.byref(p), *(FAKE,) * 6, FAKE, 256,
                                  None) == 1
    assert q(nv, 17, 16, 16, p) == 2                    # rows not a multiple of 16
    assert q(nv, 16, 24, 24, p) == 2
    assert q(nv, 16, 16, 8, p) == 2                     # ld < cols
    assert nv._lib.nvfp4_quantize(FAKE + 2, 16, 16, 16, ctypes.byref(p), *(FAKE,) * 6, FAKE, 256,
                                  None) == 3
    assert q(nv, 16, 16, 20, p) == 3                    # ld * 2 not 16-byte aligned
    p.rounding = 7
    assert q(nv, 16, 16, 16, p) == 1
    p.rounding = 0
    p.sf_layout = nv.NVFP4_SF_MMA
    assert q(nv, 16, 48, 48, p) == 2                    # tiled scales need K % 64
    p.sf_layout = 0
    assert q(nv, 16, 16, 16, p, ws=None) == 7           # amax needs the workspace
    p.outputs = 0
    assert q(nv, 16, 16, 16, p) == 1                    # nothing requested
    p.mx_outputs = nv.NVFP4_COLWISE
    assert q(nv, 16, 32, 32, p) == 2                    # MXFP8 columnwise needs rows % 32
    p.mx_outputs = 0
    p.outputs = nv.NVFP4_ROWWISE
    p.group_offsets = FAKE
    p.num_groups = 4
    assert q(nv, 16, 64, 64, p) == 1                    # grouped layout needs tiled scales


def test_gemm_argument_errors(nv):
    L = nv._lib
    args = (FAKE,) * 6
    g = L.nvfp4_gemm
    assert g(*args, 128, 128, 100, 0, FAKE, 128, None, FAKE, 256, None) == 2       # K % 256
    assert g(*args, 100, 128, 256, 0, FAKE, 128, None, FAKE, 256, None) == 2       # M % 16
    assert g(*args, 128, 128, 256, 0, FAKE, 120, None, FAKE, 256, None) == 2       # ldd < N
    assert g(*args, 128, 128, 256, 1, FAKE, 132, None, FAKE, 256, None) == 3       # ldd align
    assert g(*args, 128, 128, 256, 0, FAKE, 128, None, None, 0, None) == 7         # workspace
    assert g(*args, 128, 128, 256, 5, FAKE, 128, None, FAKE, 256, None) == 1       # dtype
    assert g(*args, 128, 128, 256, 0, FAKE, 128, FAKE + 2, FAKE, 256, None) == 3   # amax_out
    gg = L.nvfp4_grouped_gemm
    assert gg(0, FAKE, 128, *args, 128, 256, 0, FAKE, None, FAKE, 256, None) == 1
    assert gg(257, FAKE, 128, *args, 256, 256, 0, FAKE, None, FAKE, 256, None) == 1  # G > 256
    assert gg(4, FAKE, 128, *args, 100, 256, 0, FAKE, None, FAKE, 256, None) == 2
    assert gg(4, FAKE, 128, *args, 256, 256, 0, FAKE, FAKE + 1, FAKE, 256, None) == 3


def test_gather_rows_argument_errors(nv):
    L = nv._lib.nvfp4_gather_rows
    assert L(None, FAKE, 64, 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 1
    assert L(FAKE, FAKE, 64, 48, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 2  # k % 64
    assert L(FAKE, FAKE, 64, (1 << 28) + 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 2
    assert L(FAKE, FAKE, 0, 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 2   # no source
    assert L(FAKE, FAKE, 64, 64, FAKE, 64, FAKE, 0, FAKE, FAKE, FAKE, 256, None) == 1  # 0 groups
    assert L(FAKE, FAKE, 64, 64, FAKE, 64, FAKE, 300, FAKE, FAKE, FAKE, 256, None) == 1
    assert L(FAKE + 4, FAKE, 64, 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 3
    assert L(FAKE, FAKE + 2, 64, 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 256, None) == 3
    assert L(FAKE, FAKE, 64, 64, FAKE, 64, None, 0, FAKE, FAKE, FAKE, 8, None) == 7   # workspace


def test_mxfp8_and_dequant_argument_errors(nv):
    L = nv._lib
    assert L.mxfp8_quantize(FAKE, 32, 32, 32, 0, 0, 0, 0, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.mxfp8_quantize(FAKE, 32, 48, 48, 1, 0, 0, 0, FAKE, FAKE, None, None, None) == 2
    assert L.nvfp4_dequantize(FAKE, FAKE, FAKE, 16, 24, 0, 0, FAKE, None) == 2
    assert L.nvfp4_dequantize(FAKE, FAKE, FAKE, 16, 32, 0, 3, FAKE, None) == 1


def test_mxfp4_argument_errors(nv):
    L = nv._lib
    assert L.mxfp4_quantize(None, 32, 32, 32, 1, 0, FAKE, FAKE, None, None, None) == 1
    assert L.mxfp4_quantize(FAKE, 32, 32, 32, 0, 0, FAKE, FAKE, FAKE, FAKE, None) == 1   # no direction
    assert L.mxfp4_quantize(FAKE, 32, 32, 32, 4, 0, FAKE, FAKE, FAKE, FAKE, None) == 1   # unknown bit
    assert L.mxfp4_quantize(FAKE, 32, 32, 32, 2, 0, FAKE, FAKE, None, FAKE, None) == 1   # col output NULL
    assert L.mxfp4_quantize(FAKE, 48, 32, 32, 1, 0, FAKE, FAKE, None, None, None) == 2   # rows % 32
    assert L.mxfp4_quantize(FAKE, 32, 48, 48, 1, 0, FAKE, FAKE, None, None, None) == 2   # cols % 32
    assert L.mxfp4_quantize(FAKE, 32, 64, 32, 1, 0, FAKE, FAKE, None, None, None) == 2   # ld < cols
    assert L.mxfp4_quantize(FAKE + 8, 32, 32, 32, 1, 0, FAKE, FAKE, None, None, None) == 3
    assert L.mxfp4_quantize(FAKE, 32, 32, 36, 1, 0, FAKE, FAKE, None, None, None) == 3   # ld % 8
    assert L.mxfp4_quantize(FAKE, 32, 32, 32, 2, 0, None, None, FAKE + 4, FAKE, None) == 3


def test_mxfp8_gemm_argument_errors(nv):
    """The MXFP8 GEMM validates like the NVFP4 one, with K in stages of 128; the MXFP8
    tiled scale layout needs the block axis a multiple of 128."""
    L = nv._lib
    g = L.mxfp8_gemm
    args = (FAKE,) * 4
    assert g(None, FAKE, FAKE, FAKE, 128, 128, 128, 0, FAKE, 128, None, FAKE, 256, None) == 1
    assert g(*args, 128, 128, 96, 0, FAKE, 128, None, FAKE, 256, None) == 2      # K % 128
    assert g(*args, 120, 128, 128, 0, FAKE, 128, None, FAKE, 256, None) == 2     # M % 16
    assert g(*args, 128, 128, 128, 0, FAKE, 100, None, FAKE, 256, None) == 2     # ldd < N
    assert g(*args, 128, 128, 128, 1, FAKE, 132, None, FAKE, 256, None) == 3     # ldd align
    assert g(FAKE + 8, FAKE, FAKE, FAKE, 128, 128, 128, 0, FAKE, 128, None, FAKE, 256, None) == 3
    assert g(*args, 128, 128, 128, 0, FAKE, 128, None, FAKE, 8, None) == 7       # workspace
    assert g(*args, 128, 128, 128, 9, FAKE, 128, None, FAKE, 256, None) == 1     # dtype
    assert nv.mxfp8_sf_mma_bytes(128, 128) == 128 * 4
    assert nv.mxfp8_sf_mma_bytes(129, 512) == 256 * 16
    p = nv.QuantParams()
    p.mx_outputs = nv.NVFP4_ROWWISE
    p.mx_q_row = p.mx_sf_row = FAKE
    p.mx_sf_layout = nv.NVFP4_SF_MMA
    assert q(nv, 32, 96, 96, p) == 2                    # tiled MXFP8 scales need K % 128
    p.mx_sf_layout = 3
    assert q(nv, 32, 128, 128, p) == 1


def test_mxfp4_gemm_and_layout_argument_errors(nv):
    L = nv._lib
    g = L.mxfp4_gemm
    args = (FAKE,) * 4
    assert g(None, FAKE, FAKE, FAKE, 128, 128, 256, 0, FAKE, 128, None, FAKE, 256, None) == 1
    assert g(*args, 128, 128, 128, 0, FAKE, 128, None, FAKE, 256, None) == 2      # K % 256
    assert g(*args, 120, 128, 256, 0, FAKE, 128, None, FAKE, 256, None) == 2     # M % 16
    assert g(*args, 128, 128, 256, 0, FAKE, 128, None, None, 0, None) == 7       # workspace
    assert L.mxfp4_quantize(FAKE, 32, 64, 64, 1, 5, FAKE, FAKE, None, None, None) == 1  # layout
    assert L.mxfp4_quantize(FAKE, 32, 64, 64, 1, 1, FAKE, FAKE, None, None, None) == 2  # K % 128


def test_mxfp8_rowwise_alone_takes_any_row_count(nv):
    """MXFP8 rowwise without NVFP4 outputs quantises rows independently, so 17 rows pass
    validation (the call then fails only for want of a GPU); other requests keep the
    16-row rule.  And the combine validates its shapes."""
    L = nv._lib
    assert L.mxfp8_quantize(FAKE, 17, 64, 64, 1, 0, 0, 0, FAKE, FAKE, None, None, None) != 2
    assert L.mxfp8_quantize(FAKE, 17, 64, 64, 2, 0, 0, 0, None, None, FAKE, FAKE, None) == 2
    c = L.mxfp8_combine
    assert c(FAKE, FAKE, 4, 48, FAKE, FAKE, 2, 4, FAKE, None, 0, None) == 2      # cols % 32
    assert c(FAKE, FAKE, 4, 64, FAKE, FAKE, 2, 0, FAKE, None, 0, None) == 1      # k
    assert c(FAKE + 4, FAKE, 4, 64, FAKE, FAKE, 2, 4, FAKE, None, 0, None) == 3  # q alignment
    assert c(FAKE + 8, FAKE, 4, 64, FAKE, FAKE, 2, 4, FAKE, None, 0, None) == 3  # 16 bytes
    assert c(FAKE, FAKE, 4, 64, FAKE, FAKE, 0, 4, FAKE, None, 0, None) == 0      # no tokens
