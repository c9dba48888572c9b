"""The MoE expert forward at full size (64 experts, hidden 4096, FFN 1536, 16384
tokens, top-4 with Zipf(1.1) expert counts: 65536 routed rows) through the
benchmark's calls: the tokens quantised once, dispatched into the grouped layout
(nvfp4_gather_rows), the grouped up projection with amax_out, the requantisation of
its output with that amax, and -- at the down projection's full shape, on random
codes and scales -- the grouped down GEMM.  The oracle checks sampled rows; every
oracle input is generated here, never read back from the GPU."""
import numpy as np
import pytest

import workloads as W
from gpu_util import (check_gemm, cuda_available, grouped_padded_rows, host,
                      rowmajor_to_sf_mma, sf_mma_to_rowmajor, to_dev)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

T, HID, FFN, E, TOPK = 16384, 4096, 1536, 64, 4


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


@pytest.fixture(scope="module")
def moe(nv):
    import torch
    rng = np.random.default_rng(3)
    _, row_token, offsets = W.moe_routing(rng, T, E, TOPK)
    x = W.f32_to_bf16_bits(rng.standard_normal((T, HID)).astype(np.float32))
    w_up = W.f32_to_bf16_bits(rng.standard_normal((E, FFN, HID)).astype(np.float32) * 0.02)
    off = torch.from_numpy(offsets.astype(np.int32)).cuda()
    rt = torch.from_numpy(row_token.astype(np.int32)).cuda()
    mma = nv.NVFP4_SF_MMA
    tq = nv.quantize(to_dev(x), sf_layout=mma)["row"]
    A = nv.gather_rows(tq, rt, off)
    wq = [nv.quantize(to_dev(w_up[e]), sf_layout=mma)["row"] for e in range(E)]
    qb = torch.stack([t.q for t in wq])
    sfb = torch.cat([t.sf for t in wq])
    gb = torch.cat([t.g for t in wq])
    am = torch.zeros(2, dtype=torch.float32, device="cuda")
    H = nv.grouped_gemm(off, A, qb, sfb, gb, FFN, nv.NVFP4_OUT_BF16, amax_out=am)
    kw = dict(group_offsets=off, num_groups=E, sf_layout=mma)
    Hq = nv.quantize(H, amax=am, **kw)["row"]
    Hq_own = nv.quantize(H, **kw)["row"]
    return dict(x=x, w_up=w_up, offsets=offsets, row_token=row_token, A=A, H=H, am=am, Hq=Hq,
                Hq_own=Hq_own)


def _sample_rows(offsets):
    """First, middle and last routed row of the largest, the smallest non-empty and
    expert 17's groups."""
    counts = np.diff(offsets)
    nonempty = np.where(counts > 0)[0]
    experts = {int(np.argmax(counts)), int(nonempty[np.argmin(counts[nonempty])]), 17}
    rows = set()
    for e in experts:
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            rows |= {lo, hi - 1, (lo + hi) // 2}
    return sorted(rows)


def _token_row(orc, x, t, amax):
    """Oracle NVFP4 of token row t (the row repeated to a 16-row tile)."""
    xr = np.ascontiguousarray(np.tile(x[t], (16, 1)))
    return orc.nvfp4_quantize(xr, 0, amax=amax)


def test_dispatched_rows_bitexact(nv, orc, moe):
    offsets, x, rt = moe["offsets"], moe["x"], moe["row_token"]
    R = int(offsets[-1])
    am = (orc.amax(x, 0), 0.0)
    A = moe["A"]
    sf = sf_mma_to_rowmajor(host(A.sf), R, HID, grouped_padded_rows(offsets))
    for r in _sample_rows(offsets):
        q, s, g = _token_row(orc, x, rt[r], am)
        np.testing.assert_array_equal(host(A.q[r]), q[0])
        np.testing.assert_array_equal(sf[r], s[0])
        assert float(host(A.g)[0]) == g


def test_up_projection_sampled_rows(nv, orc, moe):
    offsets, x, rt, w_up = moe["offsets"], moe["x"], moe["row_token"], moe["w_up"]
    am = (orc.amax(x, 0), 0.0)
    H = W.bf16_bits_to_f32(host(moe["H"]))
    for r in _sample_rows(offsets):
        e = int(np.searchsorted(offsets, r, side="right") - 1)
        qb, sb, gb = orc.nvfp4_quantize(w_up[e], 0)
        qa, sa, ga = _token_row(orc, x, rt[r], am)
        Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, gb, rows_sel=[0])
        check_gemm(H[r:r + 1], Dr, Ar, True)


def test_up_projection_amax_out_and_requantisation(nv, moe):
    """amax_out is max |H| over the stored bf16 output; requantising H with it gives the
    bytes of the quantiser's own amax pass."""
    H = W.bf16_bits_to_f32(host(moe["H"]))
    assert host(moe["am"])[0] == np.max(np.abs(H)).astype(np.float32)
    for f in ("q", "sf", "g"):
        assert np.array_equal(host(getattr(moe["Hq"], f)), host(getattr(moe["Hq_own"], f)))


def test_down_projection_full_shape(nv, orc, moe):
    """The grouped down GEMM at its full shape (65536 routed rows, K 1536 -> N 4096) on
    random codes and in-range scale bytes, with the MoE's group offsets; sampled rows."""
    import torch
    offsets = moe["offsets"]
    R = int(offsets[-1])
    rng = np.random.default_rng(21)
    qa = rng.integers(0, 256, (R, FFN // 2), dtype=np.uint8)
    sa = rng.integers(0x28, 0x48, (R, FFN // 16), dtype=np.uint8)
    qb = rng.integers(0, 256, (E, HID, FFN // 2), dtype=np.uint8)
    sb = rng.integers(0x28, 0x48, (E, HID, FFN // 16), dtype=np.uint8)
    gb = (rng.random(E) + 0.5).astype(np.float32)
    ga = np.float32(0.75)
    pr = grouped_padded_rows(offsets)
    total_padded = int(sum(((c + 127) // 128) * 128 for c in np.diff(offsets)))
    dev = dict(device="cuda")
    A = nv.NVFP4Tensor(torch.from_numpy(qa).to(**dev),
                       torch.from_numpy(rowmajor_to_sf_mma(sa, R, FFN, pr, total_padded)).to(**dev),
                       torch.tensor([ga], **dev), R, FFN, nv.NVFP4_SF_MMA)
    sfb = np.concatenate([rowmajor_to_sf_mma(sb[e], HID, FFN) for e in range(E)])
    off = torch.from_numpy(offsets.astype(np.int32)).to(**dev)
    D = nv.grouped_gemm(off, A, torch.from_numpy(qb).to(**dev), torch.from_numpy(sfb).to(**dev),
                        torch.from_numpy(gb).to(**dev), HID, nv.NVFP4_OUT_BF16)
    D = W.bf16_bits_to_f32(host(D))
    for r in _sample_rows(offsets):
        e = int(np.searchsorted(offsets, r, side="right") - 1)
        Dr, Ar = orc.nvfp4_gemm_rows(qa[r:r + 1], sa[r:r + 1], float(ga), qb[e], sb[e],
                                     float(gb[e]), rows_sel=[0])
        check_gemm(D[r:r + 1], Dr, Ar, True)


def test_up_projection_every_expert(nv, orc, moe):
    """The first and last routed row of every non-empty expert (the group boundaries of
    the device-built tile table), against 32 columns of that expert's output: the first
    16 and 16 at an offset that moves with the expert."""
    offsets, x, rt, w_up = moe["offsets"], moe["x"], moe["row_token"], moe["w_up"]
    import torch
    am = (orc.amax(x, 0), 0.0)
    H = moe["H"]
    checked = 0
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        c1 = 256 * (e % 6) + 16 * (e % 16)
        amw = orc.amax(w_up[e], 0)
        qs = [orc.nvfp4_quantize(np.ascontiguousarray(w_up[e][c:c + 16]), 0, amax=(amw, amw))
              for c in (0, c1)]
        qb = np.concatenate([t[0] for t in qs])
        sb = np.concatenate([t[1] for t in qs])
        cols = torch.from_numpy(np.concatenate([np.arange(16), np.arange(c1, c1 + 16)])).cuda()
        for r in sorted({lo, hi - 1}):
            qa, sa, ga = _token_row(orc, x, rt[r], am)
            Dr, Ar = orc.nvfp4_gemm_rows(qa, sa, ga, qb, sb, qs[0][2], rows_sel=[0])
            got = W.bf16_bits_to_f32(host(H[r][cols]))[None, :]
            check_gemm(got, Dr, Ar, True)
            checked += 1
    assert checked >= 2 * int(np.count_nonzero(np.diff(offsets) > 1))


def test_down_projection_every_expert(nv, orc, moe):
    """The grouped down GEMM at its full shape on random codes and in-range scale bytes:
    the first and last row of every non-empty expert, every output column."""
    import torch
    offsets = moe["offsets"]
    R = int(offsets[-1])
    rng = np.random.default_rng(22)
    qa = rng.integers(0, 256, (R, FFN // 2), dtype=np.uint8)
    sa = rng.integers(0x28, 0x48, (R, FFN // 16), dtype=np.uint8)
    qb = rng.integers(0, 256, (E, HID, FFN // 2), dtype=np.uint8)
    sb = rng.integers(0x28, 0x48, (E, HID, FFN // 16), dtype=np.uint8)
    gb = (rng.random(E) + 0.5).astype(np.float32)
    ga = np.float32(1.25)
    pr = grouped_padded_rows(offsets)
    total_padded = int(sum(((c + 127) // 128) * 128 for c in np.diff(offsets)))
    dev = dict(device="cuda")
    A = nv.NVFP4Tensor(torch.from_numpy(qa).to(**dev),
                       torch.from_numpy(rowmajor_to_sf_mma(sa, R, FFN, pr, total_padded)).to(**dev),
                       torch.tensor([ga], **dev), R, FFN, nv.NVFP4_SF_MMA)
    sfb = np.concatenate([rowmajor_to_sf_mma(sb[e], HID, FFN) for e in range(E)])
    off = torch.from_numpy(offsets.astype(np.int32)).to(**dev)
    D = nv.grouped_gemm(off, A, torch.from_numpy(qb).to(**dev), torch.from_numpy(sfb).to(**dev),
                        torch.from_numpy(gb).to(**dev), HID, nv.NVFP4_OUT_BF16)
    D = W.bf16_bits_to_f32(host(D))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for r in sorted({lo, hi - 1}) if hi > lo else ():
            Dr, Ar = orc.nvfp4_gemm_rows(qa[r:r + 1], sa[r:r + 1], float(ga), qb[e], sb[e],
                                         float(gb[e]), rows_sel=[0])
            check_gemm(D[r:r + 1], Dr, Ar, True)
