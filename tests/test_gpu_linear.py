"""GPU parity of the NVFP4 linear autograd op: y, dX and dW against the oracle's FP64
GEMMs of operands the oracle quantised itself from the same bf16 x, W and dY
(x rowwise RNE; W 2D; dY rowwise SR and columnwise Hadamard SR; x columnwise
Hadamard), checked in full, plus the offset that makes stochastic rounding differ
between steps."""
import numpy as np
import pytest

import workloads as W
from gpu_util import check_gemm, cuda_available, host, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

SEED, OFFSET = 77, 5


@pytest.fixture(scope="module")
def nv():
    import nvfp4_bit_precision_b200 as nv
    return nv


@pytest.mark.parametrize("tokens,hin,hout", [(512, 256, 768), (256, 512, 256)])
def test_linear_forward_backward(nv, orc, tokens, hin, hout):
    import torch
    from nvfp4_bit_precision_b200.linear import nvfp4_linear
    rng = np.random.default_rng(tokens + hin + hout)
    x = W.f32_to_bf16_bits(rng.standard_normal((tokens, hin)).astype(np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((hout, hin)).astype(np.float32) * 0.02)
    dy = W.f32_to_bf16_bits(W.student_t(rng, (tokens, hout), 3.0, 1.0))
    xt = to_dev(x).requires_grad_(True)
    wt = to_dev(w).requires_grad_(True)
    y = nvfp4_linear(xt, wt, SEED, OFFSET)
    y.backward(to_dev(dy))
    torch.cuda.synchronize()
    f32 = lambda t: W.bf16_bits_to_f32(host(t))

    qx, sx, gx = orc.nvfp4_quantize(x, 0)
    qw, sw, gw = orc.nvfp4_quantize(w, 0, scaling=1)
    Dr, Ar = orc.nvfp4_gemm_rows(qx, sx, gx, qw, sw, gw)
    check_gemm(f32(y.detach()), Dr, Ar, True)

    qdr, sdr, gdr = orc.nvfp4_quantize(dy, 0, rounding=1, seed=SEED, offset=OFFSET)
    qwc, swc, gwc = orc.nvfp4_quantize(w, 1, scaling=1)
    Dr, Ar = orc.nvfp4_gemm_rows(qdr, sdr, gdr, qwc, swc, gwc)
    check_gemm(f32(xt.grad), Dr, Ar, True)

    qdc, sdc, gdc = orc.nvfp4_quantize(dy, 1, rounding=1, rht=1, seed=SEED, offset=OFFSET)
    qxc, sxc, gxc = orc.nvfp4_quantize(x, 1, rht=1, seed=SEED)
    Dr, Ar = orc.nvfp4_gemm_rows(qdc, sdc, gdc, qxc, sxc, gxc)
    check_gemm(f32(wt.grad), Dr, Ar, True)


def test_module_advances_the_rounding_offset(nv):
    """Two backward passes of the same layer on the same dY round differently (fresh
    Philox counters), while the forward output is unchanged."""
    import torch
    from nvfp4_bit_precision_b200.linear import NVFP4Linear
    torch.manual_seed(0)
    layer = NVFP4Linear(256, 256, device="cuda", seed=3)
    x = torch.randn((256, 256), device="cuda").to(torch.bfloat16)
    dy = torch.randn((256, 256), device="cuda").to(torch.bfloat16)
    grads, outs = [], []
    for _ in range(2):
        layer.weight.grad = None
        y = layer(x)
        y.backward(dy)
        outs.append(y.detach().clone())
        grads.append(layer.weight.grad.clone())
    assert layer.offset == 2
    assert torch.equal(outs[0], outs[1])
    assert not torch.equal(grads[0], grads[1])
