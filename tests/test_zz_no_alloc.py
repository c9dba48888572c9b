"""The allocation-free quantiser entry point, nvfp4_quantize_noalloc.

It exists for callers that must not allocate device memory at the call site (a host
framework whose GPU memory is all held by its own caching allocator, or a latency-critical
path that must never reach cudaMalloc).  Its scratch is an array compiled into the
library, shared by every call.  This test calls it twice in a row through the C ABI, on
two different tensors, and requires both results to equal the workspace-taking
nvfp4_quantize bit for bit: the second call would differ if the shared array kept the
first call's amax.  The file is named so that pytest collects it last."""
import numpy as np
import pytest

import workloads as W
from gpu_util import cuda_available, host, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def _outputs(torch, rows, cols):
    u8 = dict(dtype=torch.uint8, device="cuda")
    return [torch.empty((rows, cols // 2), **u8), torch.empty((rows, cols // 16), **u8),
            torch.empty(1, dtype=torch.float32, device="cuda"),
            torch.empty((cols, rows // 2), **u8), torch.empty((cols, rows // 16), **u8),
            torch.empty(1, dtype=torch.float32, device="cuda")]


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import nvfp4_bit_precision_b200 as nv
    rows, cols = 256, 384
    big = W.heavy_tailed(11, rows, cols, scale=1.0)     # large amax first ...
    small = W.heavy_tailed(12, rows, cols, scale=1e-3)  # ... then a much smaller one
    p = nv.QuantParams()
    p.outputs = nv.NVFP4_ROWWISE | nv.NVFP4_COLWISE
    p.rounding, p.rht_colwise, p.seed = nv.NVFP4_SR, 1, 42
    for x in (big, small):
        xd = to_dev(x)
        ref = _outputs(torch, rows, cols)
        ws = torch.empty(256, dtype=torch.uint8, device="cuda")
        nv.nvfp4_quantize(xd, rows, cols, cols, p, *ref, ws, ws.numel())
        got = _outputs(torch, rows, cols)
        nv.nvfp4_quantize_noalloc(xd, rows, cols, cols, p, *got)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            np.testing.assert_array_equal(host(a), host(b))
        assert nv.nvfp4_workspace_status(ws) == 0
        assert nv.nvfp4_quantize_noalloc_status() == 0  # the shared array's status word
