"""Host-side checks of the NVFP4 linear op: argument validation happens before any
kernel is launched.  CPU only."""
import pytest
import torch


def test_rejects_cpu_tensors_and_bad_shapes():
    from nvfp4_bit_precision_b200.linear import NVFP4LinearFunction, _check
    x = torch.zeros((256, 256), dtype=torch.bfloat16)
    w = torch.zeros((256, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        NVFP4LinearFunction.apply(x, w, 0, 0)
    # shape and dtype rules, checked without a device by a stand-in for is_cuda
    class Fake:
        def __init__(self, shape, dtype=torch.bfloat16):
            self.shape, self.dtype, self.is_cuda = torch.Size(shape), dtype, True

        def dim(self):
            return len(self.shape)

    _check(Fake((512, 256)), Fake((768, 256)))                      # accepted
    with pytest.raises(ValueError, match="multiples"):
        _check(Fake((500, 256)), Fake((768, 256)))
    with pytest.raises(ValueError, match="multiples"):
        _check(Fake((512, 256)), Fake((700, 256)))
    with pytest.raises(ValueError, match="expected"):
        _check(Fake((512, 256)), Fake((768, 512)))
    with pytest.raises(ValueError, match="bfloat16"):
        _check(Fake((512, 256), torch.float32), Fake((768, 256)))
