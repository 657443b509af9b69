"""The Python binding rejects caller-supplied buffers of the wrong dtype, shape, device or
layout before any kernel could write through their pointers (CPU only: stand-in tensors
that describe CUDA buffers, no GPU and no library call)."""
import pytest
import torch

from lm_head_linear_gemm_b200 import _abi

CUDA0 = torch.device("cuda", 0)
CUDA1 = torch.device("cuda", 1)


class Buf:
    """Describes a CUDA tensor without allocating one."""

    def __init__(self, shape, dtype, device=CUDA0, contiguous=True):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = device
        self.is_cuda = device.type == "cuda"
        self._contiguous = contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def is_contiguous(self):
        return self._contiguous

    def data_ptr(self):
        raise AssertionError("the binding must reject this buffer before using its pointer")


N, D, V = 64, 128, 1024


def inputs():
    return (Buf((N, D), torch.bfloat16), Buf((V, D), torch.bfloat16),
            Buf((N,), torch.int64))


@pytest.mark.parametrize("dX,dW,err", [
    (Buf((N, D), torch.float32), None, TypeError),            # dX must be bf16
    (None, Buf((V, D), torch.float16), TypeError),            # dW must be fp32 or bf16
    (None, Buf((V - 8, D), torch.float32), ValueError),       # dW rows must be Vpad
    (Buf((N, D + 8), torch.bfloat16), None, ValueError),      # dX shape
    (None, Buf((V, D), torch.float32, contiguous=False), ValueError),
    (None, Buf((V, D), torch.float32, device=CUDA1), ValueError),
    (None, Buf((V, D), torch.float32, device=torch.device("cpu")), ValueError),
])
def test_forward_rejects_bad_gradient_buffers(dX, dW, err):
    X, W, t = inputs()
    with pytest.raises(err):
        _abi.forward(X, W, t, 1000, 15.0, -1, True, dX=dX, dW=dW)


def test_forward_rejects_mixed_devices_and_bad_workspace():
    X, W, t = inputs()
    with pytest.raises(ValueError):
        _abi.forward(X, Buf((V, D), torch.bfloat16, device=CUDA1), t, 1000)
    with pytest.raises(ValueError):
        _abi.forward(X, W, t, 1000, workspace=Buf((1 << 20,), torch.float32))
    with pytest.raises(ValueError):
        _abi.forward(X, W, t, 1000, workspace=Buf((16, 1 << 16), torch.uint8))


def test_forward_dp_needs_a_device_count():
    X, W, t = inputs()
    with pytest.raises(TypeError):
        _abi.forward_dp(X, W, t, Buf((1,), torch.int32), 1000)
    with pytest.raises(TypeError):
        _abi.forward_dp(X, W, t, Buf((2,), torch.int64), 1000)
    with pytest.raises(TypeError):
        _abi.forward_dp(X, W, t, None, 1000)


def test_backward_checks_lse_and_upstream_gradient():
    X, W, t = inputs()
    with pytest.raises(ValueError):
        _abi.backward(X, W, t, Buf((N + 1,), torch.float32), 1000)
    with pytest.raises(TypeError):
        _abi.backward(X, W, t, Buf((N,), torch.bfloat16), 1000)
    with pytest.raises(TypeError):
        _abi.backward(X, W, t, Buf((N,), torch.float32), 1000,
                      grad_out=Buf((1,), torch.float64))


def test_fp8_forward_checks_codes_scales_and_copies():
    X, W, t = inputs()
    X8, W8 = Buf((N, D), torch.uint8), Buf((V, D), torch.uint8)
    s = Buf((), torch.float32)
    with pytest.raises(TypeError):
        _abi.forward_fp8(X8, W8, None, s, X, W, t, 1000)
    with pytest.raises(TypeError):
        _abi.forward_fp8(X8, W8, Buf((2,), torch.float32), s, X, W, t, 1000)
    with pytest.raises(ValueError):
        _abi.forward_fp8(X8, Buf((V, D + 8), torch.uint8), s, s, X, W, t, 1000)
    with pytest.raises(ValueError):   # bf16 copies must match the codes' shape
        _abi.forward_fp8(X8, W8, s, s, Buf((N, D), torch.bfloat16),
                         Buf((V - 8, D), torch.bfloat16), t, 1000, want_grads=True)


def test_rmsnorm_checks_its_buffers():
    H, g = Buf((N, D), torch.bfloat16), Buf((D,), torch.bfloat16)
    with pytest.raises(ValueError):
        _abi.rmsnorm_forward(H, Buf((D + 8,), torch.bfloat16))
    with pytest.raises(TypeError):
        _abi.rmsnorm_forward(H, g, rstd=Buf((N,), torch.float16))
    with pytest.raises(TypeError):
        _abi.rmsnorm_backward(H, g, Buf((N,), torch.float32), Buf((N, D), torch.float32))
    with pytest.raises(TypeError):
        _abi.rmsnorm_backward(H, g, Buf((N,), torch.float32), Buf((N, D), torch.bfloat16),
                              dgamma=Buf((D,), torch.bfloat16))


def test_rmsnorm_head_checks_its_buffers():
    H, g, W = Buf((N, D), torch.bfloat16), Buf((D,), torch.bfloat16), Buf((V, D), torch.bfloat16)
    t = Buf((N,), torch.int64)
    with pytest.raises(ValueError):
        _abi.forward_rmsnorm(H, Buf((D - 8,), torch.bfloat16), W, t, 1000)
    with pytest.raises(TypeError):
        _abi.forward_rmsnorm(H, g, W, t, 1000, want_grads=True, dgamma=Buf((D,), torch.bfloat16))
    with pytest.raises(ValueError):
        _abi.forward_rmsnorm(H, g, W, t, 1000, want_grads=True, dH=Buf((N, D + 8), torch.bfloat16))
    with pytest.raises(TypeError):
        _abi.forward_rmsnorm(H, g, W, t, 1000, want_grads=True, dW=Buf((V, D), torch.float16))


def test_quantiser_checks_outputs():
    x = Buf((N, D), torch.bfloat16)
    with pytest.raises(TypeError):
        _abi.quantize_e4m3(x, out=Buf((N, D), torch.int8))
    with pytest.raises(TypeError):
        _abi.quantize_e4m3(x, scale=Buf((), torch.float64))
