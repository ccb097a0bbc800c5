"""Host-side checks of the Python binding that need no GPU: an output (or any
operand) on another device than the inputs is rejected before the C call, so
a kernel never receives another GPU's pointer.  The binding's tensor checks
are exercised with the CUDA requirement lifted (tensors on 'cpu' and 'meta'
stand for two devices) and a library stub that fails if it is ever called."""
import pytest
import torch

import weight_only_bit_affine_b200 as q4


class _NoLib:
    def __getattr__(self, name):
        raise AssertionError(f"the C library was called ({name}) despite invalid arguments")


@pytest.fixture
def fake(monkeypatch):
    def want(t, name, dtype, ndim):
        if t.dtype != dtype or t.dim() != ndim:
            raise TypeError(name)
        return t

    monkeypatch.setattr(q4, "_want", want)
    monkeypatch.setattr(q4, "lib", lambda: _NoLib())
    monkeypatch.setattr(q4.torch.cuda, "device", lambda d: __import__("contextlib").nullcontext())


def _operands(M=2, N=8, K=64, dev="meta"):
    x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    c = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    s = torch.empty((N, K // 32), dtype=torch.bfloat16, device=dev)
    return x, c, s, s.clone()


def test_matmul_out_on_another_device(fake):
    x, c, s, b = _operands()
    out = torch.empty((2, 8), dtype=torch.bfloat16, device="cpu")
    with pytest.raises(ValueError, match="on"):
        q4.q4_matmul(x, c, s, b, out=out)


def test_matmul_step_out_on_another_device(fake):
    x, c, s, b = _operands(N=32)
    out = torch.empty((2, 8), dtype=torch.bfloat16, device="cpu")
    with pytest.raises(ValueError, match="on"):
        q4.q4_matmul_step(x, c, s, b, 4, 1, out=out)


def test_weights_on_another_device(fake):
    x, c, s, b = _operands()
    with pytest.raises(ValueError, match="same device"):
        q4.q4_matmul(x, torch.empty(c.shape, dtype=c.dtype, device="cpu"), s, b)


def test_dequantize_out_on_another_device(fake):
    _, c, s, b = _operands()
    out = torch.empty((8, 64), dtype=torch.bfloat16, device="cpu")
    with pytest.raises(ValueError, match="on"):
        q4.q4_dequantize(c, s, b, out=out)


def test_batch_out_on_another_device(fake):
    x, c, s, b = _operands()
    out = torch.empty((2, 8), dtype=torch.bfloat16, device="cpu")
    with pytest.raises(ValueError, match="on"):
        q4.q4_matmul_batch([(x, c, s, b, out)])


def test_empty_batch_needs_no_library(fake):
    assert q4.q4_matmul_batch([]) == []
    assert q4.q4_prepare_batch([]) is None


def test_disable_kernels_round_trip():
    """The dispatch mask is host state: set, read back, restored (no GPU)."""
    prev = q4.q4_debug_disable_kernels(q4.KERNEL_GROUP_SUM | q4.KERNEL_TILES)
    try:
        assert q4.q4_debug_disable_kernels(q4.KERNEL_WEIGHT_STREAM) == q4.KERNEL_GROUP_SUM | q4.KERNEL_TILES
        assert q4.q4_debug_disable_kernels(0) == q4.KERNEL_WEIGHT_STREAM
    finally:
        q4.q4_debug_disable_kernels(prev)
