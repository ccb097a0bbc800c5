"""Tensor-core tiles (tcgen05, M >= 16): parity with the CPU oracle.

The weights are dequantized into tensor memory as two bf16 parts (hi + lo
of fp32(s*q + b)) and multiplied with fp32 accumulation; outputs must meet
|y - y_ref| <= 4e-3 * sum|x w_hat| + 1e-6 per element.  Integer inputs
(x in [-4, 4], s = 1, b = -8) make every product and sum exact, so there the
result must equal the oracle exactly.  The group-sum kernel (which takes up to
16 rows by default) is kept out of the dispatch, so M = 16 runs on the tiles.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import bits, check_matmul, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    prev = q4.q4_debug_disable_kernels(q4.KERNEL_GROUP_SUM)
    yield
    q4.q4_debug_disable_kernels(prev)
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _packed(N, K, seed, tensor):
    return q4.q4_quantize(workloads.weight(N, K, seed, tensor, device=DEV))


def test_tc_single_tile_smoke():
    """Smallest case: one 128-row tile, 16 activation rows, one K super-chunk."""
    c, s, b = _packed(128, 256, 40, 0)
    x = workloads.activation(16, 256, 40, 1, device=DEV)
    y = q4.q4_matmul(x, c, s, b)
    torch.cuda.synchronize()
    check_matmul(x, c, s, b, y, what="tc 128x256 M=16")


@pytest.mark.parametrize("M", [16, 17, 31, 64, 100, 256, 300])
@pytest.mark.parametrize("N,K", [(1, 256), (127, 512), (129, 1024), (1000, 4096), (300, 11264)])
def test_tc_shapes(M, N, K):
    c, s, b = _packed(N, K, 41, N + K)
    x = workloads.activation(M, K, 41, 1000 + M, device=DEV)
    y = q4.q4_matmul(x, c, s, b)
    rows = sample_rows(N, 96, seed=M) if N > 96 else None
    check_matmul(x, c, s, b, y, rows=rows, what=f"tc M={M} N={N} K={K}")


def test_tc_exact_integer_inputs():
    rng = np.random.default_rng(42)
    for (M, N, K) in [(16, 128, 256), (64, 300, 4096), (256, 130, 1024), (33, 77, 11264)]:
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -8.0, dtype=torch.bfloat16, device=DEV)
        xi = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
        x = torch.from_numpy(xi).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul(x, codes, s, b)
        y_ref, _ = oracle.matmul_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b))
        exact = torch.from_numpy(y_ref).to(torch.float32).to(torch.bfloat16)
        assert torch.equal(y.cpu(), exact), (M, N, K)


def test_tc_step_slice():
    """q4_matmul_step on the tensor-core path equals q4_matmul on the slice."""
    steps, N, K, M = 4, 256, 1024, 32
    c, s, b = _packed(steps * N, K, 43, 0)
    x = workloads.activation(M, K, 43, 1, device=DEV)
    for step in (0, 3):
        y1 = q4.q4_matmul_step(x, c, s, b, steps, step)
        sl = slice(step * N, (step + 1) * N)
        y2 = q4.q4_matmul(x, c[sl].contiguous(), s[sl].contiguous(), b[sl].contiguous())
        assert torch.equal(y1, y2)
        check_matmul(x, c[sl], s[sl], b[sl], y1, rows=sample_rows(N, 32, seed=step), what=f"step {step}")


def test_tc_uses_one_launch():
    c, s, b = _packed(4096, 4096, 44, 0)
    x = workloads.activation(64, 4096, 44, 1, device=DEV)
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul(x, c, s, b)
    assert q4.q4_debug_launch_count() - n0 == 1
