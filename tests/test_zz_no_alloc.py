"""q4_matmul_batch_noalloc: the batch call whose group-sum workspace is a fixed
device array in libq4 (no device allocation).  Two consecutive calls give
exactly what q4_matmul_batch gives on the same problems (same kernels and
split; only the workspace differs), shared tiles and a SwiGLU problem
included; a call that needs more scratch than the array holds is refused
before anything is enqueued."""
import pytest
import torch

import workloads
import weight_only_bit_affine_b200 as q4
from helpers import check_matmul

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _packed(N, K, seed, tensor):
    return q4.q4_quantize(workloads.weight(N, K, seed, tensor, device=DEV))


def _problems(M, seed):
    x = workloads.activation(M, 4096, seed, 1, device=DEV)
    xd = workloads.activation(M, 11264, seed, 2, device=DEV)
    shapes = [(4096, 4096, x), (128, 4096, x), (300, 11264, xd), (1000, 4096, x)]
    probs = []
    for t, (N, K, xi) in enumerate(shapes):
        probs.append((xi, *_packed(N, K, seed, t), torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)))
    gate, up = _packed(256, 4096, seed, 10), _packed(256, 4096, seed, 11)
    probs.append((x, *gate, torch.full((M, 256), float("nan"), dtype=torch.bfloat16, device=DEV), q4.SwiGLU(*up)))
    return probs


def _fresh(probs):
    return [p[:4] + (torch.full_like(p[4], float("nan")),) + p[5:] for p in probs]


@pytest.mark.parametrize("M", [3, 8, 16])
def test_noalloc_equals_batch_on_two_consecutive_calls(M):
    probs = _problems(M, 80 + M)
    ref = [y.clone() for y in q4.q4_matmul_batch(probs)]
    for call in range(2):
        outs = q4.q4_matmul_batch_noalloc(_fresh(probs))
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(zip(outs, ref)):
            assert torch.equal(a, b), (call, i)
    x, c, s, b, y = probs[1][:5]
    check_matmul(x, c, s, b, y, what=f"noalloc 128x4096 M={M}")


def test_noalloc_refuses_a_call_larger_than_its_scratch():
    """Five launches at M = 16 (eight distinct activation tensors per launch),
    each spread over every SM with shared tiles, need more than the fixed
    array: Q4_ERR_UNSUPPORTED, and no output is written."""
    M, K, N = 16, 1024, 384
    probs = []
    for t in range(40):
        x = workloads.activation(M, K, 90, t, device=DEV)
        gate, up = _packed(N, K, 90, 2 * t), _packed(N, K, 90, 2 * t + 1)
        probs.append((x, *gate, torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV), q4.SwiGLU(*up)))
    with pytest.raises(q4.Q4Error) as err:
        q4.q4_matmul_batch_noalloc(probs)
    assert err.value.status == 4  # Q4_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert all(torch.isnan(p[4].float()).all() for p in probs)
