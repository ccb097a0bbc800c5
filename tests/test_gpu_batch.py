"""q4_matmul_batch: many independent matmuls in few launches.

On the CUDA-core GEMV (1 and 2 activation rows) each problem comes out
exactly as q4_matmul computes it alone (same kernel geometry, so
bit-identical).  The group-sum kernel (3..16 rows) spreads a launch's steps
evenly over the SMs, so where a CTA boundary falls inside a tile depends on
the whole batch and the order of the fp32 partial sums with it: there each
problem is checked against the oracle bound, and the batch against itself
(a call is deterministic).
"""
import numpy as np
import pytest
import torch

import workloads
import weight_only_bit_affine_b200 as q4
from helpers import check_matmul, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0


def _packed(N, K, seed, tensor):
    return q4.q4_quantize(workloads.weight(N, K, seed, tensor, device=DEV))


@pytest.mark.parametrize("M", [1, 2, 3])
def test_batch_matches_single_calls(M):
    shapes = [(4096, 4096), (77, 1024), (5, 256), (130, 2816), (33, 11264), (9, 288), (1, 32), (300, 768)]
    probs, singles = [], []
    for t, (N, K) in enumerate(shapes):
        c, s, b = _packed(N, K, 31, t)
        x = workloads.activation(M, K, 31, 100 + t, device=DEV)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        probs.append((x, c, s, b, out))
        singles.append(q4.q4_matmul(x, c, s, b))
    q4.q4_matmul_batch(probs)
    first = [out.clone() for *_, out in probs]
    q4.q4_matmul_batch(probs)
    torch.cuda.synchronize()
    for (x, c, s, b, out), ref, again, (N, K) in zip(probs, singles, first, shapes):
        assert torch.equal(out, again), (N, K)  # deterministic
        if M <= 2:
            assert torch.equal(out, ref), (N, K)
        check_matmul(x, c, s, b, out, rows=sample_rows(N, 32, seed=N), what=f"batch {N}x{K} M={M}")
        check_matmul(x, c, s, b, ref, rows=sample_rows(N, 32, seed=N), what=f"single {N}x{K} M={M}")


def test_batch_more_than_one_launch():
    """300 problems: more than one launch's worth of descriptors."""
    K = 1024
    probs = []
    for t in range(300):
        N = 16 + (t % 7) * 5
        c, s, b = _packed(N, K, 32, t)
        x = workloads.activation(1, K, 32, 1000 + t, device=DEV)
        probs.append((x, c, s, b, torch.empty((1, N), dtype=torch.bfloat16, device=DEV)))
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_batch(probs)
    assert q4.q4_debug_launch_count() - n0 == 2
    for t in (0, 150, 255, 256, 299):
        x, c, s, b, out = probs[t]
        assert torch.equal(out, q4.q4_matmul(x, c, s, b))
        check_matmul(x, c, s, b, out, what=f"problem {t}")


def test_tall_problem_is_split_by_rows():
    """A problem taller than one launch's per-CTA reduction buffer is split along N."""
    N, K = 80_003, 4096
    c, s, b = _packed(N, K, 33, 0)
    x = workloads.activation(1, K, 33, 1, device=DEV)
    y = q4.q4_matmul(x, c, s, b)
    check_matmul(x, c, s, b, y, rows=sample_rows(N, 64, seed=1), what="tall")
    rows = np.array([75775, 75776, 75777, N - 1])  # around the split point
    check_matmul(x, c, s, b, y, rows=rows, what="tall split")


def test_batch_validation_is_all_or_nothing():
    c, s, b = _packed(64, 1024, 34, 0)
    x = workloads.activation(1, 1024, 34, 1, device=DEV)
    good = torch.zeros((1, 64), dtype=torch.bfloat16, device=DEV)
    lib = q4.lib()
    descs = (q4.MatmulDesc * 2)()
    descs[0] = q4.MatmulDesc(x.data_ptr(), c.data_ptr(), s.data_ptr(), b.data_ptr(), good.data_ptr(), 64, 1024)
    descs[1] = q4.MatmulDesc(x.data_ptr() + 8, c.data_ptr(), s.data_ptr(), b.data_ptr(), good.data_ptr(), 64, 1024)
    import ctypes

    st = lib.q4_matmul_batch(ctypes.cast(descs, ctypes.c_void_p), 2, 1, 32,
                             torch.cuda.current_stream().cuda_stream)
    assert st == 3  # Q4_ERR_ALIGN
    assert b"[1]" in lib.q4_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(good) == 0  # nothing was enqueued
    assert lib.q4_matmul_batch(None, 0, 1, 32, None) == 0


def test_temporal_stream_layer_batched():
    """One temporal layer's seven projections as one batch (one launch)."""
    seed = workloads.seed_of("temporal_layer")
    x = workloads.activation(1, 4096, seed, 100, device=DEV)
    xd = workloads.activation(1, 11264, seed, 101, device=DEV)
    probs = []
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = _packed(p.N, p.K, seed, t)
        probs.append((xd if p.K == 11264 else x, c, s, b, torch.empty((1, p.N), dtype=torch.bfloat16, device=DEV)))
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_batch(probs)
    assert q4.q4_debug_launch_count() - n0 == 1
    for (xi, c, s, b, out), p in zip(probs, workloads.TEMPORAL_LAYER):
        check_matmul(xi, c, s, b, out, what=p.name)
