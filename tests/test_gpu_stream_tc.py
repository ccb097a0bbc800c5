"""Tensor-core weight streaming (three or four activation rows, K % 256 == 0,
16-byte aligned scale rows): parity with the CPU oracle.  The group-sum kernel
takes these problems by default; it is kept out of the dispatch here so that
the weight-streaming kernel runs.

A tile is R weight rows x (128 / R) segments of K in the MMA's 128 rows, with
R = 4, 8 or 16 depending on K (segments of K/32, K/16 or K/8 inputs); these
cases cover every segment count, segments that end in a half chunk (32
inputs), ragged last tiles, several problems of different shapes in one
launch, and a B operand rebuilt between problems.  The bound is the
acceptance bound |y - y_ref| <= 4e-3 * sum|x w_hat| + 1e-6; with integer
inputs every partial sum is exact, so the result must equal the oracle.
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

# K -> rows per tile (segments per row = 128 / rows): the fewest segments
# whose stage still fits three deep -- 8 up to K = 4096, 16 for 8192 and
# 11264, 32 for 12288 (segment lengths 32 .. 704).
ROWS_PER_TILE = {256: 16, 768: 16, 1024: 16, 2816: 16, 4096: 16, 8192: 8, 11264: 8, 12288: 4}


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


@pytest.mark.parametrize("K", sorted(ROWS_PER_TILE))
@pytest.mark.parametrize("M", [3, 4])
def test_stream_segment_shapes(K, M):
    R = ROWS_PER_TILE[K]
    for N in (1, R - 1, R + 1, 37 * R + 3):
        c, s, b = _packed(N, K, 50, K + N)
        x = workloads.activation(M, K, 50, 3000 + M, device=DEV)
        y = q4.q4_matmul(x, c, s, b)
        check_matmul(x, c, s, b, y, what=f"stream M={M} N={N} K={K}")


def test_stream_exact_integer_inputs():
    rng = np.random.default_rng(51)
    for (M, N, K) in [(3, 301, 4096), (4, 77, 11264), (4, 33, 2816), (3, 19, 256), (3, 5, 12288)]:
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -8.0, dtype=torch.bfloat16, device=DEV)
        x = torch.from_numpy(rng.integers(-4, 5, size=(M, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul(x, codes, s, b)
        y_ref, _ = oracle.matmul_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b))
        assert torch.equal(y.cpu(), torch.from_numpy(y_ref).to(torch.float32).to(torch.bfloat16)), (M, N, K)


def test_stream_tile_positions_exact():
    """One weight row with a distinct integer pattern per (row, segment):
    a misplaced segment, row or k pair changes the exact integer result."""
    rng = np.random.default_rng(52)
    for K in (1024, 4096, 11264):
        N = 3 * ROWS_PER_TILE[K] + 1
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        # group-varying scale 1 or 2, bias -q_mean: products and sums stay exact
        sc = rng.integers(1, 3, size=(N, K // 32)).astype(np.float32)
        s = torch.from_numpy(sc).to(torch.bfloat16).to(DEV)
        b = torch.from_numpy(-8.0 * sc).to(torch.bfloat16).to(DEV)
        x = torch.from_numpy(rng.integers(-2, 3, size=(3, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul(x, codes, s, b)
        y_ref, _ = oracle.matmul_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b))
        assert torch.equal(y.cpu(), torch.from_numpy(y_ref).to(torch.float32).to(torch.bfloat16)), K


@pytest.mark.parametrize("M", [3, 4])
def test_stream_mixed_batch_one_launch(M):
    """Problems of every segment count, ragged, in one launch; each equals its
    single call bit for bit."""
    shapes = [(4096, 4096), (130, 11264), (77, 1024), (1, 256), (2000, 2816), (9, 12288), (333, 4096), (4, 768)]
    probs, singles = [], []
    for t, (N, K) in enumerate(shapes):
        c, s, b = _packed(N, K, 53, t)
        x = workloads.activation(M, K, 53, 200 + t, device=DEV)
        probs.append((x, c, s, b, torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)))
        singles.append(q4.q4_matmul(x, c, s, b))
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_batch(probs)
    assert q4.q4_debug_launch_count() - n0 == 1
    for (x, c, s, b, out), ref, (N, K) in zip(probs, singles, shapes):
        assert torch.equal(out, ref), (N, K)
        check_matmul(x, c, s, b, out, rows=sample_rows(N, 48, seed=N + K), what=f"batch {N}x{K} M={M}")


def test_stream_mixed_batch_repeated():
    """The mixed launch above, 150 times over: the chunk count per tile
    changes between its problems, so an A slot's consecutive uses go to
    different MMA issuers; every repetition must equal the single calls
    (with one A-full barrier per slot shared by both issuers, a few percent
    of repetitions read a chunk before it was written)."""
    M = 3
    shapes = [(4096, 4096), (130, 11264), (77, 1024), (1, 256), (2000, 2816), (9, 12288), (333, 4096), (4, 768)]
    probs, singles = [], []
    for t, (N, K) in enumerate(shapes):
        c, s, b = _packed(N, K, 53, t)
        x = workloads.activation(M, K, 53, 200 + t, device=DEV)
        probs.append((x, c, s, b, torch.empty((M, N), dtype=torch.bfloat16, device=DEV)))
        singles.append(q4.q4_matmul(x, c, s, b))
    for rep in range(150):
        for p in probs:
            p[4].fill_(float("nan"))
        q4.q4_matmul_batch(probs)
        for (x, c, s, b, out), ref, (N, K) in zip(probs, singles, shapes):
            assert torch.equal(out, ref), (rep, N, K)


def test_stream_large_problem_sampled():
    """The text head shape (32000 x 4096) and a gate projection, every CTA busy."""
    for (N, K) in [(32000, 4096), (11264, 4096), (4096, 11264)]:
        c, s, b = _packed(N, K, 54, N)
        x = workloads.activation(4, K, 54, 1, device=DEV)
        y = q4.q4_matmul(x, c, s, b)
        check_matmul(x, c, s, b, y, rows=sample_rows(N, 256, seed=7), what=f"{N}x{K}")


@pytest.mark.parametrize("N,K", [(1024, 1024), (2816, 1024), (1024, 2816)])
def test_stream_step_slices(N, K):
    """Depformer step slices for four concurrent conversations: q4_matmul_step
    equals q4_matmul on the slice bit for bit, and the oracle within the bound."""
    steps = workloads.DEPFORMER_STEPS
    c, s, b = _packed(steps * N, K, 55, N + K)
    x = workloads.activation(4, K, 55, 7, device=DEV)
    for step in (0, 9, steps - 1):
        y1 = q4.q4_matmul_step(x, c, s, b, steps, step)
        sl = slice(step * N, (step + 1) * N)
        y2 = q4.q4_matmul(x, c[sl].contiguous(), s[sl].contiguous(), b[sl].contiguous())
        assert torch.equal(y1, y2), step
        check_matmul(x, c[sl], s[sl], b[sl], y1, rows=sample_rows(N, 64, seed=step), what=f"step {step} {N}x{K}")
