"""The group-sum tensor-core kernel (3..16 activation rows, K % 256 == 0):
parity with the CPU oracle.

The kernel forms each group's sum of (128 + q) * x on the tensor cores and
applies the group's scale and bias in fp32; a launch spreads its 128-input
steps evenly over the SMs, so a 128-row tile may be shared by several CTAs,
whose fp32 partial sums the last one to finish adds in a fixed order.  These
cases cover every register class of the epilogue (M = 3, 5, 8, 12, 16), the
smallest K (one scale run), ragged last tiles, tiles shared by two and by
thirty-two and by eighty-eight CTAs, a launch in which no tile is shared, fused SwiGLU and
residual epilogues on shared tiles, launches split by entry count and by
distinct activations, exact integer arithmetic, and determinism.
Bound: |y - y_ref| <= 4e-3 * sum|x w_hat| + 1e-6 (SwiGLU and residual: the
oracle's propagated bounds)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import bits, check_matmul, packed_to_host, sample_rows

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


def _within(y, ref, bound, what):
    yg = y.float().cpu().double().numpy()
    ok = np.abs(yg - ref) <= bound
    if not ok.all():
        m, n = np.argwhere(~ok)[0]
        raise AssertionError(f"{what}: {int((~ok).sum())} out of bound, e.g. [{m},{n}] {yg[m, n]} vs {ref[m, n]}")


@pytest.mark.parametrize("M", [3, 5, 8, 12, 16])
@pytest.mark.parametrize("N,K", [(1, 256), (127, 512), (129, 1024), (300, 4096), (77, 11264), (4096, 256)])
def test_gmma_shapes(M, N, K):
    c, s, b = _packed(N, K, 70, N + K)
    x = workloads.activation(M, K, 70, M, device=DEV)
    n0 = q4.q4_debug_launch_count()
    y = q4.q4_matmul(x, c, s, b)
    assert q4.q4_debug_launch_count() - n0 == 1
    rows = None if N <= 512 else sample_rows(N, 96, seed=N)
    check_matmul(x, c, s, b, y, rows=rows, what=f"gmma M={M} {N}x{K}")


@pytest.mark.parametrize("N,K", [(128, 4096), (256, 256), (128, 11264)])
def test_gmma_shared_tiles(N, K):
    """Fewer tiles than SMs: every tile is split over several CTAs (32 for
    128 x 4096, 2 for 256 x 256, 88 for 128 x 11264)."""
    for M in (3, 16):
        c, s, b = _packed(N, K, 71, M)
        x = workloads.activation(M, K, 71, 10 + M, device=DEV)
        y = q4.q4_matmul(x, c, s, b)
        check_matmul(x, c, s, b, y, what=f"shared M={M} {N}x{K}")


def test_gmma_no_shared_tile():
    """148 tiles of two steps each: on a 148-SM device every CTA takes exactly
    one tile (no workspace); elsewhere some tiles are shared.  Either way the
    result is checked."""
    N, K, M = 148 * 128, 256, 4
    c, s, b = _packed(N, K, 72, 0)
    x = workloads.activation(M, K, 72, 1, device=DEV)
    y = q4.q4_matmul(x, c, s, b)
    check_matmul(x, c, s, b, y, rows=sample_rows(N, 256, seed=3), what="no shared tile")


@pytest.mark.parametrize("M", [3, 4, 12])
def test_gmma_exact_integers(M):
    """Integer x in [-4, 4], s = 1, b = -8: every product, group sum, partial
    and fixup sum is an exact integer, so y equals the oracle exactly, shared
    tiles included."""
    rng = np.random.default_rng(73 + M)
    for (N, K) in [(301, 4096), (128, 1024), (19, 256), (129, 11264)]:
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -8.0, dtype=torch.bfloat16, device=DEV)
        x = torch.from_numpy(rng.integers(-4, 5, size=(M, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul(x, codes, s, b)
        y_ref, _ = oracle.matmul_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b))
        assert torch.equal(y.cpu(), torch.from_numpy(y_ref).to(torch.float32).to(torch.bfloat16)), (N, K)


@pytest.mark.parametrize("M", [3, 8, 16])
def test_gmma_swiglu_and_residual_on_shared_tiles(M):
    """One SwiGLU problem of one tile (gate and up steps spread over many
    CTAs: pieces hold gate sums, up sums or both) and one residual problem."""
    for (N, K) in [(128, 4096), (200, 1024)]:
        gate, up = _packed(N, K, 74, 1), _packed(N, K, 74, 2)
        x = workloads.activation(M, K, 74, 3, device=DEV)
        h = q4.q4_matmul_swiglu(x, gate, up)
        ref, bound = oracle.matmul_swiglu_ref(bits(x), packed_to_host(*gate), packed_to_host(*up))
        _within(h, ref, bound, f"swiglu M={M} {N}x{K}")
        r = workloads.activation(M, N, 74, 4, device=DEV)
        y = q4.q4_matmul_residual(x, *gate, r)
        ref, bound = oracle.matmul_residual_ref(bits(x), *packed_to_host(*gate), bits(r))
        _within(y, ref, bound, f"residual M={M} {N}x{K}")


def _batch(specs, seed):
    """specs: (M, N, K, x key); problems with the same key share one x."""
    xs, probs = {}, []
    for t, (M, N, K, key) in enumerate(specs):
        if key not in xs:
            xs[key] = workloads.activation(M, K, seed, 1000 + len(xs), device=DEV)
        c, s, b = _packed(N, K, seed, t)
        probs.append((xs[key], c, s, b, torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)))
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_batch(probs)
    return probs, q4.q4_debug_launch_count() - n0


@pytest.mark.parametrize("case", ["entries", "activations"])
def test_gmma_launch_splits(case):
    """A batch split into launches: 170 weights (a launch's parameter block
    holds 160), 12 distinct activation tensors (a launch holds 8 tensor
    maps)."""
    if case == "entries":
        specs, launches = [(4, 16 + 9 * (t % 11), 256, 0) for t in range(170)], 2
    else:
        specs, launches = [(3, 40 + t, 256 * (1 + t % 2), t) for t in range(12)], 2
    probs, n = _batch(specs, 75)
    assert n == launches
    for t, (x, c, s, b, out) in enumerate(probs):
        if t % 3 == 0 or t == len(probs) - 1:
            check_matmul(x, c, s, b, out, what=f"{case} problem {t}")


def test_gmma_deterministic():
    """The same call twice gives the same bits (the fixup adds the pieces of a
    shared tile in piece order, whichever CTA finishes last)."""
    c, s, b = _packed(1000, 4096, 76, 0)
    x = workloads.activation(5, 4096, 76, 1, device=DEV)
    y0 = q4.q4_matmul(x, c, s, b)
    for _ in range(3):
        assert torch.equal(q4.q4_matmul(x, c, s, b), y0)


def test_gmma_temporal_layer_m8_sampled():
    """One temporal layer (7 projections, 128 MB of packed weights) at M = 8
    as one batch, sampled rows of every projection."""
    seed = workloads.seed_of("batched_layer")
    M = 8
    x = workloads.activation(M, 4096, seed, 108, device=DEV)
    xd = workloads.activation(M, 11264, seed, 208, device=DEV)
    probs = []
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = q4.q4_quantize(workloads.weight(p.N, p.K, seed, t, device=DEV))
        probs.append((xd if p.K == 11264 else x, c, s, b, torch.empty((M, p.N), dtype=torch.bfloat16, device=DEV)))
    q4.q4_matmul_batch(probs)
    for i, (xi, c, s, b, y) in enumerate(probs):
        check_matmul(xi, c, s, b, y, rows=sample_rows(y.shape[1], 24, seed=i), what=f"layer M=8 #{i}")
