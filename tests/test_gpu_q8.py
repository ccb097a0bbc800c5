"""The 8-bit variant on the GPU: quantize and dequantize bit-exact against the
oracle (random shapes, edge values: constant groups, ties, signed zeros,
the clamped top code), and the matmul within the acceptance bound
|y - y_ref| <= 4e-3 * sum|x w_hat| + 1e-6 for one row, pairs of rows and
odd row counts, ragged N and several K (exact on integer inputs)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import bits, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _assert_q8_bitexact(W):
    c, s, b = q4.q8_quantize(W)
    oc, os_, ob = oracle.q8_quantize(bits(W))
    assert np.array_equal(bits(s), os_), "scales differ"
    assert np.array_equal(bits(b), ob), "biases differ"
    gc = c.cpu().numpy()
    assert np.array_equal(gc, oc), f"codes differ at {np.argwhere(gc != oc)[:5].tolist()}"
    Wd = q4.q8_dequantize(c, s, b)
    assert np.array_equal(bits(Wd), oracle.q8_dequantize(oc, os_, ob)), "reconstruction differs"
    return c, s, b


@pytest.mark.parametrize("N,K", [(1, 32), (7, 96), (64, 1024), (300, 2816), (33, 4096)])
def test_q8_quantize_dequantize_bitexact(N, K):
    _assert_q8_bitexact(workloads.weight(N, K, 80, N + K, device=DEV))


def test_q8_quantize_edge_values():
    rng = np.random.default_rng(81)
    K = 256
    rows = []
    rows.append(np.full(K, 0.375, np.float32))                          # constant groups
    rows.append(np.where(np.arange(K) % 2 == 0, 0.0, -0.0).astype(np.float32))  # signed zeros
    g = -1.0 + np.array([0, 255, 2.5, 3.5, 254.5] + [7] * 27) / 128.0   # ties to even
    rows.append(np.tile(g, K // 32).astype(np.float32))
    rows.append((rng.normal(0, 1, K) * 2.0 ** rng.integers(-20, 20, K)).astype(np.float32))  # wide range
    rows.append(rng.normal(0, 0.05, K).astype(np.float32))              # reaches the clamp (scale rounded down)
    W = torch.from_numpy(np.stack(rows)).to(torch.bfloat16).to(DEV)
    _assert_q8_bitexact(W)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 16])
@pytest.mark.parametrize("N,K", [(1024, 1024), (77, 2816), (300, 96), (4096, 4096), (2048, 11264)])
def test_q8_matmul_matches_oracle(M, N, K):
    W = workloads.weight(N, K, 82, N + K, device=DEV)
    c, s, b = q4.q8_quantize(W)
    x = workloads.activation(M, K, 82, 100 + M, device=DEV)
    y = q4.q8_matmul(x, c, s, b)
    rows = None if N <= 1024 else sample_rows(N, 96, seed=N)
    y_ref, absdot = oracle.q8_matmul_ref(bits(x), c.cpu().numpy(), bits(s), bits(b), rows=rows)
    yg = y.float().cpu().double().numpy()
    if rows is not None:
        yg = yg[:, rows]
    ok = oracle.tolerance_ok(yg, y_ref, absdot)
    assert ok.all(), f"{int((~ok).sum())} elements outside the bound (M={M}, {N}x{K})"


@pytest.mark.parametrize("M", [1, 2, 3])
def test_q8_matmul_exact_integers(M):
    rng = np.random.default_rng(83 + M)
    for (N, K) in [(129, 4096), (33, 1024), (5, 96)]:
        q = rng.integers(0, 256, size=(N, K))
        codes = torch.from_numpy(q.astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -128.0, dtype=torch.bfloat16, device=DEV)
        x = torch.from_numpy(rng.integers(-2, 3, size=(M, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        y = q4.q8_matmul(x, codes, s, b)
        ref, _ = oracle.q8_matmul_ref(bits(x), q.astype(np.uint8), bits(s), bits(b))
        assert torch.equal(y.cpu(), torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16)), (M, N, K)


def test_q8_empty_sizes():
    W = workloads.weight(8, 64, 84, 0, device=DEV)
    c, s, b = q4.q8_quantize(W)
    x0 = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    assert q4.q8_matmul(x0, c, s, b).shape == (0, 8)
    e = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    ce, se, be = q4.q8_quantize(e)
    assert ce.shape == (0, 64) and se.shape == (0, 2)


@pytest.mark.parametrize("M", [1, 2, 3])
def test_q8_batch_matches_single_calls(M):
    """q8_matmul_batch: the problems the bulk-copy GEMV takes (K a multiple
    of 256) share a launch and come out bit-identical to their single calls;
    a K = 96 problem runs on the warp-per-row kernel, also as alone."""
    shapes = [(4096, 4096), (77, 1024), (1, 256), (300, 2816), (33, 11264), (9, 96), (1000, 4096)]
    probs, singles = [], []
    for t, (N, K) in enumerate(shapes):
        c, s, b = q4.q8_quantize(workloads.weight(N, K, 85, t, device=DEV))
        x = workloads.activation(M, K, 85, 50 + t, device=DEV)
        probs.append((x, c, s, b, torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)))
        singles.append(q4.q8_matmul(x, c, s, b))
    n0 = q4.q4_debug_launch_count()
    q4.q8_matmul_batch(probs)
    launches = q4.q4_debug_launch_count() - n0
    # one GEMV launch per activation-row pair size, and the K = 96 problem's own launches (one per pair)
    assert launches == (2 if M != 3 else 4), launches
    for (x, c, s, b, out), ref, (N, K) in zip(probs, singles, shapes):
        assert torch.equal(out, ref), (N, K)
    x, c, s, b, y = probs[4]
    ref, absdot = oracle.q8_matmul_ref(bits(x), c.cpu().numpy(), bits(s), bits(b))
    assert oracle.tolerance_ok(y.float().cpu().double().numpy(), ref, absdot).all()


def test_q8_batch_refuses_epilogues():
    W = workloads.weight(64, 256, 86, 0, device=DEV)
    c, s, b = q4.q8_quantize(W)
    x = workloads.activation(1, 256, 86, 1, device=DEV)
    y = torch.empty((1, 64), dtype=torch.bfloat16, device=DEV)
    d = q4.MatmulDesc(x.data_ptr(), c.data_ptr(), s.data_ptr(), b.data_ptr(), y.data_ptr(), 64, 256)
    d.epilogue, d.r = q4.EPI_RESIDUAL, y.data_ptr()
    arr = (q4.MatmulDesc * 1)(d)
    import ctypes
    assert q4.lib().q8_matmul_batch(ctypes.cast(arr, ctypes.c_void_p), 1, 1, 32, None) == 4  # Q4_ERR_UNSUPPORTED


@pytest.mark.parametrize("M,K", [(1, 22528), (2, 12288), (2, 16384)])
def test_q8_widest_rows(M, K):
    """The widest rows a team of the bulk-copy GEMV holds (K = 22528 at one
    activation row, 12288 at two) and one past it at two rows (K = 16384: the
    warp-per-row kernel), against the oracle on sampled rows."""
    N = 300
    c, s, b = q4.q8_quantize(workloads.weight(N, K, 87, K + M, device=DEV))
    x = workloads.activation(M, K, 87, M, device=DEV)
    y = q4.q8_matmul(x, c, s, b)
    rows = sample_rows(N, 48, seed=K)
    y_ref, absdot = oracle.q8_matmul_ref(bits(x), c.cpu().numpy(), bits(s), bits(b), rows=rows)
    ok = oracle.tolerance_ok(y.float().cpu().double().numpy()[:, rows], y_ref, absdot)
    assert ok.all(), f"{int((~ok).sum())} elements outside the bound (M={M}, K={K})"
