"""GPU parity: libq4 (through its C ABI) against the CPU oracle.

Bit-exact for codes, scales, biases, packing and reconstruction; within
|y - y_ref| <= 4e-3 * sum|x w_hat| + 1e-6 per element for the matmul; exact
where the arithmetic is exact (integer inputs).  Inputs are the seeded
Gaussians of ``workloads`` (W ~ N(0, 0.02), x ~ N(0, 1), bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import assert_quantize_bitexact, bits, check_matmul, packed_to_host, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from weight_only_bit_affine_b200 import build

    build.build()
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _quant(W):
    c, s, b = q4.q4_quantize(W)
    torch.cuda.synchronize()
    return c, s, b


# ------------------------------------------------------------------ quantize / dequantize


def test_tiny_round_trip_bitexact():
    """1024 x 1024 (seed 0): codes, scales, biases and reconstruction equal the oracle's."""
    W = workloads.weight(1024, 1024, seed=0, tensor=0).to(DEV)
    c, s, b = _quant(W)
    assert_quantize_bitexact(W, c, s, b)
    Wh = q4.q4_dequantize(c, s, b)
    hc, hs, hb = packed_to_host(c, s, b)
    assert np.array_equal(bits(Wh), oracle.dequantize(hc, hs, hb))


@pytest.mark.parametrize("N,K", [(1, 32), (3, 96), (17, 288), (64, 1024), (33, 2816), (7, 11264)])
def test_quantize_shapes_bitexact(N, K):
    W = workloads.weight(N, K, seed=7, tensor=N).to(DEV)
    c, s, b = _quant(W)
    assert_quantize_bitexact(W, c, s, b)
    hc, hs, hb = packed_to_host(c, s, b)
    assert np.array_equal(bits(q4.q4_dequantize(c, s, b)), oracle.dequantize(hc, hs, hb))


def test_quantize_edge_values_bitexact():
    """Constant groups, signed zeros, huge and tiny magnitudes, subnormals, exact ties."""
    rng = np.random.default_rng(5)
    rows = []
    rows.append(np.full(32, 0.75, np.float32))                          # constant -> s = 0
    rows.append(np.array([0.0, -0.0] * 16, np.float32))                 # signed zeros
    rows.append(np.array([0, 15, 2.5, 3.5, 0.5, 14.5, 1, 7] * 4, np.float32))  # exact code ties
    rows.append((rng.standard_normal(32) * 1e30).astype(np.float32))    # huge
    rows.append((rng.standard_normal(32) * 1e-38).astype(np.float32))   # subnormal range
    rows.append(np.concatenate([np.full(31, -1.0), [1e-3]]).astype(np.float32))
    rows.append(np.linspace(-8.5, 8.5, 32).astype(np.float32))
    W = torch.from_numpy(np.stack(rows)).to(torch.bfloat16).to(DEV)
    c, s, b = _quant(W)
    assert_quantize_bitexact(W, c, s, b)
    hc, hs, hb = packed_to_host(c, s, b)
    assert np.array_equal(bits(q4.q4_dequantize(c, s, b)), oracle.dequantize(hc, hs, hb))


def test_dequantize_arbitrary_packed_bitexact():
    """Reconstruction of arbitrary bytes and scale/bias pairs (not produced by quantize),
    including |b| >> s and s >> |b|."""
    rng = np.random.default_rng(8)
    N, K = 64, 256
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = (rng.standard_normal((N, K // 32)) * np.exp2(rng.integers(-20, 5, size=(N, K // 32)))).astype(np.float32)
    b = (rng.standard_normal((N, K // 32)) * np.exp2(rng.integers(-20, 5, size=(N, K // 32)))).astype(np.float32)
    sb = torch.from_numpy(s).to(torch.bfloat16)
    bb = torch.from_numpy(b).to(torch.bfloat16)
    out = q4.q4_dequantize(torch.from_numpy(codes).to(DEV), sb.to(DEV), bb.to(DEV))
    assert np.array_equal(bits(out), oracle.dequantize(codes, bits(sb), bits(bb)))


# ------------------------------------------------------------------ matmul


def _packed(N, K, seed, tensor):
    W = workloads.weight(N, K, seed=seed, tensor=tensor).to(DEV)
    return _quant(W)


def test_tiny_matmul():
    W = workloads.weight(1024, 1024, seed=0, tensor=0).to(DEV)
    c, s, b = _quant(W)
    x = workloads.activation(1, 1024, seed=0, tensor=1).to(DEV)
    y = q4.q4_matmul(x, c, s, b)
    check_matmul(x, c, s, b, y, what="tiny 1024x1024")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 15])
@pytest.mark.parametrize("N,K", [(1, 32), (5, 64), (37, 256), (129, 1024), (67, 2816), (61, 4096), (9, 11264),
                                 (3, 16384), (5, 288)])
def test_matmul_shapes(M, N, K):
    """Several tiles and a ragged tail in N; K on both kernel paths (bulk-copy
    tiles when K % 256 == 0, the generic path otherwise); M across chunking."""
    c, s, b = _packed(N, K, seed=11, tensor=K + N)
    x = workloads.activation(M, K, seed=11, tensor=1000 + M).to(DEV)
    y = q4.q4_matmul(x, c, s, b)
    check_matmul(x, c, s, b, y, what=f"M={M} N={N} K={K}")


def test_matmul_many_tiles_ragged():
    """N far above the CTA count so every CTA runs many pipeline stages, N ragged."""
    N, K = 148 * 9 * 4 + 3, 1024
    c, s, b = _packed(N, K, seed=12, tensor=0)
    for M in (1, 4):
        x = workloads.activation(M, K, seed=12, tensor=M).to(DEV)
        y = q4.q4_matmul(x, c, s, b)
        check_matmul(x, c, s, b, y, what=f"ragged M={M}")


def test_matmul_unaligned_scale_rows():
    """Scales/biases only 2-byte aligned (a view offset by one group): generic path."""
    N, K = 40, 1024
    W = workloads.weight(N, K, seed=13, tensor=0).to(DEV)
    c, s, b = _quant(W)
    s2 = torch.empty(N * (K // 32) + 1, dtype=torch.bfloat16, device=DEV)
    b2 = torch.empty_like(s2)
    s2[1:].copy_(s.flatten())
    b2[1:].copy_(b.flatten())
    sv, bv = s2[1:].view(N, K // 32), b2[1:].view(N, K // 32)
    x = workloads.activation(2, K, seed=13, tensor=1).to(DEV)
    y = q4.q4_matmul(x, c, sv, bv)
    check_matmul(x, c, s, b, y, what="unaligned scales")


def test_matmul_exact_integer_inputs():
    """x integer in [-4, 4], s = 1, b = -8: every partial sum is an exact integer in fp32,
    so the GPU equals the oracle exactly, whatever the summation order."""
    rng = np.random.default_rng(21)
    for (M, N, K) in [(1, 300, 4096), (3, 77, 1024), (4, 19, 11264), (2, 9, 96)]:
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -8.0, dtype=torch.bfloat16, device=DEV)
        xi = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
        x = torch.from_numpy(xi).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul(x, codes, s, b)
        y_ref, _ = oracle.matmul_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b))
        exact_bf16 = torch.from_numpy(y_ref).to(torch.float32).to(torch.bfloat16)
        assert torch.equal(y.cpu(), exact_bf16), (M, N, K)


def test_matmul_step_equals_sliced_matmul():
    """q4_matmul_step(step) is q4_matmul on rows [step*N, (step+1)*N), bit for bit."""
    steps, N, K = 16, 1024, 1024
    c, s, b = _packed(steps * N, K, seed=3, tensor=99)
    x = workloads.activation(1, K, seed=3, tensor=98).to(DEV)
    for step in (0, 1, 7, 15):
        y1 = q4.q4_matmul_step(x, c, s, b, steps, step)
        sl = slice(step * N, (step + 1) * N)
        y2 = q4.q4_matmul(x, c[sl].contiguous(), s[sl].contiguous(), b[sl].contiguous())
        assert torch.equal(y1, y2)
    check_matmul(x, c[15 * N:], s[15 * N:], b[15 * N:], y1, what="step 15")
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_matmul_step(x, c, s, b, steps, steps)
    assert e.value.status_name == "Q4_ERR_RANGE"


def test_empty_inputs():
    c, s, b = _packed(8, 64, seed=1, tensor=1)
    x0 = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    assert q4.q4_matmul(x0, c, s, b).shape == (0, 8)
    e = torch.empty((0, 32), dtype=torch.uint8, device=DEV)
    es = torch.empty((0, 2), dtype=torch.bfloat16, device=DEV)
    x = workloads.activation(2, 64, seed=1, tensor=2).to(DEV)
    assert q4.q4_matmul(x, e, es, es).shape == (2, 0)
    cq, sq, bq = q4.q4_quantize(torch.empty((0, 64), dtype=torch.bfloat16, device=DEV))
    assert cq.shape == (0, 32)


def test_errors_on_gpu():
    c, s, b = _packed(8, 64, seed=1, tensor=3)
    x = workloads.activation(1, 64, seed=1, tensor=4).to(DEV)
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_matmul(x, c, s, b, group=64)
    assert e.value.status_name == "Q4_ERR_UNSUPPORTED"


# ------------------------------------------------------------------ the five workloads


def test_temporal_layer_m1():
    """One temporal layer at M = 1: q/k/v/o 4096x4096, gate/up 11264x4096, down 4096x11264."""
    seed = workloads.seed_of("temporal_layer")
    x = workloads.activation(1, 4096, seed, 100).to(DEV)
    x_down = workloads.activation(1, 11264, seed, 101).to(DEV)
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = _packed(p.N, p.K, seed, t)
        xi = x_down if p.K == 11264 else x
        y = q4.q4_matmul(xi, c, s, b)
        check_matmul(xi, c, s, b, y, what=p.name)


def test_depformer_steps_sampled():
    """Depformer MultiLinear: each projection stacked over 16 steps; every step of every
    projection runs through q4_matmul_step; sampled rows vs the oracle."""
    seed = workloads.seed_of("depformer_steps")
    steps = workloads.DEPFORMER_STEPS
    projs = workloads.depformer_projs()
    xs = {K: workloads.activation(1, K, seed, 500 + K).to(DEV) for K in (1024, 2816)}
    for t, p in enumerate(projs):
        W = workloads.weight(steps * p.N, p.K, seed, t, device=DEV)
        c, s, b = _quant(W)
        if t in (0, 6, len(projs) - 1):  # codes of some projections checked bit-exactly
            assert_quantize_bitexact(W, c, s, b)
        del W
        for step in range(steps):
            y = q4.q4_matmul_step(xs[p.K], c, s, b, steps, step)
            if step in (0, 15) or t % 7 == step % 7:
                sl = slice(step * p.N, (step + 1) * p.N)
                rows = sample_rows(p.N, 24, seed=t * 100 + step)
                check_matmul(xs[p.K], c[sl], s[sl], b[sl], y, rows=rows, what=f"{p.name} step {step}")


@pytest.mark.parametrize("M", workloads.BATCHED_M)
def test_batched_layer_sampled(M):
    """Batched temporal projections (concurrent conversations / prefill), M in {4, 64, 256}."""
    seed = workloads.seed_of("batched_layer")
    x = workloads.activation(M, 4096, seed, 100 + M).to(DEV)
    x_down = workloads.activation(M, 11264, seed, 200 + M).to(DEV)
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = _packed(p.N, p.K, seed, t)
        xi = x_down if p.K == 11264 else x
        y = q4.q4_matmul(xi, c, s, b)
        rows = sample_rows(p.N, 48 if M > 4 else 256, seed=t)
        check_matmul(xi, c, s, b, y, rows=rows, what=f"{p.name} M={M}")
