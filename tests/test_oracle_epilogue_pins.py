"""Pins for the oracle's fused-epilogue references (residual add, SwiGLU) and
their acceptance bounds: closed forms of silu, the derivative bound the
SwiGLU tolerance rests on, exact integer residuals, and brute force in pure
Python.  No GPU."""
import math

import numpy as np
import pytest
import torch

import workloads
from test_oracle_pins import _py_bf16_to_float, _py_matmul


# ----------------------------------------------------------------------------- silu


def test_silu_closed_forms(oracle):
    e = math.e
    assert oracle.silu(0.0) == 0.0
    # sigmoid(1) = e / (1 + e); sigmoid(ln 3) = 3/4; sigmoid(-ln 3) = 1/4
    assert oracle.silu(1.0) == pytest.approx(e / (1.0 + e), rel=2e-16)
    assert oracle.silu(-1.0) == pytest.approx(-1.0 / (1.0 + e), rel=2e-16)
    assert oracle.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=2e-16)
    assert oracle.silu(-math.log(3.0)) == pytest.approx(-0.25 * math.log(3.0), rel=2e-16)
    # limits: silu(z) -> z for large z, -> -0 for very negative z (no NaN)
    assert oracle.silu(800.0) == 800.0
    big_neg = oracle.silu(-800.0)
    assert big_neg == 0.0 and not math.isnan(big_neg)


def test_silu_odd_part_identity(oracle):
    """z sigmoid(z) - (-z) sigmoid(-z) = z (sigmoid(z) + sigmoid(-z) = 1)."""
    z = np.random.default_rng(3).normal(0, 4, size=1000)
    assert np.allclose(oracle.silu(z) - oracle.silu(-z), z, rtol=1e-14, atol=1e-14)


def test_silu_derivative_bound():
    """The SwiGLU tolerance uses |silu'| <= 1.1; the true maximum is 1.0998."""
    import oracle

    z = np.linspace(-30.0, 30.0, 600001)
    s = 1.0 / (1.0 + np.exp(-z))
    d = s * (1.0 + z * (1.0 - s))  # analytic derivative
    fd = np.gradient(z * s, z)  # and a finite difference, independent of the formula
    assert np.max(np.abs(fd - d)) < 1e-6
    assert 1.09 < np.max(np.abs(d)) <= oracle.SILU_LIPSCHITZ
    assert abs(z[np.argmax(d)] - 2.3994) < 1e-3


# ------------------------------------------------------------------------- residual


def test_residual_ref_exact_integers(oracle):
    """x in [-4, 4], s = 1, b = -8, integer r: y = x (q - 8)^T + r exactly."""
    rng = np.random.default_rng(31)
    M, N, K = 2, 13, 128
    q = rng.integers(0, 16, size=(N, K))
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    s = np.full((N, K // 32), 0x3F80, np.uint16)
    b = np.full((N, K // 32), 0xC100, np.uint16)
    xi = rng.integers(-4, 5, size=(M, K))
    ri = rng.integers(-50, 51, size=(M, N))
    xb = workloads.bf16_bits(torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16))
    rb = workloads.bf16_bits(torch.from_numpy(ri.astype(np.float32)).to(torch.bfloat16))
    y, bound = oracle.matmul_residual_ref(xb, codes, s, b, rb)
    assert np.array_equal(y, (xi @ (q - 8).T + ri).astype(np.float64))
    ad = (np.abs(xi) @ np.abs(q - 8).T).astype(np.float64)
    assert np.allclose(bound, 4e-3 * (ad + np.abs(ri)) + 1e-6, rtol=0, atol=1e-12)
    # selected rows pick the same columns of r
    rows = np.array([0, 5, 12])
    y2, _ = oracle.matmul_residual_ref(xb, codes, s, b, rb, rows=rows)
    assert np.array_equal(y2, y[:, rows])


# --------------------------------------------------------------------------- SwiGLU


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("K", [32, 64])
def test_swiglu_ref_brute_force_tiny(oracle, M, K):
    for N in range(1, 5):
        Wg = workloads.weight(N, K, seed=12, tensor=N)
        Wu = workloads.weight(N, K, seed=12, tensor=50 + N)
        x = workloads.activation(M, K, seed=12, tensor=100 + N)
        gate = oracle.quantize(workloads.bf16_bits(Wg))
        up = oracle.quantize(workloads.bf16_bits(Wu))
        xb = workloads.bf16_bits(x)
        h, _ = oracle.matmul_swiglu_ref(xb, gate, up)
        g, _ = _py_matmul(xb, *gate)
        u, _ = _py_matmul(xb, *up)
        for m in range(M):
            for n in range(N):
                gv = float(g[m, n])
                expect = gv / (1.0 + math.exp(-gv)) * float(u[m, n])
                assert h[m, n] == pytest.approx(expect, rel=1e-12, abs=1e-15)


def test_swiglu_bound_covers_product_and_rounding_errors(oracle):
    """Perturb g and u to either end of their product bounds, keep both
    unrounded (the one-pass form every kernel computes), round h to bf16: the
    result stays inside the bound the oracle returns (a check of the bound's
    derivation)."""
    rng = np.random.default_rng(77)
    K = 256
    for trial in range(20):
        N = 64
        Wg = workloads.weight(N, K, seed=13, tensor=trial)
        Wu = workloads.weight(N, K, seed=13, tensor=100 + trial)
        x = workloads.activation(1, K, seed=13, tensor=200 + trial)
        gate = oracle.quantize(workloads.bf16_bits(Wg))
        up = oracle.quantize(workloads.bf16_bits(Wu))
        xb = workloads.bf16_bits(x)
        h, bound = oracle.matmul_swiglu_ref(xb, gate, up)
        g, adg = oracle.matmul_ref(xb, *gate)
        u, adu = oracle.matmul_ref(xb, *up)
        tg, tu = 4e-3 * adg + 1e-6, 4e-3 * adu + 1e-6
        for _ in range(5):
            g1 = g + tg * rng.choice([-1.0, 1.0], size=g.shape)
            u1 = u + tu * rng.choice([-1.0, 1.0], size=u.shape)
            h1 = torch.from_numpy(oracle.silu(g1) * u1).to(torch.bfloat16).double().numpy()
            assert np.all(np.abs(h1 - h) <= bound), trial


def test_swiglu_ref_rows_selection(oracle):
    Wg = workloads.weight(20, 64, seed=14, tensor=1)
    Wu = workloads.weight(20, 64, seed=14, tensor=2)
    x = workloads.activation(2, 64, seed=14, tensor=3)
    gate = oracle.quantize(workloads.bf16_bits(Wg))
    up = oracle.quantize(workloads.bf16_bits(Wu))
    xb = workloads.bf16_bits(x)
    h, bound = oracle.matmul_swiglu_ref(xb, gate, up)
    rows = np.array([0, 7, 19])
    h2, bound2 = oracle.matmul_swiglu_ref(xb, gate, up, rows=rows)
    assert np.array_equal(h2, h[:, rows]) and np.array_equal(bound2, bound[:, rows])
    assert _py_bf16_to_float(0x3F80) == 1.0
