"""Pins for the oracle's 8-bit variant (the same affine rule with 255 levels,
one byte per code): hand-checked groups (grid recovery, ties to even,
constant groups), the exact on-grid round trip, the uniform-rounding closed
form on Gaussian weights, invariants against numpy/torch routines, a pure-
Python brute-force matmul and an exact integer case.  No GPU."""
import numpy as np
import pytest
import torch

import workloads
from test_oracle_pins import _bits_of, _py_bf16_to_float


def _group(values):
    """One row of 32 bf16 weights from exactly representable floats."""
    assert len(values) == 32
    return _bits_of(values)[None, :]


def test_q8_packed_size(oracle):
    # 1 byte per code + a bf16 scale and a bf16 bias per 32 weights = 9 bits per weight
    assert oracle.q8_packed_nbytes(4096, 4096) == 4096 * 4096 * 9 // 8
    assert oracle.q8_packed_nbytes(3, 64) == 3 * 64 + 3 * 2 * 4


def test_q8_hand_checked_groups(oracle):
    # b = -1, s = 2^-7: w = -1 + q/128 is exact in bf16 for every q in 0..255;
    # codes 0 and 255 fix min and max, so range/255 = (255/128)/255 = 2^-7 exactly.
    qs = [0, 255, 1, 2, 127, 128, 200, 254] + list(range(3, 27))
    W = _group([-1.0 + q / 128.0 for q in qs])
    c, s, b = oracle.q8_quantize(W)
    assert _py_bf16_to_float(s[0, 0]) == 2.0 ** -7
    assert _py_bf16_to_float(b[0, 0]) == -1.0
    assert c[0].tolist() == qs
    # halfway points round to even: 2.5 -> 2, 3.5 -> 4, 254.5 -> 254 (all exact in bf16)
    vals = [-1.0, -1.0 + 255 / 128.0, -1.0 + 2.5 / 128.0, -1.0 + 3.5 / 128.0, -1.0 + 254.5 / 128.0] + [-1.0] * 27
    c, s, b = oracle.q8_quantize(_group(vals))
    assert c[0, :5].tolist() == [0, 255, 2, 4, 254]
    # constant group: scale 0, every code 0, bias the value
    c, s, b = oracle.q8_quantize(_group([0.375] * 32))
    assert s[0, 0] == 0 and c[0].tolist() == [0] * 32 and _py_bf16_to_float(b[0, 0]) == 0.375


def test_q8_on_grid_round_trip_is_exact(oracle):
    rng = np.random.default_rng(8)
    N, K = 16, 256
    q = rng.integers(0, 256, size=(N, K))
    q[:, ::32] = 0
    q[:, 1::32] = 255
    e = rng.integers(-12, -3, size=(N, K // 32))  # s = 2^e, b = -128 s
    s = np.repeat(2.0 ** e, 32, axis=1)
    W = (q - 128) * s
    Wb = workloads.bf16_bits(torch.from_numpy(W.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(oracle.bf16_bits_to_f64(Wb), W)  # the grid is exact in bf16
    c, sc, bi = oracle.q8_quantize(Wb)
    assert np.array_equal(c, q.astype(np.uint8))
    assert np.array_equal(oracle.q8_dequantize(c, sc, bi), Wb)


def test_q8_gaussian_error_matches_uniform_rounding(oracle):
    W = workloads.weight(1024, 1024, seed=0, tensor=0)
    Wb = workloads.bf16_bits(W)
    c, s, b = oracle.q8_quantize(Wb)
    W64 = oracle.bf16_bits_to_f64(Wb)
    What = oracle.q8_dequantize_f64(c, s, b)
    err2 = np.mean((What - W64) ** 2)
    s64 = np.repeat(oracle.bf16_bits_to_f64(s), 32, axis=1)
    closed = np.mean(s64 ** 2) / 12.0  # uniform rounding error over a grid of spacing s
    assert abs(err2 / closed - 1.0) < 0.06
    assert oracle.nrmse(W64, What) < 0.006  # 255 levels: ~17x below the 4-bit error
    assert oracle.cosine(W64, What) > 0.9999


def test_q8_invariants_random(oracle):
    rng = np.random.default_rng(9)
    W = torch.from_numpy(rng.normal(0, 0.05, size=(64, 512)).astype(np.float32)).to(torch.bfloat16)
    Wb = workloads.bf16_bits(W)
    c, s, b = oracle.q8_quantize(Wb)
    Wf = W.float().numpy().reshape(64, 16, 32)
    # the scale is bf16(fp32(max - min) / 255): numpy fp32 arithmetic, torch bf16 rounding
    rng32 = (Wf.max(axis=2) - Wf.min(axis=2)).astype(np.float32) / np.float32(255.0)
    s_expect = workloads.bf16_bits(torch.from_numpy(rng32.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(s, s_expect)
    cg = c.reshape(64, 16, 32)
    assert np.all(cg[np.arange(64)[:, None], np.arange(16)[None, :], Wf.argmin(axis=2)] == 0)
    # the maximum: (mx - b)/s = 255 * s32/s with the bf16 s within 2^-8 (relative) of
    # s32, i.e. in [254, 256]: code 254 or 255, and the clamp at 255 binds when the
    # scale was rounded down (it never binds with 15 levels: 15 * 2^-8 < 1/2)
    top = cg[np.arange(64)[:, None], np.arange(16)[None, :], Wf.argmax(axis=2)]
    assert np.all((top == 255) | (top == 254)) and np.mean(top == 255) > 0.5
    order = np.argsort(Wf, axis=2, kind="stable")
    assert np.all(np.diff(np.take_along_axis(cg.astype(int), order, axis=2), axis=2) >= 0)
    What = oracle.q8_dequantize_f64(c, s, b).reshape(64, 16, 32)
    sg = oracle.bf16_bits_to_f64(s)[:, :, None]
    err = np.abs(What - Wf.astype(np.float64))
    clamped = (cg == 255) & (Wf > What)
    # nearest rounding: within s/2, except above the clamped top code, where the
    # excess 255 * (s32 - s) stays below 255 * 2^-8 s < s
    assert np.all(err[~clamped] <= (sg / 2 * (1 + 1e-9) + 1e-30).repeat(32, axis=2)[~clamped])
    assert np.all(err[clamped] < sg.repeat(32, axis=2)[clamped])
    assert clamped.any()  # this sample does reach the clamp
    # the bf16 reconstruction is the nearest bf16 of the exact one
    Wd = oracle.q8_dequantize(c, s, b)
    ex = oracle.q8_dequantize_f64(c, s, b)
    assert np.array_equal(Wd, np.vectorize(oracle.bf16_from_f64)(ex).astype(np.uint16))


def _py_q8_matmul(xb, codes, s, b):
    M, K = xb.shape
    N = codes.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                w = _py_bf16_to_float(s[n, k // 32]) * int(codes[n, k]) + _py_bf16_to_float(b[n, k // 32])
                acc += _py_bf16_to_float(xb[m, k]) * w
            y[m, n] = acc
    return y


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("K", [32, 96])
def test_q8_matmul_brute_force_tiny(oracle, M, K):
    for N in range(1, 4):
        W = workloads.weight(N, K, seed=18, tensor=N)
        x = workloads.activation(M, K, seed=18, tensor=100 + N)
        c, s, b = oracle.q8_quantize(workloads.bf16_bits(W))
        xb = workloads.bf16_bits(x)
        y, _ = oracle.q8_matmul_ref(xb, c, s, b)
        assert np.allclose(y, _py_q8_matmul(xb, c, s, b), rtol=1e-12, atol=1e-15)


def test_q8_matmul_exact_integer_case(oracle):
    """x in [-2, 2], s = 1, b = -128: every product and sum is an exact integer."""
    rng = np.random.default_rng(19)
    M, N, K = 2, 11, 256
    q = rng.integers(0, 256, size=(N, K))
    s = np.full((N, K // 32), 0x3F80, np.uint16)  # 1.0
    b = np.full((N, K // 32), 0xC300, np.uint16)  # -128.0
    xi = rng.integers(-2, 3, size=(M, K))
    xb = workloads.bf16_bits(torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16))
    y, ad = oracle.q8_matmul_ref(xb, q.astype(np.uint8), s, b)
    assert np.array_equal(y, (xi @ (q - 128).T).astype(np.float64))
    assert np.array_equal(ad, (np.abs(xi) @ np.abs(q - 128).T).astype(np.float64))
