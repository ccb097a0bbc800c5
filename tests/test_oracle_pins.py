"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, hand-worked examples, closed forms, textbook/library routines,
brute force in pure Python, or exact integer arithmetic.  No GPU.
"""
import json
import math
import os
import random
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits_of(values):
    """Exact bf16 bit patterns of bf16-representable floats (via torch)."""
    t = torch.tensor(values, dtype=torch.float32)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float32), t), "golden value not exactly representable in bf16"
    return workloads.bf16_bits(b)


def _py_bf16_to_float(h):
    """Independent bf16 decoding via struct (not the oracle's routine)."""
    return struct.unpack("<f", struct.pack("<I", int(h) << 16))[0]


# --------------------------------------------------------------------------- format


def test_packed_size_matches_model_card(oracle):
    """5 bits/weight: 4-bit codes + bf16 scale + bf16 bias per 32 (model card 'Release details')."""
    g = _load("format_sizes.json")
    P = g["parameters"]
    packed = oracle.packed_nbytes(1, P)
    assert round(packed / 2**30, g["gib_decimals"]) == g["packed_language_model_gib"]
    assert round(P * 2 / 2**30, g["gib_decimals"]) == g["source_weights_gib"]
    # The neighbouring readings do not reproduce the printed size.
    fp32_sb = P // 2 + (P // 32) * 8
    g64 = P // 2 + (P // 64) * 4
    assert round(fp32_sb / 2**30, 2) != g["packed_language_model_gib"]
    assert round(g64 / 2**30, 2) != g["packed_language_model_gib"]


def test_packed_nbytes_layout(oracle):
    for N, K in [(1, 32), (7, 64), (1024, 1024), (4096, 11264)]:
        assert oracle.packed_nbytes(N, K) == N * K // 2 + 4 * N * (K // 32)


# --------------------------------------------------------------------------- bf16


def test_bf16_rounding_matches_torch_on_fp32_values(oracle):
    """Nearest-even fp32 -> bf16 agrees with torch's conversion (a library routine)."""
    rng = np.random.default_rng(7)
    raw = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    f = raw.view(np.float32)
    f = f[np.isfinite(f)]
    # add exact ties and near-ties around a few magnitudes
    ties = np.array([1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-8 + 2**-20, -(2 + 2**-7), 3.0e38, 1e-39, -1e-40],
                    dtype=np.float32)
    f = np.concatenate([f, ties])
    expect = workloads.bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    got = np.array([oracle.bf16_from_f64(float(v)) for v in f], dtype=np.uint16)
    # torch may canonicalise NaN payloads; none are present here.
    assert np.array_equal(got, expect)


def _exact_bf16_round(v: float) -> int:
    """Brute-force nearest-even bf16 of a binary64 value with exact fractions."""
    fv = Fraction(v)
    best = None
    # candidates: all bf16 finite values near v -> search the bf16 grid around it
    approx = np.float32(v) if abs(v) < 3.3e38 else np.float32(np.sign(v) * 3.3e38)
    base = int(np.array([approx], np.float32).view(np.uint32)[0] >> 16)
    for h in range(max(0, base - 3), min(0xFFFF, base + 4)):
        for hh in (h, h | 0x8000, h & 0x7FFF):
            x = _py_bf16_to_float(hh)
            if not math.isfinite(x):
                continue
            d = abs(Fraction(x) - fv)
            key = (d, (hh & 1))  # ties -> even significand
            if best is None or key < best[0]:
                best = (key, hh)
    return best[1]


def test_bf16_rounding_of_binary64_is_exact_nearest_even(oracle):
    rng = random.Random(3)
    for _ in range(400):
        mant = rng.getrandbits(52) | (1 << 52)
        e = rng.randint(-60, 40)
        v = math.ldexp(mant, e - 52) * rng.choice([1, -1])
        assert oracle.bf16_from_f64(v) == _exact_bf16_round(v), v
    # exact ties between bf16 neighbours, in binary64
    for v in [1 + 2**-8, 1 + 3 * 2**-8, 0.40234375 - 2**-10, -0.599609375]:
        assert oracle.bf16_from_f64(v) == _exact_bf16_round(v)


# --------------------------------------------------------------------------- quantize


def _group_weights(g):
    if g.get("pattern") is None:
        return g["weights"]
    return g["pattern"] * 4


@pytest.mark.parametrize("name", [g["name"] for g in _load("hand_groups.json")["groups"]])
def test_hand_worked_groups(oracle, name):
    g = next(x for x in _load("hand_groups.json")["groups"] if x["name"] == name)
    w = _bits_of(_group_weights(g)).reshape(1, 32)
    codes, s, b = oracle.quantize(w)
    assert s[0, 0] == int(g["scale_bits"], 16)
    assert b[0, 0] == int(g["bias_bits"], 16)
    reps = 32 // (2 * len(g["code_bytes"])) if len(g["code_bytes"]) < 16 else 1
    exp_bytes = [int(c, 16) for c in g["code_bytes"]] * reps
    assert codes[0].tolist() == exp_bytes
    q = g["q"] * (32 // len(g["q"]))
    unpacked = [(codes[0, k // 2] >> (4 * (k & 1))) & 0xF for k in range(32)]
    assert unpacked == q
    deq = oracle.dequantize(codes, s, b)
    if g.get("dequant_equals_input"):
        assert np.array_equal(deq, w)
    if "dequant_bits" in g:
        exp = [int(h, 16) for h in g["dequant_bits"]] * (32 // len(g["dequant_bits"]))
        assert deq[0].tolist() == exp


def test_on_grid_round_trip_is_exact(oracle):
    """Weights already on a 4-bit grid (s a power of two, b = -8s, codes 0 and 15 present)
    come back bit-exactly, with the drawn codes."""
    rng = np.random.default_rng(11)
    N, K = 64, 256
    G = K // 32
    q = rng.integers(0, 16, size=(N, K))
    q[:, 0::32] = 0
    q[:, 1::32] = 15
    e = rng.integers(-12, -2, size=(N, G))
    s = np.ldexp(1.0, e)
    w = (np.repeat(s, 32, axis=1) * (q - 8)).astype(np.float32)
    wb = torch.from_numpy(w).to(torch.bfloat16)
    assert torch.equal(wb.to(torch.float32), torch.from_numpy(w))
    bits = workloads.bf16_bits(wb)
    codes, sc, bi = oracle.quantize(bits)
    got_q = np.zeros((N, K), np.int64)
    got_q[:, 0::2] = codes & 0xF
    got_q[:, 1::2] = codes >> 4
    assert np.array_equal(got_q, q)
    assert np.array_equal(oracle.bf16_bits_to_f64(sc), s)
    assert np.array_equal(oracle.bf16_bits_to_f64(bi), -8 * s)
    assert np.array_equal(oracle.dequantize(codes, sc, bi), bits)


def test_gaussian_reconstruction_meets_model_card_gates(oracle):
    """W ~ N(0, 0.02) [1024, 1024] (seed 0) passes the card's gates, and the error
    matches the closed form of uniform rounding error: E[e^2] = s^2/12 per weight
    (the group's min is exact, its max nearly so)."""
    gates = _load("acceptance_gates.json")
    W = workloads.weight(1024, 1024, seed=0, tensor=0)
    bits = workloads.bf16_bits(W)
    codes, s, b = oracle.quantize(bits)
    Wf = W.to(torch.float64).numpy()
    What = oracle.bf16_bits_to_f64(oracle.dequantize(codes, s, b))
    e = oracle.nrmse(Wf, What)
    c = oracle.cosine(Wf, What)
    assert e <= gates["max_nrmse_gate"]
    assert c >= gates["min_cosine_gate"]
    # closed form from the inputs alone: s_g = range_g / 15, 30 interior weights per group
    groups = Wf.reshape(1024, 32, 32)
    rng_g = groups.max(axis=2) - groups.min(axis=2)
    pred = math.sqrt(np.sum((30.0 / 12.0) * (rng_g / 15.0) ** 2) / np.sum(Wf**2))
    assert abs(e - pred) / pred < 0.06, (e, pred)
    assert 0.07 < e < 0.09 and c > 0.995
    # exact (unrounded) reconstruction is at least as close in this regime
    What64 = oracle.dequantize_f64(codes, s, b)
    assert oracle.nrmse(Wf, What64) <= e * 1.01


def test_quantize_invariants_random(oracle):
    """Per group: min -> code 0, max -> code 15, codes monotone in w, |w - w_hat| <= s/2,
    s = bf16(fp32(max - min) / 15) via numpy fp32 + torch bf16."""
    W = workloads.weight(96, 512, seed=5, tensor=1)
    bits = workloads.bf16_bits(W)
    codes, s, b = oracle.quantize(bits)
    Wf = W.to(torch.float32).numpy().reshape(96, 16, 32)
    q = np.zeros((96, 512), np.int64)
    q[:, 0::2] = codes & 0xF
    q[:, 1::2] = codes >> 4
    q = q.reshape(96, 16, 32)
    mn, mx = Wf.min(axis=2), Wf.max(axis=2)
    s32 = (mx - mn).astype(np.float32) / np.float32(15.0)
    s_exp = workloads.bf16_bits(torch.from_numpy(s32.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(s, s_exp)
    assert np.array_equal(b, workloads.bf16_bits(torch.from_numpy(mn).to(torch.bfloat16)))
    sd, bd = oracle.bf16_bits_to_f64(s), oracle.bf16_bits_to_f64(b)
    for n in range(96):
        for g in range(16):
            w = Wf[n, g]
            assert q[n, g, np.argmin(w)] == 0 and q[n, g, np.argmax(w)] == 15
            order = np.argsort(w, kind="stable")
            assert np.all(np.diff(q[n, g, order]) >= 0)
            err = np.abs(w.astype(np.float64) - (sd[n, g] * q[n, g] + bd[n, g]))
            # interior points: half a step; the max may sit a bf16-rounding of s away
            assert np.all(err <= sd[n, g] * 0.5 * (1 + 1e-12) + 15 * sd[n, g] * 2**-8)


def test_quantize_rejects_bad_input(oracle):
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.zeros((2, 48), np.uint16))
    w = np.zeros((1, 32), np.uint16)
    w[0, 3] = 0x7FC0  # NaN
    with pytest.raises(oracle.OracleError):
        oracle.quantize(w)
    c, s, b = oracle.quantize(np.zeros((0, 64), np.uint16))
    assert c.shape == (0, 32) and s.shape == (0, 2)


# --------------------------------------------------------------------------- matmul


def _py_matmul(xb, codes, s, b):
    """Pure-Python triple loop: decode nibbles and bf16 by hand, sum in binary64."""
    M, K = xb.shape
    N = codes.shape[0]
    y = [[0.0] * N for _ in range(M)]
    ad = [[0.0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            aacc = 0.0
            for k in range(K):
                byte = int(codes[n, k // 2])
                qv = (byte >> 4) if (k % 2) else (byte & 15)
                w = _py_bf16_to_float(s[n, k // 32]) * qv + _py_bf16_to_float(b[n, k // 32])
                p = _py_bf16_to_float(xb[m, k]) * w
                acc += p
                aacc += abs(p)
            y[m][n] = acc
            ad[m][n] = aacc
    return np.array(y), np.array(ad)


@pytest.mark.parametrize("M", [1, 2, 3])
@pytest.mark.parametrize("K", [32, 64, 96])
def test_matmul_brute_force_tiny(oracle, M, K):
    for N in range(1, 6):
        W = workloads.weight(N, K, seed=9, tensor=N)
        x = workloads.activation(M, K, seed=9, tensor=100 + N)
        codes, s, b = oracle.quantize(workloads.bf16_bits(W))
        xb = workloads.bf16_bits(x)
        y, ad = oracle.matmul_ref(xb, codes, s, b)
        y2, ad2 = _py_matmul(xb, codes, s, b)
        assert np.allclose(y, y2, rtol=1e-12, atol=1e-15)
        assert np.allclose(ad, ad2, rtol=1e-12, atol=1e-15)


def test_matmul_exact_integer_case(oracle):
    """x integers in [-4, 4], s = 1, b = -8: every product and sum is an exact integer."""
    rng = np.random.default_rng(21)
    M, N, K = 3, 17, 256
    q = rng.integers(0, 16, size=(N, K))
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    G = K // 32
    s = np.full((N, G), 0x3F80, np.uint16)  # 1.0
    b = np.full((N, G), 0xC100, np.uint16)  # -8.0
    xi = rng.integers(-4, 5, size=(M, K))
    xb = workloads.bf16_bits(torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16))
    y, ad = oracle.matmul_ref(xb, codes, s, b)
    exact = xi @ (q - 8).T
    assert np.array_equal(y, exact.astype(np.float64))
    assert np.array_equal(ad, (np.abs(xi) @ np.abs(q - 8).T).astype(np.float64))


def test_matmul_factored_form_agrees(oracle):
    """sum_k x*(s*q+b) == sum_g (s*sum x*q + b*sum x), binary64 both ways."""
    W = workloads.weight(40, 1024, seed=4, tensor=2)
    x = workloads.activation(3, 1024, seed=4, tensor=3)
    codes, s, b = oracle.quantize(workloads.bf16_bits(W))
    xb = workloads.bf16_bits(x)
    y, ad = oracle.matmul_ref(xb, codes, s, b)
    y2 = oracle.matmul_ref_factored(xb, codes, s, b)
    assert np.all(np.abs(y - y2) <= 1e-12 * ad)


def test_matmul_equals_dense_library_matmul(oracle):
    """With w_hat materialised exactly, the product is torch's fp64 matmul."""
    W = workloads.weight(300, 2048, seed=6, tensor=0)
    x = workloads.activation(4, 2048, seed=6, tensor=1)
    codes, s, b = oracle.quantize(workloads.bf16_bits(W))
    xb = workloads.bf16_bits(x)
    y, ad = oracle.matmul_ref(xb, codes, s, b)
    What = torch.from_numpy(oracle.dequantize_f64(codes, s, b))
    dense = (x.to(torch.float64) @ What.T).numpy()
    assert np.all(np.abs(y - dense) <= 1e-12 * ad)
    # row selection returns the same columns
    rows = [0, 299, 17, 17, 150]
    ys, ads = oracle.matmul_ref(xb, codes, s, b, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(ads, ad[:, rows])


def test_step_slice_reading(oracle):
    """Stacked [steps*N, K] weights: step t is rows [t*N, (t+1)*N) of codes, scales and
    biases alike (Swift/MLX blog, 'Depformer: per-step weight switching')."""
    steps, N, K = 4, 24, 256
    W = workloads.weight(steps * N, K, seed=3, tensor=0)
    x = workloads.activation(1, K, seed=3, tensor=1)
    codes, s, b = oracle.quantize(workloads.bf16_bits(W))
    xb = workloads.bf16_bits(x)
    full, _ = oracle.matmul_ref(xb, codes, s, b)
    for t in range(steps):
        sl = slice(t * N, (t + 1) * N)
        part, _ = oracle.matmul_ref(xb, codes[sl], s[sl], b[sl])
        assert np.array_equal(part, full[:, sl])
        # quantizing the slice on its own gives the same packed bytes (groups never cross rows)
        c2, s2, b2 = oracle.quantize(workloads.bf16_bits(W[sl]))
        assert np.array_equal(c2, codes[sl]) and np.array_equal(s2, s[sl]) and np.array_equal(b2, b[sl])


def test_tolerance_helper(oracle):
    y = np.array([[1.0, 2.0]])
    ref = np.array([[1.0, 2.01]])
    ad = np.array([[10.0, 1.0]])
    assert oracle.tolerance_ok(y, ref, ad).tolist() == [[True, False]]


def test_oracle_results_independent_of_thread_count(oracle):
    """Timing knob only: every output element is computed by one thread in a fixed order."""
    rng = np.random.default_rng(77)
    W = workloads.bf16_bits(torch.from_numpy(rng.standard_normal((96, 512)).astype(np.float32) * 0.02).to(torch.bfloat16))
    x = workloads.bf16_bits(torch.from_numpy(rng.standard_normal((2, 512)).astype(np.float32)).to(torch.bfloat16))
    n0 = oracle.max_threads()
    try:
        oracle.set_threads(1)
        c1, s1, b1 = oracle.quantize(W)
        y1, a1 = oracle.matmul_ref(x, c1, s1, b1)
        oracle.set_threads(4)
        c4, s4, b4 = oracle.quantize(W)
        y4, a4 = oracle.matmul_ref(x, c4, s4, b4)
    finally:
        oracle.set_threads(n0)
    assert np.array_equal(c1, c4) and np.array_equal(s1, s4) and np.array_equal(b1, b4)
    assert np.array_equal(y1, y4) and np.array_equal(a1, a4)
