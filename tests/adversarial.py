"""Adversarial inputs for the matmul tolerance (test infrastructure).

The acceptance bound |y - y_ref| <= 4e-3 * sum_k |x_k w_hat_k| + 1e-6 leaves
little room beyond the bf16 output rounding (up to 2^-8 of |y|, about 3.9e-3
of it), so it is hardest to meet when every product x_k * w_hat_k has the
same sign (then |y| = sum |x w_hat|) and every other error of the kernel
points the same way.  These families build such inputs directly as packed
weights (codes, scales, biases) -- any bytes are a valid packed weight -- and
activations:

* every output row n sees products of one sign per input k (sigma_k), so
  x_k = sigma_k * |x_k| makes all products non-negative for every row;
* each code q is chosen, among those giving w_hat = s*q + b of sign sigma_k,
  from the ones whose rounding to bf16 moves w_hat furthest away from zero
  (at least 3/4 of the group's largest such step): a kernel that rounded
  w_hat to bf16 would then err in the same direction, by nearly a full
  half-unit, on most products.

Families:
  "aligned"   groups straddling zero (b = -s * U(3, 12)), mixed signs sigma_k;
  "big_bias"  |b| >> 15 s (b = 2^U(7, 9) * s, positive): w_hat ~ b, where
              the bf16 rounding of s*q + b loses most of s*q;
  "positive"  b > 0, all w_hat and x positive: long same-sign sums (the
              accumulation's worst case at large K).

The choice of codes uses the oracle's bf16 reconstruction of every code of
every group (oracle.dequantize), so it depends on nothing in the CUDA path.
Seeds make every input reproducible.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

FAMILIES = ("aligned", "big_bias", "positive")


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """Nearest bf16 bit patterns of float32 values (ties to even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


def _pack(q: np.ndarray) -> np.ndarray:
    """Codes [N, K] (0..15) -> packed bytes [N, K/2], low nibble = even k."""
    q = q.astype(np.uint8)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)


def _scales_biases(family: str, N: int, G: int, rng) -> tuple:
    s = 2.0 ** rng.uniform(-9.0, -6.0, size=(N, G))  # 0.002 .. 0.016, the scale of N(0, 0.02) groups
    s_bits = _bf16_bits(s * (1.0 + rng.uniform(0.0, 1.0, size=(N, G))))  # all significand bits in use
    s = _f64(s_bits)
    if family == "aligned":
        b = -s * rng.uniform(3.0, 12.0, size=(N, G))
    elif family == "big_bias":
        b = s * 2.0 ** rng.uniform(7.0, 9.0, size=(N, G))
    elif family == "positive":
        b = s * rng.uniform(0.5, 4.0, size=(N, G))
    else:
        raise ValueError(family)
    return s_bits, _bf16_bits(b)


def packed_weight(family: str, N: int, K: int, seed: int, sigma: np.ndarray):
    """(codes [N, K/2], scales, biases [N, K/32]) whose w_hat[n, k] has sign
    sigma[k] (+1 or -1) wherever the group allows it, with codes chosen so the
    bf16 rounding of w_hat moves it away from zero as far as the group allows."""
    rng = np.random.default_rng(seed)
    G = K // 32
    s_bits, b_bits = _scales_biases(family, N, G, rng)
    s, b = _f64(s_bits), _f64(b_bits)
    # w_hat for every code 0..15 of every group, exactly and rounded to bf16
    # by the oracle: a probe weight whose group g holds the codes 0..15.
    probe = np.zeros((N, G, 32), np.uint8)
    probe[:, :, :16] = np.arange(16, dtype=np.uint8)
    rec = _f64(oracle.dequantize(_pack(probe.reshape(N, K)), s_bits, b_bits)).reshape(N, G, 32)[:, :, :16]
    exact = s[:, :, None] * np.arange(16.0)[None, None, :] + b[:, :, None]
    # rounding away from zero, relative to |w_hat| (up to 2^-8)
    rel_up = np.where(exact != 0, (rec - exact) / np.where(exact == 0, 1.0, exact), -1.0)
    sig = sigma.reshape(G, 32)
    q = np.zeros((N, G, 32), np.int64)
    u = rng.random((N, G, 32, 16))  # random choice among the allowed codes
    for sgn in (-1.0, 1.0):
        sign_ok = np.sign(exact) == sgn
        r = np.where(sign_ok, rel_up, -np.inf)
        best = r.max(axis=2, keepdims=True)
        # allowed: codes of this sign rounding up by at least 3/4 of the group's
        # largest such step (or, where none rounds up, any code of this sign)
        allowed = sign_ok & np.where(best > 0, r >= 0.75 * best, True)
        for j in range(32):
            pick = np.argmax(np.where(allowed, 1.0 + u[:, :, j, :], 0.0), axis=2)
            q[:, :, j] = np.where(sig[:, j][None, :] == sgn, pick, q[:, :, j])
    return _pack(q.reshape(N, K)), s_bits, b_bits


def signs(family: str, K: int, seed: int) -> np.ndarray:
    """The per-input sign pattern sigma_k of a family."""
    if family == "aligned":
        return np.where(np.random.default_rng(seed + 1).random(K) < 0.5, -1.0, 1.0)
    return np.ones(K)


def activation(M: int, K: int, seed: int, sigma: np.ndarray) -> np.ndarray:
    """x [M, K] bf16 bits: |N(0, 1)| (at least 2^-4) times sigma_k."""
    rng = np.random.default_rng(seed + 2)
    mag = np.maximum(np.abs(rng.standard_normal((M, K))), 2.0 ** -4)
    return _bf16_bits(mag * sigma[None, :])


def case(family: str, M: int, N: int, K: int, seed: int):
    """One adversarial problem: (x bits [M, K], codes, scales, biases)."""
    sigma = signs(family, K, seed)
    codes, s, b = packed_weight(family, N, K, seed, sigma)
    return activation(M, K, seed, sigma), codes, s, b


# ---- arithmetic of candidate kernels, simulated on the CPU ------------------
# (To show what the families catch; the CUDA path is tested against the oracle.)


def _bf16_round(a: np.ndarray) -> np.ndarray:
    return _f64(_bf16_bits(a.astype(np.float32)))


def simulate_bf16_operand(x_bits, codes, s_bits, b_bits) -> np.ndarray:
    """w_hat rounded once to bf16 (as oracle.dequantize), fp32 accumulation in
    a fixed order, bf16 output: a tensor-core kernel fed a bf16 operand."""
    w = _f64(oracle.dequantize(codes, s_bits, b_bits)).astype(np.float32)
    x = _f64(x_bits).astype(np.float32)
    return _bf16_round(x @ w.T)


def simulate_hi_lo_operand(x_bits, codes, s_bits, b_bits) -> np.ndarray:
    """w_hat as hi + lo: w32 = fp32(s*q + b), hi = bf16(w32), lo = bf16(w32 - hi);
    fp32 accumulation of x*hi + x*lo, bf16 output."""
    exact = oracle.dequantize_f64(codes, s_bits, b_bits)
    w32 = exact.astype(np.float32)
    hi = _bf16_round(w32).astype(np.float32)
    lo = _bf16_round(w32 - hi).astype(np.float32)
    x = _f64(x_bits).astype(np.float32)
    return _bf16_round(x @ hi.T + x @ lo.T)
