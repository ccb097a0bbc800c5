"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
call the library through its binding, and compare against the CPU oracle."""
import contextlib

import numpy as np
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4

# The matmul acceptance bound: |y_gpu - y_ref| <= REL * sum_k |x_k w_hat_k| + ABS.
REL, ABS = 4e-3, 1e-6


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t)


def packed_to_host(codes, scales, biases):
    return (codes.cpu().numpy(), bits(scales), bits(biases))


def assert_quantize_bitexact(W_dev: torch.Tensor, codes, scales, biases):
    """GPU codes/scales/biases equal the oracle's quantization of the same bf16 W."""
    oc, os_, ob = oracle.quantize(bits(W_dev))
    gc, gs, gb = packed_to_host(codes, scales, biases)
    assert np.array_equal(gs, os_), "scales differ"
    assert np.array_equal(gb, ob), "biases differ"
    assert np.array_equal(gc, oc), f"codes differ at {np.argwhere(gc != oc)[:5].tolist()}"


def check_matmul(x_dev, codes, scales, biases, y_dev, rows=None, what=""):
    """Compare y_dev [M, N] (or the selected columns) with the oracle within the bound."""
    hc, hs, hb = packed_to_host(codes, scales, biases)
    y_ref, absdot = oracle.matmul_ref(bits(x_dev), hc, hs, hb, rows=rows)
    yg = y_dev.float().cpu().double().numpy()
    if rows is not None:
        yg = yg[:, rows]
    ok = oracle.tolerance_ok(yg, y_ref, absdot, REL, ABS)
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        detail = [(int(m), int(n), float(yg[m, n]), float(y_ref[m, n]), float(absdot[m, n])) for m, n in bad]
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, e.g. {detail}")
    err = np.abs(yg - y_ref) / np.maximum(absdot, 1e-30)
    return float(err.max())


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """First, last and random rows (covers both ends of every tile grid)."""
    rng = np.random.default_rng(seed)
    pick = set([0, N - 1, N // 2]) | set(rng.integers(0, N, size=min(count, N)).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def gpu_weight(N, K, seed, tensor, device="cuda"):
    return workloads.weight(N, K, seed, tensor, device=device)


def quantize_dev(W):
    return q4.q4_quantize(W)


@contextlib.contextmanager
def kernels_disabled(mask: int):
    """Run the block with the given kernel families (q4.KERNEL_* bits) kept
    out of the matmul dispatch, to pin a problem to another kernel."""
    prev = q4.q4_debug_disable_kernels(mask)
    try:
        yield
    finally:
        q4.q4_debug_disable_kernels(prev)
