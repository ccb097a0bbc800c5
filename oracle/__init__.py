"""CPU oracle for affine 4-bit, group-32 weight-only quantization and matmul
(and its 8-bit variant, the same rule with 255 levels; the q8_* functions).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product library never imports it,
and this package imports nothing from the product.

The arithmetic lives in ``q4_oracle.c`` (plain C, binary64, OpenMP over rows);
this module builds it with gcc and marshals numpy arrays through ctypes.  bf16
tensors cross the interface as their uint16 bit patterns.

Parity pins: see the functions' docstrings and ``tests/test_oracle_pins.py``.
The reconstruction metrics below follow the acceptance gates of the model card
"personaplex-edge-q4" (section "Conversion and weight validation": maximum
normalized RMSE at most 0.12, minimum cosine similarity at least 0.985); the
card does not define "normalized RMSE", and the reading used here is
||W_hat - W||_F / ||W||_F over one tensor.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB = os.path.join(_HERE, "liboq4.so")
GROUP = 32

_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ``liboq4.so`` next to the source if missing or older than it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oq4_bf16_from_f64.restype = ctypes.c_uint16
        lib.oq4_bf16_from_f64.argtypes = [ctypes.c_double]
        lib.oq4_bf16_to_f64.restype = ctypes.c_double
        lib.oq4_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oq4_packed_nbytes.restype = i64
        lib.oq4_packed_nbytes.argtypes = [i64, i64]
        lib.oq4_quantize.restype = ctypes.c_int
        lib.oq4_quantize.argtypes = [p, i64, i64, p, p, p]
        lib.oq4_dequantize.restype = ctypes.c_int
        lib.oq4_dequantize.argtypes = [p, p, p, i64, i64, p]
        lib.oq4_dequantize_f64.restype = ctypes.c_int
        lib.oq4_dequantize_f64.argtypes = [p, p, p, i64, i64, p]
        lib.oq4_matmul_ref.restype = ctypes.c_int
        lib.oq4_matmul_ref.argtypes = [p, i64, i64, p, p, p, i64, p, i64, p, p]
        lib.oq4_matmul_ref_factored.restype = ctypes.c_int
        lib.oq4_matmul_ref_factored.argtypes = [p, i64, i64, p, p, p, i64, p]
        lib.oq8_quantize.restype = ctypes.c_int
        lib.oq8_quantize.argtypes = [p, i64, i64, p, p, p]
        lib.oq8_dequantize.restype = ctypes.c_int
        lib.oq8_dequantize.argtypes = [p, p, p, i64, i64, p]
        lib.oq8_dequantize_f64.restype = ctypes.c_int
        lib.oq8_dequantize_f64.argtypes = [p, p, p, i64, i64, p]
        lib.oq8_matmul_ref.restype = ctypes.c_int
        lib.oq8_matmul_ref.argtypes = [p, i64, i64, p, p, p, i64, p, i64, p, p]
        lib.oq4_set_threads.restype = None
        lib.oq4_set_threads.argtypes = [ctypes.c_int]
        lib.oq4_max_threads.restype = ctypes.c_int
        lib.oq4_max_threads.argtypes = []
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _check(st: int, what: str):
    if st != 0:
        raise OracleError(f"{what}: oracle status {st}")


def bf16_from_f64(v: float) -> int:
    """Nearest bf16 bit pattern to a binary64 value, ties to even."""
    return int(_load().oq4_bf16_from_f64(float(v)))


def bf16_to_f64(h: int) -> float:
    return float(_load().oq4_bf16_to_f64(int(h)))


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Widen an array of bf16 bit patterns to float64 (exact)."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def packed_nbytes(N: int, K: int) -> int:
    """Bytes of codes + scales + biases for an [N, K] weight."""
    return int(_load().oq4_packed_nbytes(N, K))


def quantize(W_bits: np.ndarray):
    """W [N, K] bf16 bits -> (codes [N, K/2] u8, scales [N, K/32] bf16 bits, biases bf16 bits)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    G = K // GROUP if K % GROUP == 0 else 0
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, max(G, 0)), np.uint16)
    biases = np.zeros((N, max(G, 0)), np.uint16)
    _check(_load().oq4_quantize(_ptr(W), N, K, _ptr(codes), _ptr(scales), _ptr(biases)), "quantize")
    return codes, scales, biases


def dequantize(codes, scales, biases) -> np.ndarray:
    """Reconstruction s*q + b rounded to bf16 (bits), [N, K]."""
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((N, K), np.uint16)
    _check(_load().oq4_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), N, K, _ptr(out)), "dequantize")
    return out


def dequantize_f64(codes, scales, biases) -> np.ndarray:
    """Reconstruction s*q + b in binary64 (not rounded), [N, K]."""
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((N, K), np.float64)
    _check(_load().oq4_dequantize_f64(_ptr(codes), _ptr(scales), _ptr(biases), N, K, _ptr(out)),
           "dequantize_f64")
    return out


def matmul_ref(x_bits, codes, scales, biases, rows=None):
    """y = x . W_hat^T in binary64 with the exact w_hat = s*q + b.

    Returns (y [M, nrows], absdot [M, nrows]) where absdot = sum_k |x*w_hat|,
    the scale of the tolerance |y_gpu - y| <= 4e-3 * absdot + 1e-6.
    ``rows`` selects output columns (indices of weight rows); None = all.
    """
    x = _c(x_bits, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    M, K = x.shape
    N = codes.shape[0]
    if codes.shape[1] * 2 != K:
        raise ValueError("x and codes disagree on K")
    if rows is None:
        rows_arr, nrows, rp = None, N, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows, rp = rows_arr.size, _ptr(rows_arr)
    y = np.zeros((M, nrows), np.float64)
    ad = np.zeros((M, nrows), np.float64)
    _check(_load().oq4_matmul_ref(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N,
                                  rp, nrows, _ptr(y), _ptr(ad)), "matmul_ref")
    return y, ad


def matmul_ref_factored(x_bits, codes, scales, biases) -> np.ndarray:
    """Same product computed per group as s*sum(x*q) + b*sum(x); all rows."""
    x = _c(x_bits, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    M, K = x.shape
    N = codes.shape[0]
    y = np.zeros((M, N), np.float64)
    _check(_load().oq4_matmul_ref_factored(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases),
                                           N, _ptr(y)), "matmul_ref_factored")
    return y


# ------------------------------------------------------------------ 8-bit codes
#
# The same affine rule with 255 levels and one byte per code (the pages'
# "standard 8-bit conversion" and INT8 bundle name the variant, not its
# arithmetic): s = bf16(fp32(mx - mn) / 255), b = bf16(mn),
# q = clamp(rne((w - b) / s), 0, 255); codes [N, K] uint8.


def q8_packed_nbytes(N: int, K: int) -> int:
    """Bytes of the 8-bit form of an [N, K] weight: 1 B per code + bf16 s and b per 32."""
    return N * K + 4 * N * (K // GROUP)


def q8_quantize(W_bits: np.ndarray):
    """W [N, K] bf16 bits -> (codes [N, K] u8, scales [N, K/32] bf16 bits, biases bf16 bits)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, K // GROUP), np.uint16)
    biases = np.zeros((N, K // GROUP), np.uint16)
    _check(_load().oq8_quantize(_ptr(W), N, K, _ptr(codes), _ptr(scales), _ptr(biases)), "q8_quantize")
    return codes, scales, biases


def q8_dequantize(codes, scales, biases) -> np.ndarray:
    """8-bit reconstruction s*q + b rounded to bf16 (bits), [N, K]."""
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    N, K = codes.shape
    out = np.zeros((N, K), np.uint16)
    _check(_load().oq8_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), N, K, _ptr(out)), "q8_dequantize")
    return out


def q8_dequantize_f64(codes, scales, biases) -> np.ndarray:
    """8-bit reconstruction s*q + b in binary64 (not rounded), [N, K]."""
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    N, K = codes.shape
    out = np.zeros((N, K), np.float64)
    _check(_load().oq8_dequantize_f64(_ptr(codes), _ptr(scales), _ptr(biases), N, K, _ptr(out)),
           "q8_dequantize_f64")
    return out


def q8_matmul_ref(x_bits, codes, scales, biases, rows=None):
    """y = x . W_hat^T over the exact 8-bit w_hat, binary64; returns (y, absdot) as matmul_ref."""
    x = _c(x_bits, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    codes = _c(codes, np.uint8)
    scales, biases = _c(scales, np.uint16), _c(biases, np.uint16)
    M, K = x.shape
    N = codes.shape[0]
    if codes.shape[1] != K:
        raise ValueError("x and codes disagree on K")
    if rows is None:
        nrows, rp = N, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows, rp = rows_arr.size, _ptr(rows_arr)
    y = np.zeros((M, nrows), np.float64)
    ad = np.zeros((M, nrows), np.float64)
    _check(_load().oq8_matmul_ref(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N,
                                  rp, nrows, _ptr(y), _ptr(ad)), "q8_matmul_ref")
    return y, ad


# --------------------------------------------------------------- output epilogues
#
# The projections feed the blocks the pages name as reused components of the
# model (Swift/MLX blog, section "Reusing the Mimi codec": KV cache, RoPE,
# SwiGLU, RMSNorm; GeekNews summary, "Arsitektur model dan konversi"): the
# attention output and down projections add into the residual stream, and the
# MLP's gate and up projections meet in SwiGLU, h = silu(gate) * up with
# silu(z) = z * sigmoid(z).  The fused forms below take the exact products
# from matmul_ref (the pinned product) as their step.

SILU_LIPSCHITZ = 1.1  # bound on |d silu / dz| = |s(z) (1 + z (1 - s(z)))|, max 1.0998 near z = 2.40


def silu(z) -> np.ndarray:
    """silu(z) = z / (1 + e^-z) in binary64, elementwise (e^-z -> inf gives -0)."""
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def matmul_residual_ref(x_bits, codes, scales, biases, r_bits, rows=None):
    """y = r + x . W_hat^T in binary64 (r [M, N] bf16 bits, the residual stream).

    Returns (y, bound): the per-element acceptance bound extends the product's
    4e-3 * sum|x w_hat| + 1e-6 to the magnitude of the sum, 4e-3 * (sum|x w_hat|
    + |r|) + 1e-6, since the one bf16 rounding of r + acc is relative to it.
    """
    y, ad = matmul_ref(x_bits, codes, scales, biases, rows=rows)
    r = bf16_bits_to_f64(_c(r_bits, np.uint16))
    if r.ndim == 1:
        r = r[None, :]
    if rows is not None:
        r = r[:, np.asarray(rows, dtype=np.int64)]
    return y + r, 4e-3 * (ad + np.abs(r)) + 1e-6


def matmul_swiglu_ref(x_bits, gate, up, rows=None):
    """h = silu(g) * u in binary64, g and u the exact products x . W_hat^T of
    the gate and up weights ((codes, scales, biases) triples).

    Returns (h, bound).  The bound carries the product bounds
    T = 4e-3 * sum|x w_hat| + 1e-6 of g and u through h to first order, for a
    computation that keeps both products unrounded until h:
    |silu(g') u' - silu(g) u| <= L Tg (|u| + Tu) + |silu(g)| Tu with
    L = SILU_LIPSCHITZ; then one bf16 rounding of h, relative 2^-8 of its
    magnitude (bf16's unit roundoff: 8 significant bits).
    """
    g, adg = matmul_ref(x_bits, *gate, rows=rows)
    u, adu = matmul_ref(x_bits, *up, rows=rows)
    tg, tu = 4e-3 * adg + 1e-6, 4e-3 * adu + 1e-6
    sg = silu(g)
    dg = SILU_LIPSCHITZ * tg
    mag_u = np.abs(u) + tu
    bound = dg * mag_u + np.abs(sg) * tu + 2.0 ** -8 * (np.abs(sg) + dg) * mag_u + 1e-6
    return sg * u, bound


def set_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops (timing only: results do not depend on it)."""
    _load().oq4_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oq4_max_threads())


def nrmse(W_ref: np.ndarray, W_hat: np.ndarray) -> float:
    """||W_hat - W_ref||_F / ||W_ref||_F over the whole tensor (binary64)."""
    a = np.asarray(W_ref, np.float64).ravel()
    b = np.asarray(W_hat, np.float64).ravel()
    return float(np.sqrt(np.sum((b - a) ** 2)) / np.sqrt(np.sum(a * a)))


def cosine(W_ref: np.ndarray, W_hat: np.ndarray) -> float:
    """<W_hat, W_ref> / (||W_hat|| ||W_ref||) over the flattened tensor."""
    a = np.asarray(W_ref, np.float64).ravel()
    b = np.asarray(W_hat, np.float64).ravel()
    return float(np.dot(a, b) / (np.sqrt(np.dot(a, a)) * np.sqrt(np.dot(b, b))))


def tolerance_ok(y_gpu: np.ndarray, y_ref: np.ndarray, absdot: np.ndarray,
                 rel: float = 4e-3, abs_: float = 1e-6) -> np.ndarray:
    """Per-element acceptance |y_gpu - y_ref| <= rel * absdot + abs_."""
    return np.abs(np.asarray(y_gpu, np.float64) - y_ref) <= rel * absdot + abs_
