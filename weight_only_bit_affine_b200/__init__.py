"""Python binding of libq4: affine 4-bit, group-32, weight-only quantized matmul
for NVIDIA B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in libq4's CUDA
kernels, reached through the C ABI declared in ``include/q4.h``; there is no
fallback of any kind.  If ``libq4.so`` is missing the first call raises.

The functions take torch tensors (device memory and the current CUDA stream
come from PyTorch) and have the same names as the C entry points:

    codes, scales, biases = q4_quantize(W)            # W [N, K] bf16, cuda
    W_hat = q4_dequantize(codes, scales, biases)        # [N, K] bf16
    y = q4_matmul(x, codes, scales, biases)             # x [M, K] -> y [M, N]
    y = q4_matmul_step(x, codes, scales, biases, num_steps, step)
    y = q4_matmul_residual(x, codes, scales, biases, r)   # r + x . w_hat^T
    h = q4_matmul_swiglu(x, (gc, gs, gb), (uc, us, ub))   # silu(gate) * up
    q4_matmul_batch([(x, codes, scales, biases, y), ...]) # one launch per kernel path
    b = q4_prepare_batch([...]); b.run()                  # the same, descriptors built once
    codes8, scales, biases = q8_quantize(W)             # 8-bit variant: codes [N, K]
    y = q8_matmul(x, codes8, scales, biases)

Layout (model card "personaplex-edge-q4", "Release details": affine Q4,
group size 32, BF16): codes [N, K/2] uint8 (low nibble = even k), scales
and biases [N, K/32] bf16, w_hat = scale * q + bias.
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional, Tuple

import torch

__all__ = [
    "Q4Error",
    "GROUP",
    "lib",
    "library_path",
    "q4_quantize",
    "q4_dequantize",
    "q4_matmul",
    "q4_matmul_step",
    "q4_matmul_residual",
    "q4_matmul_swiglu",
    "q4_matmul_batch",
    "q4_prepare_batch",
    "PreparedBatch",
    "Residual",
    "SwiGLU",
    "q8_quantize",
    "q8_dequantize",
    "q8_matmul",
    "q8_matmul_batch",
    "q4_device_status",
    "q4_check_device",
    "q4_debug_launch_count",
    "q4_debug_disable_kernels",
    "q4_matmul_batch_noalloc",
    "q4_matmul_chain",
    "q4_prepare_chain",
    "PreparedChain",
    "KERNEL_GROUP_SUM",
    "KERNEL_WEIGHT_STREAM",
    "KERNEL_TILES",
]

GROUP = 32
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libq4.so")

_STATUS = {
    0: "Q4_OK",
    1: "Q4_ERR_NULL",
    2: "Q4_ERR_SHAPE",
    3: "Q4_ERR_ALIGN",
    4: "Q4_ERR_UNSUPPORTED",
    5: "Q4_ERR_RANGE",
    6: "Q4_ERR_CUDA",
}

# Exported C symbols and their ctypes signatures.
_I64, _P, _INT = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "q4_quantize": (_INT, [_P, _I64, _I64, _INT, _P, _P, _P, _P]),
    "q4_dequantize": (_INT, [_P, _P, _P, _I64, _I64, _INT, _P, _P]),
    "q4_matmul": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _P, _P]),
    "q4_matmul_step": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _I64, _I64, _INT, _P, _P]),
    "q4_matmul_residual": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _P, _P, _P]),
    "q4_matmul_swiglu": (_INT, [_P, _I64, _I64, _P, _P, _P, _P, _P, _P, _I64, _INT, _P, _P]),
    "q4_matmul_batch": (_INT, [_P, _INT, _I64, _INT, _P]),
    "q4_matmul_batch_noalloc": (_INT, [_P, _INT, _I64, _INT, _P]),
    "q4_matmul_chain": (_INT, [_P, _INT, _P, _INT, _I64, _INT, _P]),
    "q8_quantize": (_INT, [_P, _I64, _I64, _INT, _P, _P, _P, _P]),
    "q8_dequantize": (_INT, [_P, _P, _P, _I64, _I64, _INT, _P, _P]),
    "q8_matmul": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _P, _P]),
    "q8_matmul_batch": (_INT, [_P, _INT, _I64, _INT, _P]),
    "q4_last_error": (ctypes.c_char_p, []),
    "q4_device_status": (_INT, [_INT]),
    "q4_debug_launch_count": (ctypes.c_ulonglong, []),
    "q4_debug_disable_kernels": (ctypes.c_uint, [ctypes.c_uint]),
}


EPI_NONE, EPI_RESIDUAL, EPI_SWIGLU = 0, 1, 2  # q4_epilogue


class MatmulDesc(ctypes.Structure):
    """Mirror of q4_matmul_desc (include/q4.h)."""

    _fields_ = [("x", _P), ("codes", _P), ("scales", _P), ("biases", _P), ("y", _P), ("N", _I64), ("K", _I64),
                ("epilogue", ctypes.c_int32), ("reserved", ctypes.c_int32), ("r", _P), ("up_codes", _P),
                ("up_scales", _P), ("up_biases", _P)]


class Residual(NamedTuple):
    """Batch epilogue: out = r + x . w_hat^T (r [M, N] bf16; may be out itself)."""

    r: torch.Tensor


class SwiGLU(NamedTuple):
    """Batch epilogue: out = silu(x . w_hat^T) * (x . w_hat_up^T), the problem's
    weights being the gate and these the up projection's."""

    up_codes: torch.Tensor
    up_scales: torch.Tensor
    up_biases: torch.Tensor


class Q4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.status_name = _STATUS.get(status, str(status))
        super().__init__(f"{self.status_name}: {message}")


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded libq4 (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"libq4.so not found at {_LIB_PATH}; build it with "
                "`python -m weight_only_bit_affine_b200.build` (there is no non-CUDA fallback)")
        handle = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int):
    if status != 0:
        msg = lib().q4_last_error()
        raise Q4Error(status, msg.decode() if msg else "")


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _want(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def q4_quantize(W: torch.Tensor, group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """W [N, K] bf16 -> (codes [N, K/2] uint8, scales [N, K/32] bf16, biases [N, K/32] bf16)."""
    _want(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    dev = W.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, max(K // GROUP, 0)), dtype=torch.bfloat16, device=dev)
    biases = torch.empty_like(scales)
    with torch.cuda.device(dev):
        _check(lib().q4_quantize(_ptr(W), N, K, group, _ptr(codes), _ptr(scales), _ptr(biases), _stream(dev)))
    return codes, scales, biases


def q4_dequantize(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, group: int = GROUP,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """(codes, scales, biases) -> W_hat [N, K] bf16 = bf16(scale * q + bias)."""
    _want(codes, "codes", torch.uint8, 2)
    _want(scales, "scales", torch.bfloat16, 2)
    _want(biases, "biases", torch.bfloat16, 2)
    N, K = codes.shape[0], codes.shape[1] * 2
    dev = codes.device
    if scales.shape != (N, K // GROUP) or biases.shape != (N, K // GROUP):
        raise ValueError("codes / scales / biases shapes disagree")
    out = _out(out, N, K, dev)
    with torch.cuda.device(dev):
        _check(lib().q4_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), N, K, group, _ptr(out), _stream(dev)))
    return out


def _matmul_shapes(x, codes, scales, biases, rows_per_step):
    _want(x, "x", torch.bfloat16, 2)
    _want(codes, "codes", torch.uint8, 2)
    _want(scales, "scales", torch.bfloat16, 2)
    _want(biases, "biases", torch.bfloat16, 2)
    M, K = x.shape
    if codes.shape[1] * 2 != K:
        raise ValueError(f"x has K = {K} but codes rows hold {codes.shape[1] * 2} codes")
    if scales.shape != (codes.shape[0], K // GROUP) or biases.shape != scales.shape:
        raise ValueError("scales / biases must be [rows, K/32]")
    if not (x.device == codes.device == scales.device == biases.device):
        raise ValueError("all tensors must be on the same device")
    return M, K


def q4_matmul(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
              group: int = GROUP, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = x . w_hat^T:  x [M, K] bf16, packed W with N rows -> y [M, N] bf16."""
    M, K = _matmul_shapes(x, codes, scales, biases, None)
    N = codes.shape[0]
    dev = x.device
    out = _out(out, M, N, dev)
    with torch.cuda.device(dev):
        _check(lib().q4_matmul(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N, group, _ptr(out),
                               _stream(dev)))
    return out


def q4_matmul_step(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                   num_steps: int, step: int, group: int = GROUP,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Step `step` of a stacked [num_steps * N, K] packed weight: rows [step*N, (step+1)*N)."""
    M, K = _matmul_shapes(x, codes, scales, biases, None)
    rows = codes.shape[0]
    if num_steps < 1 or rows % num_steps:
        raise ValueError(f"stacked rows {rows} not divisible by num_steps {num_steps}")
    N = rows // num_steps
    dev = x.device
    out = _out(out, M, N, dev)
    with torch.cuda.device(dev):
        _check(lib().q4_matmul_step(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N, num_steps, step,
                                    group, _ptr(out), _stream(dev)))
    return out


def _out(out, M, N, dev):
    if out is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _want(out, "out", torch.bfloat16, 2)
    if out.shape != (M, N) or out.device != dev:
        raise ValueError(f"out must be [{M}, {N}] on {dev}")
    return out


def _same_weights(codes, scales, biases, up, what):
    uc, us, ub = up
    _matmul_shapes_w(uc, us, ub, codes.shape[1] * 2, what)
    if uc.shape != codes.shape or not (uc.device == us.device == ub.device == codes.device):
        raise ValueError(f"{what}: the up weights must match the gate's shape and device")


def _matmul_shapes_w(codes, scales, biases, K, what):
    _want(codes, f"{what} codes", torch.uint8, 2)
    _want(scales, f"{what} scales", torch.bfloat16, 2)
    _want(biases, f"{what} biases", torch.bfloat16, 2)
    if codes.shape[1] * 2 != K or scales.shape != (codes.shape[0], K // GROUP) or biases.shape != scales.shape:
        raise ValueError(f"{what}: codes [N, K/2], scales and biases [N, K/32] with K = {K}")


def q4_matmul_residual(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                       r: torch.Tensor, group: int = GROUP, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = bf16(r + x . w_hat^T), summed in fp32; out=r updates r in place."""
    M, K = _matmul_shapes(x, codes, scales, biases, None)
    N = codes.shape[0]
    dev = x.device
    _want(r, "r", torch.bfloat16, 2)
    if r.shape != (M, N) or r.device != dev:
        raise ValueError(f"r must be [{M}, {N}] on {dev}")
    out = _out(out, M, N, dev)
    with torch.cuda.device(dev):
        _check(lib().q4_matmul_residual(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N, group, _ptr(r),
                                        _ptr(out), _stream(dev)))
    return out


def q4_matmul_swiglu(x: torch.Tensor, gate, up, group: int = GROUP,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """h = bf16(silu(x . w_hat_gate^T) * (x . w_hat_up^T)); gate and up are
    (codes, scales, biases) triples of the same [N, K] shape."""
    gc, gs, gb = gate
    M, K = _matmul_shapes(x, gc, gs, gb, None)
    _same_weights(gc, gs, gb, up, "up")
    N = gc.shape[0]
    dev = x.device
    out = _out(out, M, N, dev)
    uc, us, ub = up
    with torch.cuda.device(dev):
        _check(lib().q4_matmul_swiglu(_ptr(x), M, K, _ptr(gc), _ptr(gs), _ptr(gb), _ptr(uc), _ptr(us), _ptr(ub), N,
                                      group, _ptr(out), _stream(dev)))
    return out


def q4_matmul_batch(problems, group: int = GROUP):
    """Independent matmuls in as few launches as possible.

    `problems`: a sequence of (x, codes, scales, biases, out) tuples, every x
    with the same number of rows M; `out` [M, N] bf16 is written.  A sixth
    element Residual(r) or SwiGLU(up_codes, up_scales, up_biases) adds that
    epilogue.  Returns the list of outputs.
    """
    batch = q4_prepare_batch(problems, group)
    if batch is None:
        return []
    batch.run()
    return batch.outputs


def q4_matmul_batch_noalloc(problems, group: int = GROUP):
    """q4_matmul_batch through the entry point that makes no device
    allocation (its group-sum workspace is a fixed array in libq4, shared by
    all such calls on a device: serialize calls that may overlap)."""
    batch = q4_prepare_batch(problems, group)
    if batch is None:
        return []
    with torch.cuda.device(batch.device):
        _check(lib().q4_matmul_batch_noalloc(ctypes.cast(batch._descs, ctypes.c_void_p), batch._count, batch._M,
                                             batch._group, _stream(batch.device)))
    return batch.outputs


class PreparedBatch:
    """A q4_matmul_batch call whose descriptor array is built once.

    run() calls the C entry point with it on the current stream of the
    problems' device (host-side validation and the launches happen on every
    call); the tensors must stay alive and keep their storage in between, as
    for a CUDA graph.
    """

    def __init__(self, descs, count, M, group, device, outputs):
        self._descs, self._count, self._M, self._group = descs, count, M, group
        self.device, self.outputs = device, outputs

    def run(self) -> None:
        with torch.cuda.device(self.device):
            _check(lib().q4_matmul_batch(ctypes.cast(self._descs, ctypes.c_void_p), self._count, self._M, self._group,
                                         _stream(self.device)))


def q4_prepare_batch(problems, group: int = GROUP) -> Optional[PreparedBatch]:
    """Validate and marshal a q4_matmul_batch problem list once (same tuples
    as q4_matmul_batch); None for an empty list."""
    problems = list(problems)
    if not problems:
        return None
    descs = (MatmulDesc * len(problems))()
    M = None
    dev = None
    for i, prob in enumerate(problems):
        if len(prob) not in (5, 6):
            raise ValueError(f"problem {i}: (x, codes, scales, biases, out[, epilogue])")
        x, codes, scales, biases, out = prob[:5]
        epi = prob[5] if len(prob) == 6 else None
        Mi, K = _matmul_shapes(x, codes, scales, biases, None)
        if M is None:
            M, dev = Mi, x.device
        elif Mi != M or x.device != dev:
            raise ValueError("all problems of a batch need the same M and device")
        _want(out, "out", torch.bfloat16, 2)
        if out.shape != (M, codes.shape[0]) or out.device != dev:
            raise ValueError(f"out of problem {i} must be [{M}, {codes.shape[0]}] on {dev}")
        d = MatmulDesc(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
                       codes.shape[0], K)
        if isinstance(epi, Residual):
            _want(epi.r, "r", torch.bfloat16, 2)
            if epi.r.shape != out.shape or epi.r.device != dev:
                raise ValueError(f"problem {i}: r must be [{M}, {codes.shape[0]}] on {dev}")
            d.epilogue, d.r = EPI_RESIDUAL, epi.r.data_ptr()
        elif isinstance(epi, SwiGLU):
            _same_weights(codes, scales, biases, epi, f"problem {i} up")
            d.epilogue = EPI_SWIGLU
            d.up_codes, d.up_scales, d.up_biases = (epi.up_codes.data_ptr(), epi.up_scales.data_ptr(),
                                                    epi.up_biases.data_ptr())
        elif epi is not None:
            raise TypeError(f"problem {i}: epilogue must be Residual or SwiGLU")
        descs[i] = d
    return PreparedBatch(descs, len(problems), M, group, dev, [p[4] for p in problems])


def q4_matmul_chain(stages, group: int = GROUP):
    """Dependent matmuls in order: `stages` is a sequence of stages, each a
    sequence of q4_matmul_batch problem tuples (every x with the same M);
    a stage may read, as x or residual, what earlier stages write.  Computes
    exactly what q4_matmul_batch on each stage in turn computes.  Returns the
    outputs of all stages in order."""
    chain = q4_prepare_chain(stages, group)
    if chain is None:
        return []
    chain.run()
    return chain.outputs


class PreparedChain:
    """A q4_matmul_chain call whose descriptor and stage arrays are built
    once; run() calls the C entry point with them on the current stream of
    the problems' device (the tensors must stay alive in between)."""

    def __init__(self, batch: PreparedBatch, counts):
        self._batch = batch
        self._counts = (ctypes.c_int * len(counts))(*counts)
        self._n = len(counts)
        self.device, self.outputs = batch.device, batch.outputs

    def run(self) -> None:
        b = self._batch
        with torch.cuda.device(b.device):
            _check(lib().q4_matmul_chain(ctypes.cast(b._descs, ctypes.c_void_p), b._count,
                                         ctypes.cast(self._counts, ctypes.c_void_p), self._n, b._M, b._group,
                                         _stream(b.device)))


def q4_prepare_chain(stages, group: int = GROUP) -> Optional[PreparedChain]:
    """Validate and marshal a q4_matmul_chain call once; None if it has no
    problem."""
    stages = [list(st) for st in stages]
    batch = q4_prepare_batch([p for st in stages for p in st], group)
    if batch is None:
        return None
    return PreparedChain(batch, [len(st) for st in stages])


# ------------------------------------------------------------------ 8-bit codes


def q8_quantize(W: torch.Tensor, group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """W [N, K] bf16 -> (codes [N, K] uint8, scales [N, K/32] bf16, biases [N, K/32] bf16), 255 levels."""
    _want(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    dev = W.device
    codes = torch.empty((N, K), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, max(K // GROUP, 0)), dtype=torch.bfloat16, device=dev)
    biases = torch.empty_like(scales)
    with torch.cuda.device(dev):
        _check(lib().q8_quantize(_ptr(W), N, K, group, _ptr(codes), _ptr(scales), _ptr(biases), _stream(dev)))
    return codes, scales, biases


def _q8_shapes(codes, scales, biases, K, what="codes"):
    _want(codes, what, torch.uint8, 2)
    _want(scales, "scales", torch.bfloat16, 2)
    _want(biases, "biases", torch.bfloat16, 2)
    if codes.shape[1] != K or scales.shape != (codes.shape[0], K // GROUP) or biases.shape != scales.shape:
        raise ValueError(f"8-bit weights: codes [N, K], scales and biases [N, K/32] with K = {K}")


def q8_dequantize(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, group: int = GROUP,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """8-bit (codes, scales, biases) -> W_hat [N, K] bf16 = bf16(scale * q + bias)."""
    _want(codes, "codes", torch.uint8, 2)
    N, K = codes.shape
    _q8_shapes(codes, scales, biases, K)
    out = _out(out, N, K, codes.device)
    with torch.cuda.device(codes.device):
        _check(lib().q8_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), N, K, group, _ptr(out),
                                   _stream(codes.device)))
    return out


def q8_matmul(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
              group: int = GROUP, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = x . w_hat^T with 8-bit codes:  x [M, K] bf16 -> y [M, N] bf16."""
    _want(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _q8_shapes(codes, scales, biases, K)
    if not (x.device == codes.device == scales.device == biases.device):
        raise ValueError("all tensors must be on the same device")
    N = codes.shape[0]
    out = _out(out, M, N, x.device)
    with torch.cuda.device(x.device):
        _check(lib().q8_matmul(_ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), N, group, _ptr(out),
                               _stream(x.device)))
    return out


def q8_matmul_batch(problems, group: int = GROUP):
    """Independent 8-bit matmuls sharing M, in as few launches as possible:
    (x, codes, scales, biases, out) tuples with codes [N, K] uint8 (no
    epilogue).  Returns the list of outputs."""
    problems = list(problems)
    if not problems:
        return []
    descs = (MatmulDesc * len(problems))()
    M = dev = None
    for i, prob in enumerate(problems):
        if len(prob) != 5:
            raise ValueError(f"problem {i}: (x, codes, scales, biases, out)")
        x, codes, scales, biases, out = prob
        _want(x, "x", torch.bfloat16, 2)
        Mi, K = x.shape
        _q8_shapes(codes, scales, biases, K)
        if not (x.device == codes.device == scales.device == biases.device):
            raise ValueError(f"problem {i}: all tensors must be on the same device")
        if M is None:
            M, dev = Mi, x.device
        elif Mi != M or x.device != dev:
            raise ValueError("all problems of a batch need the same M and device")
        _want(out, "out", torch.bfloat16, 2)
        if out.shape != (M, codes.shape[0]) or out.device != dev:
            raise ValueError(f"out of problem {i} must be [{M}, {codes.shape[0]}] on {dev}")
        descs[i] = MatmulDesc(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
                              codes.shape[0], K)
    with torch.cuda.device(dev):
        _check(lib().q8_matmul_batch(ctypes.cast(descs, ctypes.c_void_p), len(problems), M, group, _stream(dev)))
    return [p[4] for p in problems]


def q4_device_status(clear: bool = False) -> int:
    """Kernel status flags of the current device (synchronizes); 0 means no
    bounded wait gave up.  While nonzero, results enqueued since the flags were
    last cleared are invalid (the kernels wrote NaN where they gave up)."""
    r = lib().q4_device_status(1 if clear else 0)
    if r < 0:
        raise Q4Error(6, "could not read device flags")
    return r


def q4_check_device(clear: bool = True) -> None:
    """Raise Q4Error if a kernel on the current device gave up a bounded wait
    since the flags were last cleared (synchronizes; clears them by default)."""
    r = q4_device_status(clear)
    if r != 0:
        raise Q4Error(6, f"a libq4 kernel gave up a bounded wait (flags {r:#x}); recent results are invalid")


def q4_debug_launch_count() -> int:
    """Kernel launches libq4 has enqueued in this process (host-side count)."""
    return int(lib().q4_debug_launch_count())


KERNEL_GROUP_SUM, KERNEL_WEIGHT_STREAM, KERNEL_TILES = 1, 2, 4  # Q4_KERNEL_* (include/q4.h)


def q4_debug_disable_kernels(mask: int) -> int:
    """Kernel families the matmul dispatch may not choose (KERNEL_* bits; 0 =
    all allowed); returns the previous mask.  For tests that pin a kernel."""
    return int(lib().q4_debug_disable_kernels(ctypes.c_uint(mask)))
