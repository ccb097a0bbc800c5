"""The C-ABI library builds, loads, exports every entry point include/*.h
declares, and validates arguments on the host.  No GPU needed: every call
here returns before any device work (validation precedes the device query;
on a machine without a GPU, a fully valid call stops at the device query with
Q4_ERR_CUDA)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

import weight_only_bit_affine_b200 as q4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, NULL, SHAPE, ALIGN, UNSUP, RANGE, CUDA = range(7)


@pytest.fixture(scope="module")
def lib():
    from weight_only_bit_affine_b200 import build

    build.build()
    return q4.lib()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(q[48]_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ["q4_quantize", "q4_dequantize", "q4_matmul", "q4_matmul_step", "q4_matmul_residual",
              "q4_matmul_swiglu", "q4_matmul_batch", "q4_last_error", "q8_quantize", "q8_dequantize",
              "q8_matmul"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) <= set(q4.SIGNATURES)
    out = subprocess.run(["nm", "-D", "--defined-only", q4.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (q[48]_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "q4.h"\nint main(void){ q4_status s = Q4_OK; (void)s; return 0; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-c", str(src), "-o", str(tmp_path / "t.o")])


P = 0x100000  # a fake, 16-byte aligned "device pointer": never dereferenced by validation


def _mm(lib, x=P, M=1, K=64, codes=P, s=P, b=P, N=8, group=32, y=P):
    return lib.q4_matmul(x, M, K, codes, s, b, N, group, y, None)


def test_matmul_validation(lib):
    assert _mm(lib, group=64) == UNSUP
    assert b"group" in lib.q4_last_error()
    assert _mm(lib, K=48) == SHAPE
    assert _mm(lib, K=0) == SHAPE
    assert _mm(lib, M=-1) == SHAPE
    assert _mm(lib, N=-3) == SHAPE
    assert _mm(lib, M=0) == OK  # empty: nothing to do
    assert _mm(lib, N=0) == OK
    assert _mm(lib, x=None) == NULL
    assert _mm(lib, y=None) == NULL
    assert _mm(lib, x=P + 8) == ALIGN
    assert _mm(lib, codes=P + 4) == ALIGN
    assert _mm(lib, s=P + 1) == ALIGN
    assert _mm(lib, y=P + 1) == ALIGN


def test_step_validation(lib):
    st = lambda steps, step, **kw: lib.q4_matmul_step(P, 1, 64, P, P, P, 8, steps, step, kw.get("group", 32), P, None)
    assert st(16, 16) == RANGE
    assert st(16, -1) == RANGE
    assert st(0, 0) == RANGE
    assert b"step" in lib.q4_last_error()
    assert st(16, 3, group=16) == UNSUP


def test_quantize_dequantize_validation(lib):
    assert lib.q4_quantize(P, 4, 64, 32, P + 8, P, P, None) == ALIGN
    assert lib.q4_quantize(P, 4, 40, 32, P, P, P, None) == SHAPE
    assert lib.q4_quantize(None, 4, 64, 32, P, P, P, None) == NULL
    assert lib.q4_quantize(P, 0, 64, 32, P, P, P, None) == OK
    assert lib.q4_dequantize(P, P, P, 4, 64, 8, P, None) == UNSUP
    assert lib.q4_dequantize(P, P, P, -1, 64, 32, P, None) == SHAPE
    assert lib.q4_dequantize(P, P + 1, P, 4, 64, 32, P, None) == ALIGN


def test_residual_validation(lib):
    res = lambda r=P, y=P, M=1, N=8: lib.q4_matmul_residual(P, M, 64, P, P, P, N, 32, r, y, None)
    assert res(r=None) == NULL
    assert b"residual" in lib.q4_last_error()
    assert res(r=P + 1) == ALIGN
    # r may be y itself, but no other overlap: [P + 2, P + 18) against [P, P + 16)
    assert res(r=P + 2, y=P) == SHAPE
    assert res(r=P, y=P + 2) == SHAPE
    assert res(M=0) == OK


def test_swiglu_validation(lib):
    sw = lambda uc=P, us=P, ub=P, h=P: lib.q4_matmul_swiglu(P, 1, 64, P, P, P, uc, us, ub, 8, 32, h, None)
    assert sw(uc=None) == NULL
    assert sw(us=None) == NULL
    assert sw(uc=P + 8) == ALIGN
    assert sw(ub=P + 1) == ALIGN
    assert sw(h=None) == NULL
    assert lib.q4_matmul_swiglu(P, 1, 64, P, P, P, P, P, P, 8, 16, P, None) == UNSUP


def test_batch_descriptor_validation(lib):
    def one(**kw):
        d = q4.MatmulDesc(P, P, P, P, P, 8, 64)
        for k, v in kw.items():
            setattr(d, k, v)
        arr = (q4.MatmulDesc * 1)(d)
        return lib.q4_matmul_batch(ctypes.cast(arr, ctypes.c_void_p), 1, 1, 32, None)

    assert ctypes.sizeof(q4.MatmulDesc) == 96  # the C struct (include/q4.h) on LP64
    assert one(epilogue=7) == UNSUP
    assert b"epilogue" in lib.q4_last_error()
    assert one(reserved=1) == UNSUP
    assert one(epilogue=q4.EPI_RESIDUAL) == NULL  # r missing
    assert one(epilogue=q4.EPI_RESIDUAL, r=P + 1) == ALIGN
    assert one(epilogue=q4.EPI_SWIGLU, up_codes=P, up_scales=P) == NULL
    assert one(epilogue=q4.EPI_SWIGLU, up_codes=P + 4, up_scales=P, up_biases=P) == ALIGN


def test_batch_validates_every_entry_before_the_device():
    """A bad epilogue in the last entry is reported as such (not as the device
    error a valid batch reaches on a machine without a GPU): validation of the
    whole list precedes any device work, so nothing is enqueued."""
    from weight_only_bit_affine_b200 import build

    build.build()
    lib = q4.lib()
    good = q4.MatmulDesc(P, P, P, P, P, 8, 64)
    res = q4.MatmulDesc(P, P, P, P, P + 64, 8, 64)
    res.epilogue, res.r = q4.EPI_RESIDUAL, P + 64  # in place: allowed
    bad = q4.MatmulDesc(P, P, P, P, P + 128, 8, 64)
    bad.epilogue = 9
    arr = (q4.MatmulDesc * 3)(good, res, bad)
    assert lib.q4_matmul_batch(ctypes.cast(arr, ctypes.c_void_p), 3, 1, 32, None) == UNSUP
    assert b"q4_matmul_batch[2]" in lib.q4_last_error()
    import torch

    if not torch.cuda.is_available():
        arr = (q4.MatmulDesc * 2)(good, res)
        assert lib.q4_matmul_batch(ctypes.cast(arr, ctypes.c_void_p), 2, 1, 32, None) == CUDA


def test_chain_validation_precedes_the_device(lib):
    """q4_matmul_chain: stage counts that do not add up to count, a negative
    stage count, a missing stage array and a bad descriptor in the last stage
    are reported before any device work."""
    good = q4.MatmulDesc(P, P, P, P, P, 8, 64)
    bad = q4.MatmulDesc(P, P, P, P, P + 128, 8, 64)
    bad.epilogue = 9
    arr = (q4.MatmulDesc * 3)(good, good, bad)
    vp = lambda a: ctypes.cast(a, ctypes.c_void_p)
    counts = (ctypes.c_int * 2)(1, 1)
    assert lib.q4_matmul_chain(vp(arr), 3, vp(counts), 2, 1, 32, None) == SHAPE
    neg = (ctypes.c_int * 2)(4, -1)
    assert lib.q4_matmul_chain(vp(arr), 3, vp(neg), 2, 1, 32, None) == SHAPE
    assert lib.q4_matmul_chain(vp(arr), 3, None, 2, 1, 32, None) == NULL
    ok = (ctypes.c_int * 2)(2, 1)
    assert lib.q4_matmul_chain(vp(arr), 3, vp(ok), 2, 1, 32, None) == UNSUP
    assert b"q4_matmul_chain[2] (stage 1)" in lib.q4_last_error()
    assert lib.q4_matmul_chain(vp(arr), 0, None, 0, 1, 32, None) == 0


def test_descriptor_layout_matches_c(tmp_path):
    src = tmp_path / "l.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "q4.h"\n'
                   'int main(void){ printf("%zu %zu %zu %zu %zu", sizeof(q4_matmul_desc), '
                   'offsetof(q4_matmul_desc, epilogue), offsetof(q4_matmul_desc, r), '
                   'offsetof(q4_matmul_desc, up_codes), offsetof(q4_matmul_desc, up_biases)); return 0; }\n')
    exe = tmp_path / "l"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    D = q4.MatmulDesc
    assert got == [ctypes.sizeof(D), D.epilogue.offset, D.r.offset, D.up_codes.offset, D.up_biases.offset]


def test_q8_validation(lib):
    mm = lambda x=P, M=1, K=64, codes=P, group=32: lib.q8_matmul(x, M, K, codes, P, P, 8, group, P, None)
    assert mm(K=48) == SHAPE
    assert mm(group=64) == UNSUP
    assert mm(K=196608 + 32) == UNSUP
    assert b"K" in lib.q4_last_error()
    assert mm(codes=P + 8) == ALIGN
    assert mm(x=None) == NULL
    assert mm(M=0) == OK
    assert lib.q8_quantize(P, 4, 64, 32, P + 4, P, P, None) == ALIGN
    assert lib.q8_quantize(P, -1, 64, 32, P, P, P, None) == SHAPE
    assert lib.q8_dequantize(P, P, P, 4, 64, 32, P + 8, None) == ALIGN
    assert lib.q8_dequantize(None, P, P, 4, 64, 32, P, None) == NULL


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _mm(lib) == CUDA
    assert lib.q4_last_error() != b""


def test_python_binding_raises_on_status(lib):
    import torch

    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # CPU tensors are refused before the ABI
        q4.q4_matmul(x, torch.zeros((4, 32), dtype=torch.uint8), torch.zeros((4, 2), dtype=torch.bfloat16),
                     torch.zeros((4, 2), dtype=torch.bfloat16))
    err = q4.Q4Error(RANGE, "x")
    assert err.status_name == "Q4_ERR_RANGE"
