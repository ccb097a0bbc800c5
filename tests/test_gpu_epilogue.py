"""Fused output epilogues on the GPU -- the residual add (y = r + x w_hat^T)
and SwiGLU (h = silu(x w_gate^T) * x w_up^T) -- against the CPU oracle's
references, within the bounds those references return, for every kernel the
matmul dispatches to by M: the GEMV (bulk-copy and generic kernels), the
weight-streaming kernel and the tensor-core tiles, each computing SwiGLU's
two products in one pass.  Also the structural facts: in-place residual, zero residual
equal to the plain matmul, exact integer results, batch equal to single
calls bit for bit, and launch counts."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import bits, packed_to_host, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
M_ALL = [1, 2, 3, 4, 5, 16, 64]
# (N, K): depformer MLP and attention shapes, a ragged row count, small K on
# the bulk-copy kernel (teams within a warp), K with groups not a multiple of
# 8 (generic kernel), and the temporal MLP (checked on sampled rows).
SHAPES = [(1024, 1024), (77, 2816), (300, 256), (40, 96), (11264, 4096)]
# The residual also after the temporal down projection (K = 11264).
RES_SHAPES = SHAPES + [(4096, 11264)]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _packed(N, K, seed, tensor):
    return q4.q4_quantize(workloads.weight(N, K, seed, tensor, device=DEV))


def _rows(N):
    return None if N <= 1024 else sample_rows(N, 96, seed=N)


def _assert_within(y, ref, bound, rows, what):
    yg = y.float().cpu().double().numpy()
    if rows is not None:
        yg = yg[:, rows]
    ok = np.abs(yg - ref) <= bound
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        detail = [(int(m), int(n), float(yg[m, n]), float(ref[m, n]), float(bound[m, n])) for m, n in bad]
        raise AssertionError(f"{what}: {int((~ok).sum())} outside the bound, e.g. {detail}")


# ------------------------------------------------------------------------ residual


@pytest.mark.parametrize("M", M_ALL)
@pytest.mark.parametrize("N,K", RES_SHAPES)
def test_residual_matches_oracle(M, N, K):
    c, s, b = _packed(N, K, 60, N + K)
    x = workloads.activation(M, K, 60, 1000 + M, device=DEV)
    r = workloads.activation(M, N, 60, 2000 + M, device=DEV)  # residual stream ~ N(0, 1)
    y = q4.q4_matmul_residual(x, c, s, b, r)
    rows = _rows(N)
    ref, bound = oracle.matmul_residual_ref(bits(x), *packed_to_host(c, s, b), bits(r), rows=rows)
    _assert_within(y, ref, bound, rows, f"residual M={M} {N}x{K}")


@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_residual_in_place_and_zero(M):
    N, K = 1024, 1024
    c, s, b = _packed(N, K, 61, 0)
    x = workloads.activation(M, K, 61, 1, device=DEV)
    r = workloads.activation(M, N, 61, 2, device=DEV)
    y = q4.q4_matmul_residual(x, c, s, b, r)
    r2 = r.clone()
    q4.q4_matmul_residual(x, c, s, b, r2, out=r2)  # the residual stream updated in place
    assert torch.equal(r2, y)
    z = torch.zeros_like(r)
    assert torch.equal(q4.q4_matmul_residual(x, c, s, b, z), q4.q4_matmul(x, c, s, b))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 16])
def test_residual_exact_integers(M):
    """Integer x, s = 1, b = -8 and integer r: every partial sum is exact."""
    rng = np.random.default_rng(62 + M)
    for (N, K) in [(301, 4096), (33, 1024), (19, 256)]:
        q = rng.integers(0, 16, size=(N, K))
        codes = torch.from_numpy((q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)).to(DEV)
        s = torch.ones((N, K // 32), dtype=torch.bfloat16, device=DEV)
        b = torch.full((N, K // 32), -8.0, dtype=torch.bfloat16, device=DEV)
        x = torch.from_numpy(rng.integers(-4, 5, size=(M, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        r = torch.from_numpy(rng.integers(-60, 61, size=(M, N)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        y = q4.q4_matmul_residual(x, codes, s, b, r)
        ref, _ = oracle.matmul_residual_ref(bits(x), codes.cpu().numpy(), bits(s), bits(b), bits(r))
        assert torch.equal(y.cpu(), torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16)), (M, N, K)


# -------------------------------------------------------------------------- SwiGLU


@pytest.mark.parametrize("M", M_ALL)
@pytest.mark.parametrize("N,K", SHAPES)
def test_swiglu_matches_oracle(M, N, K):
    gate = _packed(N, K, 63, N + K)
    up = _packed(N, K, 63, 7 * N + K)
    x = workloads.activation(M, K, 63, 3000 + M, device=DEV)
    h = q4.q4_matmul_swiglu(x, gate, up)
    rows = _rows(N)
    ref, bound = oracle.matmul_swiglu_ref(bits(x), packed_to_host(*gate), packed_to_host(*up), rows=rows)
    _assert_within(h, ref, bound, rows, f"swiglu M={M} {N}x{K}")


# The tile kernel's widest epilogue tiles, split over a cluster of up to
# eight CTAs: SwiGLU with 128 activation rows a tile (its two accumulators
# fill tensor memory) and with a second, ragged row tile; the residual with
# 256 rows a tile and with a second, ragged row tile.
@pytest.mark.parametrize("M", [128, 200])
@pytest.mark.parametrize("N,K", [(300, 1024), (1024, 4096)])
def test_swiglu_wide_tiles(M, N, K):
    gate = _packed(N, K, 65, N + K)
    up = _packed(N, K, 65, 7 * N + K)
    x = workloads.activation(M, K, 65, 3000 + M, device=DEV)
    h = q4.q4_matmul_swiglu(x, gate, up)
    ref, bound = oracle.matmul_swiglu_ref(bits(x), packed_to_host(*gate), packed_to_host(*up))
    _assert_within(h, ref, bound, None, f"swiglu M={M} {N}x{K}")


@pytest.mark.parametrize("M", [256, 300])
@pytest.mark.parametrize("N,K", [(300, 1024), (1024, 11264)])
def test_residual_wide_tiles(M, N, K):
    c, s, b = _packed(N, K, 66, N + K)
    x = workloads.activation(M, K, 66, 1000 + M, device=DEV)
    r = workloads.activation(M, N, 66, 2000 + M, device=DEV)
    y = q4.q4_matmul_residual(x, c, s, b, r)
    ref, bound = oracle.matmul_residual_ref(bits(x), *packed_to_host(c, s, b), bits(r))
    _assert_within(y, ref, bound, None, f"residual M={M} {N}x{K}")


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 64])
def test_swiglu_one_pass_is_one_launch(M):
    gate, up = _packed(2816, 1024, 64, 0), _packed(2816, 1024, 64, 1)
    x = workloads.activation(M, 1024, 64, 2, device=DEV)
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_swiglu(x, gate, up)
    assert q4.q4_debug_launch_count() - n0 == 1


@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_batch_with_epilogues_matches_single_calls(M):
    """A step's worth of mixed problems in one q4_matmul_batch, one launch at
    M = 1 (GEMV) and at M = 4 and 16 (group-sum kernel): on the GEMV each
    output equals its single call bit for bit; on the group-sum kernel, whose
    partial sums follow the batch's split over the SMs, both are checked
    against the oracle's bounds."""
    x = workloads.activation(M, 1024, 65, 0, device=DEV)
    x2 = workloads.activation(M, 2816, 65, 1, device=DEV)
    g1, u1 = _packed(2816, 1024, 65, 2), _packed(2816, 1024, 65, 3)
    o = _packed(1024, 1024, 65, 4)
    d = _packed(1024, 2816, 65, 5)
    q = _packed(1024, 1024, 65, 6)
    r_o = workloads.activation(M, 1024, 65, 7, device=DEV)
    r_d = workloads.activation(M, 1024, 65, 8, device=DEV)
    outs = [torch.full((M, n), float("nan"), dtype=torch.bfloat16, device=DEV) for n in (2816, 1024, 1024, 1024)]
    probs = [
        (x, *g1, outs[0], q4.SwiGLU(*u1)),
        (x, *o, outs[1], q4.Residual(r_o)),
        (x2, *d, outs[2], q4.Residual(r_d)),
        (x, *q, outs[3]),
    ]
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_batch(probs)
    launches = q4.q4_debug_launch_count() - n0
    if M in (1, 4, 16):
        assert launches == 1
    singles = [q4.q4_matmul_swiglu(x, g1, u1), q4.q4_matmul_residual(x, *o, r_o),
               q4.q4_matmul_residual(x2, *d, r_d), q4.q4_matmul(x, *q)]
    if M <= 2:
        for i, (a, b_) in enumerate(zip(outs, singles)):
            assert torch.equal(a, b_), i
        return
    hx, hx2 = bits(x), bits(x2)
    for y in (outs[0], singles[0]):
        ref, bound = oracle.matmul_swiglu_ref(hx, packed_to_host(*g1), packed_to_host(*u1))
        _assert_within(y, ref, bound, None, f"batched swiglu M={M}")
    for y in (outs[1], singles[1]):
        ref, bound = oracle.matmul_residual_ref(hx, *packed_to_host(*o), bits(r_o))
        _assert_within(y, ref, bound, None, f"batched residual o M={M}")
    for y in (outs[2], singles[2]):
        ref, bound = oracle.matmul_residual_ref(hx2, *packed_to_host(*d), bits(r_d))
        _assert_within(y, ref, bound, None, f"batched residual down M={M}")
    for y in (outs[3], singles[3]):
        ref, absdot = oracle.matmul_ref(hx, *packed_to_host(*q))
        _assert_within(y, ref, 4e-3 * absdot + 1e-6, None, f"batched plain M={M}")


def test_epilogue_empty_sizes():
    c, s, b = _packed(8, 64, 66, 0)
    x0 = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    assert q4.q4_matmul_swiglu(x0, (c, s, b), (c, s, b)).shape == (0, 8)
    r0 = torch.empty((0, 8), dtype=torch.bfloat16, device=DEV)
    assert q4.q4_matmul_residual(x0, c, s, b, r0).shape == (0, 8)
