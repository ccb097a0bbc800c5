"""Every kernel path against the oracle on adversarial inputs (tests/adversarial.py):
all products x_k * w_hat_k non-negative, so |y| = sum |x w_hat| and the bf16
output rounding alone takes up to 3.9e-3 of the 4e-3 budget, with codes chosen
so that rounding w_hat to bf16 would push nearly every product the same way.

Rows M = 1, 2 (CUDA-core GEMV), 3..16 (group-sum tensor-core kernel) and
64, 256 (tensor-core tiles) at K = 4096 and 11264, every element of every
output checked, and the fused residual and SwiGLU epilogues on the same
inputs; the weight-streaming kernel (3..8 rows) and the tiles at 16 rows are
pinned by keeping the group-sum kernel out of the dispatch."""
import numpy as np
import pytest
import torch

import adversarial
import oracle
import weight_only_bit_affine_b200 as q4
from helpers import ABS, REL, kernels_disabled

pytestmark = pytest.mark.gpu

N = 256
M_ALL = (1, 2, 3, 4, 5, 8, 12, 15, 16, 64, 256)
_cache = {}


@pytest.fixture(autouse=True)
def _device_flags():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _case(family, K, which=0):
    key = (family, K, which)
    if key not in _cache:
        seed = 1000 * which + K + adversarial.FAMILIES.index(family)
        sigma = adversarial.signs(family, K, seed=K)  # one sign pattern per (family, K): gate and up share x
        codes, s, b = adversarial.packed_weight(family, N, K, seed, sigma)
        x = adversarial.activation(max(M_ALL), K, seed=K, sigma=sigma)
        dev = [torch.from_numpy(codes).cuda(),
               torch.from_numpy(s.view(np.int16)).view(torch.bfloat16).cuda(),
               torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda()]
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        _cache[key] = (x, (codes, s, b), xd, dev)
    return _cache[key]


def _check(y_dev, ref, bound, what):
    y = y_dev.float().cpu().double().numpy()
    ok = np.abs(y - ref) <= bound
    if not ok.all():
        m, n = np.argwhere(~ok)[0]
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} out of bound, e.g. [{m},{n}] "
                             f"got {y[m, n]!r} want {ref[m, n]!r} bound {bound[m, n]!r}")


@pytest.mark.parametrize("K", [4096, 11264])
@pytest.mark.parametrize("M", M_ALL)
@pytest.mark.parametrize("family", adversarial.FAMILIES)
def test_matmul_adversarial(family, M, K):
    x, host, xd, dev = _case(family, K)
    y = q4.q4_matmul(xd[:M].contiguous(), *dev)
    torch.cuda.synchronize()
    ref, absdot = oracle.matmul_ref(x[:M], *host)
    _check(y, ref, REL * absdot + ABS, f"{family} M={M} K={K}")


@pytest.mark.parametrize("M", [1, 4, 8, 16, 64])
@pytest.mark.parametrize("family", adversarial.FAMILIES)
def test_residual_adversarial(family, M):
    K = 4096
    x, host, xd, dev = _case(family, K)
    y0, _ = oracle.matmul_ref(x[:M], *host)
    # a residual of the same sign as the product, comparable in size
    rng = np.random.default_rng(M)
    r = adversarial._bf16_bits((y0 * rng.uniform(0.2, 2.0, size=y0.shape)).astype(np.float32))
    rd = torch.from_numpy(r.view(np.int16)).view(torch.bfloat16).cuda()
    y = q4.q4_matmul_residual(xd[:M].contiguous(), *dev, rd)
    torch.cuda.synchronize()
    ref, bound = oracle.matmul_residual_ref(x[:M], *host, r)
    _check(y, ref, bound, f"residual {family} M={M}")


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 64])
@pytest.mark.parametrize("family", adversarial.FAMILIES)
def test_swiglu_adversarial(family, M):
    K = 4096
    x, gate_h, xd, gate_d = _case(family, K, which=0)
    _, up_h, _, up_d = _case(family, K, which=1)
    h = q4.q4_matmul_swiglu(xd[:M].contiguous(), tuple(gate_d), tuple(up_d))
    torch.cuda.synchronize()
    ref, bound = oracle.matmul_swiglu_ref(x[:M], gate_h, up_h)
    _check(h, ref, bound, f"swiglu {family} M={M}")


@pytest.mark.parametrize("K", [4096, 11264])
@pytest.mark.parametrize("M", [4, 8, 16])
@pytest.mark.parametrize("family", adversarial.FAMILIES)
def test_matmul_adversarial_other_kernels(family, M, K):
    """The same inputs on the weight-streaming kernel (M = 4, 8) and on the
    tensor-core tiles (M = 16)."""
    x, host, xd, dev = _case(family, K)
    with kernels_disabled(q4.KERNEL_GROUP_SUM):
        y = q4.q4_matmul(xd[:M].contiguous(), *dev)
        torch.cuda.synchronize()
    ref, absdot = oracle.matmul_ref(x[:M], *host)
    _check(y, ref, REL * absdot + ABS, f"{family} M={M} K={K} (pinned)")
