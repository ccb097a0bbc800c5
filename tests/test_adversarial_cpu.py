"""The adversarial families (tests/adversarial.py) have teeth, checked on the
CPU against the oracle: a kernel that rounds w_hat to bf16 before a bf16 MMA
breaks the acceptance bound on a large share of outputs, while the hi + lo
operand the tensor-core kernels use stays inside it everywhere.  Also pins
what the families promise: every product x_k * w_hat_k is non-negative, and
most weights round away from zero in bf16."""
import numpy as np
import pytest

import adversarial

REL, ABS = 4e-3, 1e-6


def _violations(y, ref, absdot):
    return np.abs(y - ref) > REL * absdot + ABS


@pytest.mark.parametrize("family", adversarial.FAMILIES)
def test_products_are_non_negative_and_rounding_aligned(oracle, family):
    M, N, K = 2, 64, 1024
    x, c, s, b = adversarial.case(family, M, N, K, seed=5)
    w = oracle.dequantize_f64(c, s, b)
    xf = oracle.bf16_bits_to_f64(x)
    prod = xf[:, None, :] * w[None, :, :]
    assert (prod >= 0).all(), "a product of the wrong sign"
    y, absdot = oracle.matmul_ref(x, c, s, b)
    assert np.allclose(y, absdot, rtol=1e-12, atol=0)
    # rounding w_hat to bf16 moves most weights away from zero
    wb = oracle.bf16_bits_to_f64(oracle.dequantize(c, s, b))
    up = (np.abs(wb) > np.abs(w)) | (w == 0)
    assert up.mean() > 0.7, up.mean()


@pytest.mark.parametrize("family", adversarial.FAMILIES)
@pytest.mark.parametrize("K", [4096, 11264])
def test_bf16_operand_breaks_the_bound_hi_lo_does_not(oracle, family, K):
    M, N = 4, 128
    x, c, s, b = adversarial.case(family, M, N, K, seed=11 + K)
    ref, absdot = oracle.matmul_ref(x, c, s, b)
    bad_bf16 = _violations(adversarial.simulate_bf16_operand(x, c, s, b), ref, absdot)
    bad_hilo = _violations(adversarial.simulate_hi_lo_operand(x, c, s, b), ref, absdot)
    assert bad_bf16.mean() > 0.05, f"the family should break a bf16 operand ({bad_bf16.mean():.3f})"
    assert not bad_hilo.any(), f"hi + lo out of bound on {int(bad_hilo.sum())} outputs"


def test_case_is_reproducible(oracle):
    a = adversarial.case("aligned", 2, 16, 256, seed=3)
    b = adversarial.case("aligned", 2, 16, 256, seed=3)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
