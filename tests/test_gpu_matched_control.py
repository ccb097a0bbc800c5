"""Matched control: the quantized matmul against the unquantized path on the
same inputs (model card "personaplex-edge-q4", section "Matched Q4 and BF16 control":
Q4 and the BF16 checkpoint run on the same inputs).  Here the unquantized path is
torch's dense fp32 matmul of x with the dequantized bf16 weights -- a
library cross-check beside the oracle parity tests.

Bound: W_hat rounds s*q + b to bf16 (at most 2^-8 -- bf16's unit roundoff
-- of each |x w_hat| term) and y is rounded to bf16 once (2^-8 of |y|), so
the two paths differ by at most 2 * 2^-8 = 7.8e-3 of sum|x w_hat| plus fp32
accumulation errors (~1e-7): checked against 8e-3 * sum|x w_hat| + 1e-6."""
import pytest
import torch

import workloads
import weight_only_bit_affine_b200 as q4

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _dense_check(x, W_hat, y):
    xf, wf = x.float(), W_hat.float()
    dense = xf @ wf.T
    absdot = xf.abs() @ wf.abs().T
    diff = (y.float() - dense).abs()
    assert bool((diff <= 8e-3 * absdot + 1e-6).all()), float((diff / (absdot + 1e-30)).max())


@pytest.mark.parametrize("M", [1, 2, 4, 64])
def test_q4_matmul_matches_dense_matmul_of_dequantized_weights(M):
    N, K = 1024, 4096
    c, s, b = q4.q4_quantize(workloads.weight(N, K, 90, 0, device=DEV))
    W_hat = q4.q4_dequantize(c, s, b)
    x = workloads.activation(M, K, 90, 1 + M, device=DEV)
    _dense_check(x, W_hat, q4.q4_matmul(x, c, s, b))


@pytest.mark.parametrize("M", [1, 3])
def test_q8_matmul_matches_dense_matmul_of_dequantized_weights(M):
    N, K = 512, 2816
    c, s, b = q4.q8_quantize(workloads.weight(N, K, 91, 0, device=DEV))
    W_hat = q4.q8_dequantize(c, s, b)
    x = workloads.activation(M, K, 91, 1 + M, device=DEV)
    _dense_check(x, W_hat, q4.q8_matmul(x, c, s, b))
