"""The synthetic workloads: shapes and packed sizes against the figures the
benchmark and the design quote (from the pages' architecture: 32 temporal
layers of width 4096 with an 11264-wide SwiGLU feed-forward and a 32k text
head; a 6-layer, 1024-wide depformer stacked over 16 codebook steps), and the
seeded draws' determinism and distributions.  No GPU."""
import numpy as np
import pytest

import workloads


def _packed(projs, oracle):
    return sum(oracle.packed_nbytes(p.N, p.K) for p in projs)


def test_temporal_stream_shapes_and_bytes(oracle):
    projs = workloads.stream_projs()
    assert len(projs) == 7 * 32 + 1
    params = sum(p.N * p.K for p in projs)
    assert params == 6_707_740_672  # ~7B temporal transformer incl. the text head
    assert _packed(projs, oracle) == 4_192_337_920 == params * 5 // 8
    assert _packed(workloads.TEMPORAL_LAYER, oracle) == 128_450_560
    # the down projections take the SwiGLU width, every other projection the model width
    assert {p.K for p in projs if p.name.endswith(".down")} == {11264}
    assert {p.K for p in projs if not p.name.endswith(".down")} == {4096}


def test_depformer_step_and_frame_bytes(oracle):
    projs = workloads.depformer_projs()
    assert len(projs) == 7 * 6 + 1
    step = _packed(projs, oracle)
    assert step == 49_479_680
    assert step * workloads.DEPFORMER_STEPS == 791_674_880


def test_seed_order_and_determinism():
    assert [workloads.seed_of(w) for w in workloads.WORKLOADS] == [0, 1, 2, 3, 4]
    a = workloads.weight(64, 128, seed=3, tensor=7)
    b = workloads.weight(64, 128, seed=3, tensor=7)
    c = workloads.weight(64, 128, seed=3, tensor=8)
    assert np.array_equal(workloads.bf16_bits(a), workloads.bf16_bits(b))
    assert not np.array_equal(workloads.bf16_bits(a), workloads.bf16_bits(c))


@pytest.mark.parametrize("std,make", [(workloads.W_STD, workloads.weight), (workloads.X_STD, workloads.activation)])
def test_gaussian_draws(std, make):
    t = make(512, 1024, 0, 1).float().numpy()
    assert abs(t.mean()) < 0.01 * std
    assert abs(t.std() / std - 1.0) < 0.01
    # bf16 values: the low 16 bits of every fp32 are zero
    assert np.all((t.view(np.uint32) & 0xFFFF) == 0)
