"""q4_matmul_chain: dependent matmuls (a decode step's layers) in one call.

With one or two activation rows the whole chain is one persistent launch in
which every CTA takes a share of every stage and waits, before reading a
stage's inputs, until all CTAs have finished the stage before.  The chain
must give exactly what q4_matmul_batch on each stage in turn gives (same
kernel arithmetic and the same row placement in tiles, whatever the split),
so these tests compare bit for bit with that sequence: a small decode model
(q, k, v -> o adding into the residual stream -> SwiGLU -> down adding into
the stream, several layers and a head) with in-place and out-of-place
residuals, stages of tiny problems, a chain longer than one launch holds,
a chain replayed from a CUDA graph, and the per-stage fallback at three
rows.  Stage outputs are also checked against the CPU oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_bit_affine_b200 as q4
from helpers import bits, check_matmul, packed_to_host, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q4.q4_device_status(clear=True)
    yield
    assert q4.q4_device_status() == 0, "a bounded wait gave up inside a kernel"


def _packed(N, K, seed, tensor):
    return q4.q4_quantize(workloads.weight(N, K, seed, tensor, device=DEV))


def _model(layers, d, f, vocab, seed):
    """Packed weights of a small decode model: per layer q, k, v, o [d, d],
    gate, up [f, d], down [d, f]; a head [vocab, d]."""
    W = []
    for l in range(layers):
        t = 10 * l
        W.append({"q": _packed(d, d, seed, t), "k": _packed(d, d, seed, t + 1), "v": _packed(d, d, seed, t + 2),
                  "o": _packed(d, d, seed, t + 3), "gate": _packed(f, d, seed, t + 4),
                  "up": _packed(f, d, seed, t + 5), "down": _packed(d, f, seed, t + 6)})
    return W, _packed(vocab, d, seed, 999)


def _decode_stages(W, head, h, M, in_place):
    """The stages of one decode step on the residual stream h [M, d]: per
    layer {q, k, v} -> o + residual (v's output standing in for attention)
    -> SwiGLU(gate, up) -> down + residual; then the head.  in_place: the
    residual adds update h itself; else each writes a fresh stream."""
    d = h.shape[1]
    stages, outs = [], []
    cur = h
    for P in W:
        f = P["gate"][0].shape[0]
        qkv = [torch.full((M, d), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(3)]
        stages.append([(cur, *P[n], y) for n, y in zip(("q", "k", "v"), qkv)])
        h1 = cur if in_place else torch.full((M, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        stages.append([(qkv[2], *P["o"], h1, q4.Residual(cur))])
        act = torch.full((M, f), float("nan"), dtype=torch.bfloat16, device=DEV)
        stages.append([(h1, *P["gate"], act, q4.SwiGLU(*P["up"]))])
        h2 = h1 if in_place else torch.full((M, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        stages.append([(act, *P["down"], h2, q4.Residual(h1))])
        outs += qkv + [h1, act, h2]
        cur = h2
    logits = torch.full((M, head[0].shape[0]), float("nan"), dtype=torch.bfloat16, device=DEV)
    stages.append([(cur, *head, logits)])
    return stages, outs + [logits]


def _run_both(build, M, seed):
    """build(h) -> (stages, outputs); runs the chain and the stage-by-stage
    batches from the same initial h; returns both output lists."""
    h0 = workloads.activation(M, build.d, seed, 1, device=DEV)
    h_a, h_b = h0.clone(), h0.clone()
    st_a, out_a = build(h_a)
    st_b, out_b = build(h_b)
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_chain(st_a)
    chain_launches = q4.q4_debug_launch_count() - n0
    for st in st_b:
        q4.q4_matmul_batch(st)
    torch.cuda.synchronize()
    return st_a, out_a + [h_a], out_b + [h_b], chain_launches


class _Decode:
    def __init__(self, layers, d, f, vocab, seed, M, in_place):
        self.W, self.head = _model(layers, d, f, vocab, seed)
        self.d, self.M, self.in_place = d, M, in_place

    def __call__(self, h):
        return _decode_stages(self.W, self.head, h, self.M, self.in_place)


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("in_place", [True, False])
def test_chain_equals_stagewise_batches(M, in_place):
    build = _Decode(3, 1024, 2816, 2048, 120 + M, M, in_place)
    stages, out_a, out_b, launches = _run_both(build, M, 121)
    assert launches == 1, launches
    for i, (a, b) in enumerate(zip(out_a, out_b)):
        assert not torch.isnan(a.float()).any(), i
        assert torch.equal(a, b), i
    # one plain stage against the oracle on its own (GPU-produced) input
    x, c, s, b, y = stages[-1][0][:5]
    check_matmul(x, c, s, b, y, rows=sample_rows(y.shape[1], 64, seed=M), what=f"chain head M={M}")


def test_chain_stage_outputs_against_oracle():
    """Out-of-place stream, M = 1: the o projection's residual output and
    the SwiGLU activation of the last layer, from their chain inputs."""
    M = 1
    build = _Decode(2, 1024, 2816, 512, 125, M, False)
    stages, out_a, _, _ = _run_both(build, M, 126)
    x, c, s, b, y, epi = stages[-4][0]  # last layer: o + residual
    ref, bound = oracle.matmul_residual_ref(bits(x), *packed_to_host(c, s, b), bits(epi.r))
    err = np.abs(y.float().cpu().double().numpy() - ref)
    assert (err <= bound).all(), float((err - bound).max())
    x, c, s, b, y, epi = stages[-3][0]  # last layer: SwiGLU
    ref, bound = oracle.matmul_swiglu_ref(bits(x), packed_to_host(c, s, b),
                                          packed_to_host(epi.up_codes, epi.up_scales, epi.up_biases))
    err = np.abs(y.float().cpu().double().numpy() - ref)
    assert (err <= bound).all(), float((err - bound).max())


@pytest.mark.parametrize("M", [1, 2])
def test_chain_tiny_and_mixed_stages(M):
    """Stages with fewer rows than SMs (most CTAs have nothing to do but
    still take part), several problems per stage, K from 256 to 11264."""
    seed = 130 + M
    w = [_packed(*shape, seed, t) for t, shape in
         enumerate([(7, 256), (11264, 256), (256, 11264), (300, 256), (5, 256), (256, 256)])]

    def build(h):
        y1 = torch.full((M, 11264), float("nan"), dtype=torch.bfloat16, device=DEV)
        ya = torch.full((M, 7), float("nan"), dtype=torch.bfloat16, device=DEV)
        y2 = torch.full((M, 256), float("nan"), dtype=torch.bfloat16, device=DEV)
        y3 = torch.full((M, 300), float("nan"), dtype=torch.bfloat16, device=DEV)
        y4 = torch.full((M, 5), float("nan"), dtype=torch.bfloat16, device=DEV)
        y5 = torch.full((M, 256), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = [[(h, *w[0], ya), (h, *w[1], y1)], [(y1, *w[2], y2)], [(y2, *w[3], y3), (y2, *w[4], y4)],
              [(y2, *w[5], y5, q4.Residual(h))]]
        return st, [ya, y1, y2, y3, y4, y5]

    build.d = 256
    _, out_a, out_b, launches = _run_both(build, M, seed)
    assert launches == 1
    for i, (a, b) in enumerate(zip(out_a, out_b)):
        assert torch.equal(a, b), i


def test_chain_longer_than_one_launch():
    """300 stages, each a 256 x 256 matmul of the previous stage's output
    (adding into it, but for every tenth: the values neither vanish nor
    grow without bound): two persistent launches."""
    M, n = 1, 300
    w = [_packed(256, 256, 140, t % 7) for t in range(n)]

    def build(h):
        st, outs, cur = [], [], h
        for t in range(n):
            y = torch.full((M, 256), float("nan"), dtype=torch.bfloat16, device=DEV)
            st.append([(cur, *w[t], y)] if t % 10 == 0 else [(cur, *w[t], y, q4.Residual(cur))])
            outs.append(y)
            cur = y
        return st, outs

    build.d = 256
    _, out_a, out_b, launches = _run_both(build, M, 141)
    assert launches == 2, launches
    for i, (a, b) in enumerate(zip(out_a, out_b)):
        assert torch.equal(a, b), i


def test_chain_graph_replay():
    """The chain captured in a CUDA graph and replayed twice (the stream
    reset between replays) equals a direct call."""
    M = 1
    build = _Decode(2, 1024, 2816, 1024, 150, M, True)
    h0 = workloads.activation(M, 1024, 151, 1, device=DEV)
    h = h0.clone()
    stages, outs = build(h)
    chain = q4.q4_prepare_chain(stages)
    chain.run()
    torch.cuda.synchronize()
    ref = [o.clone() for o in outs] + [h.clone()]
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    h.copy_(h0)
    torch.cuda.synchronize()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            chain.run()
    for _ in range(2):
        for o in outs:  # (the in-place stream h is among them: restored last)
            o.fill_(float("nan"))
        h.copy_(h0)
        g.replay()
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(zip(outs + [h], ref)):
            assert torch.equal(a, b), i
    del g


def test_chain_three_rows_runs_stage_by_stage():
    """M = 3: the chain is one q4_matmul_batch per stage (group-sum kernel)."""
    M = 3
    build = _Decode(2, 1024, 2816, 512, 160, M, True)
    stages, out_a, out_b, launches = _run_both(build, M, 161)
    assert launches == len(stages), launches
    for i, (a, b) in enumerate(zip(out_a, out_b)):
        assert torch.equal(a, b), i


def test_chain_off_the_bulk_copy_path_and_empty_stages():
    """A stage holding a problem the bulk-copy GEMV does not take (K = 96:
    the generic kernel) makes the whole chain run one batch per stage; empty
    stages (a zero count, or only empty problems) drop out.  Either way the
    result equals the stage-by-stage batches."""
    M = 1
    w96 = _packed(64, 96, 170, 0)
    w256 = _packed(96, 256, 170, 1)
    x = workloads.activation(M, 256, 170, 2, device=DEV)

    def build(h):
        y1 = torch.full((M, 96), float("nan"), dtype=torch.bfloat16, device=DEV)
        y2 = torch.full((M, 64), float("nan"), dtype=torch.bfloat16, device=DEV)
        return [[(h, *w256, y1)], [], [(y1, *w96, y2)]], [y1, y2]

    build.d = 256
    h0 = x.clone()
    st_a, out_a = build(h0.clone())
    st_b, out_b = build(h0.clone())
    n0 = q4.q4_debug_launch_count()
    q4.q4_matmul_chain(st_a)
    assert q4.q4_debug_launch_count() - n0 == 2  # one batch per non-empty stage
    for st in st_b:
        q4.q4_matmul_batch(st)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(out_a, out_b)):
        assert torch.equal(a, b), i

