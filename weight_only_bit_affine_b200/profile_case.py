"""Small, named workloads for profiling libq4 under ncu.

    python -m weight_only_bit_affine_b200.profile_case <case> [reps]

Cases (seeded synthetic inputs of the workload shapes; each rep runs the
whole case once, after one warm-up rep):

  stream_small   3 temporal layers + the text head (553 MB packed) as one
                 q4_matmul_batch per rep: the benchmark's kernel on a case
                 small enough for a full ncu capture.
  tc_layer       one temporal layer (7 projections, 128 MB) through q4_matmul
                 at M = 64 and then M = 256: the tensor-core kernel.
  depformer_step one depformer codebook step (43 step-sliced projections) as
                 one q4_matmul_batch.
  layer_m4       one temporal layer (7 projections) at M = 4 as one
                 q4_matmul_batch: the tensor-core streaming kernel.
  fused_layer    one temporal layer at M = 1 with its epilogues fused (o and
                 down + residual, gate/up as one SwiGLU problem), one
                 q4_matmul_batch: the GEMV's epilogue instantiation.
  q8_layer       one temporal layer with 8-bit codes at M = 1, one q8_matmul
                 per projection: the 8-bit GEMV.

Every case checks the library's bounded-wait flag at the end.
"""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _stream_small(dev):
    import torch

    import workloads
    import weight_only_bit_affine_b200 as q4

    projs = workloads.stream_projs()
    sel = [(t, p) for t, p in enumerate(projs) if p.name.startswith(("L0.", "L1.", "L2."))] + [(len(projs) - 1, projs[-1])]
    seed = workloads.seed_of("temporal_stream")
    x = workloads.activation(1, 4096, seed, 10000, device=dev)
    xd = workloads.activation(1, 11264, seed, 10001, device=dev)
    probs = []
    for t, p in sel:
        c, s, b = q4.q4_quantize(workloads.weight(p.N, p.K, seed, t, device=dev))
        probs.append((xd if p.K == 11264 else x, c, s, b, torch.empty((1, p.N), dtype=torch.bfloat16, device=dev)))
    return lambda: q4.q4_matmul_batch(probs)


def _tc_layer(dev):
    import workloads
    import weight_only_bit_affine_b200 as q4

    seed = workloads.seed_of("batched_layer")
    packed = [(p,) + tuple(q4.q4_quantize(workloads.weight(p.N, p.K, seed, t, device=dev)))
              for t, p in enumerate(workloads.TEMPORAL_LAYER)]
    xs = {M: (workloads.activation(M, 4096, seed, 100 + M, device=dev),
              workloads.activation(M, 11264, seed, 200 + M, device=dev)) for M in (64, 256)}

    def run():
        for M in (64, 256):
            for p, c, s, b in packed:
                q4.q4_matmul(xs[M][1] if p.K == 11264 else xs[M][0], c, s, b)

    return run


def _depformer_step(dev):
    import torch

    import workloads
    import weight_only_bit_affine_b200 as q4

    seed = workloads.seed_of("depformer_steps")
    steps = workloads.DEPFORMER_STEPS
    xs = {K: workloads.activation(1, K, seed, 500 + K, device=dev) for K in (1024, 2816)}
    probs = []
    for t, p in enumerate(workloads.depformer_projs()):
        c, s, b = q4.q4_quantize(workloads.weight(steps * p.N, p.K, seed, t, device=dev))
        probs.append((xs[p.K], c[:p.N], s[:p.N], b[:p.N], torch.empty((1, p.N), dtype=torch.bfloat16, device=dev)))
    return lambda: q4.q4_matmul_batch(probs)


def _layer_m4(dev):
    import torch

    import workloads
    import weight_only_bit_affine_b200 as q4

    seed = workloads.seed_of("batched_layer")
    M = 4
    x = workloads.activation(M, 4096, seed, 100 + M, device=dev)
    xd = workloads.activation(M, 11264, seed, 200 + M, device=dev)
    probs = []
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = q4.q4_quantize(workloads.weight(p.N, p.K, seed, t, device=dev))
        probs.append((xd if p.K == 11264 else x, c, s, b, torch.empty((M, p.N), dtype=torch.bfloat16, device=dev)))
    return lambda: q4.q4_matmul_batch(probs)


def _fused_layer(dev):
    import torch

    import workloads
    import weight_only_bit_affine_b200 as q4

    seed = workloads.seed_of("batched_layer")
    x = workloads.activation(1, 4096, seed, 101, device=dev)
    xd = workloads.activation(1, 11264, seed, 201, device=dev)
    w = {p.name: q4.q4_quantize(workloads.weight(p.N, p.K, seed, t, device=dev))
         for t, p in enumerate(workloads.TEMPORAL_LAYER)}
    out = lambda n: torch.empty((1, n), dtype=torch.bfloat16, device=dev)
    r_o = torch.zeros((1, 4096), dtype=torch.bfloat16, device=dev)  # two residual streams: problems of
    r_d = torch.zeros((1, 4096), dtype=torch.bfloat16, device=dev)  # one launch may not share an output
    probs = [(x, *w[n], out(4096)) for n in ("q", "k", "v")]
    probs += [(x, *w["o"], r_o, q4.Residual(r_o)), (x, *w["gate"], out(11264), q4.SwiGLU(*w["up"])),
              (xd, *w["down"], r_d, q4.Residual(r_d))]
    return lambda: q4.q4_matmul_batch(probs)


def _q8_layer(dev):
    import torch

    import workloads
    import weight_only_bit_affine_b200 as q4

    seed = workloads.seed_of("batched_layer")
    x = workloads.activation(1, 4096, seed, 101, device=dev)
    xd = workloads.activation(1, 11264, seed, 201, device=dev)
    items = []
    for t, p in enumerate(workloads.TEMPORAL_LAYER):
        c, s, b = q4.q8_quantize(workloads.weight(p.N, p.K, seed, t, device=dev))
        items.append((xd if p.K == 11264 else x, c, s, b, torch.empty((1, p.N), dtype=torch.bfloat16, device=dev)))

    def run():
        for xx, c, s, b, y in items:
            q4.q8_matmul(xx, c, s, b, out=y)

    return run


CASES = {"stream_small": _stream_small, "tc_layer": _tc_layer, "depformer_step": _depformer_step,
         "layer_m4": _layer_m4, "fused_layer": _fused_layer, "q8_layer": _q8_layer}


def main(argv=None):
    import torch

    import weight_only_bit_affine_b200 as q4

    argv = sys.argv[1:] if argv is None else argv
    if not argv or argv[0] not in CASES:
        raise SystemExit(f"usage: profile_case <{'|'.join(CASES)}> [reps]")
    reps = int(argv[1]) if len(argv) > 1 else 3
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    run = CASES[argv[0]](dev)
    torch.cuda.synchronize(dev)
    for _ in range(1 + reps):
        run()
    torch.cuda.synchronize(dev)
    if q4.q4_device_status() != 0:
        raise SystemExit("a bounded wait gave up inside a kernel")
    print(f"{argv[0]}: {reps} reps ok")


if __name__ == "__main__":
    main()
