"""Oracle for the collective primitives: plain, slow, literal CPU message passing.

TEST INFRASTRUCTURE ONLY. tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
leg are the only callers; the CUDA library and its Python binding never import it, and
it imports nothing from them.

What it does: N simulated ranks each own numpy arrays; the schedules the collective pages
describe (ring reduce-scatter + allgather, double binary tree, binomial broadcast,
alltoall / alltoallv, DDP buckets) run step by step as send / recv on a mesh of FIFO
channels, with per-rank byte counters. Floating point: binary32 folds in exactly the
order each schedule implies (the pages fix binary32 in the ring experiment, lecture 09
§7.1); bf16 inputs are widened exactly to binary32 first.

Modules:
  mesh         LockstepMesh (deterministic) and ThreadedMesh (timeouts, fault injection)
  layout       ring chunk rule, double-binary-tree shapes, binomial tree
  collectives  ring allreduce / reduce-scatter / allgather, tree allreduce, broadcast,
               reduce, scatter, gather, alltoall
  moe          top-2 routing and the alltoallv dispatch / combine
  ddp          bucket assignment, flatten, averaged allreduce, unflatten

Pins (tests/test_oracle_*.py): the pages' worked examples (tests/golden/), the per-rank
byte counts the pages derive, allreduce == allgather(reduce_scatter) bit for bit, the
N = 1 identity, int32 against brute-force sums, fp32 against an independent left-fold /
recursive evaluator and against an fp64 error bound, tree-shape invariants and hand-derived
tree shapes for N = 5, 6, 8, 13 (tests/golden/tree_shapes.json), the binomial reduce's
bracketing against an evaluator built from the broadcast's rounds, alltoallv round trip and
count conservation, and gloo (int32) on CPU processes.
Parity unpinned: the per-rank byte figures the pages give for the tree (they disagree with
one another; the oracle counts what its own schedule moves).
"""
from . import collectives, ddp, layout, mesh, moe  # noqa: F401
