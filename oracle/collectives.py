"""The collective schedules, executed literally as message passing on per-rank arrays.

TEST INFRASTRUCTURE (see oracle/__init__.py).

Every function takes one host array per simulated rank and returns one array per rank,
plus the Mesh that ran it (byte counters: mesh.sent / mesh.recvd, bytes per rank).

Arithmetic. Element values are numpy float32, int32, or uint16 bf16 bit patterns.
  SUM  one IEEE-754 binary32 add, round to nearest even (numpy float32 `+`), or a
       wrapping two's-complement int32 add. The receiver folds "local (+) incoming"
       (lecture 09 §7.1 experiment 1: chunks[recv][c] += val); binary32 addition is
       commutative, so only the bracketing matters, and the schedule fixes it.
  PROD one binary32 (or wrapping int32) multiply, folded like SUM.
  MAX / MIN  with -0 ordered below +0, so that the result never depends on operand
       order (lecture 09 §3.4 names SUM, MAX, MIN, PROD).
  bf16 input is widened exactly (bits << 16) on the rank that holds it, and all partial
  sums travel and fold in binary32.
  scale: the rank that completes a reduction multiplies the full result once by the
  binary32 `scale` (DDP divides the sum by the rank count, lecture 09 §3.5; reading: one
  multiply after the fold). int32 requires scale == 1 and never multiplies.

Sampling. `positions` (sorted element indices, default all) lets a caller run any
schedule on a subset of a buffer of `count` elements: chunk and half membership is
decided from the full count, so each sampled element sees exactly the operations it
sees in the full run. That is how full-size GPU outputs are checked element by element.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .layout import BinaryTree, binomial_children, binomial_parent, chunk_bounds, tree_half_split
from .mesh import LockstepMesh, _MeshBase

SUM, MAX, MIN, PROD = "sum", "max", "min", "prod"


# ---- element arithmetic ---------------------------------------------------------------------

def widen(x: np.ndarray, in_dtype: str) -> np.ndarray:
    """Rank-local conversion of an input buffer to its accumulation type."""
    if in_dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    if in_dtype == "f32":
        return np.array(x, dtype=np.float32, copy=True)
    if in_dtype == "i32":
        return np.array(x, dtype=np.int32, copy=True)
    raise ValueError(f"unknown dtype {in_dtype}")


def combine(local: np.ndarray, incoming: np.ndarray, op: str) -> np.ndarray:
    """local (op) incoming, one elementwise operation."""
    if op == SUM:
        return local + incoming
    if op == PROD:
        return local * incoming
    if op in (MAX, MIN):
        a, b = (local, incoming) if op == MAX else (incoming, local)
        # a < b in the order of values with -0 below +0; MAX keeps b when a < b, MIN keeps
        # (with the operands swapped) the smaller one the same way.
        lt = a < b
        if a.dtype == np.float32:
            lt = lt | ((a == b) & np.signbit(a) & ~np.signbit(b))
        return np.where(lt, b, a) if op == MAX else np.where(lt, a, b)
    raise ValueError(f"unknown op {op}")


def apply_scale(x: np.ndarray, scale: float) -> np.ndarray:
    if x.dtype == np.int32:
        if scale != 1:
            raise ValueError("int32 reductions take scale 1")
        return x
    return x * np.float32(scale)


def _local_slices(bounds, positions: Optional[np.ndarray]) -> list[slice]:
    """Map [start, stop) ranges of the full buffer onto the (sorted) sampled positions."""
    if positions is None:
        return [slice(a, b) for a, b in bounds]
    return [slice(int(np.searchsorted(positions, a)), int(np.searchsorted(positions, b)))
            for a, b in bounds]


def _prep(xs: Sequence[np.ndarray], in_dtype: str) -> list[np.ndarray]:
    return [widen(x, in_dtype) for x in xs]


# ---- ring allreduce, reduce-scatter, allgather ------------------------------------------------
# Lecture 09 §4.3 (two phases of N-1 steps each) and §7.1 experiment 1; the multi-node page
# §4.3.1 pseudocode; the from-scratch page "两趟实现 ring allreduce". In reduce-scatter
# step s, rank r sends chunk (r - s) mod N to rank r + 1, which folds it into its own copy;
# after N-1 steps rank r holds the full reduction of chunk (r + 1) mod N, i.e. chunk c is
# folded starting at rank c: ((x_c (+) x_{c+1}) (+) ...) (+) x_{c-1}. In allgather step s,
# rank r sends chunk (r - s + 1) mod N and the receiver overwrites.

def _ring_rs_phase(ctx, buf, sl, op):
    r, n = ctx.rank, ctx.n
    right, left = (r + 1) % n, (r - 1) % n
    for s in range(n - 1):
        ctx.send(right, buf[sl[(r - s) % n]], tag=("rs", s))
        c_in = (r - s - 1) % n
        incoming = yield from ctx.recv(left, tag=("rs", s))
        buf[sl[c_in]] = combine(buf[sl[c_in]], incoming, op)


def _ring_ag_phase(ctx, buf, sl, first_owned_offset):
    """first_owned_offset = 1 after reduce-scatter (rank r owns chunk r+1), 0 for a plain
    allgather (rank r owns chunk r)."""
    r, n = ctx.rank, ctx.n
    right, left = (r + 1) % n, (r - 1) % n
    for s in range(n - 1):
        ctx.send(right, buf[sl[(r - s + first_owned_offset) % n]], tag=("ag", s))
        c_in = (r - s - 1 + first_owned_offset) % n
        buf[sl[c_in]] = yield from ctx.recv(left, tag=("ag", s))


def ring_allreduce(xs: Sequence[np.ndarray], *, op: str = SUM, scale: float = 1.0,
                   in_dtype: str = "f32", count: Optional[int] = None,
                   positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    """Ring allreduce = ring reduce-scatter (N-1 steps) + ring allgather (N-1 steps)."""
    n = len(xs)
    bufs = _prep(xs, in_dtype)
    count = bufs[0].size if count is None else count
    sl = _local_slices(chunk_bounds(count, n), positions)
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        buf = bufs[ctx.rank]
        yield from _ring_rs_phase(ctx, buf, sl, op)
        own = sl[(ctx.rank + 1) % n]
        buf[own] = apply_scale(buf[own], scale)
        yield from _ring_ag_phase(ctx, buf, sl, 1)

    mesh.run(program)
    return bufs, mesh


def ring_reduce_scatter(xs: Sequence[np.ndarray], *, op: str = SUM, scale: float = 1.0,
                        in_dtype: str = "f32", count: Optional[int] = None,
                        positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    """The reduce-scatter half of the ring. Returns shard c (the reduction of chunk c) as
    rank c's output. The ring completes chunk c on rank c-1; handing it to output c is a
    relabelling of which rank is called the chunk's owner, and moves no bytes (reading:
    it keeps the fold order identical to the allreduce's, so allreduce equals
    reduce-scatter followed by allgather bit for bit, lecture 09 §3.9)."""
    n = len(xs)
    bufs = _prep(xs, in_dtype)
    count = bufs[0].size if count is None else count
    sl = _local_slices(chunk_bounds(count, n), positions)
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        buf = bufs[ctx.rank]
        yield from _ring_rs_phase(ctx, buf, sl, op)
        own = sl[(ctx.rank + 1) % n]
        buf[own] = apply_scale(buf[own], scale)

    mesh.run(program)
    shards = [bufs[(c - 1) % n][sl[c]].copy() for c in range(n)]
    return shards, mesh


def ring_allgather(shards: Sequence[np.ndarray], *, count: Optional[int] = None,
                   positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    """Rank r contributes chunk r of a count-element output; N-1 ring steps, overwrite."""
    n = len(shards)
    if count is None:
        count = sum(s.size for s in shards)
    sl = _local_slices(chunk_bounds(count, n), positions)
    total = count if positions is None else len(positions)
    bufs = []
    for r in range(n):
        b = np.zeros(total, dtype=shards[0].dtype)
        b[sl[r]] = shards[r]
        bufs.append(b)
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        yield from _ring_ag_phase(ctx, bufs[ctx.rank], sl, 0)

    mesh.run(program)
    return bufs, mesh


# ---- hierarchical allreduce -------------------------------------------------------------------
# Lecture 09 §9.3 design question 1 and appendix A Q4: with N = M nodes x G ranks per node
# (rank = node * G + local), (1) each node runs a ring reduce-scatter over its G ranks,
# (2) the G ranks that hold the same shard (one per node) run a ring allreduce across the M
# nodes, G such rings in parallel, (3) each node runs a ring allgather over its G ranks.
# Each phase is the ring of the section above on a sub-group (same send indices, same
# "local (+) incoming" fold), so element e of local chunk c and of sub-chunk j (the chunk
# rule applied to chunk c with M parts) folds, within every node, x_{m,c} (+) x_{m,c+1} ...
# and across nodes, starting at node j: (S_j (+) S_{j+1}) (+) ... (reading: the nodes are
# ordered by index, the inter-node ring is node j -> j + 1).

def _group_ring_rs(ctx, group, pos, buf, sl, op, tag):
    g = len(group)
    right, left = group[(pos + 1) % g], group[(pos - 1) % g]
    for s in range(g - 1):
        ctx.send(right, buf[sl[(pos - s) % g]], tag=(tag, s))
        c_in = (pos - s - 1) % g
        incoming = yield from ctx.recv(left, tag=(tag, s))
        buf[sl[c_in]] = combine(buf[sl[c_in]], incoming, op)


def _group_ring_ag(ctx, group, pos, buf, sl, first_owned_offset, tag):
    g = len(group)
    right, left = group[(pos + 1) % g], group[(pos - 1) % g]
    for s in range(g - 1):
        ctx.send(right, buf[sl[(pos - s + first_owned_offset) % g]], tag=(tag, s))
        c_in = (pos - s - 1 + first_owned_offset) % g
        buf[sl[c_in]] = yield from ctx.recv(left, tag=(tag, s))


def hierarchical_allreduce(xs: Sequence[np.ndarray], ranks_per_node: int, *, op: str = SUM, scale: float = 1.0,
                           in_dtype: str = "f32", count: Optional[int] = None,
                           positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    n = len(xs)
    G = ranks_per_node
    if G < 1 or n % G:
        raise ValueError("the rank count must be a multiple of ranks_per_node")
    M = n // G
    bufs = _prep(xs, in_dtype)
    count = bufs[0].size if count is None else count
    local_bounds = chunk_bounds(count, G)
    sl_local = _local_slices(local_bounds, positions)
    # sub-chunks of every local chunk, for the inter-node rings
    sl_sub = [_local_slices([(a + p, a + q) for p, q in chunk_bounds(b - a, M)], positions) for a, b in local_bounds]
    mesh = mesh or LockstepMesh(n, ranks_per_node=G)

    def program(ctx):
        m, l = divmod(ctx.rank, G)
        buf = bufs[ctx.rank]
        node = [m * G + k for k in range(G)]
        yield from _group_ring_rs(ctx, node, l, buf, sl_local, op, "h1")
        c = (l + 1) % G  # the local chunk this rank now holds complete for its node
        peers = [k * G + l for k in range(M)]
        yield from _group_ring_rs(ctx, peers, m, buf, sl_sub[c], op, "h2rs")
        own = sl_sub[c][(m + 1) % M]
        buf[own] = apply_scale(buf[own], scale)
        yield from _group_ring_ag(ctx, peers, m, buf, sl_sub[c], 1, "h2ag")
        yield from _group_ring_ag(ctx, node, l, buf, sl_local, 1, "h3")

    mesh.run(program)
    return bufs, mesh


# ---- multi-ring allreduce ---------------------------------------------------------------------
# Lecture 09 §5.3: for large cross-node messages the library runs several rings side by side,
# one per NIC rail. Reading (the page names the algorithm only): K rings; the message is cut
# into K contiguous parts by the chunk rule (K parts) and ring k runs the ring allreduce of
# §4.3 on part k, with the chunk rule over N inside the part. Even-numbered rings pass chunks
# to rank r + 1 exactly as above; odd-numbered rings run the same schedule the other way round:
# in reduce-scatter step s rank r sends chunk (r + s) mod N to rank r - 1, which folds it, so
# chunk c completes on rank c + 1 and its allgather starts there. With K >= 2 both directions
# of every link carry traffic. Chunk c of part k folds
#   ((x_c (+) x_{c+1}) (+) ...) (+) x_{c-1}   for even k,
#   ((x_c (+) x_{c-1}) (+) ...) (+) x_{c+1}   for odd k.
# The rings touch disjoint elements and use their own message tags, so running them one
# after another, as below, gives the same values and byte counts as running them side by side.

def _ring_rs_dir(ctx, buf, sl, op, d, tag):
    """Reduce-scatter phase of a ring whose chunks travel from rank r to rank r + d."""
    r, n = ctx.rank, ctx.n
    to, frm = (r + d) % n, (r - d) % n
    for s in range(n - 1):
        ctx.send(to, buf[sl[(r - d * s) % n]], tag=(tag, "rs", s))
        c_in = (r - d * s - d) % n
        incoming = yield from ctx.recv(frm, tag=(tag, "rs", s))
        buf[sl[c_in]] = combine(buf[sl[c_in]], incoming, op)


def _ring_ag_dir(ctx, buf, sl, d, tag):
    """Allgather phase after _ring_rs_dir: rank r starts with chunk r + d, complete."""
    r, n = ctx.rank, ctx.n
    to, frm = (r + d) % n, (r - d) % n
    for s in range(n - 1):
        ctx.send(to, buf[sl[(r - d * s + d) % n]], tag=(tag, "ag", s))
        c_in = (r - d * s) % n
        buf[sl[c_in]] = yield from ctx.recv(frm, tag=(tag, "ag", s))


def multiring_allreduce(xs: Sequence[np.ndarray], nrings: int, *, op: str = SUM, scale: float = 1.0,
                        in_dtype: str = "f32", count: Optional[int] = None,
                        positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    n = len(xs)
    if nrings < 1:
        raise ValueError("at least one ring")
    bufs = _prep(xs, in_dtype)
    count = bufs[0].size if count is None else count
    parts = chunk_bounds(count, nrings)
    sls = [_local_slices([(a + p, a + q) for p, q in chunk_bounds(b - a, n)], positions) for a, b in parts]
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        buf = bufs[ctx.rank]
        for k in range(nrings):
            d = 1 if k % 2 == 0 else -1
            yield from _ring_rs_dir(ctx, buf, sls[k], op, d, ("mr", k))
            own = sls[k][(ctx.rank + d) % n]
            buf[own] = apply_scale(buf[own], scale)
            yield from _ring_ag_dir(ctx, buf, sls[k], d, ("mr", k))

    mesh.run(program)
    return bufs, mesh


# ---- double binary tree allreduce -------------------------------------------------------------
# Lecture 09 §5.2 (reduce leaves -> root, then broadcast root -> leaves; 2 log2 N steps) and
# the multi-node page §4.3.2 (two trees, one per half of the data). Shapes: layout.BinaryTree.
# A node folds ((S_left (+) x_self) (+) S_right), skipping absent children (reading).

def tree_allreduce(xs: Sequence[np.ndarray], *, op: str = SUM, scale: float = 1.0,
                   in_dtype: str = "f32", count: Optional[int] = None,
                   positions: Optional[np.ndarray] = None, mesh: Optional[_MeshBase] = None):
    n = len(xs)
    bufs = _prep(xs, in_dtype)
    count = bufs[0].size if count is None else count
    mid = tree_half_split(count)
    halves = _local_slices([(0, mid), (mid, count)], positions)
    trees = [BinaryTree(n, mirrored=False), BinaryTree(n, mirrored=True)]
    mesh = mesh or LockstepMesh(n)

    def one_tree(ctx, t, tree, sl):
        r = ctx.rank
        buf = bufs[r]
        left, right, parent = tree.left[r], tree.right[r], tree.parent[r]
        acc = buf[sl].copy()
        if left is not None:
            s_left = yield from ctx.recv(left, tag=(t, "up"))
            acc = combine(s_left, acc, op)
        if right is not None:
            s_right = yield from ctx.recv(right, tag=(t, "up"))
            acc = combine(acc, s_right, op)
        if parent is not None:
            ctx.send(parent, acc, tag=(t, "up"))
            result = yield from ctx.recv(parent, tag=(t, "down"))
        else:
            result = apply_scale(acc, scale)
        buf[sl] = result
        for ch in tree.children(r):
            ctx.send(ch, result, tag=(t, "down"))

    def program(ctx):
        for t in range(2):
            yield from one_tree(ctx, t, trees[t], halves[t])

    mesh.run(program)
    return bufs, mesh


# ---- broadcast, reduce, scatter, gather -------------------------------------------------------

def broadcast(x_root: np.ndarray, n: int, root: int = 0, *, mesh: Optional[_MeshBase] = None):
    """Binomial-tree broadcast (from-scratch page: broadcast over a log2(N) tree; lecture 09
    §3.1). Every non-root receives the root's buffer exactly once."""
    bufs: list[Optional[np.ndarray]] = [None] * n
    bufs[root] = np.array(x_root, copy=True)
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        v = (ctx.rank - root) % n
        p = binomial_parent(v)
        if p is not None:
            bufs[ctx.rank] = yield from ctx.recv((p + root) % n, tag="bc")
        for ch in binomial_children(v, n):
            ctx.send((ch + root) % n, bufs[ctx.rank], tag="bc")

    mesh.run(program)
    return bufs, mesh


def reduce(xs: Sequence[np.ndarray], root: int = 0, *, op: str = SUM, in_dtype: str = "f32",
           mesh: Optional[_MeshBase] = None):
    """Reduce to root over the binomial tree (the broadcast tree run upward; lecture 09 §3.4).
    Node v folds its own buffer first, then each child's partial in the order it would send
    to them: ((x_v (+) S_c1) (+) S_c2) ... (reading). Only the root's result is defined."""
    n = len(xs)
    bufs = _prep(xs, in_dtype)
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        v = (ctx.rank - root) % n
        acc = bufs[ctx.rank]
        for ch in binomial_children(v, n):
            part = yield from ctx.recv((ch + root) % n, tag="rd")
            acc = combine(acc, part, op)
        p = binomial_parent(v)
        if p is not None:
            ctx.send((p + root) % n, acc, tag="rd")
        bufs[ctx.rank] = acc

    mesh.run(program)
    return bufs[root], mesh


def scatter(x_root: np.ndarray, n: int, root: int = 0, *, mesh: Optional[_MeshBase] = None):
    """Root sends block r of its buffer (chunk rule) straight to rank r (lecture 09 §3.2)."""
    sl = _local_slices(chunk_bounds(x_root.size, n), None)
    out: list[Optional[np.ndarray]] = [None] * n
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        if ctx.rank == root:
            for r in range(n):
                if r != root:
                    ctx.send(r, x_root[sl[r]], tag="sc")
            out[root] = x_root[sl[root]].copy()
        else:
            out[ctx.rank] = yield from ctx.recv(root, tag="sc")

    mesh.run(program)
    return out, mesh


def gather(xs: Sequence[np.ndarray], root: int = 0, *, mesh: Optional[_MeshBase] = None):
    """Every rank sends its block straight to root, which concatenates them in rank order
    (lecture 09 §3.3)."""
    n = len(xs)
    parts: list[Optional[np.ndarray]] = [None] * n
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        if ctx.rank != root:
            ctx.send(root, xs[ctx.rank], tag="ga")
            return
        for r in range(n):
            if r == root:
                parts[r] = np.array(xs[r], copy=True)
            else:
                parts[r] = yield from ctx.recv(r, tag="ga")

    mesh.run(program)
    return np.concatenate(parts), mesh


def alltoall(blocks: Sequence[Sequence[np.ndarray]], *, mesh: Optional[_MeshBase] = None):
    """blocks[i][j] = what rank i sends to rank j; rank j receives [blocks[0][j], ...,
    blocks[N-1][j]] (lecture 09 §3.8 and §7.4 experiment 4: recv[j][i] = send[i][j])."""
    n = len(blocks)
    recv: list[list] = [[None] * n for _ in range(n)]
    mesh = mesh or LockstepMesh(n)

    def program(ctx):
        i = ctx.rank
        for j in range(n):
            ctx.send(j, blocks[i][j], tag="a2a")
        for src in range(n):
            recv[i][src] = yield from ctx.recv(src, tag="a2a")

    mesh.run(program)
    return recv, mesh
