"""Pins of two oracle readings that the order-free checks cannot see: the double binary
tree's exact shape for N other than 8, and the fp32 bracketing of the binomial reduce.

Tree shapes: tests/golden/tree_shapes.json holds tree A and tree B for N = 5, 6, 8, 13,
derived by hand from the shape reading (the multi-node training page §4.3.2 gives only
"two trees, one per half"; lecture 09 §5.2 the leaves-to-root-and-back order). The oracle's
layout must reproduce them, and its tree allreduce must equal a recursive evaluation over
the golden shapes (not over the oracle's own layout).

Binomial reduce (lecture 09 §3.4 gives only the sum): the reading is the binomial broadcast
tree run upward, each node folding its own value first and then each child's partial in the
order the broadcast sends to that child. The evaluator here derives the send order by
simulating the broadcast's rounds (in round k every rank below 2^k that already holds the
data sends to rank + 2^k), which is a different construction from the oracle's
children formula, and folds recursively. Inputs whose magnitudes span 2^-20..2^20 make the
bracketing visible; planted mistakes (children in reverse order, the node's own value folded
last) must fail the pin.
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import layout as L

SHAPES = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tree_shapes.json")))["cases"]


def _bits(a):
    return np.ascontiguousarray(a).view(np.uint32)


def _spread_f32(seed, n, count):
    out = []
    for r in range(n):
        u = synth.uniform_f32(seed, r, count)
        e = synth.int32_uniform(seed, r, count, -20, 20, stream=1)
        out.append((u * np.exp2(e).astype(np.float32)).astype(np.float32))
    return out


# ---- double binary tree shapes -------------------------------------------------------------------

def _golden_tree(case, which):
    t = case[which]
    left = {int(k): v for k, v in t["left"].items()}
    right = {int(k): v for k, v in t["right"].items()}
    return t["root"], left, right


@pytest.mark.parametrize("case", SHAPES, ids=[f"n{c['n']}" for c in SHAPES])
def test_layout_reproduces_hand_derived_tree_shapes(case):
    n = case["n"]
    for which, mirrored in (("tree_a", False), ("tree_b", True)):
        root, left, right = _golden_tree(case, which)
        t = L.BinaryTree(n, mirrored)
        assert t.root == root, which
        assert {r: t.left[r] for r in range(n) if t.left[r] is not None} == left, which
        assert {r: t.right[r] for r in range(n) if t.right[r] is not None} == right, which


def _golden_fold(xs, e, root, left, right):
    """((S_left + x_v) + S_right) over a golden shape, one binary32 add at a time."""
    def val(v):
        acc = np.float32(xs[v][e])
        if v in left:
            acc = np.float32(val(left[v]) + acc)
        if v in right:
            acc = np.float32(acc + val(right[v]))
        return acc
    return val(root)


@pytest.mark.parametrize("case", SHAPES, ids=[f"n{c['n']}" for c in SHAPES])
def test_tree_allreduce_folds_over_the_golden_shapes(case):
    n = case["n"]
    count = 4 * n + 3
    xs = _spread_f32(41, n, count)
    out, _ = C.tree_allreduce(xs)
    mid = (count + 1) // 2
    ta, tb = _golden_tree(case, "tree_a"), _golden_tree(case, "tree_b")
    for e in range(count):
        want = np.float32(_golden_fold(xs, e, *(ta if e < mid else tb))).view(np.uint32)
        for o in out:
            assert _bits(o[e:e + 1])[0] == want


# ---- binomial reduce bracketing ---------------------------------------------------------------------

def _broadcast_send_lists(n):
    """Relative rank -> the ranks it sends to, in send order, from the broadcast's rounds:
    in round k = 0, 1, ... every relative rank u < 2^k sends to u + 2^k when that is < n."""
    sends = {u: [] for u in range(n)}
    k = 0
    while (1 << k) < n:
        for u in range(min(1 << k, n)):
            if u + (1 << k) < n:
                sends[u].append(u + (1 << k))
        k += 1
    return sends


def _binomial_reduce_expected(xs, root):
    n = len(xs)
    sends = _broadcast_send_lists(n)

    def partial(v):  # relative rank v: own value first, then each child's partial in send order
        acc = np.asarray(xs[(v + root) % n], dtype=np.float32).copy()
        for c in sends[v]:
            acc = (acc + partial(c)).astype(np.float32)
        return acc
    return partial(0)


CASES = [(n, root) for n in (3, 4, 5, 8, 13, 64) for root in sorted({0, 1, n // 2, n - 1})]


@pytest.mark.parametrize("n,root", CASES)
def test_binomial_reduce_bracketing_matches_independent_evaluator(n, root):
    xs = _spread_f32(43 + n, n, 257)
    got, _ = C.reduce(xs, root)
    assert np.array_equal(_bits(got), _bits(_binomial_reduce_expected(xs, root)))


def test_broadcast_rounds_give_each_non_root_one_sender():
    for n in range(1, 70):
        senders = [u for lst in _broadcast_send_lists(n).values() for u in lst]
        assert sorted(senders) == list(range(1, n))


def _pin_holds():
    return all(np.array_equal(_bits(C.reduce(xs, root)[0]), _bits(_binomial_reduce_expected(xs, root)))
               for n, root in ((4, 0), (8, 3), (13, 5))
               for xs in [_spread_f32(47, n, 257)])


def test_planted_reversed_children_order_is_caught(monkeypatch):
    real = C.binomial_children
    monkeypatch.setattr(C, "binomial_children", lambda v, n: list(reversed(real(v, n))))
    assert not _pin_holds()


def test_planted_own_value_folded_last_is_caught(monkeypatch):
    """A reduce that folds the children's partials first and the node's own value last."""
    def wrong_reduce(xs, root=0, *, op=C.SUM, in_dtype="f32", mesh=None):
        n = len(xs)
        bufs = C._prep(xs, in_dtype)
        mesh = mesh or C.LockstepMesh(n)

        def program(ctx):
            v = (ctx.rank - root) % n
            acc = None
            for ch in C.binomial_children(v, n):
                part = yield from ctx.recv((ch + root) % n, tag="rd")
                acc = part if acc is None else C.combine(acc, part, op)
            acc = bufs[ctx.rank] if acc is None else C.combine(acc, bufs[ctx.rank], op)
            p = C.binomial_parent(v)
            if p is not None:
                ctx.send((p + root) % n, acc, tag="rd")
            bufs[ctx.rank] = acc

        mesh.run(program)
        return bufs[root], mesh

    assert _pin_holds()
    monkeypatch.setattr(C, "reduce", wrong_reduce)
    assert not _pin_holds()
