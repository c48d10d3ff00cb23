"""Oracle against the worked examples the collective pages print (tests/golden/)."""
import json
import os

import numpy as np
import pytest

from oracle import collectives as C

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")))["cases"]


def _f32(rows):
    return [np.asarray(r, dtype=np.float32) for r in rows]


@pytest.mark.parametrize("case", GOLDEN, ids=[c["op"] + ":" + c["cite"][:40] for c in GOLDEN])
def test_page_example(case):
    op = case["op"]
    if op == "broadcast":
        out, _ = C.broadcast(np.asarray(case["input"], np.float32), case["n"], case["root"])
        assert [o.tolist() for o in out] == case["expected"]
    elif op == "scatter":
        out, _ = C.scatter(np.asarray(case["input"], np.float32), case["n"], case["root"])
        assert [o.tolist() for o in out] == case["expected"]
    elif op == "gather":
        out, _ = C.gather(_f32(case["inputs"]), case["root"])
        assert out.tolist() == case["expected"]
    elif op == "reduce":
        out, _ = C.reduce(_f32(case["inputs"]), case["root"])
        assert out.tolist() == case["expected"]
    elif op == "allreduce":
        for fn in (C.ring_allreduce, C.tree_allreduce):
            out, _ = fn(_f32(case["inputs"]))
            assert [o.tolist() for o in out] == case["expected"]
    elif op == "reduce_scatter":
        out, _ = C.ring_reduce_scatter(_f32(case["inputs"]))
        assert [o.tolist() for o in out] == case["expected"]
    elif op == "allgather":
        out, _ = C.ring_allgather(_f32(case["inputs"]))
        assert [o.tolist() for o in out] == case["expected"]
    elif op == "alltoall":
        blocks = [[np.asarray([v]) for v in row] for row in case["send"]]
        recv, _ = C.alltoall(blocks)
        assert [[int(b[0]) for b in row] for row in recv] == case["expected"]
    elif op == "allreduce_fill":
        n, size = case["n"], case["size"]
        xs = [np.full(size, r + 1, dtype=np.float32) for r in range(n)]
        for fn in (C.ring_allreduce, C.tree_allreduce):
            out, _ = fn(xs)
            for o in out:
                assert np.all(o == np.float32(case["expected_value"]))
    else:
        raise AssertionError(f"unknown golden op {op}")


def test_int32_examples_match_too():
    """The same allreduce / reduce-scatter examples in int32 (order-free arithmetic)."""
    xs = [np.full(4, r + 1, dtype=np.int32) for r in range(4)]
    out, _ = C.ring_allreduce(xs, in_dtype="i32")
    assert all(o.tolist() == [10] * 4 for o in out)
    sh, _ = C.ring_reduce_scatter(xs, in_dtype="i32")
    assert [s.tolist() for s in sh] == [[10]] * 4
