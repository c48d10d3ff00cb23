"""MoE expert-parallel alltoallv: top-2 routing, dispatch and the inverse combine.

TEST INFRASTRUCTURE (see oracle/__init__.py).

Lecture 09 §6.4: the router picks an expert for each token, a first AllToAll sends each
token to the GPU that holds its expert, the experts run, and a second AllToAll returns the
outputs to the original GPU in input order. §3.8 / §7.4 experiment 4: rank j receives
[from rank 0, from rank 1, ...] (recv[j][i] = send[i][j]).

Readings (the page gives only the dataflow):
  routing   top-2 of the router logits: the two largest values, ties to the lower expert
            id; slot k = 0 holds the larger. Expert e lives on rank e // experts_per_rank,
            as local expert e % experts_per_rank. Both slots send a row, also when both
            experts are on one rank.
  order     the rows rank s sends to rank d are ordered by (local expert, token, slot);
            rank d's receive buffer is the concatenation of the blocks from ranks 0..N-1.
  combine   each row goes back to slot [token][k] of a [tokens, topk, hidden] buffer on its
            source rank (no gate weighting: that is model compute).
Experts are the identity, so the combine input is the dispatch output.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .collectives import alltoall
from .mesh import _MeshBase


def route_topk(logits: np.ndarray, topk: int = 2) -> np.ndarray:
    """[tokens, experts] fp32 logits -> [tokens, topk] int32 expert ids (stable sort on
    the negated logits: larger first, equal values keep the lower id first)."""
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :topk].astype(np.int32)


def send_lists(expert_ids: np.ndarray, n: int, experts_per_rank: int) -> list[np.ndarray]:
    """For one source rank: per destination, the flat row ids i = token * topk + k in send
    order (local expert, token, slot)."""
    flat = expert_ids.reshape(-1).astype(np.int64)
    rows = np.arange(flat.size, dtype=np.int64)
    dst = flat // experts_per_rank
    local = flat % experts_per_rank
    out = []
    for d in range(n):
        sel = rows[dst == d]
        key = local[sel]
        out.append(sel[np.lexsort((sel, key))])
    return out


def dispatch(tokens: Sequence[np.ndarray], expert_ids: Sequence[np.ndarray], experts_per_rank: int,
             *, mesh: Optional[_MeshBase] = None):
    """tokens[s]: [T, H] rows (any dtype, moved as bytes); expert_ids[s]: [T, topk].
    Returns per destination rank the received [rows, H] buffer, and the mesh."""
    n = len(tokens)
    topk = expert_ids[0].shape[1]
    lists = [send_lists(expert_ids[s], n, experts_per_rank) for s in range(n)]
    blocks = [[tokens[s][lists[s][d] // topk] for d in range(n)] for s in range(n)]
    recv, mesh = alltoall(blocks, mesh=mesh)
    h = tokens[0].shape[1]
    out = [np.concatenate(recv[d], axis=0) if recv[d] else np.zeros((0, h), tokens[0].dtype)
           for d in range(n)]
    return out, mesh


def combine(expert_out: Sequence[np.ndarray], expert_ids: Sequence[np.ndarray], experts_per_rank: int,
            *, mesh: Optional[_MeshBase] = None):
    """Inverse of dispatch: expert_out[d] is rank d's [rows, H] buffer in dispatch order.
    Returns per source rank a [T, topk, H] buffer."""
    n = len(expert_out)
    topk = expert_ids[0].shape[1]
    lists = [send_lists(expert_ids[s], n, experts_per_rank) for s in range(n)]
    # rank d cuts its buffer back into the per-source blocks it received
    blocks = []
    for d in range(n):
        sizes = [lists[s][d].size for s in range(n)]
        cuts = np.cumsum([0] + sizes)
        blocks.append([expert_out[d][cuts[s]:cuts[s + 1]] for s in range(n)])
    recv, mesh = alltoall(blocks, mesh=mesh)
    outs = []
    for s in range(n):
        t = expert_ids[s].shape[0]
        h = expert_out[0].shape[1]
        o = np.zeros((t * topk, h), dtype=expert_out[0].dtype)
        for d in range(n):
            o[lists[s][d]] = recv[s][d]
        outs.append(o.reshape(t, topk, h))
    return outs, mesh


def count_table(expert_ids: Sequence[np.ndarray], experts_total: int) -> np.ndarray:
    """[N, experts_total] int64: rows source rank s sends to each global expert."""
    return np.stack([np.bincount(e.reshape(-1), minlength=experts_total) for e in expert_ids])
