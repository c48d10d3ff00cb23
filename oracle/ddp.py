"""DDP gradient buckets: assignment, flatten, ring allreduce with the 1/N scale, unflatten.

TEST INFRASTRUCTURE (see oracle/__init__.py).

Lecture 09 §6.1 and the from-scratch page ("allreduce 前先把梯度 bucket 起来"): gradients
are packed into buckets of about 25 MB, in the reverse order of the layers (the order
backward produces them), small tensors ride with large ones, one allreduce per bucket,
then each rank divides by the rank count.

Readings: the cap is 25 MiB; tensors are taken in reverse registration order and never
split; a new bucket starts when the next tensor would push a non-empty bucket over the
cap (so a tensor larger than the cap forms a bucket of its own); inside a bucket the
tensors lie in the order they were taken. The average is one binary32 multiply of the
ring sum by fl(1/N) (exact division for N = 8).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .collectives import SUM, ring_allreduce, tree_allreduce

CAP_BYTES = 25 * 1024 * 1024


def assign_buckets(numels: Sequence[int], elem_bytes: int = 4, cap_bytes: int = CAP_BYTES) -> list[list[int]]:
    """Tensor indices per bucket (indices into registration order), buckets in launch order."""
    buckets: list[list[int]] = []
    cur: list[int] = []
    cur_bytes = 0
    for i in reversed(range(len(numels))):
        b = numels[i] * elem_bytes
        if cur and cur_bytes + b > cap_bytes:
            buckets.append(cur)
            cur, cur_bytes = [], 0
        cur.append(i)
        cur_bytes += b
    if cur:
        buckets.append(cur)
    return buckets


def flatten(grads: Sequence[np.ndarray], members: Sequence[int]) -> np.ndarray:
    return np.concatenate([np.asarray(grads[i]).reshape(-1) for i in members])


def unflatten(flat: np.ndarray, grads_like: Sequence[np.ndarray], members: Sequence[int]) -> dict[int, np.ndarray]:
    out, off = {}, 0
    for i in members:
        n = grads_like[i].size
        out[i] = flat[off:off + n].reshape(grads_like[i].shape)
        off += n
    return out


def ddp_allreduce(grads: Sequence[Sequence[np.ndarray]], *, scale: Optional[float] = None,
                  cap_bytes: int = CAP_BYTES, algo: str = "ring", buckets=None):
    """grads[r][i] = rank r's gradient tensor i (registration order). Returns the averaged
    gradients per rank and the list of per-bucket meshes."""
    n = len(grads)
    scale = (1.0 / n) if scale is None else scale
    numels = [g.size for g in grads[0]]
    buckets = assign_buckets(numels, grads[0][0].itemsize, cap_bytes) if buckets is None else buckets
    outs: list[list[Optional[np.ndarray]]] = [[None] * len(numels) for _ in range(n)]
    meshes = []
    reduce_fn = ring_allreduce if algo == "ring" else tree_allreduce
    for members in buckets:
        flats = [flatten(grads[r], members) for r in range(n)]
        res, mesh = reduce_fn(flats, op=SUM, scale=scale)
        meshes.append(mesh)
        for r in range(n):
            for i, t in unflatten(res[r], grads[r], members).items():
                outs[r][i] = t
    return outs, meshes
