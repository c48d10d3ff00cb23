"""Index layouts the schedules use: ring chunks, the double binary tree, the binomial tree.

TEST INFRASTRUCTURE (see oracle/__init__.py).

Readings (the pages leave these open; each is stated where it is used):
  chunk rule   lecture 09 §7.1 experiment 1 asserts that the tensor length divides by
               the GPU count. For any count: q = count // N, r = count % N; chunk c has
               q + (1 if c < r else 0) elements and starts at c*q + min(c, r).
  tree shape   the multi-node training page §4.3.2 says only "two trees, one for the
               first half of the data, one for the second"; lecture 09 §5.2 says leaves
               reduce to the root, then the root broadcasts. Tree A is an in-order binary
               tree over positions 0..N-1 with 1-based label q = position + 1 and height
               h = ctz(q): left child q - 2^(h-1), right child q + 2^(j-1) for the
               largest j <= h with q + 2^(j-1) <= N; the root is the largest power of two
               <= N. Tree B is the mirror (rank r sits at position N-1-r). Tree A reduces
               elements [0, ceil(count/2)), tree B the rest.
  binomial     the from-scratch page's table gives broadcast as a log2(N) tree. Relative
               rank v = (r - root) mod N receives from v - 2^floor(log2 v) and sends to
               v + 2^k for every 2^k > v with v + 2^k < N, k ascending.
"""
from __future__ import annotations

from typing import Optional


def chunk_bounds(count: int, n: int) -> list[tuple[int, int]]:
    """[start, stop) of each of the n ring chunks of a count-element buffer."""
    q, r = divmod(count, n)
    out = []
    for c in range(n):
        start = c * q + min(c, r)
        out.append((start, start + q + (1 if c < r else 0)))
    return out


def tree_half_split(count: int) -> int:
    """First element of tree B's half: ceil(count / 2)."""
    return (count + 1) // 2


def _ctz(q: int) -> int:
    return (q & -q).bit_length() - 1


class BinaryTree:
    """One of the two trees of the double binary tree, in rank terms."""

    def __init__(self, n: int, mirrored: bool):
        self.n = n
        self.mirrored = mirrored
        self.left: list[Optional[int]] = [None] * n
        self.right: list[Optional[int]] = [None] * n
        self.parent: list[Optional[int]] = [None] * n
        for pos in range(n):
            q = pos + 1
            h = _ctz(q)
            if h == 0:
                continue
            lq = q - (1 << (h - 1))
            self._link(q, lq, "left")
            for j in range(h, 0, -1):
                rq = q + (1 << (j - 1))
                if rq <= n:
                    self._link(q, rq, "right")
                    break
        root_q = 1 << (n.bit_length() - 1)
        self.root = self.rank_of(root_q - 1)

    def rank_of(self, pos: int) -> int:
        return self.n - 1 - pos if self.mirrored else pos

    def _link(self, q: int, child_q: int, side: str) -> None:
        p, c = self.rank_of(q - 1), self.rank_of(child_q - 1)
        getattr(self, side)[p] = c
        self.parent[c] = p

    def children(self, rank: int) -> list[int]:
        return [c for c in (self.left[rank], self.right[rank]) if c is not None]

    def depth(self, rank: int) -> int:
        d = 0
        while self.parent[rank] is not None:
            rank = self.parent[rank]
            d += 1
        return d


def binomial_parent(v: int) -> Optional[int]:
    """Parent of relative rank v in the binomial broadcast tree (None for the root)."""
    if v == 0:
        return None
    return v - (1 << (v.bit_length() - 1))


def binomial_children(v: int, n: int) -> list[int]:
    """Children of relative rank v, in the order v sends to them."""
    out = []
    k = 0 if v == 0 else v.bit_length()
    while v + (1 << k) < n:
        out.append(v + (1 << k))
        k += 1
    return out
