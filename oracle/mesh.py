"""Message-passing mesh for the oracle: N ranks, tagged FIFO point-to-point channels,
per-rank byte counters.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
leg may import this package. The product path never does.

Model (collective pages: lecture 09 "网络通信基础与集合通信" §2.1 Send/Recv; the
"从零实现集合通信" page, "用队列 mesh 替代 NCCL", one ordered single-producer /
single-consumer queue per edge, send(dst, t) / recv(src)):
  * every rank runs the same program (a Python generator) on its own buffers;
  * send() copies the payload (a snapshot taken at send time, so all sends of a step
    see the values from before that step's adds, as in lecture 09 §7.1 experiment 1)
    and charges its bytes to the sender's `sent` and the receiver's `recvd` counters;
  * recv() returns the oldest undelivered message on (src, dst, tag).

Two drivers run the programs:
  * LockstepMesh: one thread, round-robin over the rank programs; a program that must
    wait for a message yields. A full round without progress is a deadlock and raises
    ProtocolError. This is the default (deterministic, no timing).
  * ThreadedMesh: one thread per rank, channels are queue.Queue with a receive timeout
    (the page's `recv_timeout_ms` exercise): a rank that waits longer raises
    MeshTimeout instead of hanging. Messages carry per-channel sequence numbers, so a
    dropped, duplicated or reordered message is reported as ProtocolError or
    MeshTimeout. A `fault` hook can drop, delay or duplicate a chosen message.
"""
from __future__ import annotations

import queue
import threading
import time
from collections import defaultdict, deque
from typing import Callable, Generator, Optional

import numpy as np


class ProtocolError(RuntimeError):
    """A message arrived out of sequence, twice, or was never consumed; or a deadlock."""


class MeshTimeout(RuntimeError):
    """A rank waited longer than the receive timeout for a message."""


class _Ctx:
    """What a rank program sees: its rank, the world size, send and recv."""

    def __init__(self, mesh: "_MeshBase", rank: int):
        self.mesh = mesh
        self.rank = rank
        self.n = mesh.n

    def send(self, dst: int, payload: np.ndarray, tag=0) -> None:
        self.mesh._send(self.rank, dst, tag, np.array(payload, copy=True))

    def recv(self, src: int, tag=0) -> Generator[None, None, np.ndarray]:
        return (yield from self.mesh._recv(src, self.rank, tag))


class _MeshBase:
    def __init__(self, n: int, ranks_per_node: Optional[int] = None):
        if n < 1:
            raise ValueError("a mesh needs at least one rank")
        self.n = n
        self.sent = [0] * n
        self.recvd = [0] * n
        # bytes a rank sends to ranks of other nodes (ranks r and s share a node when
        # r // ranks_per_node == s // ranks_per_node; default: every rank is its own node)
        self.ranks_per_node = ranks_per_node or 1
        self.sent_off_node = [0] * n
        # bytes per directed link (src, dst)
        self.link_bytes: dict = defaultdict(int)
        self.messages = 0
        self.delivered = 0
        self._seq_out: dict = defaultdict(int)
        self._seq_in: dict = defaultdict(int)

    def _count(self, src: int, dst: int, payload: np.ndarray) -> None:
        if src != dst:
            self.sent[src] += int(payload.nbytes)
            self.recvd[dst] += int(payload.nbytes)
            self.link_bytes[(src, dst)] += int(payload.nbytes)
            if src // self.ranks_per_node != dst // self.ranks_per_node:
                self.sent_off_node[src] += int(payload.nbytes)
        self.messages += 1

    def _check_seq(self, key, seq: int) -> None:
        want = self._seq_in[key]
        if seq != want:
            raise ProtocolError(f"channel {key}: got message #{seq}, expected #{want}")
        self._seq_in[key] = want + 1


class LockstepMesh(_MeshBase):
    """Single-threaded round-robin driver (deterministic)."""

    def __init__(self, n: int, ranks_per_node: Optional[int] = None):
        super().__init__(n, ranks_per_node)
        self._chan: dict = defaultdict(deque)

    def _send(self, src, dst, tag, payload):
        key = (src, dst, tag)
        self._count(src, dst, payload)
        self._chan[key].append((self._seq_out[key], payload))
        self._seq_out[key] += 1

    def _recv(self, src, dst, tag):
        key = (src, dst, tag)
        while not self._chan[key]:
            yield
        seq, payload = self._chan[key].popleft()
        self._check_seq(key, seq)
        self.delivered += 1
        return payload

    def run(self, program: Callable[[_Ctx], Generator], ranks: Optional[list[int]] = None) -> None:
        live = {r: program(_Ctx(self, r)) for r in (ranks if ranks is not None else range(self.n))}
        while live:
            before = (self.messages, self.delivered, len(live))
            for r in list(live):
                try:
                    next(live[r])
                except StopIteration:
                    del live[r]
            if live and (self.messages, self.delivered, len(live)) == before:
                raise ProtocolError(f"deadlock: ranks {sorted(live)} wait for messages never sent")
        left = {k: len(v) for k, v in self._chan.items() if v}
        if left:
            raise ProtocolError(f"undelivered messages left on channels {left}")


class ThreadedMesh(_MeshBase):
    """One thread per rank; receive with a timeout; optional fault injection.

    fault(src, dst, tag, seq) may return None, "drop", "dup" or ("delay", seconds).
    """

    def __init__(self, n: int, recv_timeout_s: float = 2.0, fault=None):
        super().__init__(n)
        self.timeout = recv_timeout_s
        self.fault = fault
        self._chan: dict = defaultdict(queue.Queue)
        self._lock = threading.Lock()

    def _send(self, src, dst, tag, payload):
        key = (src, dst, tag)
        with self._lock:
            seq = self._seq_out[key]
            self._seq_out[key] += 1
            self._count(src, dst, payload)
            q = self._chan[key]
        action = self.fault(src, dst, tag, seq) if self.fault else None
        if action == "drop":
            return
        if isinstance(action, tuple) and action[0] == "delay":
            time.sleep(action[1])
        q.put((seq, payload))
        if action == "dup":
            q.put((seq, payload))

    def _recv(self, src, dst, tag):
        key = (src, dst, tag)
        with self._lock:
            q = self._chan[key]
        try:
            seq, payload = q.get(timeout=self.timeout)
        except queue.Empty:
            raise MeshTimeout(f"rank {dst} waited {self.timeout}s for a message from rank {src} (tag {tag})")
        with self._lock:
            self._check_seq(key, seq)
        return payload
        yield  # makes this a generator; never reached

    def run(self, program: Callable[[_Ctx], Generator], ranks: Optional[list[int]] = None) -> None:
        errors: dict[int, BaseException] = {}

        def body(r):
            try:
                for _ in program(_Ctx(self, r)):
                    pass
            except BaseException as e:  # reported to the caller below
                errors[r] = e

        threads = [threading.Thread(target=body, args=(r,), daemon=True)
                   for r in (ranks if ranks is not None else range(self.n))]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        if errors:
            r = min(errors)
            raise errors[r]
        left = {k: q.qsize() for k, q in self._chan.items() if q.qsize()}
        if left:
            raise ProtocolError(f"undelivered messages left on channels {left}")
