"""Host side of the one-rank-per-process slice calls, without a GPU: argument validation of
the C entry points, and PeerGroup's handle exchange over a 2-rank gloo group with the IPC
calls replaced by a fake (the CUDA part runs in the GPU tests)."""
import ctypes
import os
import socket

import pytest

import collective_communication_primitives_rank_b200 as cc

FAKE = [0x10000 * (i + 1) for i in range(8)]


def _pp(vals):
    return (ctypes.c_void_p * len(vals))(*vals)


def test_slice_entry_points_validate():
    lib = cc.get_lib()
    p4 = _pp(FAKE[:4])
    f32, sm, ring = cc.CC_F32, cc.CC_SUM, cc.CC_ALGO_RING
    # rank outside [0, nranks)
    assert lib.cc_allreduce_slice(p4, p4, 4, 4, 10, f32, f32, sm, ring, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_allreduce_slice(p4, p4, 4, -1, 10, f32, f32, sm, ring, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_reduce_scatter_slice(p4, FAKE[0], 4, 4, 10, f32, f32, sm, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_allgather_slice(FAKE[0], p4, 4, 9, 10, f32, None) == cc.CC_ERR_INVALID_ARG
    # dtype pair, algo
    assert lib.cc_allreduce_slice(p4, p4, 4, 0, 10, f32, cc.CC_I32, sm, ring, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_allreduce_slice(p4, p4, 4, 0, 10, f32, f32, sm, 7, 1.0, None) == cc.CC_ERR_INVALID_ARG
    # nothing to do: count 0, or this rank's chunk is empty (count 2 over 4 ranks, rank 3)
    assert lib.cc_allreduce_slice(p4, p4, 4, 1, 0, f32, f32, sm, ring, 1.0, None) == cc.CC_OK
    assert lib.cc_allreduce_slice(p4, p4, 4, 3, 2, f32, f32, sm, ring, 1.0, None) == cc.CC_OK
    assert lib.cc_reduce_scatter_slice(p4, None, 4, 3, 2, f32, f32, sm, 1.0, None) == cc.CC_OK
    assert lib.cc_allgather_slice(None, p4, 4, 3, 2, f32, None) == cc.CC_OK
    # a non-empty chunk needs its shard
    assert lib.cc_reduce_scatter_slice(p4, None, 4, 0, 10, f32, f32, sm, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_allgather_slice(None, p4, 4, 0, 10, f32, None) == cc.CC_ERR_INVALID_ARG


def test_ipc_entry_points_validate():
    lib = cc.get_lib()
    assert lib.cc_ipc_handle_bytes() == 64
    off = ctypes.c_size_t()
    h = ctypes.create_string_buffer(64)
    assert lib.cc_ipc_export(None, h, ctypes.byref(off)) == cc.CC_ERR_INVALID_ARG
    p = ctypes.c_void_p()
    assert lib.cc_ipc_open(None, 0, ctypes.byref(p)) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_ipc_close(FAKE[0]) == cc.CC_ERR_INVALID_ARG  # never opened


def test_slice_binding_checks_shapes():
    import torch
    x = [torch.zeros(8) for _ in range(2)]
    with pytest.raises(ValueError):
        cc.cc_allreduce_slice(x, x, 2)  # rank out of range
    with pytest.raises(ValueError):
        cc.cc_allreduce_slice([FAKE[0], x[1]], x, 0)  # this rank's entry is not a tensor


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _FakeIpc:
    """cc_ipc_* stand-ins: a handle names (rank, tensor index); opening it returns a fake
    address 0x10000000 * (rank + 1) + 0x100000 * index + offset."""

    def __init__(self, rank):
        self.rank = rank
        self.opened, self.closed = [], []

    def cc_ipc_handle_bytes(self):
        return 64

    def cc_ipc_export(self, ptr, h, off):
        idx = ptr & 0xFF  # the fake _dev_ptr encodes the tensor index in the low byte
        ctypes.memmove(h, f"r{self.rank}i{idx}".encode().ljust(64, b"."), 64)
        off._obj.value = 16 * idx
        return 0

    def cc_ipc_open(self, h, off, out):
        r, i = h.rstrip(b".").decode()[1:].split("i")
        addr = 0x10000000 * (int(r) + 1) + 0x100000 * int(i) + off
        out._obj.value = addr
        self.opened.append(addr)
        return 0

    def cc_ipc_close(self, p):
        self.closed.append(p)
        return 0

    def cc_status_string(self, st):
        return b"fake"


def _worker(rank, world, port, bad, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    fake = _FakeIpc(rank)
    cc.lib = fake
    ts = [torch.zeros(5 + (1 if (bad and rank == 1 and i == 1) else 0)) for i in range(3)]
    cc._dev_ptr = lambda t: 0x7000000 + [id(x) for x in ts].index(id(t))
    try:
        g = cc.PeerGroup(ts)
        out = []
        for i in range(3):
            b = g.buffers(i)
            out.append([("own", b[r] is ts[i]) if r == rank else ("peer", b[r]) for r in range(world)])
        g.close()
        q.put((rank, "ok", out, sorted(fake.opened), sorted(fake.closed)))
    except ValueError as e:
        q.put((rank, "error", str(e), sorted(fake.opened), sorted(fake.closed)))
    dist.barrier()
    dist.destroy_process_group()


def _run(bad):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, bad, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        item = q.get(timeout=150)
        res[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.timeout(180)
def test_peer_group_exchanges_handles_over_gloo():
    res = _run(bad=False)
    for rank in range(2):
        status, bufs, opened, closed = res[rank]
        assert status == "ok"
        peer = 1 - rank
        for i in range(3):
            assert bufs[i][rank] == ("own", True)
            # the peer's allocation for tensor i, at the offset it exported
            assert bufs[i][peer] == ("peer", 0x10000000 * (peer + 1) + 0x100000 * i + 16 * i)
        assert opened == closed and len(opened) == 3  # close() unmaps every open


@pytest.mark.timeout(180)
def test_peer_group_rejects_mismatched_tensors():
    res = _run(bad=True)
    for rank in range(2):
        status, msg, opened, closed = res[rank]
        assert status == "error" and "differs on rank" in msg
        assert opened == closed  # what was opened before the mismatch is closed again
