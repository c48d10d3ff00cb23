"""Shared test helpers: host <-> device transfer of per-rank arrays, bit views, guard bands."""
import numpy as np

GUARD = 1024  # elements of canary before and after every guarded output


def bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    return a.view({4: np.uint32, 2: np.uint16}[a.itemsize])


def torch_dtype(np_dtype):
    import torch
    return {np.dtype(np.float32): torch.float32, np.dtype(np.int32): torch.int32,
            np.dtype(np.uint16): torch.bfloat16}[np.dtype(np_dtype)]


def to_dev(a: np.ndarray):
    """numpy array -> CUDA tensor with the same bits (uint16 arrays become bfloat16)."""
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def to_host(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


class Guarded:
    """An output tensor with canary-filled guard bands on both sides; .check() asserts that
    no kernel wrote outside the tensor."""

    def __init__(self, numel: int, dtype, shape=None, misalign: int = 0):
        import torch
        self.full = torch.empty(numel + 2 * GUARD + misalign, dtype=dtype, device="cuda")
        if dtype == torch.bfloat16:
            self.full.view(torch.int16).fill_(0x5A5A)
        elif dtype == torch.int32:
            self.full.fill_(0x5A5A5A5A)
        else:
            self.full.view(torch.int32).fill_(0x7FC5A5A5)
        self.off = GUARD + misalign
        self.t = self.full[self.off:self.off + numel]
        if shape is not None:
            self.t = self.t.view(shape)
        self.numel = numel
        self._canary = self.full[:1].clone()

    def check(self):
        import torch
        head = self.full[:self.off]
        tail = self.full[self.off + self.numel:]
        c = self._canary
        if self.full.dtype in (torch.float32,):
            head, tail, c = head.view(torch.int32), tail.view(torch.int32), c.view(torch.int32)
        elif self.full.dtype == torch.bfloat16:
            head, tail, c = head.view(torch.int16), tail.view(torch.int16), c.view(torch.int16)
        assert bool((head == c).all()) and bool((tail == c).all()), "write outside the output tensor"


def misaligned(a: np.ndarray):
    """A CUDA tensor holding `a` whose address is one element past a 16-byte boundary."""
    import torch
    full = to_dev(np.concatenate([np.zeros(1, a.dtype), a]))
    t = full[1:]
    assert t.data_ptr() % 16 != 0
    return t
