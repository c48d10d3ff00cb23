"""Seeded synthetic inputs shared by the oracle tests, the GPU tests, smoke() and bench.py.

Every value is a pure function of (seed, rank, stream, index): a counter-based
SplitMix64 stream (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the output mix is the published SplitMix64 finaliser).
Nothing in this module knows about collectives: it only produces host arrays.
Both sides of a parity test read the same host array, so bit-identity of the
inputs never depends on the floating-point behaviour of the transforms below.

Distributions (the workloads of the collective pages):
  uniform_f32    U[lo, hi) from the top 24 bits, exact in fp32 for [-1, 1)
  normal_f32     Box-Muller in fp64 from one 64-bit draw, rounded to fp32
  int32_uniform  uniform integers in [lo, hi] (inclusive)
  to_bf16_bits   round-to-nearest-even fp32 -> bf16, returned as uint16 bits
The same definitions are compiled from synth/synth.c (OpenMP) for speed; build_native()
makes synth/_synth.so with gcc. Without it the numpy code below runs (slower, same
definitions; normal values may then differ from the C ones in the last bit of the fp64
transform, which never matters: each test feeds one host array to both sides).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_synth.so")
_lib = None


def build_native(force: bool = False) -> str:
    """Compile synth/synth.c into synth/_synth.so (gcc, OpenMP, no fast-math)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _native():
    global _lib
    if _lib is None:
        try:
            lib = ctypes.CDLL(build_native())
        except (OSError, subprocess.CalledProcessError, FileNotFoundError):
            _lib = False
            return None
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_stream_key.restype = u64
        lib.synth_stream_key.argtypes = [u64, i64, i64]
        lib.synth_uniform_f32.argtypes = [u64, u64, i64, dbl, dbl, vp]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_int32.argtypes = [u64, u64, i64, i64, i64, vp]
        lib.synth_to_bf16.argtypes = [vp, i64, vp]
        _lib = lib
    return _lib or None

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_SLICE = 1 << 22
_THREADS = max(1, min(32, os.cpu_count() or 1))


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, rank: int, stream: int = 0) -> np.uint64:
    """Start state of the (seed, rank, stream) sequence."""
    with np.errstate(over="ignore"):
        s = _mix(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))
        s = _mix(s + np.uint64(rank + 1) * GOLDEN + np.uint64(stream & 0xFFFFFFFF))
    return s[0]


def raw_u64(seed: int, rank: int, index: np.ndarray, stream: int = 0) -> np.ndarray:
    """The index-th output of the (seed, rank, stream) SplitMix64 sequence."""
    k = stream_key(seed, rank, stream)
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(k + (idx + np.uint64(1)) * GOLDEN)


def _fill(out: np.ndarray, fn) -> np.ndarray:
    n = out.size
    if n <= _SLICE:
        fn(0, n, out)
        return out
    starts = range(0, n, _SLICE)
    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(lambda a: fn(a, min(n, a + _SLICE), out[a:min(n, a + _SLICE)]), starts))
    return out


def uniform_f32(seed: int, rank: int, count: int, lo: float = -1.0, hi: float = 1.0,
                stream: int = 0, native: bool = True, start: int = 0) -> np.ndarray:
    """fp32 values lo + (hi - lo) * u, u = top-24-bit fraction; [-1, 1) is exact.
    Values start..start+count-1 of the sequence."""
    out = np.empty(count, dtype=np.float32)
    lib = _native() if native else None
    if lib:
        lib.synth_uniform_f32(int(stream_key(seed, rank, stream)), start, count, lo, hi, out.ctypes.data)
        return out

    def fn(a, b, dst):
        u = (raw_u64(seed, rank, np.arange(start + a, start + b, dtype=np.uint64), stream) >> np.uint64(40))
        f = u.astype(np.float32) * np.float32(2.0 ** -24)
        if lo == -1.0 and hi == 1.0:
            dst[:] = f * np.float32(2.0) - np.float32(1.0)
        else:
            dst[:] = (lo + (hi - lo) * f.astype(np.float64)).astype(np.float32)
    return _fill(out, fn)


def normal_f32(seed: int, rank: int, count: int, std: float = 1.0, stream: int = 0,
               native: bool = True, start: int = 0) -> np.ndarray:
    """fp32 normal(0, std): Box-Muller on the two 32-bit halves of one draw, in fp64.
    Values start..start+count-1 of the sequence."""
    out = np.empty(count, dtype=np.float32)
    lib = _native() if native else None
    if lib:
        lib.synth_normal_f32(int(stream_key(seed, rank, stream)), start, count, std, out.ctypes.data)
        return out

    def fn(a, b, dst):
        z = raw_u64(seed, rank, np.arange(start + a, start + b, dtype=np.uint64), stream)
        u1 = ((z >> np.uint64(32)).astype(np.float64) + 1.0) * (2.0 ** -32)
        u2 = (z & np.uint64(0xFFFFFFFF)).astype(np.float64) * (2.0 ** -32)
        g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        dst[:] = (g * std).astype(np.float32)
    return _fill(out, fn)


def int32_uniform(seed: int, rank: int, count: int, lo: int, hi: int, stream: int = 0,
                  native: bool = True, start: int = 0) -> np.ndarray:
    """int32 values uniform on [lo, hi] (modulo reduction of a 64-bit draw).
    Values start..start+count-1 of the sequence."""
    span = np.uint64(hi - lo + 1)
    out = np.empty(count, dtype=np.int32)
    lib = _native() if native else None
    if lib:
        lib.synth_int32(int(stream_key(seed, rank, stream)), start, count, lo, hi, out.ctypes.data)
        return out

    def fn(a, b, dst):
        z = raw_u64(seed, rank, np.arange(start + a, start + b, dtype=np.uint64), stream)
        dst[:] = ((z % span).astype(np.int64) + lo).astype(np.int32)
    return _fill(out, fn)


def to_bf16_bits(x: np.ndarray, native: bool = True) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    lib = _native() if native else None
    if lib:
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(x.shape, dtype=np.uint16)
        lib.synth_to_bf16(x.ctypes.data, x.size, out.ctypes.data)
        return out
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (for building expected inputs)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---- workload shapes -------------------------------------------------------------------------

def transformer_grad_shapes(layers: int = 12, d: int = 768, ffn: int = 3072,
                            vocab: int = 32000) -> list[tuple[str, tuple[int, ...]]]:
    """Parameter list of the 12-layer d=768 transformer, in registration order.

    Token embedding (tied with the LM head), then per layer ln1.{w,b}, qkv.{w,b},
    proj.{w,b}, ln2.{w,b}, fc1.{w,b}, fc2.{w,b}, then the final lnf.{w,b}.
    """
    shapes: list[tuple[str, tuple[int, ...]]] = [("emb", (vocab, d))]
    for i in range(layers):
        p = f"h{i}."
        shapes += [
            (p + "ln1.w", (d,)), (p + "ln1.b", (d,)),
            (p + "qkv.w", (d, 3 * d)), (p + "qkv.b", (3 * d,)),
            (p + "proj.w", (d, d)), (p + "proj.b", (d,)),
            (p + "ln2.w", (d,)), (p + "ln2.b", (d,)),
            (p + "fc1.w", (d, ffn)), (p + "fc1.b", (ffn,)),
            (p + "fc2.w", (ffn, d)), (p + "fc2.b", (d,)),
        ]
    shapes += [("lnf.w", (d,)), ("lnf.b", (d,))]
    return shapes


def numel(shape: tuple[int, ...]) -> int:
    n = 1
    for s in shape:
        n *= s
    return n
