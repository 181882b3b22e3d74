"""Seeded synthetic inputs for the Q4_0 GEMV path (shared by the oracle tests,
the GPU tests and the benchmark).

Holds none of the dequantise-and-multiply arithmetic: it only draws
splitmix64 numbers and encodes them as GGUF Q4_0 blocks or f16 vectors.  The
definitions live in ``synth.c``; this wrapper builds it on first use (plain
gcc) and loads it with ctypes.

Workload recipe (value distributions of the 27B-shaped decode workload):
  * Q4_0 scale d ~ U[0.002, 0.05] with a random sign, rounded to f16;
    nibbles q ~ U{0..15};
  * activations x ~ N(0, 1) rounded to f16;
  * seeds: ``workload_seed(w) = 0x5EED0000 + w`` with w = 0 for the single
    1024 x 1024 GEMV, 1 for the 5120 x 5120 GEMV, 2 for the FFN GEMVs (gate+up
    34816 x 5120, down 5120 x 17408), 3 for the small-M batches on those
    shapes, 4 for the 64-layer decode step;
  * tensor ids: weight matrix j -> ``weight_id(j)``, activation row m ->
    ``act_id(m)`` (separate id spaces, so every tensor is its own stream).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, no fused FP ops)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64 = ctypes.c_uint64, ctypes.c_int64
            vp = ctypes.c_void_p
            lib.synth_splitmix64_at.argtypes = [u64, u64]
            lib.synth_splitmix64_at.restype = u64
            lib.synth_stream_key.argtypes = [u64, u64]
            lib.synth_stream_key.restype = u64
            lib.synth_f64_to_f16.argtypes = [ctypes.c_double]
            lib.synth_f64_to_f16.restype = ctypes.c_uint16
            lib.synth_f64_to_f16_array.argtypes = [vp, i64, vp]
            lib.synth_f64_to_f16_array.restype = None
            lib.synth_q4_0_rows.argtypes = [u64, u64, i64, i64, i64, vp]
            lib.synth_q4_0_rows.restype = None
            lib.synth_normal_f16.argtypes = [u64, u64, i64, i64, vp]
            lib.synth_q8_0_rows.argtypes = [u64, u64, i64, i64, i64, vp]
            lib.synth_q8_0_rows.restype = None
            lib.synth_normal_f16.restype = None
            _lib = lib
    return _lib


def workload_seed(w: int) -> int:
    return 0x5EED0000 + int(w)


def weight_id(j: int) -> int:
    return (1 << 32) | int(j)


def act_id(m: int) -> int:
    return (2 << 32) | int(m)


def splitmix64_at(state: int, i: int) -> int:
    return int(_load().synth_splitmix64_at(state & (2**64 - 1), i & (2**64 - 1)))


def f64_to_f16_bits(v) -> np.ndarray:
    """binary64 -> binary16 bit patterns (round to nearest even)."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.uint16)
    _load().synth_f64_to_f16_array(a.ctypes.data, a.size, out.ctypes.data)
    return out


def block_bytes(K: int) -> int:
    return (K // 32) * 18


def _threads(n_items: int, threads: int | None) -> int:
    t = threads or min(32, os.cpu_count() or 1)
    return max(1, min(t, n_items))


def q4_0_rows(seed: int, tensor_id: int, K: int, row0: int, nrows: int,
              out: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """GGUF Q4_0 bytes of rows [row0, row0+nrows) of a K-column matrix,
    shape (nrows, K/32*18) uint8."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    rb = block_bytes(K)
    if out is None:
        out = np.empty((nrows, rb), dtype=np.uint8)
    assert out.flags.c_contiguous and out.dtype == np.uint8 and out.size == nrows * rb
    lib = _load()
    t = _threads(nrows, threads)
    if t == 1 or nrows * rb < (1 << 20):
        lib.synth_q4_0_rows(seed, tensor_id, K, row0, nrows, out.ctypes.data)
        return out
    chunk = (nrows + t - 1) // t
    base = out.ctypes.data

    def work(i):
        r0 = i * chunk
        n = min(chunk, nrows - r0)
        if n > 0:
            lib.synth_q4_0_rows(seed, tensor_id, K, row0 + r0, n, base + r0 * rb)

    with ThreadPoolExecutor(t) as ex:
        list(ex.map(work, range(t)))
    return out


def q4_0_matrix(seed: int, tensor_id: int, N: int, K: int,
                out: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    return q4_0_rows(seed, tensor_id, K, 0, N, out=out, threads=threads)


def q4_0_row_list(seed: int, tensor_id: int, K: int, rows) -> np.ndarray:
    """GGUF bytes of an arbitrary list of rows (random access by row)."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, block_bytes(K)), dtype=np.uint8)
    lib = _load()
    for i, r in enumerate(rows):
        lib.synth_q4_0_rows(seed, tensor_id, K, int(r), 1, out[i].ctypes.data)
    return out


def q8_0_block_bytes(K: int) -> int:
    return (K // 32) * 34


def q8_0_rows(seed: int, tensor_id: int, K: int, row0: int, nrows: int,
              threads: int | None = None) -> np.ndarray:
    """GGUF Q8_0 bytes of rows [row0, row0+nrows) of a K-column matrix,
    shape (nrows, K/32*34) uint8."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    rb = q8_0_block_bytes(K)
    out = np.empty((nrows, rb), dtype=np.uint8)
    lib = _load()
    t = _threads(nrows, threads)
    if t == 1 or nrows * rb < (1 << 20):
        lib.synth_q8_0_rows(seed, tensor_id, K, row0, nrows, out.ctypes.data)
        return out
    chunk = (nrows + t - 1) // t
    base = out.ctypes.data

    def work(i):
        r0 = i * chunk
        n = min(chunk, nrows - r0)
        if n > 0:
            lib.synth_q8_0_rows(seed, tensor_id, K, row0 + r0, n, base + r0 * rb)

    with ThreadPoolExecutor(t) as ex:
        list(ex.map(work, range(t)))
    return out


def q8_0_matrix(seed: int, tensor_id: int, N: int, K: int, threads: int | None = None) -> np.ndarray:
    return q8_0_rows(seed, tensor_id, K, 0, N, threads=threads)


def normal_f16(seed: int, tensor_id: int, n: int, i0: int = 0) -> np.ndarray:
    """f16 bit patterns (uint16) of elements [i0, i0+n) of an N(0,1) vector."""
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_f16(seed, tensor_id, i0, n, out.ctypes.data)
    return out


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """x[M][K] as f16 bit patterns, row m drawn from stream act_id(m)."""
    return np.stack([normal_f16(seed, act_id(m), K) for m in range(M)])
