"""q4_quantized_decode_b200 -- B200-native Q4_0 GEMV for memory-bound decode.

A thin ctypes binding over the C-ABI library ``libq4gemv.so`` (declared in
``include/q4gemv.h``).  The functions below carry the ABI's names and only
marshal arguments: every step of the computation runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams (``Q4Gemv`` accepts
tensors); nothing here computes on the CPU, and there is no fallback: if the
library is missing or fails to load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4gemv.so")

Q4_OK = 0
Q4_EINVAL = -1
Q4_ESHAPE = -2
Q4_EALIGN = -3
Q4_ENOMEM = -4
Q4_ECUDA = -5
Q4_EUNSUPPORTED = -6
Q4_ETIMEOUT = -7
Q4_EFAULTINJ = -8
Q4_ECONCURRENT = -9
MAX_M = 256        # vectors per q4gemv_run call
MAX_M_GEMV = 16    # above this, the tensor-core GEMM path


class Q4Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"q4gemv status {status}: {msg}")
        self.status = status


class q4gemv_layer(ctypes.Structure):
    _fields_ = [("qkv", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p)]


def _load_library():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
            "or `python q4_quantized_decode_b200/build_ext.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sigs = {
        "q4gemv_version": ([], ci),
        "q4gemv_create": ([ctypes.POINTER(vp), ci], ci),
        "q4gemv_destroy": ([vp], ci),
        "q4gemv_gguf_bytes": ([i64, i64], ctypes.c_size_t),
        "q4gemv_packed_bytes": ([i64, i64], ctypes.c_size_t),
        "q4gemv_validate": ([ci, i64, i64, vp, vp, vp], ci),
        "q4gemv_repack": ([vp, vp, vp, i64, i64, vp], ci),
        "q4gemv_run": ([vp, vp, vp, vp, ci, i64, i64, vp], ci),
        "q4gemv_run_swiglu": ([vp, vp, vp, vp, i64, i64, vp], ci),
        "q4gemv_shard_rows": ([i64, ci, ci, ctypes.POINTER(i64), ctypes.POINTER(i64),
                               ctypes.POINTER(i64)], ci),
        "q4gemv_comm_unique_id": ([ctypes.c_char_p], ci),
        "q4gemv_comm_init": ([vp, ci, ci, ctypes.c_char_p], ci),
        "q4gemv_run_stack_sharded": ([vp, ctypes.POINTER(q4gemv_layer), ci, i64, i64, i64, vp, vp,
                                      vp], ci),
        "q4gemv_peer_layout": ([ci, i64, i64, i64, ctypes.POINTER(i64)], ci),
        "q4gemv_peer_check": ([ctypes.c_char_p, ci], ci),
        "q4gemv_peer_export": ([vp, ci, ci, i64, i64, i64, ctypes.c_char_p], ci),
        "q4gemv_peer_open": ([vp, ctypes.c_char_p], ci),
        "q4gemv_peer_close": ([vp], ci),
        "q4gemv_run_stack": ([vp, ctypes.POINTER(q4gemv_layer), ci, i64, i64, i64,
                              vp, vp, vp, vp, vp], ci),
        "q4gemv_run_stack_gated": ([vp, ctypes.POINTER(q4gemv_layer), ci, i64, i64, i64,
                                    vp, vp, vp], ci),
        "q4gemv_sync_status": ([vp, vp], ci),
        "q4gemv_strerror": ([ci], ctypes.c_char_p),
        "q4gemv_last_error": ([vp], ctypes.c_char_p),
        "q4gemv_set_fault": ([vp, ctypes.c_char_p], ci),
        "q4gemv_run_noalloc": ([vp, vp, vp, ci, i64, i64, vp], ci),
        "q4gemv_q8_0_gguf_bytes": ([i64, i64], ctypes.c_size_t),
        "q4gemv_q8_0_packed_bytes": ([i64, i64], ctypes.c_size_t),
        "q4gemv_q8_0_repack": ([vp, vp, vp, i64, i64, vp], ci),
        "q4gemv_q8_0_validate": ([ci, i64, i64, vp, vp, vp], ci),
        "q4gemv_q8_0_run": ([vp, vp, vp, vp, ci, i64, i64, vp], ci),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load_library()
lib = _lib


def q4gemv_version() -> int:
    return _lib.q4gemv_version()


def q4gemv_strerror(status: int) -> str:
    return _lib.q4gemv_strerror(status).decode()


def q4gemv_last_error(h) -> str:
    return _lib.q4gemv_last_error(h).decode()


def q4gemv_gguf_bytes(N: int, K: int) -> int:
    return _lib.q4gemv_gguf_bytes(N, K)


def q4gemv_packed_bytes(N: int, K: int) -> int:
    return _lib.q4gemv_packed_bytes(N, K)


def q4gemv_validate(M, N, K, W, x, y) -> int:
    return _lib.q4gemv_validate(M, N, K, W, x, y)


def q4gemv_create(device: int = 0):
    h = ctypes.c_void_p()
    st = _lib.q4gemv_create(ctypes.byref(h), device)
    return st, h


def q4gemv_destroy(h) -> int:
    return _lib.q4gemv_destroy(h)


def q4gemv_repack(h, gguf, packed, N, K, stream) -> int:
    return _lib.q4gemv_repack(h, gguf, packed, N, K, stream)


def q4gemv_run(h, W, x, y, M, N, K, stream) -> int:
    return _lib.q4gemv_run(h, W, x, y, M, N, K, stream)


def q4gemv_run_swiglu(h, W, gate_up, y, N, K, stream) -> int:
    return _lib.q4gemv_run_swiglu(h, W, gate_up, y, N, K, stream)


def q4gemv_run_stack(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out,
                     trace_x, trace_y, stream) -> int:
    return _lib.q4gemv_run_stack(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out,
                                 trace_x, trace_y, stream)


def q4gemv_run_stack_gated(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, stream) -> int:
    return _lib.q4gemv_run_stack_gated(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, stream)


def q4gemv_sync_status(h, stream) -> int:
    return _lib.q4gemv_sync_status(h, stream)


def q4gemv_set_fault(h, which: str) -> int:
    return _lib.q4gemv_set_fault(h, which.encode())


def q4gemv_shard_rows(N: int, world: int, rank: int):
    """(status, row0, rows, chunk) of rank's row slice of an N-row matrix."""
    r0, n, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    st = _lib.q4gemv_shard_rows(N, world, rank, ctypes.byref(r0), ctypes.byref(n), ctypes.byref(c))
    return st, r0.value, n.value, c.value


def q4gemv_comm_unique_id():
    """(status, 128-byte NCCL unique id)."""
    buf = ctypes.create_string_buffer(128)
    st = _lib.q4gemv_comm_unique_id(buf)
    return st, buf.raw


def q4gemv_comm_init(h, world: int, rank: int, uid: bytes) -> int:
    return _lib.q4gemv_comm_init(h, world, rank, ctypes.create_string_buffer(uid, 128))


PEER_BLOB_BYTES = 128
PEER_MAX_WORLD = 8


def q4gemv_peer_layout(world: int, hidden: int, qkv_n: int, ffn: int):
    """(status, [6 byte offsets]) of the peer exchange buffer (see the header)."""
    off = (ctypes.c_int64 * 6)()
    st = _lib.q4gemv_peer_layout(world, hidden, qkv_n, ffn, off)
    return st, list(off)


def q4gemv_peer_check(blobs: bytes, world: int) -> int:
    return _lib.q4gemv_peer_check(ctypes.create_string_buffer(blobs, len(blobs)), world)


def q4gemv_peer_export(h, world: int, rank: int, hidden: int, qkv_n: int, ffn: int):
    """(status, this rank's 128-byte exchange blob)."""
    buf = ctypes.create_string_buffer(PEER_BLOB_BYTES)
    st = _lib.q4gemv_peer_export(h, world, rank, hidden, qkv_n, ffn, buf)
    return st, buf.raw


def q4gemv_peer_open(h, blobs: bytes) -> int:
    return _lib.q4gemv_peer_open(h, ctypes.create_string_buffer(blobs, len(blobs)))


def q4gemv_peer_close(h) -> int:
    return _lib.q4gemv_peer_close(h)


def q4gemv_run_stack_sharded(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, stream) -> int:
    return _lib.q4gemv_run_stack_sharded(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, stream)


def q4gemv_run_noalloc(W, x, y, M, N, K, stream) -> int:
    """The M <= 2 GEMV without a handle or any allocation (see the header)."""
    return _lib.q4gemv_run_noalloc(W, x, y, M, N, K, stream)


def q4gemv_q8_0_gguf_bytes(N: int, K: int) -> int:
    return _lib.q4gemv_q8_0_gguf_bytes(N, K)


def q4gemv_q8_0_packed_bytes(N: int, K: int) -> int:
    return _lib.q4gemv_q8_0_packed_bytes(N, K)


def q4gemv_q8_0_repack(h, gguf, packed, N, K, stream) -> int:
    return _lib.q4gemv_q8_0_repack(h, gguf, packed, N, K, stream)


def q4gemv_q8_0_validate(M, N, K, W, x, y) -> int:
    return _lib.q4gemv_q8_0_validate(M, N, K, W, x, y)


def q4gemv_q8_0_run(h, W, x, y, M, N, K, stream) -> int:
    return _lib.q4gemv_q8_0_run(h, W, x, y, M, N, K, stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Q4Gemv:
    """Owns one library handle on one device; methods take torch tensors."""

    def __init__(self, device: int = 0):
        st, h = q4gemv_create(device)
        if st != Q4_OK:
            raise Q4Error(st, q4gemv_strerror(st))
        self.h = h
        self.device = device

    def close(self):
        if self.h:
            q4gemv_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st: int):
        if st != Q4_OK:
            raise Q4Error(st, q4gemv_last_error(self.h) or q4gemv_strerror(st))

    def packed_bytes(self, N: int, K: int) -> int:
        return q4gemv_packed_bytes(N, K)

    def repack(self, gguf, N: int, K: int, out=None, stream=None):
        """gguf: uint8 CUDA tensor of N*(K/32)*18 bytes -> packed uint8 tensor."""
        import torch
        if out is None:
            out = torch.empty(q4gemv_packed_bytes(N, K), dtype=torch.uint8, device=gguf.device)
        self._check(q4gemv_repack(self.h, _ptr(gguf), _ptr(out), N, K, _stream(stream)))
        return out

    def run(self, W_packed, x, N: int, K: int, out=None, stream=None):
        """x: f16 CUDA tensor [M][K] (or [K]) -> y f16 [M][N]."""
        import torch
        x2 = x.reshape(-1, K)
        M = x2.shape[0]
        if out is None:
            out = torch.empty((M, N), dtype=torch.float16, device=x.device)
        self._check(q4gemv_run(self.h, _ptr(W_packed), _ptr(x2), _ptr(out), M, N, K,
                               _stream(stream)))
        return out

    def run_swiglu(self, W_packed, gate_up, N: int, K: int, out=None, stream=None):
        """gate_up: f16 CUDA tensor [2K] ([gate | up]) -> y f16 [N] = W (SiLU(gate) * up)."""
        import torch
        if out is None:
            out = torch.empty(N, dtype=torch.float16, device=gate_up.device)
        self._check(q4gemv_run_swiglu(self.h, _ptr(W_packed), _ptr(gate_up), _ptr(out), N, K,
                                      _stream(stream)))
        return out

    def repack_q8_0(self, gguf, N: int, K: int, out=None, stream=None):
        """gguf: uint8 CUDA tensor of N*(K/32)*34 bytes -> packed Q8_0 tensor."""
        import torch
        if out is None:
            out = torch.empty(q4gemv_q8_0_packed_bytes(N, K), dtype=torch.uint8, device=gguf.device)
        self._check(q4gemv_q8_0_repack(self.h, _ptr(gguf), _ptr(out), N, K, _stream(stream)))
        return out

    def run_q8_0(self, W_packed, x, N: int, K: int, out=None, stream=None):
        """x: f16 CUDA tensor [M][K] (M <= 256) -> y f16 [M][N] for a packed Q8_0 W."""
        import torch
        x2 = x.reshape(-1, K)
        M = x2.shape[0]
        if out is None:
            out = torch.empty((M, N), dtype=torch.float16, device=x.device)
        self._check(q4gemv_q8_0_run(self.h, _ptr(W_packed), _ptr(x2), _ptr(out), M, N, K,
                                    _stream(stream)))
        return out

    def run_stack(self, layers, x_in, hidden: int, qkv_n: int, ffn: int, x_out=None,
                  trace_x=None, trace_y=None, stream=None):
        """layers: list of (qkv, o, gate_up, down) packed tensors."""
        import torch
        if x_out is None:
            x_out = torch.empty(hidden, dtype=torch.float16, device=x_in.device)
        arr = (q4gemv_layer * len(layers))()
        for i, (a, b, c, d) in enumerate(layers):
            arr[i] = q4gemv_layer(_ptr(a), _ptr(b), _ptr(c), _ptr(d))
        self._check(q4gemv_run_stack(self.h, arr, len(layers), hidden, qkv_n, ffn, _ptr(x_in),
                                     _ptr(x_out), _ptr(trace_x), _ptr(trace_y), _stream(stream)))
        return x_out

    def run_stack_gated(self, layers, x_in, hidden: int, qkv_n: int, ffn: int, x_out=None, stream=None):
        """The step with each down GEMV fed SiLU(gate) * up (see the header)."""
        import torch
        if x_out is None:
            x_out = torch.empty(hidden, dtype=torch.float16, device=x_in.device)
        arr = (q4gemv_layer * len(layers))()
        for i, (a, b, c, d) in enumerate(layers):
            arr[i] = q4gemv_layer(_ptr(a), _ptr(b), _ptr(c), _ptr(d))
        self._check(q4gemv_run_stack_gated(self.h, arr, len(layers), hidden, qkv_n, ffn, _ptr(x_in),
                                           _ptr(x_out), _stream(stream)))
        return x_out

    def init_comm(self, world: int, rank: int, uid: bytes):
        """Joins the `world`-GPU communicator of the row-sharded step as `rank`."""
        self._check(q4gemv_comm_init(self.h, world, rank, uid))

    def peer_export(self, world: int, rank: int, hidden: int, qkv_n: int, ffn: int) -> bytes:
        """Allocates this rank's exchange buffer for the peer-memory sharded step
        and returns the blob every rank must receive (e.g. all_gather_object)."""
        st, blob = q4gemv_peer_export(self.h, world, rank, hidden, qkv_n, ffn)
        self._check(st)
        return blob

    def peer_open(self, blobs):
        """Maps every rank's exchange buffer; `blobs`: the world's blobs in rank order.
        run_stack_sharded then gathers over peer memory for these shapes."""
        self._check(q4gemv_peer_open(self.h, b"".join(blobs)))

    def peer_close(self):
        self._check(q4gemv_peer_close(self.h))

    def run_stack_sharded(self, layers_local, x_in, hidden: int, qkv_n: int, ffn: int, x_out=None,
                          stream=None):
        """layers_local: this rank's (qkv, o, gate_up, down) row slices (packed tensors, or
        None for a slice of 0 rows)."""
        import torch
        if x_out is None:
            x_out = torch.empty(hidden, dtype=torch.float16, device=x_in.device)
        arr = (q4gemv_layer * len(layers_local))()
        for i, (a, b, c, d) in enumerate(layers_local):
            arr[i] = q4gemv_layer(_ptr(a), _ptr(b), _ptr(c), _ptr(d))
        self._check(q4gemv_run_stack_sharded(self.h, arr, len(layers_local), hidden, qkv_n, ffn,
                                             _ptr(x_in), _ptr(x_out), _stream(stream)))
        return x_out

    def sync_status(self, stream=None) -> int:
        return q4gemv_sync_status(self.h, _stream(stream))

    def set_fault(self, which: str):
        self._check(q4gemv_set_fault(self.h, which))


def stack_trace_dims(hidden: int, qkv_n: int, ffn: int):
    """Row strides of the trace_x / trace_y buffers of q4gemv_run_stack."""
    return max(hidden, ffn), max(qkv_n, hidden, 2 * ffn)
