"""The row-sharded decode step's host logic on CPU.

q4gemv_shard_rows (host-only, through the C ABI) must partition every matrix
into whole 32-row tiles of equal-size pieces; and the sharded chain -- each
rank computing its rows of every GEMV, then an all-gather of every rank's
rows before the next GEMV -- run by two gloo ranks with the fp64 oracle
standing in for each rank's kernel, must reproduce the unsharded oracle chain
bit for bit (each output row depends only on its own row of W, so the split
changes nothing).  This checks the row ranges, the padding of the last
rank's piece, the gather order and the reading of the first K gathered
entries -- the bookkeeping the GPU path uses.

For the peer-memory exchange: q4gemv_peer_layout's offsets, q4gemv_peer_check
on hand-built blobs (each kind of mismatch refused), and the exchange's
protocol -- every row stored into every rank's buffer as a word carrying a
16-bit stamp (steps run x GEMVs per step + GEMV index), each reader polling
the words it needs for the previous GEMV's stamp, across the 16-bit wrap --
run by two or three processes over shared memory with the oracle standing
in for the kernels, reproducing the unsharded oracle chain over three
steps."""
import os
import sys

import numpy as np
import pytest

import oracle
import synth
import q4_quantized_decode_b200 as q4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N", [1, 31, 32, 33, 100, 5120, 7168, 34816, 17408])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_rows_partition(N, world):
    covered = np.zeros(N, dtype=np.int64)
    chunks = set()
    for r in range(world):
        st, row0, rows, chunk = q4.q4gemv_shard_rows(N, world, r)
        assert st == q4.Q4_OK
        chunks.add(chunk)
        assert chunk % 32 == 0 and 0 <= rows <= chunk
        if rows:
            assert row0 == r * chunk and row0 % 32 == 0
            covered[row0:row0 + rows] += 1
    assert len(chunks) == 1 and chunks.pop() * world >= N
    assert np.all(covered == 1)


def test_shard_rows_rejects_bad_arguments():
    assert q4.q4gemv_shard_rows(0, 2, 0)[0] == q4.Q4_EINVAL
    assert q4.q4gemv_shard_rows(64, 0, 0)[0] == q4.Q4_EINVAL
    assert q4.q4gemv_shard_rows(64, 2, 2)[0] == q4.Q4_EINVAL
    assert q4.q4gemv_shard_rows(64, 2, -1)[0] == q4.Q4_EINVAL


L, HIDDEN, QKV_N, FFN, SEED = 2, 128, 224, 160, 7070
DIMS = [(QKV_N, HIDDEN), (HIDDEN, HIDDEN), (2 * FFN, HIDDEN), (HIDDEN, FFN)]


def _sharded_chain(rank, world, gather):
    """The sharded step of one rank: its rows of each GEMV from the oracle,
    f16-rounded, padded to the common piece size and all-gathered."""
    keep = [HIDDEN, HIDDEN, FFN, HIDDEN]
    x = synth.normal_f16(SEED, synth.act_id(0), HIDDEN)
    s = 1.0
    for l in range(L):
        for t, (N, K) in enumerate(DIMS):
            _, row0, rows, chunk = q4.q4gemv_shard_rows(N, world, rank)
            piece = np.zeros(chunk, dtype=np.uint16)
            if rows:
                W = synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), N, K)[row0:row0 + rows]
                y = s * oracle.q4_gemv(W, K, x.reshape(1, K))[0]
                piece[:rows] = oracle.f64_to_f16(y)
            full = gather(piece)                 # world * chunk entries, rank order
            x = np.ascontiguousarray(full[:keep[t]])
            s = oracle.unit_rms_scale(x)
    return oracle.renorm(x)


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def gather(piece):
            t = torch.from_numpy(piece.view(np.float16).copy())   # bits moved unchanged
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            return torch.cat(parts).numpy().view(np.uint16)

        out.put((rank, _sharded_chain(rank, world, gather)))
    finally:
        dist.destroy_process_group()


def test_sharded_chain_two_gloo_ranks_equals_unsharded_oracle():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + os.getpid() % 1000
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = oracle.stack_step(
        lambda l, t: synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), *DIMS[t]),
        synth.normal_f16(SEED, synth.act_id(0), HIDDEN), L, HIDDEN, QKV_N, FFN)
    # the last rank's QKV piece is padded (224 rows = 128 + 96)
    assert q4.q4gemv_shard_rows(QKV_N, world, 1)[2] < q4.q4gemv_shard_rows(QKV_N, world, 1)[3]
    for r in range(world):
        assert np.array_equal(got[r], want), r


def test_sharded_chain_single_rank_is_the_plain_chain():
    got = _sharded_chain(0, 1, lambda piece: piece)
    want = oracle.stack_step(
        lambda l, t: synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), *DIMS[t]),
        synth.normal_f16(SEED, synth.act_id(0), HIDDEN), L, HIDDEN, QKV_N, FFN)
    assert np.array_equal(got, want)


# ---- the peer-memory exchange's host logic ----------------------------------

PEER_MAGIC, PEER_VERSION = 0x51345045, 1


def _blob(world, rank, hidden, qkv_n, ffn, nbytes=None, magic=PEER_MAGIC, version=PEER_VERSION,
          handle=b""):
    """A blob as the header lays it out (little-endian), built here by hand."""
    import struct
    if nbytes is None:
        nbytes = q4.q4gemv_peer_layout(world, hidden, qkv_n, ffn)[1][5]
    b = struct.pack("<IIiiqqqQ", magic, version, world, rank, hidden, qkv_n, ffn, nbytes)
    b += handle.ljust(64, b"\0")
    return b.ljust(q4.PEER_BLOB_BYTES, b"\0")


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("hidden,qkv_n,ffn", [(5120, 7168, 17408), (96, 160, 224), (32, 32, 32)])
def test_peer_layout(world, hidden, qkv_n, ffn):
    st, off = q4.q4gemv_peer_layout(world, hidden, qkv_n, ffn)
    assert st == q4.Q4_OK
    assert off[0] == 0 and all(o % 256 == 0 for o in off)
    for t, N in enumerate([qkv_n, hidden, 2 * ffn, hidden]):
        chunk = q4.q4gemv_shard_rows(N, world, 0)[3]
        assert off[t + 1] - off[t] >= 4 * world * chunk     # world * chunk stamped words
        assert off[t + 1] - off[t] < 4 * world * chunk + 256
    assert off[5] - off[4] >= 8                             # step count, arrival-count epoch


def test_peer_layout_rejects_bad_arguments():
    for args in [(0, 64, 64, 64), (q4.PEER_MAX_WORLD + 1, 64, 64, 64), (2, 0, 64, 64),
                 (2, 64, -1, 64), (2, 64, 64, 0)]:
        assert q4.q4gemv_peer_layout(*args)[0] == q4.Q4_EINVAL


def test_peer_check_accepts_one_exchange_and_rejects_each_mismatch():
    w, dims = 3, (256, 384, 512)
    good = [_blob(w, r, *dims) for r in range(w)]
    assert q4.q4gemv_peer_check(b"".join(good), w) == q4.Q4_OK
    bad_cases = [
        [good[1], good[0], good[2]],                                  # not in rank order
        [good[0], _blob(w, 1, *dims, magic=0), good[2]],              # magic
        [good[0], _blob(w, 1, *dims, version=2), good[2]],            # version
        [good[0], _blob(2, 1, *dims), good[2]],                       # another world
        [good[0], _blob(w, 1, 256, 384, 1024), good[2]],              # another shape
        [good[0], good[1], _blob(w, 2, *dims, nbytes=1 << 20)],       # size off the layout
    ]
    for case in bad_cases:
        assert q4.q4gemv_peer_check(b"".join(case), w) == q4.Q4_EINVAL
    assert q4.q4gemv_peer_check(b"".join(good), 0) == q4.Q4_EINVAL
    assert q4.q4gemv_peer_check(b"".join(good), q4.PEER_MAX_WORLD + 1) == q4.Q4_EINVAL


def _peer_rank(rank, world, shms, steps, dist):
    """One rank of the peer exchange, emulated on the host: every rank's
    exchange buffer is a shared-memory block laid out by q4gemv_peer_layout.
    GEMV g of a step stores each of its rows (the fp64 oracle standing in for
    the kernel) into every rank's gather buffer at rank * chunk as one word,
    the binary16 value in the low half and the stamp
    (steps run x GEMVs per step + g) mod 2^16 in the high half; GEMV g > 0
    and the final renorm poll the words they read until each carries the
    previous GEMV's stamp."""
    import random
    import time

    st, off = q4.q4gemv_peer_layout(world, HIDDEN, QKV_N, FFN)
    blobs = [None] * world
    dist.all_gather_object(blobs, _blob(world, rank, HIDDEN, QKV_N, FFN, handle=shms[rank].name.encode()))
    assert q4.q4gemv_peer_check(b"".join(blobs), world) == q4.Q4_OK

    def words(p, t, first, n):
        return np.frombuffer(shms[p].buf, dtype=np.uint32, count=n, offset=off[t] + 4 * first)

    seq = np.frombuffer(shms[rank].buf, dtype=np.uint32, count=2, offset=off[4])
    keep = [HIDDEN, HIDDEN, FFN, HIDDEN]
    per_step = 4 * L
    rng = random.Random(rank)

    def read_stamped(t, n, stamp):
        deadline = time.monotonic() + 60
        while True:
            w = words(rank, t, 0, n).copy()
            if np.all(w >> 16 == stamp):
                return (w & 0xFFFF).astype(np.uint16)
            assert time.monotonic() < deadline, "stamp wait ran out"
            time.sleep(1e-4)

    x = synth.normal_f16(SEED, synth.act_id(0), HIDDEN)
    results = []
    for _ in range(steps):
        seq[0] = (int(seq[0]) + 1) & 0xFFFFFFFF
        stamp = lambda g: (int(seq[0]) * per_step + g) & 0xFFFF  # noqa: E731
        s = 1.0
        for i in range(per_step):
            l, t = divmod(i, 4)
            N, K = DIMS[t]
            if i > 0:
                x = np.ascontiguousarray(read_stamped((t + 3) % 4, keep[(t + 3) % 4], stamp(i - 1)))
                s = oracle.unit_rms_scale(x)
            _, row0, rows, chunk = q4.q4gemv_shard_rows(N, world, rank)
            if rows:
                W = synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), N, K)[row0:row0 + rows]
                y = oracle.f64_to_f16(s * oracle.q4_gemv(W, K, x.reshape(1, K))[0])
                w = (np.uint32(stamp(i)) << np.uint32(16)) | y.astype(np.uint32)
                order = list(range(rows))
                rng.shuffle(order)                      # rows land in any order
                for p in range(world):
                    dst = words(p, t, rank * chunk, rows)
                    for r in order:
                        dst[r] = w[r]
            time.sleep(rng.random() * 2e-3)            # ranks out of step
        x = oracle.renorm(read_stamped(3, HIDDEN, stamp(per_step - 1)))
        results.append(x.copy())
    return results


def _peer_worker(rank, world, port, shm_names, out, steps):
    import gc
    from multiprocessing import shared_memory

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    shms = [shared_memory.SharedMemory(name=n) for n in shm_names]
    try:
        results = _peer_rank(rank, world, shms, steps, dist)
        dist.barrier()
        out.put((rank, results))
    finally:
        gc.collect()                               # the views into the blocks go first
        for m in shms:
            m.close()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_peer_exchange_ranks_chain_the_unsharded_oracle(world):
    """Two or three ranks (spawned processes, gloo for the blob exchange)
    run three chained steps through the peer-exchange bookkeeping; every
    step on every rank must equal the unsharded oracle step of the previous
    output bit for bit, the step count starting where the 16-bit stamps wrap
    inside the first step.  With three ranks the last holds no rows of the
    128-row matrices (64 + 64 + 0) and writes nothing for them."""
    import torch.multiprocessing as mp
    from multiprocessing import shared_memory
    steps = 3
    if world == 3:
        assert q4.q4gemv_shard_rows(HIDDEN, 3, 2)[2] == 0
    st, off = q4.q4gemv_peer_layout(world, HIDDEN, QKV_N, FFN)
    shms = [shared_memory.SharedMemory(create=True, size=off[5]) for _ in range(world)]
    try:
        for m in shms:
            m.buf[:off[5]] = bytes(off[5])
            # step count 8190: the first step's stamps (8191 * 8 + g) cross 2^16
            np.frombuffer(m.buf, dtype=np.uint32, count=2, offset=off[4])[:] = [8190, 0]
        ctx = mp.get_context("spawn")
        q = ctx.Queue()
        port = 29700 + 10 * world + os.getpid() % 1000
        procs = [ctx.Process(target=_peer_worker, args=(r, world, port, [m.name for m in shms], q, steps))
                 for r in range(world)]
        for p in procs:
            p.start()
        got = dict(q.get(timeout=300) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for m in shms:
            m.close()
            m.unlink()
    get = lambda l, t: synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), *DIMS[t])  # noqa: E731
    x = synth.normal_f16(SEED, synth.act_id(0), HIDDEN)
    for k in range(steps):
        x = oracle.stack_step(get, x, L, HIDDEN, QKV_N, FFN)
        for r in range(world):
            assert np.array_equal(got[r][k], x), (r, k)
