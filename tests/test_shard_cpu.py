"""The row-sharded decode step's host logic on CPU.

q4gemv_shard_rows (host-only, through the C ABI) must partition every matrix
into whole 32-row tiles of equal-size pieces; and the sharded chain -- each
rank computing its rows of every GEMV, then an all-gather of every rank's
rows before the next GEMV -- run by two gloo ranks with the fp64 oracle
standing in for each rank's kernel, must reproduce the unsharded oracle chain
bit for bit (each output row depends only on its own row of W, so the split
changes nothing).  This checks the row ranges, the padding of the last
rank's piece, the gather order and the reading of the first K gathered
entries -- the bookkeeping the GPU path uses."""
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
