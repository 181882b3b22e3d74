"""The layer-range pipeline's host logic on CPU (bench.py --pipeline, the
pages' multi-device split, used as the comparison for the row-sharded step).

bench.layer_range must give every rank a contiguous range, together all
layers once; and two gloo ranks, each running its range of the fp64 oracle
chain and passing the f16 hidden state on with send/recv (the last rank back
to the first, for the next token of one autoregressive stream), must
reproduce the same chain run range by range in one process, bit for bit,
over two tokens.  Against the unsharded chain the only difference is one
more f16 rounding of the renormalised hidden state per range boundary (the
next range takes it as its input as it is), checked at the boundary."""
import os
import sys

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L, HIDDEN, QKV_N, FFN, SEED = 4, 128, 192, 160, 4242
DIMS = [(QKV_N, HIDDEN), (HIDDEN, HIDDEN), (2 * FFN, HIDDEN), (HIDDEN, FFN)]


def _rows(l, t):
    return synth.q4_0_matrix(SEED, synth.weight_id(4 * l + t), *DIMS[t])


def _range_step(l0, l1, x):
    return oracle.stack_step(lambda l, t: _rows(l0 + l, t), x, l1 - l0, HIDDEN, QKV_N, FFN)


@pytest.mark.parametrize("n_layers", [1, 2, 7, 64])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_layer_ranges_cover_every_layer_once(world, n_layers):
    sys.path.insert(0, ROOT)
    import bench
    covered = []
    prev = 0
    for r in range(world):
        l0, l1 = bench.layer_range(world, r, n_layers)
        assert l0 == prev and l1 >= l0 and l1 - l0 in (n_layers // world, -(-n_layers // world))
        covered += list(range(l0, l1))
        prev = l1
    assert covered == list(range(n_layers))


def _worker(rank, world, port, out, tokens):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        l0, l1 = bench.layer_range(world, rank, L)
        buf = torch.empty(HIDDEN, dtype=torch.int16)
        x = synth.normal_f16(SEED, synth.act_id(0), HIDDEN)
        outs = []
        for _ in range(tokens):
            if rank > 0:
                dist.recv(buf, src=rank - 1)
                x = buf.numpy().view(np.uint16).copy()
            y = _range_step(l0, l1, x)
            dist.send(torch.from_numpy(y.view(np.int16).copy()), dst=(rank + 1) % world)
            if rank == 0:
                dist.recv(buf, src=world - 1)
                x = buf.numpy().view(np.uint16).copy()
                outs.append(x)
        out.put((rank, outs))
    finally:
        dist.destroy_process_group()


def test_pipeline_two_gloo_ranks_two_tokens():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29800 + os.getpid() % 1000
    world, tokens = 2, 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, tokens)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = synth.normal_f16(SEED, synth.act_id(0), HIDDEN)
    for k in range(tokens):
        first = _range_step(0, L // 2, x)
        ranged = _range_step(L // 2, L, first)
        assert np.array_equal(got[0][k], ranged), k
        # the first range is the unsharded chain's first layers, and the
        # hidden state handed on is that chain's input to layer L/2, rounded
        # to f16 after its unit-RMS scale (the unsharded chain keeps the
        # scale exact inside the GEMV): the pipeline's one difference
        seen = {}
        oracle.stack_step(_rows, x, L, HIDDEN, QKV_N, FFN,
                          record=lambda i, xf, s, y: seen.setdefault(i, (xf.copy(), s)))
        xf, s = seen[4 * (L // 2)]
        assert np.array_equal(first, oracle.renorm(xf))
        assert s == oracle.unit_rms_scale(xf)
        x = ranged
