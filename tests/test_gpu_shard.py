"""The row-sharded decode step through the C ABI on one GPU (world = 1), on
both exchanges: a real NCCL communicator, and the peer-memory exchange (the
GEMV kernels store their rows into every rank's gather buffer and stamp
them; the next GEMV waits for the stamps).  Each must match the fp64 oracle
chain end to end and q4gemv_run_stack within the GEMV tolerance, the two
exchanges must give the same bits, steps must chain (the stamps advance
every step), a stamp that never comes must end in Q4_ETIMEOUT with the
handle still usable, and a handle without a communicator or an exchange for
the shapes must refuse.  The host bookkeeping for more ranks is covered on
CPU (tests/test_shard_cpu.py)."""
import os

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, bits_of, f16_dev, packed_on_gpu, rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import q4_quantized_decode_b200 as q4  # noqa: E402


def _stack(eng, L, hidden, qkv_n, ffn, seed):
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    layers = [tuple(packed_on_gpu(eng, synth.q4_0_matrix(seed, synth.weight_id(4 * l + t), *dims[t]), *dims[t])
                    for t in range(4)) for l in range(L)]
    get = lambda l, t: synth.q4_0_matrix(seed, synth.weight_id(4 * l + t), *dims[t])  # noqa: E731
    return layers, get


@pytest.fixture(scope="module")
def eng():
    e = q4.Q4Gemv(0)
    st, uid = q4.q4gemv_comm_unique_id()
    assert st == q4.Q4_OK
    e.init_comm(1, 0, uid)
    yield e
    e.close()


@pytest.mark.parametrize("L,hidden,qkv_n,ffn", [(2, 256, 384, 512), (1, 5120, 7168, 17408)])
def test_sharded_step_matches_oracle_and_single_gpu_step(eng, L, hidden, qkv_n, ffn):
    layers, get = _stack(eng, L, hidden, qkv_n, ffn, 1234)
    x = synth.normal_f16(1234, synth.act_id(0), hidden)
    xd = f16_dev(x)
    got = bits_of(eng.run_stack_sharded(layers, xd, hidden, qkv_n, ffn))
    assert eng.sync_status() == q4.Q4_OK
    want = oracle.stack_step(get, x, L, hidden, qkv_n, ffn, threads=8)
    assert rel_err(got, oracle.f16_to_f64(want)) <= TOL
    single = bits_of(eng.run_stack(layers, xd, hidden, qkv_n, ffn))
    assert rel_err(got, single.view(np.float16).astype(np.float64)) <= TOL


def test_sharded_step_replay_follows_input(eng):
    L, hidden, qkv_n, ffn = 1, 128, 192, 256
    layers, get = _stack(eng, L, hidden, qkv_n, ffn, 99)
    xa = synth.normal_f16(99, synth.act_id(0), hidden)
    xb = synth.normal_f16(99, synth.act_id(1), hidden)
    xin = f16_dev(xa)
    out = torch.empty(hidden, dtype=torch.float16, device="cuda")
    eng.run_stack_sharded(layers, xin, hidden, qkv_n, ffn, x_out=out)
    oa = bits_of(out)
    xin.copy_(f16_dev(xb))
    eng.run_stack_sharded(layers, xin, hidden, qkv_n, ffn, x_out=out)
    ob = bits_of(out)
    assert eng.sync_status() == q4.Q4_OK
    assert rel_err(oa, oracle.f16_to_f64(oracle.stack_step(get, xa, L, hidden, qkv_n, ffn))) <= TOL
    assert rel_err(ob, oracle.f16_to_f64(oracle.stack_step(get, xb, L, hidden, qkv_n, ffn))) <= TOL


def test_sharded_step_needs_a_communicator():
    e = q4.Q4Gemv(0)
    layers, _ = _stack(e, 1, 64, 96, 128, 5)
    with pytest.raises(q4.Q4Error) as err:
        e.run_stack_sharded(layers, f16_dev(synth.normal_f16(5, synth.act_id(0), 64)), 64, 96, 128)
    assert err.value.status == q4.Q4_EINVAL
    e.close()


def _peer_engine(hidden, qkv_n, ffn):
    e = q4.Q4Gemv(0)
    blob = e.peer_export(1, 0, hidden, qkv_n, ffn)
    assert len(blob) == q4.PEER_BLOB_BYTES and q4.q4gemv_peer_check(blob, 1) == q4.Q4_OK
    e.peer_open([blob])
    return e


@pytest.mark.parametrize("L,hidden,qkv_n,ffn", [(2, 256, 384, 512), (1, 5120, 7168, 17408),
                                                (2, 96, 160, 224), (1, 96, 200, 224)])
def test_peer_step_matches_oracle_and_nccl_bits(eng, L, hidden, qkv_n, ffn):
    """(1, 96, 200, 224): QKV of 200 rows, a ragged last tile whose missing
    rows are never written nor read."""
    pe = _peer_engine(hidden, qkv_n, ffn)
    layers, get = _stack(pe, L, hidden, qkv_n, ffn, 4321)
    x = synth.normal_f16(4321, synth.act_id(0), hidden)
    xd = f16_dev(x)
    got = bits_of(pe.run_stack_sharded(layers, xd, hidden, qkv_n, ffn))
    assert pe.sync_status() == q4.Q4_OK
    want = oracle.stack_step(get, x, L, hidden, qkv_n, ffn, threads=8)
    assert rel_err(got, oracle.f16_to_f64(want)) <= TOL
    nccl = bits_of(eng.run_stack_sharded(layers, xd, hidden, qkv_n, ffn))
    assert eng.sync_status() == q4.Q4_OK
    assert np.array_equal(got, nccl)
    # at world 1 the row split is the whole matrix: the per-GEMV kernels of
    # the single-GPU step (same kernel, split and combine order), so their
    # bits; the persistent step splits small shapes over more warps, so it
    # agrees within the tolerance (and bit for bit at full width)
    old = os.environ.get("Q4GEMV_STACK_MODE")
    os.environ["Q4GEMV_STACK_MODE"] = "kernels"
    try:
        ek = q4.Q4Gemv(0)
    finally:
        if old is None:
            os.environ.pop("Q4GEMV_STACK_MODE", None)
        else:
            os.environ["Q4GEMV_STACK_MODE"] = old
    kern = bits_of(ek.run_stack(layers, xd, hidden, qkv_n, ffn))
    assert ek.sync_status() == q4.Q4_OK
    ek.close()
    assert np.array_equal(got, kern)
    single = bits_of(pe.run_stack(layers, xd, hidden, qkv_n, ffn))
    assert rel_err(got, single.view(np.float16).astype(np.float64)) <= TOL
    if hidden == 5120:
        assert np.array_equal(got, single)
    pe.close()


def test_peer_steps_chain(eng):
    """Five steps in a row, each fed the previous output: the stamp base
    advances by the step's GEMV count every step, and every step must read
    its own GEMVs' rows -- the same bits as the NCCL exchange on the same
    input, and the oracle step of that input within the GEMV tolerance (one
    layer: longer chains are gated GEMV by GEMV, see test_gpu_parity)."""
    L, hidden, qkv_n, ffn = 1, 256, 384, 512
    pe = _peer_engine(hidden, qkv_n, ffn)
    layers, get = _stack(pe, L, hidden, qkv_n, ffn, 77)
    x = synth.normal_f16(77, synth.act_id(0), hidden)
    xin = f16_dev(x)
    out = torch.empty(hidden, dtype=torch.float16, device="cuda")
    for _ in range(5):
        pe.run_stack_sharded(layers, xin, hidden, qkv_n, ffn, x_out=out)
        y = bits_of(out)
        assert pe.sync_status() == q4.Q4_OK
        assert np.array_equal(y, bits_of(eng.run_stack_sharded(layers, xin, hidden, qkv_n, ffn)))
        assert rel_err(y, oracle.f16_to_f64(oracle.stack_step(get, x, L, hidden, qkv_n, ffn))) <= TOL
        x = y
        xin.copy_(out)
    pe.close()


def test_peer_layer_count_change():
    """The split tiles' arrival counts run on across layers and steps with
    the layer count in their arithmetic: a step of another depth on the same
    exchange (counts zeroed, graph recaptured) must still be right, and so
    must the first depth again."""
    hidden, qkv_n, ffn = 256, 384, 512
    pe = _peer_engine(hidden, qkv_n, ffn)
    layers, get = _stack(pe, 3, hidden, qkv_n, ffn, 55)
    x = synth.normal_f16(55, synth.act_id(0), hidden)
    xd = f16_dev(x)
    for L in (1, 3, 1, 1):
        y = bits_of(pe.run_stack_sharded(layers[:L], xd, hidden, qkv_n, ffn))
        assert pe.sync_status() == q4.Q4_OK
        single = bits_of(pe.run_stack(layers[:L], xd, hidden, qkv_n, ffn))
        assert pe.sync_status() == q4.Q4_OK
        assert rel_err(y, single.view(np.float16).astype(np.float64)) <= TOL
        if L == 1:
            assert rel_err(y, oracle.f16_to_f64(oracle.stack_step(get, x, L, hidden, qkv_n, ffn))) <= TOL
    pe.close()


def test_peer_wait_timeout_is_reported_and_recoverable():
    """Every stamp wait of the step given a stamp no rank writes and a short
    poll budget (the "timeout" test knob): the kernels must return, the
    error word read Q4_ETIMEOUT, and the next step on the same handle run
    normally."""
    L, hidden, qkv_n, ffn = 1, 256, 384, 512
    pe = _peer_engine(hidden, qkv_n, ffn)
    layers, get = _stack(pe, L, hidden, qkv_n, ffn, 31)
    x = synth.normal_f16(31, synth.act_id(0), hidden)
    xd = f16_dev(x)
    want = bits_of(pe.run_stack_sharded(layers, xd, hidden, qkv_n, ffn))
    assert pe.sync_status() == q4.Q4_OK
    out = torch.zeros(hidden, dtype=torch.float16, device="cuda")
    pe.set_fault("timeout")
    pe.run_stack_sharded(layers, xd, hidden, qkv_n, ffn, x_out=out)
    torch.cuda.synchronize()                      # every wait gave up and returned
    assert pe.sync_status() == q4.Q4_ETIMEOUT
    assert pe.sync_status() == q4.Q4_OK
    pe.set_fault("none")
    got = bits_of(pe.run_stack_sharded(layers, xd, hidden, qkv_n, ffn, x_out=out))
    assert pe.sync_status() == q4.Q4_OK
    assert np.array_equal(got, want)
    assert rel_err(got, oracle.f16_to_f64(oracle.stack_step(get, x, L, hidden, qkv_n, ffn))) <= TOL
    pe.close()


def test_peer_exchange_argument_errors():
    hidden, qkv_n, ffn = 64, 96, 128
    e = q4.Q4Gemv(0)
    with pytest.raises(q4.Q4Error) as err:              # nothing exported yet
        e.peer_open([bytes(q4.PEER_BLOB_BYTES)])
    assert err.value.status == q4.Q4_EINVAL
    for world, rank in [(0, 0), (2, 2), (q4.PEER_MAX_WORLD + 1, 0), (2, -1)]:
        with pytest.raises(q4.Q4Error) as err:
            e.peer_export(world, rank, hidden, qkv_n, ffn)
        assert err.value.status == q4.Q4_EINVAL
    blob = e.peer_export(1, 0, hidden, qkv_n, ffn)
    bad = bytearray(blob)
    bad[24] ^= 1                                        # another QKV size
    with pytest.raises(q4.Q4Error) as err:
        e.peer_open([bytes(bad)])
    assert err.value.status == q4.Q4_EINVAL
    e.peer_open([blob])
    layers, _ = _stack(e, 1, hidden, qkv_n, ffn, 5)
    x = f16_dev(synth.normal_f16(5, synth.act_id(0), hidden))
    e.run_stack_sharded(layers, x, hidden, qkv_n, ffn)
    assert e.sync_status() == q4.Q4_OK
    with pytest.raises(q4.Q4Error) as err:              # shapes without an exchange or NCCL
        e.run_stack_sharded(layers, x, hidden, qkv_n, 2 * ffn)
    assert err.value.status == q4.Q4_EINVAL
    e.peer_close()
    with pytest.raises(q4.Q4Error) as err:              # closed
        e.run_stack_sharded(layers, x, hidden, qkv_n, ffn)
    assert err.value.status == q4.Q4_EINVAL
    e.close()
