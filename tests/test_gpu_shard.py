"""The row-sharded decode step through the C ABI on one GPU (world = 1, a
real NCCL communicator): it must match the fp64 oracle chain end to end and
q4gemv_run_stack within the GEMV tolerance, follow a new input on graph
replay, and refuse to run without a communicator.  The host bookkeeping for
more ranks is covered on CPU (tests/test_shard_cpu.py)."""
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
