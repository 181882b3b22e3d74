"""The decode step with the feed-forward activation (q4gemv_run_stack_gated:
each down GEMV fed SiLU(gate) * up of the gate+up output, scaled to unit RMS)
through the C ABI, against the fp64 oracle's gated chain, on both step modes
(the persistent kernel, whose staging combines the gate and up halves, and
the per-GEMV kernels, whose down GEMV is the gated GEMV kernel)."""
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


def _engine(mode):
    old = os.environ.get("Q4GEMV_STACK_MODE")
    os.environ["Q4GEMV_STACK_MODE"] = mode
    try:
        return q4.Q4Gemv(0)
    finally:
        if old is None:
            os.environ.pop("Q4GEMV_STACK_MODE", None)
        else:
            os.environ["Q4GEMV_STACK_MODE"] = old


def _stack(eng, L, hidden, qkv_n, ffn, seed):
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    get = lambda l, t: synth.q4_0_matrix(seed, synth.weight_id(4 * l + t), *dims[t])  # noqa: E731
    layers = [tuple(packed_on_gpu(eng, get(l, t), *dims[t]) for t in range(4)) for l in range(L)]
    return layers, get


@pytest.mark.parametrize("mode", ["persistent", "kernels"])
@pytest.mark.parametrize("L,hidden,qkv_n,ffn", [(1, 256, 384, 512), (1, 96, 160, 224)])
def test_gated_step_matches_oracle(mode, L, hidden, qkv_n, ffn):
    """One layer end to end (longer chains compound single-ulp differences
    past the GEMV tolerance even for an ideal fp32 kernel; see
    tests/test_chain_drift_cpu.py)."""
    eng = _engine(mode)
    layers, get = _stack(eng, L, hidden, qkv_n, ffn, 606)
    x = synth.normal_f16(606, synth.act_id(0), hidden)
    got = bits_of(eng.run_stack_gated(layers, f16_dev(x), hidden, qkv_n, ffn))
    assert eng.sync_status() == q4.Q4_OK
    want = oracle.stack_step(get, x, L, hidden, qkv_n, ffn, threads=8, gated=True)
    assert rel_err(got, oracle.f16_to_f64(want)) <= TOL
    plain = bits_of(eng.run_stack(layers, f16_dev(x), hidden, qkv_n, ffn))
    assert not np.array_equal(got, plain)          # the activation changes the step
    eng.close()


def test_gated_step_full_width_modes_agree_and_match_oracle():
    """One 27B-shaped layer: every output row against the oracle, and the
    two step modes (same split at full width) give the same bits."""
    L, hidden, qkv_n, ffn = 1, 5120, 7168, 17408
    outs = {}
    for mode in ("persistent", "kernels"):
        eng = _engine(mode)
        if mode == "persistent":
            layers, get = _stack(eng, L, hidden, qkv_n, ffn, 707)
        x = synth.normal_f16(707, synth.act_id(0), hidden)
        outs[mode] = bits_of(eng.run_stack_gated(layers, f16_dev(x), hidden, qkv_n, ffn))
        assert eng.sync_status() == q4.Q4_OK
        eng.close()
    assert np.array_equal(outs["persistent"], outs["kernels"])
    want = oracle.stack_step(get, x, L, hidden, qkv_n, ffn, threads=8, gated=True)
    assert rel_err(outs["persistent"], oracle.f16_to_f64(want)) <= TOL


@pytest.mark.parametrize("hidden,qkv_n,ffn,exact", [(256, 384, 512, False), (5120, 7168, 17408, True)])
def test_gated_two_layers_modes_agree(hidden, qkv_n, ffn, exact):
    """Two layers, so the plain staging after a gated GEMV runs too: the
    persistent step and the per-GEMV kernels agree -- bit for bit at full
    width (the same split), within the GEMV tolerance on small shapes (the
    persistent step splits them over more warps, so its fp32 sums run in
    another order)."""
    L = 2
    outs = {}
    for mode in ("persistent", "kernels"):
        eng = _engine(mode)
        if mode == "persistent":
            layers, _ = _stack(eng, L, hidden, qkv_n, ffn, 909)
        x = synth.normal_f16(909, synth.act_id(0), hidden)
        outs[mode] = bits_of(eng.run_stack_gated(layers, f16_dev(x), hidden, qkv_n, ffn))
        assert eng.sync_status() == q4.Q4_OK
        eng.close()
    if exact:
        assert np.array_equal(outs["persistent"], outs["kernels"])
    else:
        assert rel_err(outs["persistent"], outs["kernels"].view(np.float16).astype(np.float64)) <= TOL


def test_gated_and_plain_steps_alternate_on_one_handle():
    """The gated and plain steps keep separate descriptors and graphs: calls
    alternating on one handle give each step's own result."""
    L, hidden, qkv_n, ffn = 1, 128, 192, 256
    eng = q4.Q4Gemv(0)
    layers, get = _stack(eng, L, hidden, qkv_n, ffn, 808)
    x = synth.normal_f16(808, synth.act_id(0), hidden)
    xd = f16_dev(x)
    wp = oracle.f16_to_f64(oracle.stack_step(get, x, L, hidden, qkv_n, ffn))
    wg = oracle.f16_to_f64(oracle.stack_step(get, x, L, hidden, qkv_n, ffn, gated=True))
    for _ in range(2):
        assert rel_err(bits_of(eng.run_stack(layers, xd, hidden, qkv_n, ffn)), wp) <= TOL
        assert rel_err(bits_of(eng.run_stack_gated(layers, xd, hidden, qkv_n, ffn)), wg) <= TOL
    assert eng.sync_status() == q4.Q4_OK
    eng.close()


def test_gated_step_host_vectors_and_errors():
    """Host (pinned) input and output vectors, staged inside the call, give
    the device-vector result; null and misaligned arguments are refused."""
    L, hidden, qkv_n, ffn = 1, 128, 192, 256
    eng = q4.Q4Gemv(0)
    layers, _ = _stack(eng, L, hidden, qkv_n, ffn, 1010)
    x = synth.normal_f16(1010, synth.act_id(0), hidden)
    dev = bits_of(eng.run_stack_gated(layers, f16_dev(x), hidden, qkv_n, ffn))
    xh = torch.from_numpy(x.view(np.float16).copy()).pin_memory()
    oh = torch.empty(hidden, dtype=torch.float16).pin_memory()
    eng.run_stack_gated(layers, xh, hidden, qkv_n, ffn, x_out=oh)
    torch.cuda.synchronize()
    assert eng.sync_status() == q4.Q4_OK
    assert np.array_equal(oh.view(torch.int16).numpy().view(np.uint16), dev)
    arr = (q4.q4gemv_layer * 1)()
    arr[0] = q4.q4gemv_layer(None, None, None, None)
    out = torch.empty(hidden, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    xd = f16_dev(x)
    assert q4.q4gemv_run_stack_gated(eng.h, arr, 1, hidden, qkv_n, ffn, xd.data_ptr(), out.data_ptr(),
                                     st) == q4.Q4_EINVAL
    a, b, c, d = layers[0]
    arr[0] = q4.q4gemv_layer(a.data_ptr(), b.data_ptr() + 8, c.data_ptr(), d.data_ptr())
    assert q4.q4gemv_run_stack_gated(eng.h, arr, 1, hidden, qkv_n, ffn, xd.data_ptr(), out.data_ptr(),
                                     st) == q4.Q4_EALIGN
    eng.close()
