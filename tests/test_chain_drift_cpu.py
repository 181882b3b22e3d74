"""Why the decode-step chain is gated teacher-forced (no GPU).

An emulation of an ideal fp32 kernel (exact f16 inputs, fp32 accumulation,
f16 outputs, fp32 unit-RMS scale) drifts from the fp64 oracle chain by more than the
2e-3 GEMV tolerance after a few layers (four here), because single-ulp rounding
differences in the f16 intermediate vectors compound through the chain.  So
no implementation short of bit-identity to the oracle passes an end-to-end
2e-3 gate on a multi-layer chain; each GEMV and renorm is gated instead,
from the GPU's own inputs."""
import numpy as np

import oracle
import synth
from tests.gpu_util import rel_err


def _f16(v):
    return v.astype(np.float16).astype(np.float64)


def _fp32_gemv(rows, K, x):
    N = rows.shape[0]
    b = rows.reshape(N, K // 32, 18)
    d = (b[:, :, 0].astype(np.uint16) | (b[:, :, 1].astype(np.uint16) << 8)).view(np.float16)
    q = np.concatenate([b[:, :, 2:] & 15, b[:, :, 2:] >> 4], axis=2).astype(np.float64) - 8
    blk = np.einsum("nbj,bj->nb", q, x.reshape(K // 32, 32)) * d.astype(np.float64)
    acc = np.zeros(N, np.float32)
    for j in range(K // 32):
        acc = (acc + blk[:, j].astype(np.float32)).astype(np.float32)
    return acc.astype(np.float64)


def _fp32_scale(v):
    v32 = v.astype(np.float32)
    return np.float32(1) / np.sqrt(np.sum(v32 * v32, dtype=np.float32) / np.float32(len(v)))


def test_fp32_emulation_drifts_past_gemv_tolerance():
    L, hidden, qkv_n, ffn = 4, 256, 384, 512
    dims = [(qkv_n, hidden), (hidden, hidden), (2 * ffn, hidden), (hidden, ffn)]
    keep = [hidden, hidden, ffn, hidden]
    mats = {(l, t): synth.q4_0_matrix(4321, synth.weight_id(4 * l + t), *dims[t])
            for l in range(L) for t in range(4)}
    worst = 0.0
    for seed in range(3):
        xb = synth.normal_f16(4321 + seed, synth.act_id(0), hidden)
        ref = oracle.stack_step(lambda l, t: mats[(l, t)], xb, L, hidden, qkv_n, ffn)
        x = xb.view(np.float16).astype(np.float64)
        s = np.float32(1)
        for l in range(L):
            for t in range(4):
                y = _f16((s * _fp32_gemv(mats[(l, t)], dims[t][1], x).astype(np.float32)).astype(np.float64))
                x = y[:keep[t]]
                s = _fp32_scale(x)
        out = _f16((x.astype(np.float32) * s).astype(np.float64))
        worst = max(worst, rel_err(out.astype(np.float16).view(np.uint16), oracle.f16_to_f64(ref)))
    assert worst > 2e-3
