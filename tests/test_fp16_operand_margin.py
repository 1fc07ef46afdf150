"""The small-m GEMM's operand rounding, emulated on the CPU against the fp64
oracle: levels fp16(fp16(256 c[code]) * d), activations x' = R x scaled per
row by a power of two 2^-e (sqrt(32) max|x| in [2^13, 2^14)) and rounded to
fp16, exact products accumulated, then y = bf16(sum * 2^e / 256).  The error
of this design must sit well inside the layer's tolerance (max_rel 2e-2,
mean_rel 2e-3), also for activations of very large and very small magnitude
where the per-row scale does the work."""
import numpy as np
import pytest

import oracle
import synth
from tests._parity import errors


def _f16(a):
    return a.astype(np.float16).astype(np.float64)


def _emulate(x_bits, codes, scales, seed):
    lv32 = oracle.codebook()[2]
    table = _f16(lv32.astype(np.float32) * np.float32(256.0))        # fp16(256 c)
    n, kb = codes.shape
    k = 2 * kb
    c = np.empty((n, k), np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    d = scales.view(np.float16).astype(np.float64)
    A = _f16(table[c] * np.repeat(d, 16, axis=1))                      # one fp16 product
    mask = oracle.sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    H = oracle.hadamard32().astype(np.float64)
    x = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    r = float(np.float32(1.0 / np.sqrt(32.0)))
    xr = ((x.reshape(x.shape[0], -1, 32) * s) @ H.T * r).reshape(x.shape)
    mx = np.abs(x).max(axis=1, keepdims=True)
    e = np.floor(np.log2(mx * np.sqrt(32.0))) + 1 - 14                 # sqrt(32) mx in [2^13, 2^14)
    sc = 2.0 ** e
    y = (_f16(xr / sc) @ A.T) * sc / 256.0
    return synth.f32_to_bf16_bits(y.astype(np.float32))


@pytest.mark.parametrize("m,n,k,x_std,seed", [
    (16, 256, 1024, 1.0, 70),
    (5, 128, 512, 3000.0, 71),
    (8, 128, 512, 1e-5, 72),
])
def test_fp16_operands_stay_well_inside_the_tolerance(m, n, k, x_std, seed):
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.f32_to_bf16_bits(synth.student_t_f32((m, k), seed + 1, 5.0, x_std))
    codes, scales, _ = oracle.quantize(W, seed)
    y_ref, _ = oracle.linear(x, codes, scales, seed)
    e = errors(_emulate(x, codes, scales, seed), y_ref)
    assert e["mean_rel"] < 1e-3 and e["max_rel"] < 1.5e-2, e
