"""GPU parity of the MLX-style affine group format (the MLX port's README,
section "Quantization (6-bit, scheme mixed_v1)"; 4/6/8-bit family), the
second format of the bytes-versus-accuracy comparison with TQ4_1S: codes,
bf16 scales and biases bit for bit against the CPU oracle, the dequantized
weight bit for bit, and the linear within the stated tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("shape,seed", [((64, 256), 180), ((7, 1024), 181), ((512, 2688), 182)])
def test_affine_quantize_and_dequantize_bit_exact(bits, shape, seed):
    W = synth.student_t_f32(shape, seed, 5.0, 0.02)
    W[0, 64:128] = 0.25                                   # a constant group
    a = tq.tq4_1s_affine_quantize(torch.from_numpy(W).to(DEV), bits)
    Wd = tq.tq4_1s_affine_dequantize(a)
    torch.cuda.synchronize()
    codes, scales, biases = oracle.affine_quantize(W, bits)
    assert np.array_equal(a.codes.cpu().numpy(), codes)
    assert np.array_equal(a.scales.cpu().numpy().view(np.uint16), scales)
    assert np.array_equal(a.biases.cpu().numpy().view(np.uint16), biases)
    Wo = oracle.affine_dequantize(codes, scales, biases, bits)
    assert np.array_equal(Wd.cpu().numpy().view(np.uint32), Wo.view(np.uint32))


@pytest.mark.parametrize("bits,m,n,k,seed", [(6, 16, 512, 1024, 183), (4, 1, 256, 256, 184),
                                             (8, 200, 384, 512, 185)])
def test_affine_linear_parity(bits, m, n, k, seed):
    W = synth.normal_f32((n, k), seed, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    a = tq.tq4_1s_affine_quantize(torch.from_numpy(W).to(DEV), bits)
    y = tq.tq4_1s_affine_linear(torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), a)
    torch.cuda.synchronize()
    codes, scales, biases = oracle.affine_quantize(W, bits)
    y_ref = oracle.linear_f64(x, oracle.affine_dequantize(codes, scales, biases, bits))
    assert_close(_bits(y), y_ref, f"affine linear {bits}-bit m={m}")
    assert tq.tq4_1s_get_status() == 0
