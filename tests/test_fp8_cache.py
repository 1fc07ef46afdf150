"""GPU parity of the fp8-resident weight cache (model card
"Nemotron-TheHobbit-30B-A3B", section "Help wanted": dequantize once, keep
the weights resident in fp8): the TQ4_1S -> fp8 conversion bit for bit
against the CPU oracle (E4M3 codes and the fp32 row scales), and the fp8
linear against the oracle's fp64 product with the same cache, in the decode
kernel (m <= 32) and the large-m path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


@pytest.mark.parametrize("shape,seed", [((256, 256), 160), ((200, 96), 161), ((3, 64, 160), 162),
                                        ((4096, 4096), 2)])
def test_to_fp8_bit_exact(shape, seed):
    W = synth.student_t_f32(shape, seed, 5.0, 0.02)
    W.reshape(-1, shape[-1])[1] = 0.0                      # a zero row: scale 0, codes 0
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    f = tq.tq4_1s_to_fp8(p)
    torch.cuda.synchronize()
    codes, scales, _ = oracle.quantize(W.reshape(-1, shape[-1]), seed)
    q, s = oracle.to_fp8(codes, scales, seed)
    assert np.array_equal(f.q.cpu().numpy(), q)
    assert np.array_equal(f.wscale.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert tq.tq4_1s_get_status() == 0


@pytest.mark.parametrize("m,n,k,seed", [
    (16, 4096, 4096, 2),      # the decode block: 4-CTA clusters, 1 byte per weight streamed
    (1, 256, 256, 163),
    (17, 512, 1024, 164),     # two 16-token blocks
    (16, 200, 2080, 165),     # ragged rows and k
    (48, 512, 1024, 166),     # large-m path: bf16 weight + tensor-core GEMM
    (300, 520, 224, 167),
])
def test_linear_fp8_parity(m, n, k, seed):
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    f = tq.tq4_1s_to_fp8(p)
    y = tq.tq4_1s_linear_fp8(_bf16_dev(x), f)
    torch.cuda.synchronize()
    codes, scales, _ = oracle.quantize(W, seed)
    q, s = oracle.to_fp8(codes, scales, seed)
    y_ref, _ = oracle.linear_fp8(x, q, s)
    assert_close(_bits(y), y_ref, f"fp8 linear m={m} n={n} k={k}")
    assert tq.tq4_1s_get_status() == 0


def test_linear_fp8_static_flag_same_bits():
    p = tq.tq4_1s_quantize(synth.normal_f32_device((2048, 2048), 168, 0.02, DEV), seed=168)
    f = tq.tq4_1s_to_fp8(p)
    torch.cuda.synchronize()
    fs = tq.Fp8Weight(f.q, f.wscale, f.n, f.k, flags=tq.TQ_WEIGHT_STATIC)
    x = _bf16_dev(synth.activations_bf16(16, 2048, 169))
    y0, y1 = tq.tq4_1s_linear_fp8(x, f), tq.tq4_1s_linear_fp8(x, fs)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
