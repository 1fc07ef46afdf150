"""GPU parity at the full size of one layer of the 52-layer denoise sweep.

One layer is a 128-expert top-6 MoE block (up 2688 -> 1856, squared ReLU,
down 1856 -> 2688) plus a dense 2688 -> 4096 and a 4096 -> 2688 projection,
run on 512 tokens (32 sequences x one 16-token denoise block).  The CUDA path
runs the whole layer in the launch configuration the benchmark times; the
oracle recomputes sampled tokens and rows, which are independent of the
others (a token's MoE output depends only on its own row and routing, a
linear output row only on its input row)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
WL = synth.WORKLOADS["denoise_sweep_52"]
LAYER = 37


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


def test_denoise_layer_moe_512_tokens_sampled():
    E, H, I, m, topk = WL["num_experts"], WL["hidden"], WL["inter"], WL["m"], WL["topk"]
    s_up, s_dn = synth.sweep_seed(LAYER, 0), synth.sweep_seed(LAYER, 1)
    up = synth.normal_f32_device((E, I, H), s_up, WL["w_std"], DEV)
    dn = synth.normal_f32_device((E, H, I), s_dn, WL["w_std"], DEV)
    pu = tq.tq4_1s_quantize(up, seed=s_up)
    pd = tq.tq4_1s_quantize(dn, seed=s_dn)
    x = synth.activations_bf16(m, H, synth.sweep_seed(LAYER, 4))
    ids, w = synth.gumbel_topk_router(m, E, topk, synth.sweep_seed(LAYER, 5))
    y = tq.tq4_1s_moe(_bf16_dev(x), torch.from_numpy(ids).to(DEV), torch.from_numpy(w).to(DEV), pu, pd)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    # every expert is active at 512 tokens x top-6 (3072 pairs over 128 experts)
    assert len(set(ids.ravel().tolist())) == E

    tokens = np.array([0, 131, 302, 511])
    used = sorted(set(int(e) for e in ids[tokens].ravel()))
    remap = {e: i for i, e in enumerate(used)}
    # the oracle quantizes the sampled tokens' experts from the same fp32 draws
    uc = np.zeros((len(used), I, H // 2), np.uint8); us = np.zeros((len(used), I, H // 16), np.uint16)
    dc = np.zeros((len(used), H, I // 2), np.uint8); ds = np.zeros((len(used), H, I // 16), np.uint16)
    for e in used:
        uc[remap[e]], us[remap[e]], _ = oracle.quantize(up[e].cpu().numpy(), s_up)
        dc[remap[e]], ds[remap[e]], _ = oracle.quantize(dn[e].cpu().numpy(), s_dn)
    ids_s = np.vectorize(remap.get)(ids[tokens]).astype(np.int32)
    y_ref, _, bad = oracle.moe(x[tokens], ids_s, w[tokens], uc, us, s_up, dc, ds, s_dn)
    assert bad == 0
    e = assert_close(_bits(y)[tokens], y_ref, "denoise layer moe, 512 tokens")
    print("moe 512 errors", e)


@pytest.mark.parametrize("which", [0, 1])
def test_denoise_layer_dense_512_tokens_sampled(which):
    n, k = WL["dense"][which]
    m = WL["m"]
    s_w = synth.sweep_seed(LAYER, 2 + which)
    W = synth.normal_f32_device((n, k), s_w, WL["w_std"], DEV)
    p = tq.tq4_1s_quantize(W, seed=s_w)
    x = synth.activations_bf16(m, k, synth.sweep_seed(LAYER, 4 if which == 0 else 6))
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    rows = np.array([0, 77, 255, 256, 400, 511])
    codes, scales, _ = oracle.quantize(W.cpu().numpy(), s_w)
    y_ref = oracle.linear_f64(x[rows], oracle.dequantize(codes, scales, s_w))
    e = assert_close(_bits(y)[rows], y_ref, f"denoise layer dense {n}x{k}, 512 tokens")
    print("dense 512 errors", e)
