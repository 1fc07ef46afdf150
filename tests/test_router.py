"""GPU parity of the device-side MoE router and of the MoE that routes from
logits (model card "Nemotron-TheHobbit-30B-A3B", sections "The model
underneath" -- top-6 of 128 experts -- and "Performance" -- the sync-free
MoE), against the CPU oracle's router on the same fp32 logits.  Expert ids
are compared bit for bit; router weights within 1e-6 relative."""
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


@pytest.mark.parametrize("m,E,topk,seed", [
    (16, 128, 6, 7),       # the decode block's routing
    (512, 128, 6, 1005),   # one layer of the denoise sweep (32 sequences x 16 tokens)
    (33, 1000, 8, 71),     # ragged token count, experts not a multiple of 32
    (5, 7, 7, 72),         # every expert chosen
    (3, 32, 1, 73),        # top-1
])
def test_router_topk_matches_oracle(m, E, topk, seed):
    z = synth.router_logits_f32(m, E, seed)
    ids, w = tq.tq4_1s_router_topk(torch.from_numpy(z).to(DEV), topk)
    ids_ref, w_ref = oracle.router_topk(z, topk)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    wg = w.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(wg - w_ref) / w_ref) <= 1e-6
    assert tq.tq4_1s_get_status() == 0


def test_router_ties_and_special_values():
    # equal logits (ties to the lower id), -inf logits (chosen last), and a
    # row whose logits are all equal
    z = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, -np.inf, 0.0, 2.0],
                  [0.0] * 8,
                  [-np.inf, -np.inf, 3.0, -1.0, -np.inf, -np.inf, -np.inf, -np.inf]], np.float32)
    ids, w = tq.tq4_1s_router_topk(torch.from_numpy(z).to(DEV), 3)
    ids_ref, w_ref = oracle.router_topk(z, 3)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.allclose(w.cpu().numpy(), w_ref, rtol=1e-6, atol=0)
    assert tq.tq4_1s_get_status() == 0
    # a NaN logit is never chosen and is reported
    zn = z.copy()
    zn[0, 1] = np.nan
    ids, _ = tq.tq4_1s_router_topk(torch.from_numpy(zn).to(DEV), 3)
    assert 1 not in ids.cpu().numpy()[0].tolist()
    assert tq.tq4_1s_get_status() & tq.TQ_DEV_NONFINITE


@pytest.mark.parametrize("E,H,I,m,topk,seeds", [
    (8, 256, 128, 4, 2, (90, 91, 92, 93)),
    (32, 512, 256, 16, 6, (94, 95, 96, 97)),
])
def test_moe_from_logits_matches_oracle(E, H, I, m, topk, seeds):
    up_seed, dn_seed, x_seed, r_seed = seeds
    up = synth.normal_f32((E, I, H), up_seed, 0.02)
    dn = synth.normal_f32((E, H, I), dn_seed, 0.02)
    z = synth.router_logits_f32(m, E, r_seed)
    x = synth.activations_bf16(m, H, x_seed)
    pu = tq.tq4_1s_quantize(torch.from_numpy(up).to(DEV), seed=up_seed)
    pd = tq.tq4_1s_quantize(torch.from_numpy(dn).to(DEV), seed=dn_seed)
    zd = torch.from_numpy(z).to(DEV)
    y = tq.tq4_1s_moe_logits(_bf16_dev(x), zd, topk, pu, pd)
    # the same layer with the router's decisions handed in: bit-identical
    ids_d, w_d = tq.tq4_1s_router_topk(zd, topk)
    y2 = tq.tq4_1s_moe(_bf16_dev(x), ids_d, w_d, pu, pd)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    ids, w = oracle.router_topk(z, topk)
    used = sorted(set(int(e) for e in ids.ravel()))
    uc = np.zeros((E, I, H // 2), np.uint8); us = np.zeros((E, I, H // 16), np.uint16)
    dc = np.zeros((E, H, I // 2), np.uint8); ds = np.zeros((E, H, I // 16), np.uint16)
    for e in used:
        uc[e], us[e], _ = oracle.quantize(up[e], up_seed)
        dc[e], ds[e], _ = oracle.quantize(dn[e], dn_seed)
    y_ref, _, bad = oracle.moe(x, ids, w, uc, us, up_seed, dc, ds, dn_seed)
    assert bad == 0
    assert_close(_bits(y), y_ref, f"moe from logits E={E}")
    assert tq.tq4_1s_get_status() == 0
