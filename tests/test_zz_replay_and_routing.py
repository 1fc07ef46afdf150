"""Later GPU checks of the MoE path: CUDA-graph replays over changing inputs,
and tokens that name one expert in several slots.  (Kept in their own file,
run after the core parity tests.)"""
import numpy as np
import pytest
import torch

import synth
from tests._parity import assert_close
from tests.test_gpu_parity import _bits, _moe_case

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


@pytest.mark.parametrize("m", [16, 20])
def test_moe_repeated_expert_ids_in_a_token(m):
    # a token that names the same expert in several slots (a top-k router
    # never does, but the call accepts it): every slot contributes, and an
    # expert's rows (here 3 per token, up to 60) are split into segments no
    # wider than the accumulators
    ids = np.tile(np.array([3, 3, 5, 3, 5, 1], np.int32), (m, 1))
    y, y_ref, bad = _moe_case(8, 256, 128, m, 6, (50, 51, 52, 53), ids=ids)
    assert bad == 0
    assert_close(_bits(y), y_ref, f"moe repeated ids m={m}")
    assert tq.tq4_1s_get_status() == 0


def test_moe_graph_replays_follow_their_inputs():
    # a captured MoE call replayed over three different activation blocks
    # must reproduce each block's eager result: a split tile left unfinished
    # by a replay would leave the previous block's intermediate values behind
    E, H, I, m, topk = 32, 512, 256, 16, 6
    up = tq.tq4_1s_quantize(synth.normal_f32_device((E, I, H), 86, 0.02, DEV), seed=86)
    dn = tq.tq4_1s_quantize(synth.normal_f32_device((E, H, I), 87, 0.02, DEV), seed=87)
    ids, w = synth.gumbel_topk_router(m, E, topk, 88)
    ids_d, w_d = torch.from_numpy(ids).to(DEV), torch.from_numpy(w).to(DEV)
    xs = [_bf16_dev(synth.activations_bf16(m, H, 89 + i)) for i in range(3)]
    ws = torch.empty(tq.tq4_1s_moe_workspace(m, topk, up, dn), dtype=torch.uint8, device=DEV)
    refs = [tq.tq4_1s_moe(x, ids_d, w_d, up, dn, workspace=ws).clone() for x in xs]
    x_in = xs[0].clone()
    y = torch.empty((m, H), dtype=torch.bfloat16, device=DEV)
    tq.tq4_1s_moe(x_in, ids_d, w_d, up, dn, out=y, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    with torch.cuda.graph(g, stream=s):
        tq.tq4_1s_moe(x_in, ids_d, w_d, up, dn, out=y, workspace=ws)
    bad = 0
    for r in range(30):
        i = r % 3
        x_in.copy_(xs[i])
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        bad += int(not torch.equal(y.view(torch.int16), refs[i].view(torch.int16)))
    del g
    assert bad == 0, f"{bad} of 30 MoE graph replays differ from their eager results"
    assert tq.tq4_1s_get_status() == 0
