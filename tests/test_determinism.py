"""Run-to-run determinism of the CUDA path: bit-identical outputs over 100
repetitions, eager and replayed from a CUDA graph.

Every reduction in the kernels has a fixed order (the four dequant groups'
accumulators in group order; split-tile partials summed by the last
contributor in CTA order; the cluster split-K reduction in rank order; the
MoE's slots in slot order); the only atomics count arrivals and routing
buckets, which are integers.  So repeated calls must agree bit for bit, and a
race (a stage or partial read before it is complete) would show up as a
difference."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
REPS = 100


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


@pytest.mark.parametrize("m,n,k,seed", [
    (16, 4096, 4096, 2),      # decode shape: fused cluster split-K
    (48, 4096, 4096, 71),     # TMA-fed stream-K with split tiles
    (256, 1024, 2048, 72),    # large-m GEMM path
])
def test_linear_bit_identical_over_repeats(m, n, k, seed):
    p = tq.tq4_1s_quantize(synth.normal_f32_device((n, k), seed, 0.02, DEV), seed=seed)
    x = _bf16_dev(synth.activations_bf16(m, k, seed + 1))
    ws = torch.empty(tq.tq4_1s_linear_workspace(m, p), dtype=torch.uint8, device=DEV)
    ref = tq.tq4_1s_linear(x, p, workspace=ws).clone()
    outs = torch.empty((REPS, m, n), dtype=torch.bfloat16, device=DEV)
    for i in range(REPS):
        tq.tq4_1s_linear(x, p, out=outs[i], workspace=ws)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    same = (outs.view(torch.int16) == ref.view(torch.int16)).all(dim=2).all(dim=1)
    assert bool(same.all()), f"{int((~same).sum())} of {REPS} eager repeats differ"

    # the same call captured once and replayed
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    tq.tq4_1s_linear(x, p, out=y, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    with torch.cuda.graph(g, stream=s):
        tq.tq4_1s_linear(x, p, out=y, workspace=ws)
    bad = 0
    for _ in range(REPS):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        bad += int(not torch.equal(y.view(torch.int16), ref.view(torch.int16)))
    del g
    assert bad == 0, f"{bad} of {REPS} graph replays differ"
    assert tq.tq4_1s_get_status() == 0


def test_moe_bit_identical_over_repeats():
    wl = synth.WORKLOADS["moe_128x_top6"]
    E, H, I, m, topk = wl["num_experts"], wl["hidden"], wl["inter"], wl["m"], wl["topk"]
    up = tq.tq4_1s_quantize(synth.normal_f32_device((E, I, H), 81, 0.02, DEV), seed=81)
    dn = tq.tq4_1s_quantize(synth.normal_f32_device((E, H, I), 82, 0.02, DEV), seed=82)
    ids, w = synth.gumbel_topk_router(m, E, topk, 83)
    ids_d, w_d = torch.from_numpy(ids).to(DEV), torch.from_numpy(w).to(DEV)
    x = _bf16_dev(synth.activations_bf16(m, H, 84))
    ws = torch.empty(tq.tq4_1s_moe_workspace(m, topk, up, dn), dtype=torch.uint8, device=DEV)
    ref = tq.tq4_1s_moe(x, ids_d, w_d, up, dn, workspace=ws).clone()
    outs = torch.empty((REPS, m, H), dtype=torch.bfloat16, device=DEV)
    for i in range(REPS):
        tq.tq4_1s_moe(x, ids_d, w_d, up, dn, out=outs[i], workspace=ws)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    same = (outs.view(torch.int16) == ref.view(torch.int16)).all(dim=2).all(dim=1)
    assert bool(same.all()), f"{int((~same).sum())} of {REPS} MoE repeats differ"


def test_quantize_bit_identical_over_repeats():
    W = synth.normal_f32_device((1024, 2048), 85, 0.02, DEV)
    ref = tq.tq4_1s_quantize(W, seed=85)
    out = tq.tq4_1s_quantize(W, seed=85)
    for _ in range(REPS):
        tq.tq4_1s_quantize(W, seed=85, out=out)
        assert torch.equal(out.codes, ref.codes) and torch.equal(out.scales, ref.scales)
    assert tq.tq4_1s_get_status() == 0

