"""GPU checks of the decode-block kernel of tq4_1s_linear (m <= 32 tokens, one
launch per call, the CTAs of a row tile in a cluster): parity with the CPU
oracle on the shapes and splits it runs (odd cluster sizes, uneven k ranges,
ragged rows and k, two 16-token blocks), the static-weight flag (the weight
read before the dependency wait) giving the same bits, and a chain of calls
-- each consuming the previous call's output, as a layer stack does --
replayed from a CUDA graph giving the eager bits."""
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


@pytest.mark.parametrize("m,n,k,seed", [
    (16, 4096, 2688, 1002),   # dense hidden -> 4096 projection: 4-CTA clusters, 5 or 6 iterations each
    (16, 2688, 4096, 1003),   # dense 4096 -> hidden: 21 row tiles, 7-CTA clusters
    (16, 640, 768, 101),      # 6 k iterations: 6-CTA clusters, one iteration each
    (17, 512, 1024, 102),     # two 16-token blocks, the second with one token
    (31, 200, 384, 103),      # ragged rows and tokens
    (2, 128, 96, 104),        # one partial k iteration, no cluster
    (16, 1024, 2080, 105),    # ragged k (65 slices): a partial last iteration in the last CTA of a tile
])
def test_decode_parity(m, n, k, seed):
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    codes, scales, _ = oracle.quantize(W, seed)
    assert np.array_equal(p.codes[0].cpu().numpy(), codes)
    y_ref, _ = oracle.linear(x, codes, scales, seed)
    assert_close(_bits(y), y_ref, f"decode m={m} n={n} k={k}")
    assert tq.tq4_1s_get_status() == 0


def test_static_weight_flag_gives_the_same_bits():
    n, k, m = 4096, 4096, 16
    p = tq.tq4_1s_quantize(synth.normal_f32_device((n, k), 110, 0.02, DEV), seed=110)
    torch.cuda.synchronize()   # the contract of the flag: the planes' writer has finished
    ps = tq.Packed(p.codes, p.scales, n, k, 1, 110, flags=tq.TQ_WEIGHT_STATIC)
    x = _bf16_dev(synth.activations_bf16(m, k, 111))
    y0 = tq.tq4_1s_linear(x, p)
    y1 = tq.tq4_1s_linear(x, ps)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert tq.tq4_1s_get_status() == 0


@pytest.mark.parametrize("static", [False, True])
def test_chained_calls_in_a_graph_reproduce_eager(static):
    # 16 calls, call j reading call j-1's output, over 4 distinct weights:
    # the graph replays (dependent launches overlapping the previous call's
    # tail) must give the eager chain's bits, call by call
    n = k = 2048
    m, calls = 16, 16
    ws = []
    for i in range(4):
        p = tq.tq4_1s_quantize(synth.normal_f32_device((n, k), 120 + i, 0.02, DEV), seed=120 + i)
        ws.append(tq.Packed(p.codes, p.scales, n, k, 1, 120 + i, flags=tq.TQ_WEIGHT_STATIC if static else 0))
    torch.cuda.synchronize()
    x0 = _bf16_dev(synth.activations_bf16(m, k, 130))
    ys = torch.empty((calls, m, n), dtype=torch.bfloat16, device=DEV)

    def chain():
        x = x0
        for j in range(calls):
            tq.tq4_1s_linear(x, ws[j % 4], out=ys[j])
            x = ys[j]

    chain()
    torch.cuda.synchronize()
    ref = ys.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    with torch.cuda.graph(g, stream=s):
        chain()
    bad = 0
    for _ in range(10):
        ys.zero_()
        g.replay()
        torch.cuda.synchronize()
        bad += int(not torch.equal(ys.view(torch.int16), ref.view(torch.int16)))
    del g
    assert bad == 0, f"{bad} of 10 chained-graph replays differ from the eager chain"
    assert tq.tq4_1s_get_status() == 0
