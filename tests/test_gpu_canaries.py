"""Output canaries: every path of the linear layer and the MoE writes its
output inside a buffer with guard rows before and after it (a fixed 16-bit
pattern), and the guards must come back untouched.  A kernel that wrote a row
or column past its output would change them.  This stands in for a bounds
checker, which this environment does not provide; the outputs are also
checked against the oracle, so a write that landed inside the output in the
wrong place shows up there."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
GUARD = 0x5A5A
GUARD_ROWS = 3


def _guarded(rows, cols):
    """(whole buffer, the output view in its middle) as int16; the view's
    first byte stays 16-byte aligned when cols * 2 is a multiple of 16."""
    buf = torch.full((rows + 2 * GUARD_ROWS, cols), GUARD, dtype=torch.int16, device=DEV)
    return buf, buf[GUARD_ROWS:GUARD_ROWS + rows]


def _guards_intact(buf, rows):
    head = buf[:GUARD_ROWS]
    tail = buf[GUARD_ROWS + rows:]
    return bool((head == GUARD).all()) and bool((tail == GUARD).all())


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


@pytest.mark.parametrize("m,n,k,seed,path", [
    (16, 4096, 4096, 70, "decode kernel, 4-CTA clusters"),
    (5, 200, 96, 71, "decode kernel, ragged rows, columns and k"),
    (32, 384, 512, 72, "decode kernel, two 16-token blocks"),
    (48, 256, 544, 73, "TMA-fed stream-K, ragged k"),
    (100, 640, 384, 74, "TMA-fed stream-K, four segments"),
    (16, 19072, 256, 75, "fused stream-K past one wave"),
    (200, 520, 224, 76, "large m: dequantize + GEMM, ragged"),
])
def test_linear_writes_only_its_output(m, n, k, seed, path):
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    buf, y = _guarded(m, n)
    tq.tq4_1s_linear(_bf16_dev(x), p, out=y.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert _guards_intact(buf, m), path
    assert tq.tq4_1s_get_status() == 0
    codes, scales, _ = oracle.quantize(W, seed)
    y_ref, _ = oracle.linear(x, codes, scales, seed)
    assert_close(y.cpu().numpy().view(np.uint16), y_ref, path)


def test_moe_writes_only_its_output():
    E, H, I, m, topk = 8, 256, 128, 12, 2
    up = synth.normal_f32((E, I, H), 77, 0.02)
    dn = synth.normal_f32((E, H, I), 78, 0.02)
    ids, w = synth.gumbel_topk_router(m, E, topk, 79)
    x = synth.f32_to_bf16_bits(synth.normal_f32((m, H), 80, 1.0))
    pu = tq.tq4_1s_quantize(torch.from_numpy(up).to(DEV), seed=77)
    pd = tq.tq4_1s_quantize(torch.from_numpy(dn).to(DEV), seed=78)
    buf, y = _guarded(m, H)
    tq.tq4_1s_moe(_bf16_dev(x), torch.from_numpy(ids).to(DEV), torch.from_numpy(w).to(DEV), pu, pd,
                  out=y.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert _guards_intact(buf, m)
    assert tq.tq4_1s_get_status() == 0
    uc = np.zeros((E, I, H // 2), np.uint8)
    us = np.zeros((E, I, H // 16), np.uint16)
    dc = np.zeros((E, H, I // 2), np.uint8)
    ds = np.zeros((E, H, I // 16), np.uint16)
    for e in sorted(set(int(v) for v in ids.ravel())):
        uc[e], us[e], _ = oracle.quantize(up[e], 77)
        dc[e], ds[e], _ = oracle.quantize(dn[e], 78)
    y_ref, _, _ = oracle.moe(x, ids, w, uc, us, 77, dc, ds, 78)
    assert_close(y.cpu().numpy().view(np.uint16), y_ref, "moe")
