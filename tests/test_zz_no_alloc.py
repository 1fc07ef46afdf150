"""tq4_1s_linear_static -- the linear layer for callers that cannot allocate.

Plugin hosts and serving runtimes that fix their device memory at start-up
cannot hand tq4_1s_linear a workspace; tq4_1s_linear_static keeps its scratch
in a fixed array inside the library instead.  This test calls it through the
C ABI twice in a row (the second call runs on the scratch the first one left
behind) and checks each result against the CPU oracle and against
tq4_1s_linear, which uses a caller workspace, with the same tolerances as the
parity tests.  It lives in a file of its own that pytest collects last.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _to_dev(bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def test_static_scratch_linear_matches_workspace_linear():
    dev = torch.device("cuda:0")
    lib = tq.load_library()
    fn = lib.tq4_1s_linear_static
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(tq._Weight), ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    Wh = synth.student_t_f32((4096, 4096), 2, 5.0, 0.02)
    p = tq.tq4_1s_quantize(torch.from_numpy(Wh).to(dev), seed=2)
    codes, scales, _ = oracle.quantize(Wh, 2)
    wst = p.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for call, (m, seed) in enumerate([(16, 3), (13, 5)]):
        xh = synth.activations_bf16(m, 4096, seed)
        x = _to_dev(xh, dev)
        ref = tq.tq4_1s_linear(x, p)
        y = torch.empty((m, 4096), dtype=torch.bfloat16, device=dev)
        rc = fn(ctypes.c_void_p(x.data_ptr()), m, ctypes.byref(wst), ctypes.c_void_p(y.data_ptr()), stream)
        assert rc == 0, tq.tq4_1s_error_string(rc)
        torch.cuda.synchronize()
        y_ref, _ = oracle.linear(xh, codes, scales, 2)
        assert_close(_bits(y), y_ref, f"static call {call} vs oracle")
        ref_f = _bits(ref).astype(np.uint32) << 16
        assert_close(_bits(y), ref_f.view(np.float32).astype(np.float64), f"static call {call}")
    assert tq.tq4_1s_get_status() == 0
    # shapes beyond the fixed scratch are refused without a launch
    big = tq.Packed(p.codes, p.scales, 4096, 4096, 1, 2)
    x40 = torch.zeros((40, 4096), dtype=torch.bfloat16, device=dev)
    y40 = torch.empty((40, 4096), dtype=torch.bfloat16, device=dev)
    bst = big.c_struct()
    assert fn(ctypes.c_void_p(x40.data_ptr()), 40, ctypes.byref(bst), ctypes.c_void_p(y40.data_ptr()), stream) == 9


@pytest.mark.parametrize("m,n,k,seed", [
    (32, 8192, 8192, 60),   # too long per CTA for the fused modes: rotation kernel + TMA-fed stream-K
    (7, 4096, 128, 61),     # one k iteration: fused stream-K without a cluster
])
def test_static_scratch_other_modes(m, n, k, seed):
    dev = torch.device("cuda:0")
    lib = tq.load_library()
    fn = lib.tq4_1s_linear_static
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(tq._Weight), ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    Wh = synth.normal_f32((n, k), seed, 0.02)
    p = tq.tq4_1s_quantize(torch.from_numpy(Wh).to(dev), seed=seed)
    wst = p.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    xh = synth.activations_bf16(m, k, seed + 1)
    x = _to_dev(xh, dev)
    ref = tq.tq4_1s_linear(x, p)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    rc = fn(ctypes.c_void_p(x.data_ptr()), m, ctypes.byref(wst), ctypes.c_void_p(y.data_ptr()), stream)
    assert rc == 0, tq.tq4_1s_error_string(rc)
    torch.cuda.synchronize()
    codes, scales, _ = oracle.quantize(Wh, seed)
    y_ref, _ = oracle.linear(xh, codes, scales, seed)
    assert_close(_bits(y), y_ref, f"static m={m} n={n} k={k} vs oracle")
    ref_f = _bits(ref).astype(np.uint32) << 16
    assert_close(_bits(y), ref_f.view(np.float32).astype(np.float64), f"static m={m} n={n} k={k}")
    assert tq.tq4_1s_get_status() == 0


def _static_fn():
    lib = tq.load_library()
    fn = lib.tq4_1s_linear_static
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(tq._Weight), ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def test_static_scratch_takes_no_memory_and_replays_in_a_graph():
    # After one warm-up call (which may load the library's device code and
    # with it the fixed array), further calls change neither the device's
    # free memory nor torch's allocations; a captured call replayed over
    # changing inputs reproduces each input's eager result.
    dev = torch.device("cuda:0")
    fn = _static_fn()
    n, k, m = 2048, 2048, 16
    p = tq.tq4_1s_quantize(synth.normal_f32_device((n, k), 62, 0.02, dev), seed=62)
    wst = p.c_struct()
    xs = [_to_dev(synth.activations_bf16(m, k, 63 + i), dev) for i in range(3)]
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)

    def call(x, st=stream):
        assert fn(ctypes.c_void_p(x.data_ptr()), m, ctypes.byref(wst), ctypes.c_void_p(y.data_ptr()), st) == 0

    refs = torch.empty((3, m, n), dtype=torch.bfloat16, device=dev)
    call(xs[0])
    torch.cuda.synchronize()
    # (the collector is paused over the measured calls: objects of earlier
    # tests freed or finalised meanwhile would move torch's counters)
    gc.collect()
    gc.disable()
    try:
        free0, alloc0 = torch.cuda.mem_get_info(dev)[0], torch.cuda.memory_allocated(dev)
        for i, x in enumerate(xs):
            call(x)
            torch.cuda.synchronize()
            refs[i].copy_(y)
        free1, alloc1 = torch.cuda.mem_get_info(dev)[0], torch.cuda.memory_allocated(dev)
    finally:
        gc.enable()
    assert free1 == free0 and alloc1 == alloc0
    x_in = xs[0].clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    with torch.cuda.graph(g, stream=s):
        call(x_in, ctypes.c_void_p(s.cuda_stream))
    bad = 0
    for r in range(9):
        x_in.copy_(xs[r % 3])
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        bad += int(not torch.equal(y.view(torch.int16), refs[r % 3].view(torch.int16)))
    del g
    assert bad == 0
    assert tq.tq4_1s_get_status() == 0


def test_static_scratch_at_its_limits():
    # m = 32, k = 8192, n = 32768 (the last tile counter): sampled output
    # columns against the oracle, and guard rows around y left untouched
    dev = torch.device("cuda:0")
    fn = _static_fn()
    m, n, k, seed = 32, 32768, 8192, 64
    W = synth.normal_f32_device((n, k), seed, 0.02, dev)
    p = tq.tq4_1s_quantize(W, seed=seed)
    xh = synth.activations_bf16(m, k, seed + 1)
    x = _to_dev(xh, dev)
    guard = 0x5A5A
    buf = torch.full((m + 2, n), guard, dtype=torch.int16, device=dev)
    y = buf[1:m + 1].view(torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    wst = p.c_struct()
    for _ in range(2):
        assert fn(ctypes.c_void_p(x.data_ptr()), m, ctypes.byref(wst), ctypes.c_void_p(y.data_ptr()), stream) == 0
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    assert bool((buf[0] == guard).all()) and bool((buf[m + 1] == guard).all())
    rows = np.array(sorted(set([0, 1, 127, 128, n - 129, n - 1] + list(range(5, n, 997)))))
    Ws = W[torch.from_numpy(rows).to(dev)].cpu().numpy()
    codes, scales, _ = oracle.quantize(Ws, seed)
    y_ref, _ = oracle.linear(xh, codes, scales, seed)
    assert_close(_bits(y)[:, rows], y_ref, "static at its limits, sampled columns")
