"""Failure handling on the GPU, made without faulting it.

Host-injected failures (the library's test hook makes the next launching call
fail before it launches, as a failed launch would), a workspace that is too
small, and a bounded device wait that runs out: a test hook shortens the
wait limit to 2 ms and makes one rotation warp of the decode kernel withhold
its arrival, so the MMA issuers' and the epilogue's waits run out; the kernel
must report TQ_DEV_TIMEOUT, wind down (copies landed, MMAs finished, tensor
memory freed) and leave the context usable.  Kept in a file that runs after
the parity tests."""
import time

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
def _restore_hooks():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, 0)
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_WITHHOLD_ARRIVAL, 0)
    if torch.cuda.is_available():
        tq.tq4_1s_debug_hook(tq.TQ_HOOK_WAIT_NS, 0)


def _case(m=16, n=512, k=1024, seed=140):
    W = synth.normal_f32((n, k), seed, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    codes, scales, _ = oracle.quantize(W, seed)
    y_ref, _ = oracle.linear(x, codes, scales, seed)
    return p, x, y_ref


def test_injected_launch_failure_returns_cuda_error_without_launching():
    p, x, y_ref = _case()
    xd = _bf16_dev(x)
    torch.cuda.synchronize()
    for call in (lambda: tq.tq4_1s_linear(xd, p),
                 lambda: tq.tq4_1s_quantize(torch.zeros((64, 64), device=DEV), seed=1),
                 lambda: tq.tq4_1s_router_topk(torch.zeros((4, 32), device=DEV), 2)):
        tq.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, 1)
        n0 = tq.tq4_1s_launch_count()
        with pytest.raises(tq.TQ4Error) as e:
            call()
        assert e.value.code == 5                                  # TQ_ERR_CUDA
        assert tq.tq4_1s_launch_count() == n0                      # nothing was launched
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    y = tq.tq4_1s_linear(xd, p)                                    # the hook is spent: a normal call
    torch.cuda.synchronize()
    assert_close(_bits(y), y_ref, "after injected failures")


def test_workspace_too_small_is_refused_without_launching():
    p, x, _ = _case(m=48)          # the TMA-fed path needs a workspace
    xd = _bf16_dev(x)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    n0 = tq.tq4_1s_launch_count()
    with pytest.raises(tq.TQ4Error) as e:
        tq.tq4_1s_linear(xd, p, workspace=small)
    assert e.value.code == 4                                      # TQ_ERR_WORKSPACE
    E, H, I = 4, 256, 128
    up = tq.tq4_1s_quantize(synth.normal_f32_device((E, I, H), 141, 0.02, DEV), seed=141)
    dn = tq.tq4_1s_quantize(synth.normal_f32_device((E, H, I), 142, 0.02, DEV), seed=142)
    ids, w = synth.gumbel_topk_router(3, E, 2, 143)
    n0 = tq.tq4_1s_launch_count()
    with pytest.raises(tq.TQ4Error) as e:
        tq.tq4_1s_moe(_bf16_dev(synth.activations_bf16(3, H, 144)), torch.from_numpy(ids).to(DEV),
                      torch.from_numpy(w).to(DEV), up, dn, workspace=small)
    assert e.value.code == 4 and tq.tq4_1s_launch_count() == n0


@pytest.mark.parametrize("n,k", [(256, 256), (4096, 4096)])
def test_device_wait_runs_out_and_kernel_winds_down(n, k):
    p, x, y_ref = _case(n=n, k=k, seed=145)
    xd = _bf16_dev(x)
    torch.cuda.synchronize()
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_WAIT_NS, 2_000_000)            # 2 ms
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_WITHHOLD_ARRIVAL, 1)
    t0 = time.perf_counter()
    tq.tq4_1s_linear(xd, p)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_WITHHOLD_ARRIVAL, 0)
    tq.tq4_1s_debug_hook(tq.TQ_HOOK_WAIT_NS, 0)
    assert tq.tq4_1s_get_status() & tq.TQ_DEV_TIMEOUT
    assert elapsed < 1.0, f"the timed-out call took {elapsed:.3f} s"
    # the context is still usable and the kernel gives the right answer again
    y = tq.tq4_1s_linear(xd, p)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    assert_close(_bits(y), y_ref, "after a timed-out call")
