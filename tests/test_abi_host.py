"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol the header declares, and its host-only logic (sizes, sign mask,
codebook, argument validation) behaves as documented.  No GPU compute."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import bit_rotated_weight_b200 as tq
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq4_1s.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq4_1s_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = tq.load_library()
    names = declared_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {tq.LIB_PATH}").read()
    exported = set(re.findall(r" T (tq4_1s_\w+)", out))
    assert exported == set(names), exported ^ set(names)


def test_version_and_error_strings():
    assert tq.tq4_1s_version() == 102
    for code in range(0, 9):
        s = tq.tq4_1s_error_string(code)
        assert s and s != "unknown error code"
    assert tq.tq4_1s_error_string(99) == "unknown error code"


def test_packed_bytes_is_five_bits_per_weight():
    c, s = tq.tq4_1s_packed_bytes(4096, 4096)
    assert (c, s) == (8_388_608, 2_097_152) and c + s == 10_485_760
    c, s = tq.tq4_1s_packed_bytes(1856, 2688, 128)
    assert (c + s) * 8 == 5 * 128 * 1856 * 2688
    with pytest.raises(tq.TQ4Error):
        tq.tq4_1s_packed_bytes(4096, 4016)   # k % 32 != 0


def test_sign_mask_matches_oracle_and_published_value():
    assert tq.tq4_1s_sign_mask(0) == 0x7B1DCDAF
    for seed in [1, 2, 3, 1000, 2 ** 63 + 5, 2 ** 64 - 1]:
        assert tq.tq4_1s_sign_mask(seed) == oracle.sign_mask(seed)


def test_library_codebook_equals_oracle_codebook():
    # two independent Lloyd iterations (positive half vs full) agree in fp32
    lv, th = tq.tq4_1s_codebook()
    _, _, c32, t32 = oracle.codebook()
    assert np.array_equal(lv.numpy().view(np.uint32), c32.view(np.uint32))
    assert np.array_equal(th.numpy().view(np.uint32), t32.view(np.uint32))


def _weight(n=64, k=64, e=1, codes=16, scales=16):
    return tq._Weight(n, k, e, 0, 0, codes, scales)


def test_validation_rejects_before_any_launch():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    good = ctypes.c_void_p(4096)
    w = _weight(k=48)                                          # k % 32 != 0
    assert lib.tq4_1s_linear(good, 16, ctypes.byref(w), good, good, 1 << 20, null) == 1
    w = _weight(codes=0)                                       # null codes
    assert lib.tq4_1s_linear(good, 16, ctypes.byref(w), good, good, 1 << 20, null) == 1
    w = _weight(codes=4104)                                    # misaligned codes
    assert lib.tq4_1s_linear(good, 16, ctypes.byref(w), good, good, 1 << 20, null) == 2
    w = _weight()
    assert lib.tq4_1s_linear(good, -1, ctypes.byref(w), good, good, 1 << 20, null) == 1
    assert lib.tq4_1s_linear(good, 0, ctypes.byref(w), good, good, 0, null) == 0     # m == 0: no-op
    assert lib.tq4_1s_linear(null, 16, ctypes.byref(w), good, good, 1 << 20, null) == 1
    assert lib.tq4_1s_linear(ctypes.c_void_p(4100), 16, ctypes.byref(w), good, good, 1 << 20, null) == 2
    w2 = _weight(e=2)                                          # linear wants a dense weight
    assert lib.tq4_1s_linear(good, 16, ctypes.byref(w2), good, good, 1 << 20, null) == 1
    assert lib.tq4_1s_quantize(good, 7, ctypes.byref(w), null) == 1          # bad dtype
    assert lib.tq4_1s_quantize(null, 0, ctypes.byref(w), null) == 1
    assert lib.tq4_1s_dequantize(ctypes.byref(w), null, null) == 1
    assert lib.tq4_1s_get_status(null, None) == 1
    up, dn = _weight(n=128, k=64, e=4), _weight(n=64, k=96, e=4)            # up.n != down.k
    assert lib.tq4_1s_moe(good, 4, good, good, 2, ctypes.byref(up), ctypes.byref(dn), good, good, 1 << 20,
                          null) == 1
    assert lib.tq4_1s_moe_workspace(4, 2, ctypes.byref(up), ctypes.byref(dn)) == 0
    assert lib.tq4_1s_moe_route(good, 4, 0, 8, good, good, null) == 1


def test_static_entry_validation_and_scratch_limits():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    good = ctypes.c_void_p(4096)
    assert lib.tq4_1s_linear_static(good, 16, None, good, null) == 1                # no weight
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(k=48)), good, null) == 1
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(e=2)), good, null) == 1
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(codes=0)), good, null) == 1
    # the fixed scratch bounds: m <= 32, k <= 8192, n <= 32768 (TQ_ERR_SCRATCH_LIMIT)
    assert lib.tq4_1s_linear_static(good, 33, ctypes.byref(_weight()), good, null) == 9
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(k=8224)), good, null) == 9
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(n=32769)), good, null) == 9
    assert lib.tq4_1s_linear_static(good, 0, ctypes.byref(_weight()), good, null) == 0   # m == 0: no-op
    assert lib.tq4_1s_linear_static(null, 16, ctypes.byref(_weight()), good, null) == 1
    assert lib.tq4_1s_linear_static(ctypes.c_void_p(4100), 16, ctypes.byref(_weight()), good, null) == 2
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(_weight(scales=24)), good, null) == 2
    assert tq.tq4_1s_error_string(9).startswith("shape exceeds the fixed scratch")


def test_fp8_cache_validation():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    good = ctypes.c_void_p(4096)
    assert lib.tq4_1s_to_fp8(ctypes.byref(_weight()), null, good, null) == 1
    assert lib.tq4_1s_to_fp8(ctypes.byref(_weight()), ctypes.c_void_p(4104), good, null) == 2
    assert lib.tq4_1s_to_fp8(ctypes.byref(_weight(k=48)), good, good, null) == 1
    assert lib.tq4_1s_linear_fp8_workspace(16, 4096, 4096) == 4096 * 4096 * 2
    assert lib.tq4_1s_linear_fp8_workspace(16, 4096, 4016) == 0            # k % 32 != 0
    assert lib.tq4_1s_linear_fp8(good, 0, good, good, 64, 64, 0, good, null, 0, null) == 0   # m == 0
    assert lib.tq4_1s_linear_fp8(good, 16, good, good, 64, 48, 0, good, null, 0, null) == 1
    assert lib.tq4_1s_linear_fp8(good, 16, good, good, 64, 64, 2, good, null, 0, null) == 1  # unknown flag
    assert lib.tq4_1s_linear_fp8(null, 16, good, good, 64, 64, 0, good, null, 0, null) == 1
    assert lib.tq4_1s_linear_fp8(good, 16, ctypes.c_void_p(4097), good, 64, 64, 0, good, null, 0, null) == 2


def test_affine_validation():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    good = ctypes.c_void_p(4096)

    def aw(n=64, k=128, bits=6, codes=16, scales=16, biases=16):
        return tq._AffineWeight(n, k, bits, 0, codes, scales, biases)

    assert lib.tq4_1s_affine_quantize(good, ctypes.byref(aw(bits=5)), null) == 1      # bits not 4/6/8
    assert lib.tq4_1s_affine_quantize(good, ctypes.byref(aw(k=96)), null) == 1        # k % 64 != 0
    assert lib.tq4_1s_affine_quantize(null, ctypes.byref(aw()), null) == 1
    assert lib.tq4_1s_affine_quantize(good, ctypes.byref(aw(biases=0)), null) == 1
    assert lib.tq4_1s_affine_quantize(good, ctypes.byref(aw(scales=24)), null) == 2
    assert lib.tq4_1s_affine_linear_workspace(16, ctypes.byref(aw(n=4096, k=4096))) == 4096 * 4096 * 2
    assert lib.tq4_1s_affine_linear(good, 0, ctypes.byref(aw()), good, null, 0, null) == 0        # m == 0


def test_debug_hooks_validation():
    lib = tq.load_library()
    assert lib.tq4_1s_debug_hook(99, 0) == 1                       # unknown hook
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, -1) == 1
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, 0) == 0
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_WITHHOLD_ARRIVAL, 2) == 1
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_WITHHOLD_ARRIVAL, 0) == 0
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_WAIT_NS, -5) == 1
    if not torch.cuda.is_available():
        assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_WAIT_NS, 1000) == 3     # needs a device
    # an armed failure is not consumed by calls that fail validation first
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, 1) == 0
    null = ctypes.c_void_p(0)
    assert lib.tq4_1s_linear(null, 16, ctypes.byref(_weight()), null, null, 0, null) == 1
    assert lib.tq4_1s_debug_hook(tq.TQ_HOOK_FAIL_NEXT_CALLS, 0) == 0


def test_router_and_moe_logits_validation():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    good = ctypes.c_void_p(4096)
    assert lib.tq4_1s_router_topk(good, 0, 128, 6, good, good, null) == 0      # m == 0: no-op
    assert lib.tq4_1s_router_topk(good, -1, 128, 6, good, good, null) == 1
    assert lib.tq4_1s_router_topk(good, 4, 1025, 6, good, good, null) == 1     # more than 1024 experts
    assert lib.tq4_1s_router_topk(good, 4, 128, 33, good, good, null) == 1     # topk > 32
    assert lib.tq4_1s_router_topk(good, 4, 4, 5, good, good, null) == 1        # topk > E
    assert lib.tq4_1s_router_topk(null, 4, 128, 6, good, good, null) == 1
    assert lib.tq4_1s_router_topk(good, 4, 128, 6, good, null, null) == 1
    up, dn = _weight(n=128, k=64, e=4), _weight(n=64, k=128, e=4)
    assert lib.tq4_1s_moe_logits(good, 4, null, 2, ctypes.byref(up), ctypes.byref(dn), good, good, 1 << 20,
                                 null) == 1                                    # no logits
    assert lib.tq4_1s_moe_logits(good, 4, good, 5, ctypes.byref(up), ctypes.byref(dn), good, good, 1 << 20,
                                 null) == 1                                    # topk > E
    assert lib.tq4_1s_moe_logits(good, 4, ctypes.c_void_p(4100), 2, ctypes.byref(up), ctypes.byref(dn), good,
                                 good, 1 << 20, null) == 2                     # misaligned logits
    big_u, big_d = _weight(n=128, k=64, e=1025), _weight(n=64, k=128, e=1025)
    assert lib.tq4_1s_moe_logits(good, 4, good, 2, ctypes.byref(big_u), ctypes.byref(big_d), good, good,
                                 1 << 20, null) == 1                           # router limit: 1024 experts
    assert lib.tq4_1s_moe_logits(good, 0, good, 2, ctypes.byref(up), ctypes.byref(dn), good, good, 0,
                                 null) == 0                                    # m == 0: no-op


def test_quantize_batched_validation():
    lib = tq.load_library()
    null = ctypes.c_void_p(0)
    ws = (tq._Weight * 2)(_weight(), _weight())
    ptrs = (ctypes.c_void_p * 2)(4096, 8192)
    cw, cp = ctypes.cast(ws, ctypes.c_void_p), ctypes.cast(ptrs, ctypes.c_void_p)
    assert lib.tq4_1s_quantize_batched(cp, 0, cw, 0, null) == 0           # count 0: no-op
    assert lib.tq4_1s_quantize_batched(cp, 0, cw, -1, null) == 1
    assert lib.tq4_1s_quantize_batched(null, 0, cw, 2, null) == 1         # no pointer array
    assert lib.tq4_1s_quantize_batched(cp, 0, null, 2, null) == 1         # no descriptors
    assert lib.tq4_1s_quantize_batched(cp, 5, cw, 2, null) == 1           # bad dtype
    bad = (tq._Weight * 2)(_weight(), _weight(k=48))                       # second one invalid
    assert lib.tq4_1s_quantize_batched(cp, 0, ctypes.cast(bad, ctypes.c_void_p), 2, null) == 1
    mis = (ctypes.c_void_p * 2)(4096, 8200)                                # second W misaligned
    assert lib.tq4_1s_quantize_batched(ctypes.cast(mis, ctypes.c_void_p), 0, cw, 2, null) == 2
    nul = (ctypes.c_void_p * 2)(4096, 0)
    assert lib.tq4_1s_quantize_batched(ctypes.cast(nul, ctypes.c_void_p), 0, cw, 2, null) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_fails_loudly():
    lib = tq.load_library()
    good = ctypes.c_void_p(4096)
    w = _weight()
    need = lib.tq4_1s_linear_workspace(16, ctypes.byref(w))
    assert need > 0
    assert lib.tq4_1s_linear(good, 16, ctypes.byref(w), good, good, need, ctypes.c_void_p(0)) == 3
    assert lib.tq4_1s_quantize(good, 0, ctypes.byref(w), ctypes.c_void_p(0)) == 3
    ws1, p1 = (tq._Weight * 1)(w), (ctypes.c_void_p * 1)(4096)
    assert lib.tq4_1s_quantize_batched(ctypes.cast(p1, ctypes.c_void_p), 0, ctypes.cast(ws1, ctypes.c_void_p), 1,
                                       ctypes.c_void_p(0)) == 3
    assert lib.tq4_1s_linear_static(good, 16, ctypes.byref(w), good, ctypes.c_void_p(0)) == 3


def test_workspace_queries():
    lib = tq.load_library()
    w = _weight(n=4096, k=4096)
    small = lib.tq4_1s_linear_workspace(16, ctypes.byref(w))
    large = lib.tq4_1s_linear_workspace(8192, ctypes.byref(w))
    assert 0 < small < large and large >= 4096 * 4096 * 2
    assert lib.tq4_1s_linear_workspace(0, ctypes.byref(w)) == 0
    up, dn = _weight(n=1856, k=2688, e=128), _weight(n=2688, k=1856, e=128)
    assert lib.tq4_1s_moe_workspace(16, 6, ctypes.byref(up), ctypes.byref(dn)) > 0


def test_missing_library_raises(tmp_path):
    import importlib
    with pytest.raises(ImportError):
        tq._lib_saved = tq._lib
        tq._lib = None
        try:
            tq.load_library(str(tmp_path / "nope.so"))
        finally:
            tq._lib = tq._lib_saved


def test_bucket_threshold_search_counts_like_the_full_search():
    # The quantize kernel, on finite half blocks of a symmetric codebook, takes
    # a code from |u|'s bucket (bits >> 19 = exponent and top 4 mantissa bits,
    # 2^-5 .. 2^3 in 128 buckets, one bucket below and one above): the number
    # of positive thresholds below the bucket, plus the one inside it if
    # |u| passes it, compared as float bits (> for u > 0, >= for u <= 0).
    # Built here as the kernel builds it from the library's fp32 thresholds,
    # and checked against the strict count t < u on every float of every
    # bucket that holds a threshold, both signs, and at both ends of the others.
    _, th = tq.tq4_1s_codebook()
    t = th.numpy().astype(np.float32)
    p = t[8:15]
    q0, nb = 122 << 4, 130

    def bucket_of_bits(bits):
        q = (bits >> 19).astype(np.int64) - (q0 - 1)
        return np.clip(q, 0, nb - 1)

    pb = p.view(np.uint32)
    assert len(set(bucket_of_bits(pb).tolist())) == 7          # one threshold per bucket at most
    inside = np.full(nb, 0x7F800000, np.uint64)
    below = np.zeros(nb, np.int64)
    for i in range(nb):
        lo = 0.0 if i == 0 else np.array([(q0 + i - 1) << 19], np.uint32).view(np.float32)[0]
        hi = np.inf if i == nb - 1 else np.array([(q0 + i) << 19], np.uint32).view(np.float32)[0]
        for pj in p:
            if pj < lo:
                below[i] += 1
            elif pj < hi:
                inside[i] = int(np.array([pj], np.float32).view(np.uint32)[0])

    def bucket_code(u):
        pos = u > 0
        ab = u.view(np.uint32) & np.uint32(0x7FFFFFFF)
        q = bucket_of_bits(ab)
        c = below[q] + ((ab.astype(np.uint64) + np.where(pos, 0, 1).astype(np.uint64)) > inside[q]).astype(np.int64)
        return np.where(pos, 8 + c, 7 - c)

    def full_code(u):
        return (t[None, :] < u[:, None]).sum(axis=1)

    for pj in pb:
        b = int(pj >> 19)
        bits = np.arange(b << 19, (b + 1) << 19, dtype=np.uint64).astype(np.uint32)
        for sgn in (0, 0x80000000):
            u = (bits | np.uint32(sgn)).view(np.float32)
            for chunk in range(0, len(u), 1 << 16):
                uu = u[chunk:chunk + (1 << 16)]
                assert np.array_equal(bucket_code(uu), full_code(uu))
    ends = []
    for i in range(nb):
        for bits in ((q0 + i - 1) << 19, ((q0 + i) << 19) - 1):
            if 0 < bits < 0x7F800000:
                ends.append(bits)
    ends += [0, 1, 0x00800000, 0x3D000000 - 1, 0x3D000000, 0x41000000 - 1, 0x41000000, 0x7F7FFFFF]
    e = np.array(ends, np.uint32)
    u = np.concatenate([e, e | np.uint32(0x80000000)]).view(np.float32)
    assert np.array_equal(bucket_code(u), full_code(u))
