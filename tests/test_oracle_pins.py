"""Pins that tie the CPU oracle to facts other than itself.

Each test checks one oracle function against a closed form, a textbook or
published value, a library routine used independently, or brute force, so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails here.  CPU only.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.stats import norm

import oracle
import synth


def test_hadamard_is_orthogonal_and_symmetric():
    # Closed form: the 32-point Sylvester Hadamard matrix satisfies H H^T = 32 I.
    H = oracle.hadamard32().astype(np.int64)
    assert np.array_equal(H @ H.T, 32 * np.eye(32, dtype=np.int64))
    assert np.array_equal(H, H.T)
    assert np.all(H[0] == 1) and np.all(H[:, 0] == 1)
    # Sylvester recursion H_2n = [[H_n, H_n], [H_n, -H_n]] in natural order.
    h = np.array([[1]])
    for _ in range(5):
        h = np.block([[h, h], [h, -h]])
    assert np.array_equal(H, h)


def test_fwht_matches_matrix_product():
    H = oracle.hadamard32().astype(np.float64)
    for i in range(32):   # unit vectors: exact columns of H
        e = np.zeros(32, np.float32); e[i] = 1.0
        assert np.array_equal(oracle.fwht32(e).astype(np.float64), H[:, i])
    a = synth.normal_f32(32, 11)
    ref = H @ a.astype(np.float64)
    got = oracle.fwht32(a).astype(np.float64)
    # five fp32 additions per output: |err| <= 5 * 2^-24 * sum|a| (generous)
    assert np.max(np.abs(got - ref)) <= 5 * 2.0 ** -24 * np.abs(a).sum() * 4


def test_rotate_block_applies_signs_then_hadamard():
    mask = 0b1011_0000_0000_0000_0000_0000_0000_0101
    H = oracle.hadamard32().astype(np.float64)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    w = synth.normal_f32(32, 12)
    ref = (H @ (s * w.astype(np.float64))) / np.sqrt(32.0)
    got = oracle.rotate_block(w, mask).astype(np.float64)
    assert np.max(np.abs(got - ref)) < 1e-5 * np.abs(w).max()


def test_codebook_is_lloyd_fixed_point():
    c, t, c32, t32 = oracle.codebook()
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    # centroid condition, with scipy's normal pdf/cdf (independent library)
    cent = (norm.pdf(edges[:-1]) - norm.pdf(edges[1:])) / (norm.cdf(edges[1:]) - norm.cdf(edges[:-1]))
    assert np.max(np.abs(cent - c)) < 1e-9
    # midpoint (nearest-neighbour) condition
    assert np.max(np.abs(t - 0.5 * (c[:-1] + c[1:]))) < 1e-15
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(c[::-1], -c) and t[7] == 0.0
    assert np.array_equal(c32, c.astype(np.float32)) and np.array_equal(t32, t.astype(np.float32))


def test_codebook_matches_max_1960_table(golden_dir):
    c, t, _, _ = oracle.codebook()
    outs, ths = {}, {}
    for line in open(os.path.join(golden_dir, "max1960_gaussian_16_levels.txt")):
        if line.startswith("#") or not line.strip():
            continue
        kind, idx, val = line.split()
        (outs if kind == "output" else ths)[int(idx)] = float(val)
    for i, v in outs.items():
        assert abs(c[7 + i] - v) <= 6e-4, (i, c[7 + i], v)
    for i, v in ths.items():
        assert abs((0.0 if i == 1 else t[6 + i]) - v) <= 6e-4, (i, v)


def test_codebook_distortion():
    # MSE of the 16-level Lloyd-Max quantizer of N(0,1) by numerical integration.
    c, t, _, _ = oracle.codebook()
    from scipy.integrate import quad
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    mse = sum(quad(lambda x, cj=cj: (x - cj) ** 2 * norm.pdf(x), a, b)[0]
              for cj, a, b in zip(c, edges[:-1], edges[1:]))
    assert 0.0094 < mse < 0.0096


def test_sign_mask_published_splitmix64(golden_dir):
    for line in open(os.path.join(golden_dir, "splitmix64_first_outputs.txt")):
        if line.startswith("#") or not line.strip():
            continue
        state, hx = line.split()
        assert oracle.splitmix64_first(int(state)) == int(hx, 16)
        assert oracle.sign_mask(int(state)) == int(hx, 16) & 0xFFFFFFFF


def test_f16_rounding_matches_numpy():
    g = synth.rng(21)
    vals = np.concatenate([
        (g.standard_normal(20000) * 10.0 ** g.uniform(-9, 4.8, 20000)).astype(np.float32),
        np.array([0.0, -0.0, 6.1035156e-05, 5.9604645e-08, 2.9802322e-08, 65504.0, 65519.0, 1e-3], np.float32),
    ])
    vals = vals[np.abs(vals) < 65520.0]   # numpy overflows to inf beyond; saturation is checked below
    for v in vals:
        assert oracle.f32_to_f16_sat(float(v)) == int(np.array(v, np.float32).astype(np.float16).view(np.uint16))
    # saturation instead of overflow to infinity
    for v, bits in [(65520.0, 0x7BFF), (1e6, 0x7BFF), (-np.inf, 0xFBFF), (np.inf, 0x7BFF)]:
        assert oracle.f32_to_f16_sat(v) == bits
    for h in [0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x8001, 0xBC00]:
        assert oracle.f16_to_f32(h) == float(np.array(h, np.uint16).view(np.float16))


def _bf16_brute(x: float) -> int:
    """Round x to bf16 by enumerating bf16 neighbours in exact rational arithmetic."""
    f = Fraction(x)
    sign = 0x8000 if x < 0 else 0
    f = abs(f)
    # bracket by the float32 neighbours: find bf16 values just below/above
    b = np.array(abs(x), np.float64).astype(np.float32).view(np.uint32) >> 16
    cands = [int(b) - 1, int(b), int(b) + 1, int(b) + 2]
    best = None
    for cb in cands:
        if cb < 0 or cb > 0x7F80:
            continue
        val = Fraction(float(np.array(cb << 16, np.uint32).view(np.float32)))
        d = abs(val - f)
        key = (d, cb & 1)
        if best is None or key < best[0]:
            best = (key, cb)
    return sign | best[1]


def test_bf16_rounding_from_double_brute_force():
    g = synth.rng(22)
    vals = list(g.standard_normal(3000) * 10.0 ** g.uniform(-30, 30, 3000))
    # exact ties between two bf16 values: must go to the even one
    vals += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -40]
    for v in vals:
        assert oracle.f64_to_bf16(float(v)) == _bf16_brute(float(v)), v


def test_threshold_search_equals_nearest_level():
    _, _, c32, t32 = oracle.codebook()
    u = synth.rng(23).standard_normal(1_000_000).astype(np.float32) * 1.3
    by_threshold = (u[:, None] > t32[None, :]).sum(axis=1)
    by_distance = np.argmin(np.abs(u[:, None].astype(np.float64) - c32[None, :].astype(np.float64)), axis=1)
    near = np.min(np.abs(u[:, None].astype(np.float64) - t32[None, :].astype(np.float64)), axis=1) < 1e-6
    assert np.all((by_threshold == by_distance) | near)
    assert near.sum() < 20


def _unpack(codes):
    lo = codes & 0xF
    hi = codes >> 4
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def test_quantize_brute_force_tiny():
    """Codes and scales against an independent formulation: explicit Hadamard
    matrix in fp64, numpy's fp16 rounding, argmin over the 16 levels."""
    c, t, c32, t32 = oracle.codebook()
    H = oracle.hadamard32().astype(np.float64)
    seed = 5
    mask = oracle.sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    W = np.concatenate([synth.normal_f32((6, 96), 31, 0.02), synth.student_t_f32((6, 96), 32, 5.0, 0.3)])
    codes, scales, bad = oracle.quantize(W, seed)
    assert bad == 0 and codes.shape == (12, 48) and scales.shape == (12, 6)
    q = _unpack(codes)
    boundary, midpoint = 0, 0
    for r in range(W.shape[0]):
        for kb in range(3):
            v = (H @ (s * W[r, 32 * kb:32 * kb + 32].astype(np.float64))) / np.sqrt(32.0)
            for h in range(2):
                vh = v[16 * h:16 * h + 16]
                rms = np.sqrt(np.mean(vh * vh))
                d16 = np.array(rms, np.float64).astype(np.float16)
                got_d = scales[r, 2 * kb + h]
                if got_d != int(d16.view(np.uint16)):
                    # only allowed within 1e-6 (relative) of an fp16 rounding midpoint
                    lo = float(np.array(got_d, np.uint16).view(np.float16))
                    ref = float(d16)
                    assert abs(rms - 0.5 * (lo + ref)) <= 1e-6 * rms
                    midpoint += 1
                    continue
                d = float(d16)
                u = vh / d
                want = np.argmin(np.abs(u[:, None] - c32[None, :].astype(np.float64)), axis=1)
                got = q[r, 32 * kb + 16 * h:32 * kb + 16 * h + 16]
                for i in range(16):
                    if got[i] != want[i]:
                        assert np.min(np.abs(u[i] - t)) < 1e-6
                        boundary += 1
    assert boundary + midpoint <= 2


def test_quantize_special_blocks():
    W = np.zeros((2, 64), np.float32)
    W[1, 32:] = synth.normal_f32(32, 41)
    W[1, 3] = np.nan
    codes, scales, bad = oracle.quantize(W, 0)
    assert bad == 1
    # all-zero block: both scales 0 and every code is 7
    assert np.all(scales[0] == 0) and np.all(codes[0] == 0x77)
    # a NaN spreads through the butterfly: scale is the fp16 NaN, codes 0
    assert np.all(scales[1, :2] == 0x7E00) and np.all(codes[1, :16] == 0)
    assert np.all(scales[1, 2:] != 0)


def test_levels_and_dequantize_closed_form():
    _, _, c32, _ = oracle.codebook()
    seed = 77
    mask = oracle.sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    H = oracle.hadamard32().astype(np.float64)
    g = synth.rng(42)
    codes = g.integers(0, 256, (5, 48), dtype=np.uint8)
    scales = np.array(g.uniform(0.001, 2.0, (5, 6)), np.float32).astype(np.float16).view(np.uint16)
    q = _unpack(codes)
    d = scales.view(np.float16).astype(np.float64)
    wn_ref = c32[q].astype(np.float64) * np.repeat(d, 16, axis=1)
    wn = oracle.levels(codes, scales)
    assert np.allclose(wn, wn_ref, rtol=2 ** -23, atol=0)
    W = oracle.dequantize(codes, scales, seed).astype(np.float64)
    for kb in range(3):
        blk = wn_ref[:, 32 * kb:32 * kb + 32]
        ref = (blk @ H.T) / np.sqrt(32.0) * s[None, :]
        assert np.max(np.abs(W[:, 32 * kb:32 * kb + 32] - ref)) < 1e-5 * np.abs(ref).max()
    # constant codes: H * (level * 1) = 32 * level * e_0, so only element 0 survives
    codes_c = np.full((1, 16), 0xFF, np.uint8)
    scales_c = np.array([[0x3C00, 0x3C00]], np.uint16)  # d = 1.0
    Wc = oracle.dequantize(codes_c, scales_c, seed)[0]
    expect0 = np.float32(np.float32(np.float32(32.0) * c32[15]) * np.float32(1 / np.sqrt(32.0)))
    assert Wc[0] == pytest.approx(s[0] * float(expect0), rel=1e-6)
    assert np.all(Wc[1:] == 0.0)


def test_bits_per_weight_is_five():
    codes_b, scales_b = oracle.packed_bytes(4096, 4096)
    assert codes_b + scales_b == 10_485_760           # "~10.5 MB" packed
    assert (codes_b + scales_b) * 8 / (4096 * 4096) == 5.0
    W = synth.normal_f32((4, 64), 1, 0.02)
    codes, scales, _ = oracle.quantize(W, 0)
    assert (codes.nbytes + scales.nbytes) * 8 / W.size == 5.0


@pytest.mark.parametrize("dist", ["normal", "student_t5", "laplace"])
def test_reconstruction_cosine(dist):
    if dist == "normal":
        W = synth.normal_f32((128, 1024), 51, 0.02)
    elif dist == "student_t5":
        W = synth.student_t_f32((128, 1024), 52, 5.0, 0.02)
    else:
        W = (synth.rng(53).laplace(0.0, 0.02, (128, 1024))).astype(np.float32)
    codes, scales, _ = oracle.quantize(W, 9)
    Wh = oracle.dequantize(codes, scales, 9).astype(np.float64)
    W = W.astype(np.float64)
    cos = (W * Wh).sum() / np.sqrt((W * W).sum() * (Wh * Wh).sum())
    assert cos >= 0.99


def test_rotation_equivalence_route_a_equals_route_b():
    """x * W_hat^T == (R x) * w_n^T per 32-slice, with R = r H diag(s) orthogonal."""
    seed = 13
    W = synth.normal_f32((8, 128), 61, 0.02)
    codes, scales, _ = oracle.quantize(W, seed)
    x = synth.activations_bf16(3, 128, 62)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    wn = oracle.levels(codes, scales).astype(np.float64)
    mask = oracle.sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    H = oracle.hadamard32().astype(np.float64)
    R = (H * s[None, :]) / np.sqrt(32.0)
    xr = np.concatenate([xf[:, 32 * b:32 * b + 32] @ R.T for b in range(4)], axis=1)
    route_b = xr @ wn.T
    # route A with the exactly inverse-rotated (fp64) weights
    What = np.concatenate([wn[:, 32 * b:32 * b + 32] @ R for b in range(4)], axis=1)
    route_a = xf @ What.T
    assert np.max(np.abs(route_a - route_b)) < 1e-12 * np.abs(route_a).max()
    # and the oracle's linear (fp32 inverse rotation) agrees to fp32 accuracy
    y, _ = oracle.linear(x, codes, scales, seed)
    assert np.max(np.abs(y - route_b)) < 1e-5 * np.abs(route_b).max()


def test_linear_matches_library_matmul_and_rounding():
    W = synth.normal_f32((40, 96), 71, 0.02)
    codes, scales, _ = oracle.quantize(W, 3)
    x = synth.activations_bf16(5, 96, 72)
    Wh = oracle.dequantize(codes, scales, 3)
    y, yb = oracle.linear(x, codes, scales, 3)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ Wh.astype(np.float64).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    flat = y.ravel()
    for i in range(0, flat.size, 7):
        assert yb.ravel()[i] == _bf16_brute(float(flat[i]))


def test_moe_route_brute_force():
    ids, _ = synth.gumbel_topk_router(16, 128, 6, 7)
    offsets, pairs, bad = oracle.moe_route(ids, 128)
    assert bad == 0
    flat = ids.ravel()
    want = sorted(range(flat.size), key=lambda p: (flat[p], p))
    assert list(pairs) == want
    counts = np.bincount(flat, minlength=128)
    assert np.array_equal(np.diff(offsets), counts)
    ids2 = ids.copy(); ids2[3, 2] = 128; ids2[5, 0] = -1
    offsets2, pairs2, bad2 = oracle.moe_route(ids2, 128)
    assert bad2 == 2 and len(pairs2) == flat.size - 2 and 3 * 6 + 2 not in pairs2


def test_router_weights_are_normalised():
    ids, w = synth.gumbel_topk_router(16, 128, 6, 7)
    assert ids.shape == (16, 6) and np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert all(len(set(r)) == 6 for r in ids)


def test_router_topk_invariants_on_gumbel_logits():
    # Selection: distinct ids in descending logit order, every chosen logit at
    # least every unchosen one; weights positive, descending, summing to 1.
    z = synth.router_logits_f32(64, 128, 7)
    ids, w = oracle.router_topk(z, 6)
    assert ids.shape == (64, 6) and w.dtype == np.float32
    for t in range(64):
        sel = z[t, ids[t]]
        assert len(set(ids[t].tolist())) == 6
        assert np.all(np.diff(sel) <= 0)
        rest = np.delete(z[t], ids[t])
        assert sel.min() >= rest.max()
        assert np.all(w[t] > 0) and np.all(np.diff(w[t]) <= 0)
        assert abs(float(w[t].astype(np.float64).sum()) - 1.0) < 1e-6
    # the Gumbel-perturbed selection of the input generator chooses the same
    # experts from the unrounded logits (no fp32 near-ties in this draw)
    ids_g, w_g = synth.gumbel_topk_router(64, 128, 6, 7)
    assert np.array_equal(ids, ids_g)
    assert np.allclose(w, w_g, rtol=1e-6, atol=0)


def test_router_topk_special_cases():
    # equal logits: the lowest ids in order, weights exactly 1/k
    ids, w = oracle.router_topk(np.zeros((3, 16), np.float32), 4)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (3, 1)))
    assert np.all(w == np.float32(0.25))
    # ties inside the selection: equal logits ranked by id
    z = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, -3.0]], np.float32)
    ids, w = oracle.router_topk(z, 4)
    assert ids.tolist() == [[1, 3, 2, 4]]
    assert w[0, 0] == w[0, 1] and w[0, 2] == w[0, 3]
    # one choice: weight exactly 1
    ids, w = oracle.router_topk(synth.router_logits_f32(5, 32, 3), 1)
    assert np.all(w == 1.0)
    # k = E: the full softmax (scipy, independent of the oracle's loop)
    from scipy.special import softmax
    z = synth.router_logits_f32(4, 24, 9)
    ids, w = oracle.router_topk(z, 24)
    ref = softmax(z.astype(np.float64), axis=1)
    for t in range(4):
        assert np.array_equal(ids[t], np.argsort(-z[t], kind="stable"))
        assert np.allclose(w[t], ref[t, ids[t]], rtol=2e-7, atol=0)


def test_moe_composes_linear_relu2_and_slot_sum():
    E, H, I, m, topk = 4, 64, 96, 5, 2
    up = synth.normal_f32((E, I, H), 81, 0.05)
    dn = synth.normal_f32((E, H, I), 82, 0.05)
    uq = [oracle.quantize(up[e], 4)[:2] for e in range(E)]
    dq = [oracle.quantize(dn[e], 5)[:2] for e in range(E)]
    uc = np.stack([a for a, _ in uq]); us = np.stack([b for _, b in uq])
    dc = np.stack([a for a, _ in dq]); ds = np.stack([b for _, b in dq])
    ids, w = synth.gumbel_topk_router(m, E, topk, 83)
    ids[1, 1] = E + 3  # out of range: skipped
    x = synth.activations_bf16(m, H, 84)
    y, yb, bad = oracle.moe(x, ids, w, uc, us, 4, dc, ds, 5)
    assert bad == 1
    ref = np.zeros((m, H))
    for t in range(m):
        for j in range(topk):
            e = ids[t, j]
            if not 0 <= e < E:
                continue
            u = oracle.linear_f64(x[t:t + 1], oracle.dequantize(uc[e], us[e], 4))
            h = oracle.round_bf16(np.maximum(u, 0.0) ** 2)
            z = oracle.linear_f64(h, oracle.dequantize(dc[e], ds[e], 5))
            ref[t] += float(w[t, j]) * z[0]
    assert np.array_equal(y, ref)
    assert np.array_equal(yb, oracle.round_bf16(ref))


# ----------------------------------------------------------- boundary-near count
def _rotate_inverse_f64(v, seed):
    """w with R w = v for one 32-block (R = r H diag(s), exact inverse in fp64)."""
    mask = oracle.sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    H = oracle.hadamard32().astype(np.float64)
    r = float(np.float32(1.0 / np.sqrt(32.0)))
    return s * (H @ np.asarray(v, np.float64)) / (32.0 * r)


def test_boundary_near_explains_every_fp32_fp64_code_difference():
    # codes taken in fp64 from the definition (explicit H, exact division)
    # against the stored scale may differ from the oracle's fp32 codes only
    # where the count flags a decision within 1e-6 of a threshold
    W = synth.student_t_f32((512, 1024), 91, 5.0, 0.02)
    codes, scales, _ = oracle.quantize(W, 91)
    near = oracle.boundary_near(W, 91, scales)
    mask = oracle.sign_mask(91)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
    H = oracle.hadamard32().astype(np.float64)
    r = float(np.float32(1.0 / np.sqrt(32.0)))
    v = ((W.astype(np.float64).reshape(-1, 32) * s) @ H.T * r).reshape(-1, 16)
    d = scales.reshape(-1).view(np.float16).astype(np.float64)
    _, _, _, t32 = oracle.codebook()
    u = v / d[:, None]
    ideal = (u[:, :, None] > t32.astype(np.float64)[None, None, :]).sum(axis=2).reshape(W.shape)
    diff = ideal != oracle.unpack_codes(codes)
    assert not np.any(diff & ~near["code_mask"])
    assert near["codes"] < 1e-4 * W.size
    # the mask marks the right elements: scaling u by (1 + 1e-4) moves a code
    # only where u was within |t_j| * 1e-4 <= 2.5e-4 of threshold t_j, so every
    # moved code lies inside the mask taken at tol = 3e-4 (and some do move)
    wide = oracle.boundary_near(W, 91, scales, tol=3e-4)
    moved = ((u * (1 + 1e-4))[:, :, None] > t32.astype(np.float64)[None, None, :]).sum(axis=2).reshape(W.shape)
    moved = moved != ideal
    assert moved.sum() >= 10
    assert not np.any(moved & ~wide["code_mask"])
    assert wide["codes"] < 20 * moved.sum()


def test_boundary_near_flags_a_value_on_a_threshold_and_a_scale_on_a_midpoint():
    seed = 5
    _, _, _, t32 = oracle.codebook()
    D = 1.5   # an fp16 value: the stored scale of the first half
    tj = float(t32[11])
    a = D * np.sqrt((16.0 - tj * tj) / 15.0)
    v = np.empty(32)
    v[0] = tj * D                       # u = t_11 exactly
    v[1:16] = a                         # half-block RMS exactly D
    M = 1.0 + 2.0 ** -11                # midpoint of fp16 1.0 and 1 + 2^-10
    v[16:32] = M                        # second half: RMS exactly on a midpoint
    W = _rotate_inverse_f64(v, seed).astype(np.float32).reshape(1, 32)
    codes, scales, _ = oracle.quantize(W, seed)
    assert scales[0, 0] == np.float16(D).view(np.uint16)
    near = oracle.boundary_near(W, seed, scales)
    assert near["code_mask"][0, 0] and near["codes"] == 1
    assert near["scale_mask"][0, 1] and not near["scale_mask"][0, 0] and near["scales"] == 1
    # nudged off the boundaries, nothing is flagged
    v[0] = float(t32[11] + t32[12]) / 2 * D
    v[1:16] = D * np.sqrt((16.0 - (v[0] / D) ** 2) / 15.0)
    v[16:32] = 1.0 + 2.0 ** -12
    W = _rotate_inverse_f64(v, seed).astype(np.float32).reshape(1, 32)
    near = oracle.boundary_near(W, seed)
    assert near["codes"] == 0 and near["scales"] == 0


# ----------------------------------------------------------------- fp8 cache
def test_e4m3_format_values_and_round_trips():
    # OCP E4M3: largest finite 448 (0x7E), smallest subnormal 2^-9 (0x01),
    # smallest normal 2^-6 (0x08), 0x7F is NaN; every finite code decodes and
    # re-encodes to itself
    assert oracle.e4m3_to_f64(0x7E) == 448.0 and oracle.e4m3_to_f64(0xFE) == -448.0
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9 and oracle.e4m3_to_f64(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_f64(0x38) == 1.0 and oracle.e4m3_to_f64(0x3F) == 1.875
    assert np.isnan(oracle.e4m3_to_f64(0x7F))
    for b in range(256):
        if b & 0x7F == 0x7F:
            continue
        v = oracle.e4m3_to_f64(b)
        assert oracle.f32_to_e4m3(v) == b
    # saturation and ties to even (1 + 1/16 lies between 1 and 1.125: even is 1)
    assert oracle.f32_to_e4m3(1e6) == 0x7E and oracle.f32_to_e4m3(-500.0) == 0xFE
    assert oracle.f32_to_e4m3(1.0625) == 0x38 and oracle.f32_to_e4m3(1.1875) == 0x3A
    assert oracle.f32_to_e4m3(2.0 ** -10) == 0x00 and oracle.f32_to_e4m3(3 * 2.0 ** -10) == 0x02


def test_e4m3_rounding_matches_torch_float8():
    import torch
    x = np.concatenate([synth.normal_f32(20000, 150, 3.0), synth.normal_f32(5000, 151, 0.01),
                        np.float32([0.0, 447.0, -447.9, 2.0 ** -9, 5 * 2.0 ** -11])]).astype(np.float32)
    mine = np.array([oracle.f32_to_e4m3(v) for v in x], np.uint8)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_fp8_cache_conversion_bounds():
    W = synth.student_t_f32((40, 256), 152, 5.0, 0.02)
    W[7] = 0.0
    codes, scales, _ = oracle.quantize(W, 152)
    q, s = oracle.to_fp8(codes, scales, 152)
    Wh = oracle.dequantize(codes, scales, 152).astype(np.float64)
    Wc = oracle.fp8_dequantize(q, s)
    amax = np.abs(Wh).max(axis=1)
    # the row scale maps the row's largest |w| to 448 exactly once rounded
    assert np.array_equal(s, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    assert s[7] == 0.0 and np.all(q[7] == 0)
    nz = [i for i in range(40) if i != 7]
    assert all(np.any((q[i] & 0x7F) == 0x7E) for i in nz)
    # E4M3 keeps 3 mantissa bits: relative error at most 2^-4 above the
    # subnormal range, absolute error at most 2^-10 s below it
    err = np.abs(Wc - Wh)
    bound = np.maximum(np.abs(Wh) * 2.0 ** -4, s[:, None].astype(np.float64) * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    # cosine of the cached weight against the TQ4_1S reconstruction
    for i in nz:
        c = Wh[i] @ Wc[i] / np.linalg.norm(Wh[i]) / np.linalg.norm(Wc[i])
        assert c > 0.998


def test_fp8_linear_matches_numpy_matmul():
    W = synth.normal_f32((24, 96), 153, 0.02)
    codes, scales, _ = oracle.quantize(W, 153)
    q, s = oracle.to_fp8(codes, scales, 153)
    x = synth.activations_bf16(5, 96, 154)
    y, yb = oracle.linear_fp8(x, q, s)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ oracle.fp8_dequantize(q, s).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------- affine (MLX-style) format
def _unpack_bits(codes, bits):
    # an independent reading of the little-endian bit stream (numpy's unpackbits)
    b = np.unpackbits(codes, axis=1, bitorder="little")
    n, nbits = b.shape
    b = b.reshape(n, nbits // bits, bits).astype(np.uint32)
    return (b << np.arange(bits, dtype=np.uint32)).sum(axis=2)


def _bf16(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, np.uint16)).astype(np.float64)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_affine_codes_are_nearest_grid_points(bits):
    W = synth.student_t_f32((16, 256), 170 + bits, 5.0, 0.02)
    codes, scales, biases = oracle.affine_quantize(W, bits)
    q = _unpack_bits(codes, bits)
    sc = np.repeat(_bf16(scales), 64, axis=1)
    bi = np.repeat(_bf16(biases), 64, axis=1)
    qmax = 2 ** bits - 1
    grid = sc[..., None] * np.arange(qmax + 1)[None, None, :] + bi[..., None]
    dist = np.abs(grid - W[..., None].astype(np.float64))
    best = dist.argmin(axis=2)
    d_sel = np.take_along_axis(dist, q[..., None].astype(np.int64), axis=2)[..., 0]
    # the chosen point is a nearest one (up to fp32 rounding of the quotient)
    assert np.all(d_sel <= dist.min(axis=2) + 1e-6 * sc)
    assert np.mean(q == best) > 0.999
    # scale = (max - min) / (2^b - 1) and bias = min, rounded to bf16
    g = W.reshape(16, 4, 64).astype(np.float32)
    lo, hi = g.min(axis=2), g.max(axis=2)
    assert np.array_equal(scales, synth.f32_to_bf16_bits((hi - lo) / np.float32(qmax)))
    assert np.array_equal(biases, synth.f32_to_bf16_bits(lo))
    # the dequantized weight is the chosen grid point, and within half a step
    Wd = oracle.affine_dequantize(codes, scales, biases, bits).astype(np.float64)
    assert np.allclose(Wd, sc * q + bi, rtol=1e-6, atol=1e-9)
    # (bf16 rounding of the bias shifts the grid, of the scale stretches it:
    # the extremes of a group may lie that much beyond the grid's ends)
    slack = np.abs(bi - np.repeat(lo.astype(np.float64), 64, axis=1))
    slack += qmax * np.abs(sc - np.repeat(((hi - lo) / np.float32(qmax)).astype(np.float64), 64, axis=1))
    assert np.all(np.abs(Wd - W) <= 0.5 * sc + slack + 1e-7)


def test_affine_exact_grid_constant_group_and_packing():
    bits = 6
    rng = np.random.default_rng(175)
    q = rng.integers(0, 64, size=(3, 128))
    q[:, 0], q[:, 1] = 0, 63          # each group spans the full range
    q[:, 64], q[:, 65] = 0, 63
    sc, bi = np.float32(2.0 ** -9), np.float32(-0.0625)
    W = (bi + sc * q).astype(np.float32)
    W[2, 64:] = np.float32(0.3)       # a constant group: zero scale, codes 0
    codes, scales, biases = oracle.affine_quantize(W, bits)
    got = _unpack_bits(codes, bits)
    assert np.array_equal(got[:2], q[:2]) and np.array_equal(got[2, :64], q[2, :64])
    assert np.all(got[2, 64:] == 0) and _bf16(scales)[2, 1] == 0.0
    Wd = oracle.affine_dequantize(codes, scales, biases, bits)
    assert np.array_equal(Wd[:2], W[:2]) and np.array_equal(Wd[2, :64], W[2, :64])
    assert np.all(Wd[2, 64:] == _bf16(synth.f32_to_bf16_bits(np.float32([0.3])))[0])
    # 4 and 8 bits: the stream is plain nibbles (even element low) and bytes
    c4, _, _ = oracle.affine_quantize(W, 4)
    assert np.array_equal(_unpack_bits(c4, 4)[:, 0::2], (c4 & 0xF)) and np.array_equal(_unpack_bits(c4, 4)[:, 1::2], c4 >> 4)
    c8, _, _ = oracle.affine_quantize(W, 8)
    assert np.array_equal(_unpack_bits(c8, 8), c8)
