"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Packing, unpacking and routing are compared bit for bit;
GEMM outputs against the stated max/mean relative tolerances."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import assert_close, errors

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("bit_rotated_weight_b200")
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _quantize_both(W, seed):
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=seed)
    torch.cuda.synchronize()
    codes, scales, bad = oracle.quantize(W.reshape(-1, W.shape[-1]), seed)
    return p, codes.reshape(p.codes.shape), scales.reshape(p.scales.shape), bad


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        tq.tq4_1s_get_status()
    yield


# ----------------------------------------------------------------- quantize
@pytest.mark.parametrize("shape,seed,dist", [
    ((256, 256), 0, "normal"),             # tiny single linear
    ((200, 96), 11, "student_t"),          # ragged rows, 3 blocks per row
    ((1, 32), 12, "normal"),               # one block
    ((4096, 4096), 2, "student_t"),        # dense decode-block weight
    ((4, 64, 160), 13, "normal"),          # expert stack
])
def test_quantize_bit_exact(shape, seed, dist):
    W = (synth.normal_f32(shape, seed, 0.02) if dist == "normal"
         else synth.student_t_f32(shape, seed, 5.0, 0.02))
    p, codes, scales, _ = _quantize_both(W, seed)
    g_codes = p.codes.cpu().numpy()
    g_scales = p.scales.cpu().numpy().view(np.uint16)
    # both sides take every decision in fp32 with the same operation order,
    # so codes and scales match bit for bit; the decisions within 1e-6 of a
    # threshold or of an fp16 rounding midpoint are counted and reported
    k = W.shape[-1]
    near = oracle.boundary_near(W.reshape(-1, k), seed, scales.reshape(-1, k // 16))
    n_code = int((oracle.unpack_codes(g_codes.reshape(-1, k // 2)) != oracle.unpack_codes(codes.reshape(-1, k // 2))).sum())
    n_scale = int((g_scales != scales).sum())
    print(f"quantize {shape}: {n_code} codes, {n_scale} scales differ; within 1e-6 of a boundary: "
          f"{near['codes']} codes, {near['scales']} scales")
    assert np.array_equal(g_codes, codes)
    assert np.array_equal(g_scales, scales)
    assert tq.tq4_1s_get_status() == 0


def test_quantize_bf16_input_bit_exact():
    Wb = synth.f32_to_bf16_bits(synth.normal_f32((128, 256), 21, 0.05))
    Wf = synth.bf16_bits_to_f32(Wb)
    p = tq.tq4_1s_quantize(_bf16_dev(Wb), seed=21)
    codes, scales, _ = oracle.quantize(Wf, 21)
    assert np.array_equal(p.codes[0].cpu().numpy(), codes)
    assert np.array_equal(p.scales[0].cpu().numpy().view(np.uint16), scales)


def test_quantize_batched_bit_exact_against_oracle():
    # tensors of different shapes, seeds and block counts (one not a multiple
    # of 32 blocks, so a warp chunk ends inside it) quantized in one launch
    shapes = [(200, 96), (1, 32), (3, 64, 160), (257, 128), (64, 4096)]
    Ws = [synth.normal_f32(s, 50 + i, 0.02) for i, s in enumerate(shapes)]
    seeds = [50 + i for i in range(len(shapes))]
    outs = tq.tq4_1s_quantize_batched([torch.from_numpy(W).to(DEV) for W in Ws], seeds)
    torch.cuda.synchronize()
    for W, seed, p in zip(Ws, seeds, outs):
        codes, scales, _ = oracle.quantize(W.reshape(-1, W.shape[-1]), seed)
        assert np.array_equal(p.codes.cpu().numpy().reshape(codes.shape), codes)
        assert np.array_equal(p.scales.cpu().numpy().view(np.uint16).reshape(scales.shape), scales)
    # bf16 inputs, batched
    Wb = [synth.f32_to_bf16_bits(synth.normal_f32((96, 192), 60 + i, 0.05)) for i in range(3)]
    outs = tq.tq4_1s_quantize_batched([_bf16_dev(b) for b in Wb], [60, 61, 62])
    for b, seed, p in zip(Wb, [60, 61, 62], outs):
        codes, scales, _ = oracle.quantize(synth.bf16_bits_to_f32(b), seed)
        assert np.array_equal(p.codes[0].cpu().numpy(), codes)
        assert np.array_equal(p.scales[0].cpu().numpy().view(np.uint16), scales)
    assert tq.tq4_1s_get_status() == 0


def test_quantize_special_blocks_and_status():
    W = np.zeros((3, 64), np.float32)
    W[1, 32:] = synth.normal_f32(32, 41)
    W[2, 3] = np.nan
    W[2, 40] = np.inf
    p, codes, scales, bad = _quantize_both(W, 0)
    assert bad == 2
    assert np.array_equal(p.codes.cpu().numpy(), codes)
    assert np.array_equal(p.scales.cpu().numpy().view(np.uint16), scales)
    assert tq.tq4_1s_get_status() & tq.TQ_DEV_NONFINITE
    assert tq.tq4_1s_get_status() == 0     # read clears


# ----------------------------------------------------------------- dequantize
@pytest.mark.parametrize("shape,seed", [((256, 256), 0), ((77, 320), 5), ((3, 64, 96), 6)])
def test_dequantize_bit_exact(shape, seed):
    W = synth.student_t_f32(shape, seed, 5.0, 0.02)
    p, codes, scales, _ = _quantize_both(W, seed)
    Wg = tq.tq4_1s_dequantize(p).cpu().numpy()
    Wo = oracle.dequantize(codes.reshape(-1, codes.shape[-1]), scales.reshape(-1, scales.shape[-1]), seed)
    assert np.array_equal(Wg.reshape(Wo.shape).view(np.uint32), Wo.view(np.uint32))


# ----------------------------------------------------------------- linear
LINEAR_CASES = [
    # (m, n, k, seed)  -- small-m stream-K path
    (16, 256, 256, 0),      # tiny single linear: split tiles on a 4-CTA grid
    (1, 128, 128, 30),
    (5, 200, 96, 31),       # ragged rows and a ragged k tail (96 = 0.75 of a 128 k step)
    (16, 1000, 544, 32),
    (32, 384, 512, 33),     # two 16-row boxes per operand
    (33, 256, 256, 34),     # two segments, the second with one row
    (100, 640, 384, 35),    # four segments
    (16, 4096, 4096, 2),    # dense decode-block linear, full size
    (16, 256, 8192, 36),    # wide k: four rotation warps per activation row
    (8, 128, 16416, 37),    # wider k: eight rotation warps, lanes with 2-3 slices
    # large-m path (dequantize + GEMM)
    (129, 256, 256, 40),
    (300, 520, 224, 41),    # ragged m, n, k
    (512, 1024, 512, 42),
]


@pytest.mark.parametrize("m,n,k,seed", LINEAR_CASES)
def test_linear_parity(m, n, k, seed):
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.activations_bf16(m, k, seed + 1)
    p, codes, scales, _ = _quantize_both(W, seed)
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
    assert_close(_bits(y), y_ref, f"linear m={m} n={n} k={k}")
    assert tq.tq4_1s_get_status() == 0


@pytest.mark.parametrize("m,n,k,seed", [
    (16, 512, 1024, 43),    # fused cluster split-K
    (48, 512, 1024, 44),    # TMA-fed stream-K (two segments)
    (200, 512, 1024, 45),   # large-m GEMM
])
def test_linear_degenerate_rows_and_blocks(m, n, k, seed):
    # the method's degenerate inputs: all-zero weight rows and 32-blocks
    # (scale 0, codes 7), a zero half-block, and all-zero activation rows;
    # zero rows of x give exactly zero output rows, zero rows of W exactly
    # zero output columns, the rest matches the oracle
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    W[[0, 7, n - 1]] = 0.0
    W[3, 64:96] = 0.0
    W[5, 128:144] = 0.0
    x = synth.activations_bf16(m, k, seed + 1)
    zero_rows = [0, m // 2, m - 1]
    x[zero_rows] = 0
    p, codes, scales, _ = _quantize_both(W, seed)
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    yf = y.float().cpu().numpy()
    assert np.all(yf[zero_rows] == 0.0)
    assert np.all(yf[:, [0, 7, n - 1]] == 0.0)
    y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
    assert_close(_bits(y), y_ref, f"linear degenerate m={m}")


def test_moe_zero_token_rows():
    y, y_ref, _ = _moe_case(8, 256, 128, 12, 2, (46, 47, 48, 49), zero_rows=(0, 5, 11))
    yf = y.float().cpu().numpy()
    assert np.all(yf[[0, 5, 11]] == 0.0)
    assert_close(_bits(y), y_ref, "moe zero rows")
    assert tq.tq4_1s_get_status() == 0


@pytest.mark.parametrize("x_std", [3000.0, 1e-5])
def test_linear_activation_range(x_std):
    # activations far outside (and far inside) the fp16 range: the per-row
    # power-of-two scaling of the rotated activations keeps full precision
    m, n, k, seed = 16, 384, 512, 38
    W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
    x = synth.f32_to_bf16_bits(synth.student_t_f32((m, k), seed + 1, 5.0, x_std))
    p, codes, scales, _ = _quantize_both(W, seed)
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    assert np.all(np.isfinite(y.float().cpu().numpy()))
    y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
    assert_close(_bits(y), y_ref, f"linear range x_std={x_std}")
    assert tq.tq4_1s_get_status() == 0


def test_linear_any_finite_scale_decode_path():
    # half-block scales far above ~93.6 (one row x 20000) and far below 2e-6
    # (one row x 1e-5, fp16 subnormal scales): the decode kernel scales each
    # dequant group's levels by a per-row power of two, so every output,
    # those rows' columns included, matches the oracle and nothing is flagged
    m, n, k, seed = 16, 256, 256, 39
    W = synth.normal_f32((n, k), seed, 0.02)
    W[3] *= 20000.0
    W[9] *= 1e-5
    x = synth.activations_bf16(m, k, seed + 1)
    p, codes, scales, _ = _quantize_both(W, seed)
    assert scales[0][3].view(np.float16).astype(np.float32).max() > 94.0
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
    yb = _bits(y)
    keep = np.array([c for c in range(n) if c not in (3, 9)])
    assert_close(yb[:, keep], y_ref[:, keep], "decode: ordinary rows")
    assert_close(yb[:, [3]], y_ref[:, [3]], "decode: scales above the fp16 level range")
    assert_close(yb[:, [9]], y_ref[:, [9]], "decode: subnormal scales")


@pytest.mark.parametrize("m,n,k,seed", [
    (48, 256, 256, 39),      # TMA-fed stream-K (two segments)
    (48, 256, 544, 46),      # ragged k: rows of scales not 16-byte aligned
    (16, 19072, 256, 47),    # 149 row tiles: past the decode kernel's one wave (fused
                             # stream-K: x' only in the CTA's shared memory)
])
def test_linear_any_finite_scale_stream_k(m, n, k, seed):
    # scales far above ~93.6 (one row x 20000) overflow the stream-K
    # kernel's fp16 levels; the row's sums come out non-finite and the
    # epilogue recomputes them exactly, so every column matches the oracle
    # and nothing is flagged; scales far below 2e-6 (one row x 1e-5) give
    # fp16-subnormal levels, still within the tolerance
    W = synth.normal_f32((n, k), seed, 0.02)
    W[3] *= 20000.0
    W[9] *= 1e-5
    x = synth.activations_bf16(m, k, seed + 1)
    p, codes, scales, _ = _quantize_both(W, seed)
    assert scales[0][3].view(np.float16).astype(np.float32).max() > 94.0
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    assert tq.tq4_1s_get_status() == 0
    y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
    yb = _bits(y)
    keep = np.array([c for c in range(n) if c not in (3, 9)])
    assert_close(yb[:, keep], y_ref[:, keep], "stream-K: ordinary rows")
    assert_close(yb[:, [3]], y_ref[:, [3]], "stream-K: scales above the unscaled fp16 level range")
    assert_close(yb[:, [9]], y_ref[:, [9]], "stream-K: subnormal scales")


def test_linear_shared_workspace_across_shapes_and_paths():
    # one workspace reused by small-m calls of different shapes (different
    # tile counts and activation sizes) stays valid: each call clears its own
    # counters; a large-m call in between uses the binding's large-m workspace
    cases = [(16, 256, 256, 50), (16, 4096, 1024, 51), (300, 520, 224, 52), (8, 1000, 544, 53), (16, 256, 256, 50)]
    ws = None
    for m, n, k, seed in cases:
        W = synth.student_t_f32((n, k), seed, 5.0, 0.02)
        x = synth.activations_bf16(m, k, seed + 1)
        p, codes, scales, _ = _quantize_both(W, seed)
        if m <= 128:
            need = tq.tq4_1s_linear_workspace(m, p)
            if ws is None or ws.numel() < need:
                ws = torch.full((max(need, 4 << 20),), 0x5A, dtype=torch.uint8, device=DEV)   # not zeroed
            y = tq.tq4_1s_linear(_bf16_dev(x), p, workspace=ws)
        else:
            y = tq.tq4_1s_linear(_bf16_dev(x), p)
        torch.cuda.synchronize()
        y_ref, _ = oracle.linear(x, codes[0], scales[0], seed)
        assert_close(_bits(y), y_ref, f"shared workspace m={m} n={n} k={k}")


def test_linear_deterministic_repeats():
    W = synth.student_t_f32((4096, 4096), 2, 5.0, 0.02)
    x = synth.activations_bf16(16, 4096, 3)
    p = tq.tq4_1s_quantize(torch.from_numpy(W).to(DEV), seed=2)
    xd = _bf16_dev(x)
    first = _bits(tq.tq4_1s_linear(xd, p))
    for _ in range(20):
        assert np.array_equal(_bits(tq.tq4_1s_linear(xd, p)), first)


def test_linear_prefill_8192_sampled_rows():
    """M=8192 x K=4096 against W 14336 x 4096: sampled output rows vs oracle."""
    m, n, k, seed = 8192, 14336, 4096, 8
    W = synth.normal_f32((n, k), seed, 0.02)
    x = synth.activations_bf16(m, k, 9)
    p, codes, scales, _ = _quantize_both(W, seed)
    y = tq.tq4_1s_linear(_bf16_dev(x), p)
    torch.cuda.synchronize()
    rows = np.sort(synth.rng(99).choice(m, 12, replace=False))
    rows = np.concatenate([rows, [0, m - 1]])
    Wh = oracle.dequantize(codes[0], scales[0], seed)
    y_ref = oracle.linear_f64(x[rows], Wh)
    assert_close(_bits(y)[rows], y_ref, "prefill sampled rows")


# ----------------------------------------------------------------- MoE
def test_moe_route_bit_exact():
    for m, E, topk, seed in [(16, 128, 6, 7), (512, 128, 6, 77), (3, 8, 2, 78)]:
        ids, _ = synth.gumbel_topk_router(m, E, topk, seed)
        off, pairs = tq.tq4_1s_moe_route(torch.from_numpy(ids).to(DEV), E)
        o_off, o_pairs, _ = oracle.moe_route(ids, E)
        assert np.array_equal(off.cpu().numpy(), o_off)
        assert np.array_equal(pairs.cpu().numpy()[: len(o_pairs)], o_pairs)


def test_moe_route_bad_ids_flagged():
    ids, _ = synth.gumbel_topk_router(8, 16, 2, 5)
    ids[2, 1] = 16
    ids[5, 0] = -3
    off, pairs = tq.tq4_1s_moe_route(torch.from_numpy(ids).to(DEV), 16)
    o_off, o_pairs, bad = oracle.moe_route(ids, 16)
    assert bad == 2
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(pairs.cpu().numpy()[: len(o_pairs)], o_pairs)
    assert tq.tq4_1s_get_status() & tq.TQ_DEV_BAD_ROUTING


def _moe_case(E, H, I, m, topk, seeds, dist_std=0.02, bad_ids=False, x_std=1.0, zero_rows=(), ids=None,
              mutate=None):
    up_seed, dn_seed, x_seed, r_seed = seeds
    up = synth.normal_f32((E, I, H), up_seed, dist_std)
    dn = synth.normal_f32((E, H, I), dn_seed, dist_std)
    routed, w = synth.gumbel_topk_router(m, E, topk, r_seed)
    ids = routed if ids is None else np.ascontiguousarray(ids, np.int32)
    if mutate is not None:
        mutate(up, dn, ids)
    if bad_ids:
        ids[0, 1] = E + 1
    x = synth.f32_to_bf16_bits(synth.normal_f32((m, H), x_seed, x_std))
    x[list(zero_rows)] = 0
    pu = tq.tq4_1s_quantize(torch.from_numpy(up).to(DEV), seed=up_seed)
    pd = tq.tq4_1s_quantize(torch.from_numpy(dn).to(DEV), seed=dn_seed)
    y = tq.tq4_1s_moe(_bf16_dev(x), torch.from_numpy(ids).to(DEV), torch.from_numpy(w).to(DEV), pu, pd)
    torch.cuda.synchronize()
    # the oracle quantizes only the experts the routing touches (others cannot
    # influence y); unused experts keep zero planes on the oracle side
    used = sorted(set(int(e) for e in ids.ravel() if 0 <= e < E))
    uc = np.zeros((E, I, H // 2), np.uint8); us = np.zeros((E, I, H // 16), np.uint16)
    dc = np.zeros((E, H, I // 2), np.uint8); ds = np.zeros((E, H, I // 16), np.uint16)
    for e in used:
        uc[e], us[e], _ = oracle.quantize(up[e], up_seed)
        dc[e], ds[e], _ = oracle.quantize(dn[e], dn_seed)
    y_ref, _, bad = oracle.moe(x, ids, w, uc, us, up_seed, dc, ds, dn_seed)
    return y, y_ref, bad


def test_moe_small_parity():
    y, y_ref, _ = _moe_case(8, 256, 128, 4, 2, (4, 5, 6, 7))
    assert_close(_bits(y), y_ref, "moe small")
    assert tq.tq4_1s_get_status() == 0


def test_moe_many_tokens_per_expert():
    # 40 tokens, 4 experts, top-2: 20 rows per expert on average, some experts
    # take more than one 32-row segment
    y, y_ref, _ = _moe_case(4, 256, 192, 40, 2, (14, 15, 16, 17))
    assert_close(_bits(y), y_ref, "moe segments")


def test_moe_bad_id_skipped():
    y, y_ref, bad = _moe_case(8, 128, 96, 5, 2, (24, 25, 26, 27), bad_ids=True)
    assert bad == 1
    assert_close(_bits(y), y_ref, "moe bad id")
    assert tq.tq4_1s_get_status() & tq.TQ_DEV_BAD_ROUTING


@pytest.mark.parametrize("x_std,w_std", [(3000.0, 0.0005), (1e-5, 30.0)])
def test_moe_activation_range(x_std, w_std):
    # activations far outside (and far inside) the fp16 range: the per-row
    # power-of-two scaling of the rotated activations keeps full precision
    y, y_ref, _ = _moe_case(4, 128, 96, 6, 2, (34, 35, 36, 37), dist_std=w_std, x_std=x_std)
    assert np.all(np.isfinite(y.float().cpu().numpy()))
    assert_close(_bits(y), y_ref, f"moe range x_std={x_std}")


def test_moe_any_finite_scale():
    # one routed expert with its whole up projection x 20000 and one down row
    # x 20000 (half-block scales far above ~93.6), another with an up row
    # x 1e-5 (fp16 subnormal scales): the stream-K kernel's exact recompute of
    # the rows whose sums overflowed keeps every output finite and matching
    # the oracle, unflagged, in both projections.  (The
    # whole up projection is scaled, not one row: a single dominant
    # h = bf16(relu(u)^2) would make a whole token row hinge on one bf16
    # rounding, which the fp16 operands may legitimately flip.)  Outputs of
    # different magnitude are compared apart: the tokens routed to the big
    # expert (its column 2 on its own), and the other tokens.
    routed = {}

    def mutate(up, dn, ids):
        e = routed["e"] = int(ids[0, 0])
        routed["ids"] = ids.copy()
        up[e] *= 20000.0
        dn[e, 2] *= 20000.0
        small = next(int(v) for v in ids.ravel() if int(v) != e)
        up[small, 7] *= 1e-5

    m = 16
    y, y_ref, _ = _moe_case(8, 256, 128, m, 2, (54, 55, 56, 57), mutate=mutate)
    assert tq.tq4_1s_get_status() == 0
    assert np.all(np.isfinite(y.float().cpu().numpy()))
    yb = _bits(y)
    big = np.array([t for t in range(m) if routed["e"] in routed["ids"][t]])
    other = np.array([t for t in range(m) if t not in big])
    assert len(big) and len(other)
    keep = np.array([c for c in range(256) if c != 2])
    assert_close(yb[np.ix_(big, keep)], y_ref[np.ix_(big, keep)], "moe large scales: tokens of the big expert")
    assert_close(yb[big][:, [2]], y_ref[big][:, [2]], "moe large scales: the big down row")
    assert_close(yb[other], y_ref[other], "moe large scales: the other tokens")


def test_moe_128_experts_top6_full():
    """128 experts (up 2688->1856, down 1856->2688), 16 tokens, top-6."""
    y, y_ref, _ = _moe_case(128, 2688, 1856, 16, 6, (4, 5, 6, 7))
    e = assert_close(_bits(y), y_ref, "moe 128x top6")
    print("moe errors", e)
