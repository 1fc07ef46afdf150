"""TQ4_1S CPU oracle -- test infrastructure, not part of the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It wraps ``tq4_1s_oracle.c`` (plain scalar C,
compiled with gcc without FMA contraction or fast-math) through ctypes and
shares nothing with the CUDA path.

Every function follows the Nemotron-TheHobbit-30B-A3B model card, section
"What Config-I means" (per-32-block Walsh-Hadamard rotation, 16-level
Lloyd-Max codes, two half-block scales, ~5 bits/weight), with the readings
listed at the top of the C file.  Parity status of each function:

- codebook, sign_mask, hadamard32, fwht32, quantize, dequantize, levels,
  linear, moe_route: pinned by ``tests/test_oracle_pins.py``.
- router_topk: pinned by invariants (distinct ids, descending order, every
  chosen logit >= every other, weights positive summing to 1), equal-logit
  and single-choice special cases, and k = E against scipy's softmax.
- f32_to_e4m3, e4m3_to_f64, to_fp8, fp8_dequantize, linear_fp8 (the fp8
  weight cache of the model card's "Help wanted"): pinned by the format's
  published values (largest finite 448, smallest subnormal 2^-9), round
  trips of every code, ties to even, torch's float8_e4m3fn conversion,
  the conversion's scale and error bounds, and numpy matmul.
- affine_quantize, affine_dequantize (the MLX-style affine group format of
  the MLX port's README, for the bytes-versus-accuracy comparison): pinned
  by brute-force nearest grid points, the half-step error bound, exactly
  representable grids, constant groups and the bit-stream packing.
- moe: pinned through closed-form special cases (single slot, constant-level
  experts) and composition with the pinned linear; the squared-ReLU and the
  bf16 rounding of the hidden activation are fixed by the workload
  definition, not by the pages.
- boundary_near (which code and scale decisions lie within 1e-6 of a
  threshold or of an fp16 rounding midpoint; a reporting aid beside the
  bit-exact comparison): pinned by constructed blocks that land exactly on a
  threshold and on a midpoint, and by perturbed-decision containment.
- reconstruction cosine 0.997 quoted on the model card for real weights:
  parity unpinned (real weights are not available; synthetic weights are
  checked against the >= 0.99 bound instead).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq4_1s_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_tq4.so")
CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fexcess-precision=standard", "-fno-fast-math",
          "-shared", "-fPIC"]
_lock = threading.Lock()
_lib = None

BLOCK = 32
HALF = 16


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.orc_codebook.argtypes = [P, P, P, P]
            lib.orc_codebook.restype = ctypes.c_int
            lib.orc_splitmix64_first.argtypes = [ctypes.c_uint64]
            lib.orc_splitmix64_first.restype = ctypes.c_uint64
            lib.orc_sign_mask.argtypes = [ctypes.c_uint64]
            lib.orc_sign_mask.restype = ctypes.c_uint32
            lib.orc_hadamard32.argtypes = [P]
            lib.orc_fwht32_f32.argtypes = [P]
            lib.orc_rotate_block.argtypes = [P, ctypes.c_uint32, P]
            lib.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
            lib.orc_f16_to_f32.restype = ctypes.c_float
            lib.orc_f32_to_f16_sat.argtypes = [ctypes.c_float]
            lib.orc_f32_to_f16_sat.restype = ctypes.c_uint16
            lib.orc_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.orc_f64_to_bf16.restype = ctypes.c_uint16
            lib.orc_quantize.argtypes = [P, I64, I64, ctypes.c_uint64, P, P]
            lib.orc_quantize.restype = I64
            lib.orc_dequantize.argtypes = [P, P, I64, I64, ctypes.c_uint64, P]
            lib.orc_levels.argtypes = [P, P, I64, I64, P]
            lib.orc_linear.argtypes = [P, I64, I64, P, I64, P]
            lib.orc_round_bf16.argtypes = [P, I64, P]
            lib.orc_moe_route.argtypes = [P, I64, ctypes.c_int, ctypes.c_int, P, P]
            lib.orc_moe_route.restype = I64
            lib.orc_moe.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, ctypes.c_int,
                                    P, P, ctypes.c_uint64, P, P, ctypes.c_uint64, P]
            lib.orc_moe.restype = I64
            lib.orc_router_topk.argtypes = [P, I64, ctypes.c_int, ctypes.c_int, P, P]
            lib.orc_f32_to_e4m3_sat.argtypes = [ctypes.c_float]
            lib.orc_f32_to_e4m3_sat.restype = ctypes.c_uint8
            lib.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_to_f64.restype = ctypes.c_double
            lib.orc_to_fp8.argtypes = [P, P, I64, I64, ctypes.c_uint64, P, P]
            lib.orc_linear_fp8.argtypes = [P, I64, I64, P, P, I64, P]
            lib.orc_affine_quantize.argtypes = [P, I64, I64, ctypes.c_int, P, P, P]
            lib.orc_affine_dequantize.argtypes = [P, P, P, I64, I64, ctypes.c_int, P]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
def codebook():
    """Lloyd-Max levels of N(0,1), 16 levels.  Returns (c, t, c32, t32)."""
    c = np.zeros(16); t = np.zeros(15)
    c32 = np.zeros(16, np.float32); t32 = np.zeros(15, np.float32)
    it = _load().orc_codebook(_ptr(c), _ptr(t), _ptr(c32), _ptr(t32))
    if it < 0:
        raise RuntimeError("Lloyd iteration did not converge")
    return c, t, c32, t32


def splitmix64_first(state: int) -> int:
    return int(_load().orc_splitmix64_first(state))


def sign_mask(seed: int) -> int:
    return int(_load().orc_sign_mask(seed))


def hadamard32() -> np.ndarray:
    H = np.zeros((32, 32), np.int8)
    _load().orc_hadamard32(_ptr(H))
    return H


def fwht32(a) -> np.ndarray:
    a = _c(a, np.float32).copy()
    assert a.shape == (32,)
    _load().orc_fwht32_f32(_ptr(a))
    return a


def rotate_block(w, mask: int) -> np.ndarray:
    w = _c(w, np.float32)
    v = np.zeros(32, np.float32)
    _load().orc_rotate_block(_ptr(w), mask, _ptr(v))
    return v


def f16_to_f32(h: int) -> float:
    return float(_load().orc_f16_to_f32(h))


def f32_to_f16_sat(x: float) -> int:
    return int(_load().orc_f32_to_f16_sat(x))


def f64_to_bf16(x: float) -> int:
    return int(_load().orc_f64_to_bf16(x))


def quantize(W, seed: int):
    """W fp32 [n][k] -> (codes uint8 [n][k/2], scales uint16 [n][k/16], nonfinite_blocks)."""
    W = _c(W, np.float32)
    n, k = W.shape
    assert k % BLOCK == 0
    codes = np.zeros((n, k // 2), np.uint8)
    scales = np.zeros((n, k // HALF), np.uint16)
    bad = _load().orc_quantize(_ptr(W), n, k, seed, _ptr(codes), _ptr(scales))
    return codes, scales, int(bad)


def unpack_codes(codes) -> np.ndarray:
    """codes plane [n][k/2] -> one code per element [n][k] (even k in the low nibble)."""
    codes = _c(codes, np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


def boundary_near(W, seed: int, scales=None, tol: float = 1e-6):
    """Which quantization decisions of W sit within ``tol`` of a boundary.

    Two correct fp32 implementations of the quantizer may disagree only on
    these, so parity of codes and scales is exact everywhere else and the
    count here is what gets reported beside it.  Computed in fp64 from the
    definition (explicit Hadamard matrix, not the butterfly): with v = R w
    per 32-block (r = fp32(1/sqrt(32))) and d the stored fp16 scale of the
    half block, a code is near when min_j |v/d - t32_j| <= tol; a half-block
    scale is near when the fp64 RMS of its 16 rotated values lies within
    ``tol`` (relative) of the midpoint between the two fp16 values around it.

    Returns {"codes": count, "scales": count, "code_mask": bool [n][k],
    "scale_mask": bool [n][k/16]}."""
    W = _c(W, np.float32)
    n, k = W.shape
    assert k % BLOCK == 0
    if scales is None:
        _, scales, _ = quantize(W, seed)
    mask = sign_mask(seed)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(BLOCK)])
    H = hadamard32().astype(np.float64)
    r = float(np.float32(1.0 / np.sqrt(32.0)))
    v = (W.astype(np.float64).reshape(-1, BLOCK) * s) @ H.T * r          # [blocks][32]
    vh = v.reshape(-1, HALF)                                              # [halves][16]
    d = _c(scales, np.uint16).reshape(-1).view(np.float16).astype(np.float64)
    _, _, _, t32 = codebook()
    t = t32.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = vh / d[:, None]
    idx = np.clip(np.searchsorted(t, u), 1, len(t) - 1)
    dist = np.minimum(np.abs(u - t[idx - 1]), np.abs(u - t[idx]))
    code_near = (d[:, None] > 0) & np.isfinite(u) & (dist <= tol)
    rms = np.sqrt(np.mean(vh * vh, axis=1))
    h = rms.astype(np.float16)
    lo = np.where(h.astype(np.float64) > rms, np.nextafter(h, np.float16(-np.inf)), h)
    hi = np.nextafter(lo, np.float16(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2.0
    scale_near = (rms > 0) & (rms < 65504.0) & (np.abs(rms - mid) <= tol * rms)
    code_mask = code_near.reshape(n, k)
    scale_mask = scale_near.reshape(n, k // HALF)
    return {"codes": int(code_mask.sum()), "scales": int(scale_mask.sum()),
            "code_mask": code_mask, "scale_mask": scale_mask}


def dequantize(codes, scales, seed: int) -> np.ndarray:
    codes = _c(codes, np.uint8); scales = _c(scales, np.uint16)
    n, k = codes.shape[0], codes.shape[1] * 2
    W = np.zeros((n, k), np.float32)
    _load().orc_dequantize(_ptr(codes), _ptr(scales), n, k, seed, _ptr(W))
    return W


def levels(codes, scales) -> np.ndarray:
    """Rotated-domain dequantized values (codebook level times half-block scale)."""
    codes = _c(codes, np.uint8); scales = _c(scales, np.uint16)
    n, k = codes.shape[0], codes.shape[1] * 2
    wn = np.zeros((n, k), np.float32)
    _load().orc_levels(_ptr(codes), _ptr(scales), n, k, _ptr(wn))
    return wn


def linear_f64(x_bf16, W_hat) -> np.ndarray:
    """y = x * W_hat^T in fp64 (x as bf16 bits [m][k], W_hat fp32 [n][k])."""
    x = _c(x_bf16, np.uint16); W = _c(W_hat, np.float32)
    m, k = x.shape
    n = W.shape[0]
    assert W.shape[1] == k
    y = np.zeros((m, n), np.float64)
    _load().orc_linear(_ptr(x), m, k, _ptr(W), n, _ptr(y))
    return y


def round_bf16(y) -> np.ndarray:
    y = _c(y, np.float64)
    out = np.zeros(y.shape, np.uint16)
    _load().orc_round_bf16(_ptr(y), y.size, _ptr(out))
    return out


def linear(x_bf16, codes, scales, seed: int):
    """The TQ4_1S linear layer: returns (y_f64, y_bf16_bits)."""
    y = linear_f64(x_bf16, dequantize(codes, scales, seed))
    return y, round_bf16(y)


def moe_route(ids, num_experts: int):
    ids = _c(ids, np.int32)
    m, topk = ids.shape
    offsets = np.zeros(num_experts + 1, np.int32)
    pairs = np.full(m * topk, -1, np.int32)
    bad = _load().orc_moe_route(_ptr(ids), m, topk, num_experts, _ptr(offsets), _ptr(pairs))
    return offsets, pairs[: offsets[-1]], int(bad)


def router_topk(z, topk: int):
    """MoE router: fp32 logits z [m][E] -> (ids int32 [m][topk], w float32 [m][topk]).

    Softmax over all experts (fp64), the topk largest chosen in descending
    order (equal logits: lower expert id first), their probabilities
    renormalised to sum to 1 and rounded to fp32."""
    z = _c(z, np.float32)
    m, E = z.shape
    assert 1 <= topk <= E
    ids = np.zeros((m, topk), np.int32)
    w = np.zeros((m, topk), np.float32)
    _load().orc_router_topk(_ptr(z), m, E, topk, _ptr(ids), _ptr(w))
    return ids, w


def f32_to_e4m3(x: float) -> int:
    """fp32 -> OCP E4M3 bits, round to nearest even, saturating at +-448."""
    return int(_load().orc_f32_to_e4m3_sat(float(np.float32(x))))


def e4m3_to_f64(b: int) -> float:
    return float(_load().orc_e4m3_to_f64(int(b)))


def to_fp8(codes, scales, seed: int):
    """fp8-resident cache of a TQ4_1S weight [n][k]: (q uint8 [n][k] E4M3 bits,
    row scales float32 [n]); the cached weight is s[n] * q[n][k]."""
    codes = _c(codes, np.uint8); scales = _c(scales, np.uint16)
    n, k = codes.shape[0], codes.shape[1] * 2
    q = np.zeros((n, k), np.uint8)
    s = np.zeros(n, np.float32)
    _load().orc_to_fp8(_ptr(codes), _ptr(scales), n, k, seed, _ptr(q), _ptr(s))
    return q, s


def fp8_dequantize(q, s) -> np.ndarray:
    """The cached weight s[n] * e4m3(q[n][k]) in fp64."""
    q = _c(q, np.uint8)
    lut = np.array([e4m3_to_f64(b) for b in range(256)], np.float64)
    return np.asarray(s, np.float64)[:, None] * lut[q]


def linear_fp8(x_bf16, q, s):
    """y = x * (s q)^T with the sum in fp64: returns (y_f64, y_bf16_bits)."""
    x = _c(x_bf16, np.uint16); q = _c(q, np.uint8); s = _c(s, np.float32)
    m, k = x.shape
    n = q.shape[0]
    y = np.zeros((m, n), np.float64)
    _load().orc_linear_fp8(_ptr(x), m, k, _ptr(q), _ptr(s), n, _ptr(y))
    return y, round_bf16(y)


AFFINE_GROUP = 64


def affine_quantize(W, bits: int):
    """MLX-style affine group quantization of W fp32 [n][k] (groups of 64 along
    k): returns (codes uint8 [n][k*bits/8] bit stream, scales bf16 bits
    [n][k/64], biases bf16 bits [n][k/64])."""
    W = _c(W, np.float32)
    n, k = W.shape
    assert bits in (4, 6, 8) and k % AFFINE_GROUP == 0
    codes = np.zeros((n, k * bits // 8), np.uint8)
    scales = np.zeros((n, k // AFFINE_GROUP), np.uint16)
    biases = np.zeros((n, k // AFFINE_GROUP), np.uint16)
    _load().orc_affine_quantize(_ptr(W), n, k, bits, _ptr(codes), _ptr(scales), _ptr(biases))
    return codes, scales, biases


def affine_dequantize(codes, scales, biases, bits: int) -> np.ndarray:
    codes = _c(codes, np.uint8); scales = _c(scales, np.uint16); biases = _c(biases, np.uint16)
    n = codes.shape[0]
    k = codes.shape[1] * 8 // bits
    W = np.zeros((n, k), np.float32)
    _load().orc_affine_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), n, k, bits, _ptr(W))
    return W


def moe(x_bf16, ids, w, up_codes, up_scales, up_seed, dn_codes, dn_scales, dn_seed):
    """MoE layer.  up_*: [E][I][H/2], [E][I][H/16]; dn_*: [E][H][I/2], [E][H][I/16].

    Returns (y_f64 [m][H], y_bf16_bits, skipped_pairs)."""
    x = _c(x_bf16, np.uint16); ids = _c(ids, np.int32); w = _c(w, np.float32)
    uc = _c(up_codes, np.uint8); us = _c(up_scales, np.uint16)
    dc = _c(dn_codes, np.uint8); ds = _c(dn_scales, np.uint16)
    m, H = x.shape
    E, I = uc.shape[0], uc.shape[1]
    topk = ids.shape[1]
    assert uc.shape == (E, I, H // 2) and dc.shape == (E, H, I // 2)
    y = np.zeros((m, H), np.float64)
    bad = _load().orc_moe(_ptr(x), m, H, I, _ptr(ids), _ptr(w), topk, E, _ptr(uc), _ptr(us), up_seed,
                          _ptr(dc), _ptr(ds), dn_seed, _ptr(y))
    return y, round_bf16(y), int(bad)


def packed_bytes(n: int, k: int, num_experts: int = 1):
    """Bytes of the two planes: codes 4 bits/weight, scales 2 x fp16 per 32."""
    return num_experts * n * k // 2, num_experts * n * (k // HALF) * 2
