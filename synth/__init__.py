"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA-side tests/bench.

This module draws random numbers and nothing else: it holds none of the
TQ4_1S arithmetic (no rotation, no codebook, no packing).  Every workload the
pages describe is stood in for by arrays from here, because the real
TwoTower weights and activations are not available.

Generator: numpy's ``Generator(Philox(seed))`` -- the Philox4x32-10
counter-based generator of Salmon, Moraes, Dror and Shaw, "Parallel random
numbers: as easy as 1, 2, 3" (SC 2011).  Normal variates come from numpy's
``standard_normal``; Student-t from ``standard_t``.

Shapes and distributions follow the workloads of the Nemotron-TheHobbit model
card ("What Config-I means": 32-element blocks; "The model underneath":
128-expert top-6 MoE) and the Nemotron-Labs-TwoTower news page ("How it
works": 16-token denoise blocks, 16 denoising steps).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng", "normal_f32", "student_t_f32", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "activations_bf16", "gumbel_topk_router", "router_logits_f32", "normal_f32_device", "sweep_seed", "WORKLOADS",
]


def rng(seed: int) -> np.random.Generator:
    """A Philox4x32-10 stream keyed by ``seed``."""
    return np.random.Generator(np.random.Philox(int(seed)))


def normal_f32(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """i.i.d. N(0, std^2), drawn in float64 and rounded once to float32."""
    return (rng(seed).standard_normal(shape) * std).astype(np.float32)


def student_t_f32(shape, seed: int, nu: float = 5.0, scale: float = 1.0) -> np.ndarray:
    """i.i.d. scale * t(nu), drawn in float64 and rounded once to float32."""
    return (rng(seed).standard_t(nu, shape) * scale).astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); return the uint16 bits.

    Inputs are stored as bf16 because the layer consumes bf16 activations; this
    is input preparation, done once, identically for both sides.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations_bf16(m: int, k: int, seed: int) -> np.ndarray:
    """bf16 activations x[m][k] ~ N(0,1), as uint16 bits."""
    return f32_to_bf16_bits(normal_f32((m, k), seed))


def gumbel_topk_router(m: int, num_experts: int, topk: int, seed: int):
    """Router decisions for m tokens: top-k of Gumbel-perturbed logits.

    logits l ~ N(0,1) [m][E]; Gumbel noise g = -ln(-ln U), U ~ U(0,1);
    the k largest z = l + g are selected (ties broken toward the lower expert
    id); weights are the softmax of the selected z, renormalised to sum to 1.
    Returns (ids int32 [m][k], weights float32 [m][k]).
    """
    g = rng(seed)
    logits = g.standard_normal((m, num_experts))
    u = g.random((m, num_experts))
    u = np.clip(u, np.finfo(np.float64).tiny, 1.0 - 2.0 ** -53)
    z = logits - np.log(-np.log(u))
    order = np.argsort(-z, axis=1, kind="stable")[:, :topk]
    sel = np.take_along_axis(z, order, axis=1)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = e / e.sum(axis=1, keepdims=True)
    w = w / w.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def router_logits_f32(m: int, num_experts: int, seed: int) -> np.ndarray:
    """Router logits for m tokens as the layer receives them: fp32 [m][E],
    z = l + g with l ~ N(0,1) and Gumbel noise g = -ln(-ln U), U ~ U(0,1),
    drawn in float64 exactly as :func:`gumbel_topk_router` draws them (same
    seed, same stream) and rounded to float32."""
    g = rng(seed)
    logits = g.standard_normal((m, num_experts))
    u = g.random((m, num_experts))
    u = np.clip(u, np.finfo(np.float64).tiny, 1.0 - 2.0 ** -53)
    return (logits - np.log(-np.log(u))).astype(np.float32)


def normal_f32_device(shape, seed: int, std: float, device):
    """i.i.d. N(0, std^2) float32 drawn on a CUDA device by torch's Philox
    generator keyed by ``seed``.

    For tensors too large to draw on the host in reasonable time (a
    128-expert stack is 638M weights).  Deterministic for a given seed, shape
    and device type; a different stream from :func:`normal_f32` with the same
    seed."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32).mul_(std)


def sweep_seed(layer: int, tensor: int) -> int:
    """Seed of one tensor of layer ``layer`` of the 52-layer denoise sweep.

    tensor: 0 up-projection stack, 1 down-projection stack, 2 dense
    hidden -> 4096 weight, 3 dense 4096 -> hidden weight, 4 activations of the
    MoE and first dense projection, 5 router, 6 activations of the second
    dense projection.  The RHT seed of each weight equals its seed here."""
    if not (0 <= tensor < 8):
        raise ValueError("tensor index must be in [0, 8)")
    return WORKLOADS["denoise_sweep_52"]["seed_base"] + 8 * int(layer) + int(tensor)


# Seeds and shapes of the five workloads.  The RHT seed of each quantized
# tensor equals the seed its weights were drawn with.
WORKLOADS = {
    "tiny_linear_256": dict(n=256, k=256, m=16, w_seed=0, x_seed=1, w_dist="normal", w_std=0.02),
    "decode_linear_4096": dict(n=4096, k=4096, m=16, w_seed=2, x_seed=3, w_dist="student_t", w_std=0.02,
                               calls=16),
    "moe_128x_top6": dict(num_experts=128, hidden=2688, inter=1856, m=16, topk=6, up_seed=4, down_seed=5,
                          x_seed=6, router_seed=7, w_std=0.02),
    "prefill_linear_8192": dict(n=14336, k=4096, m=8192, w_seed=8, x_seed=9, w_dist="normal", w_std=0.02),
    "denoise_sweep_52": dict(layers=52, m=512, steps=16, num_experts=128, hidden=2688, inter=1856, topk=6,
                             # dense weights as [out][in]: hidden -> 4096, then 4096 -> hidden
                             dense=((4096, 2688), (2688, 4096)), seed_base=1000, w_std=0.02),
}
