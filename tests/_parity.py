"""Parity metrics shared by the GPU tests.

Tolerances (stated for the GEMM outputs): with y_ref the fp64 oracle result
and R = rms(y_ref),
  max_rel  = max_i |y_gpu,i - bf16(y_ref,i)| / max(|y_ref,i|, R)  <= 2e-2
  mean_rel = mean_i |y_gpu,i - bf16(y_ref,i)| / R                   <= 2e-3
A per-element |dy|/|y| is not usable because y crosses zero.
"""
import numpy as np

import oracle

MAX_REL = 2e-2
MEAN_REL = 2e-3


def bf16_bits_to_f64(bits):
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def errors(y_gpu_bits, y_ref):
    y_ref = np.asarray(y_ref, np.float64)
    g = bf16_bits_to_f64(y_gpu_bits).reshape(y_ref.shape)
    yb = bf16_bits_to_f64(oracle.round_bf16(y_ref)).reshape(y_ref.shape)
    R = float(np.sqrt(np.mean(y_ref ** 2)))
    d = np.abs(g - yb)
    return {
        "max_rel": float(np.max(d / np.maximum(np.abs(y_ref), R))),
        "mean_rel": float(np.mean(d) / R),
        "mean_rel_unrounded": float(np.mean(np.abs(g - y_ref)) / R),
        "exact_frac": float(np.mean(d == 0)),
    }


def assert_close(y_gpu_bits, y_ref, what=""):
    e = errors(y_gpu_bits, y_ref)
    assert e["max_rel"] <= MAX_REL and e["mean_rel"] <= MEAN_REL, (what, e)
    return e
