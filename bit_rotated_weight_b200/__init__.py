"""Python binding of libtq4_1s.so, the B200 (sm_100a) TQ4_1S layer.

Argument marshalling only: PyTorch supplies device memory and the current
stream; every step of quantize, dequantize, linear and MoE runs in the CUDA
kernels behind the C ABI declared in ``include/tq4_1s.h``.  There is no CPU
or PyTorch fallback: if the shared library is missing or the device is not
an sm_100 GPU, the calls raise.

TQ4_1S ("Config-I") is the weight format of the Nemotron-TheHobbit-30B-A3B
model card, section "What Config-I means": a randomized Walsh-Hadamard
rotation per 32-element block, 4-bit codes into a 16-level Lloyd-Max
codebook, two half-block scales, about 5 bits per weight.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

__all__ = [
    "LIB_PATH", "TQ4Error", "Packed", "load_library",
    "tq4_1s_version", "tq4_1s_error_string", "tq4_1s_packed_bytes", "tq4_1s_sign_mask", "tq4_1s_codebook",
    "tq4_1s_quantize", "tq4_1s_quantize_batched", "tq4_1s_dequantize", "tq4_1s_linear_workspace", "tq4_1s_linear",
    "tq4_1s_moe_workspace", "tq4_1s_moe", "tq4_1s_moe_logits", "tq4_1s_router_topk", "tq4_1s_moe_route", "tq4_1s_get_status", "tq4_1s_launch_count",
    "tq4_1s_linear_static", "tq4_1s_debug_hook", "Fp8Weight", "tq4_1s_to_fp8", "tq4_1s_linear_fp8",
    "AffineWeight", "tq4_1s_affine_quantize", "tq4_1s_affine_dequantize", "tq4_1s_affine_linear",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq4_1s.so")

TQ_OK = 0
TQ_DTYPE_F32, TQ_DTYPE_BF16 = 0, 1
TQ_DEV_TIMEOUT, TQ_DEV_BAD_ROUTING, TQ_DEV_NONFINITE, TQ_DEV_SCALE_RANGE = 1, 2, 4, 8
TQ_WEIGHT_STATIC = 1
TQ_HOOK_FAIL_NEXT_CALLS, TQ_HOOK_WAIT_NS, TQ_HOOK_WITHHOLD_ARRIVAL = 1, 2, 3


class TQ4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {tq4_1s_error_string(code)} (code {code})")


class _Weight(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("num_experts", ctypes.c_int32),
        ("flags", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
    ]


class _AffineWeight(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("bits", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
    ]


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtq4_1s.so (built by ``__graft_entry__.build()``); raise if absent."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError(f"libtq4_1s.so not built (expected at {path}); run __graft_entry__.build()")
            lib = ctypes.CDLL(path)
            P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
            W = ctypes.POINTER(_Weight)
            sig = {
                "tq4_1s_version": ([], ctypes.c_int),
                "tq4_1s_error_string": ([ctypes.c_int], ctypes.c_char_p),
                "tq4_1s_packed_bytes": ([I64, I64, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ)], ctypes.c_int),
                "tq4_1s_sign_mask": ([ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
                "tq4_1s_codebook": ([P, P], ctypes.c_int),
                "tq4_1s_quantize": ([P, ctypes.c_int, W, P], ctypes.c_int),
                "tq4_1s_quantize_batched": ([P, ctypes.c_int, P, I32, P], ctypes.c_int),
                "tq4_1s_dequantize": ([W, P, P], ctypes.c_int),
                "tq4_1s_linear_workspace": ([I64, W], SZ),
                "tq4_1s_linear": ([P, I64, W, P, P, SZ, P], ctypes.c_int),
                "tq4_1s_linear_static": ([P, I64, W, P, P], ctypes.c_int),
                "tq4_1s_moe_workspace": ([I64, I32, W, W], SZ),
                "tq4_1s_moe": ([P, I64, P, P, I32, W, W, P, P, SZ, P], ctypes.c_int),
                "tq4_1s_moe_route": ([P, I64, I32, I32, P, P, P], ctypes.c_int),
                "tq4_1s_moe_logits": ([P, I64, P, I32, W, W, P, P, SZ, P], ctypes.c_int),
                "tq4_1s_router_topk": ([P, I64, I32, I32, P, P, P], ctypes.c_int),
                "tq4_1s_get_status": ([P, ctypes.POINTER(I32)], ctypes.c_int),
                "tq4_1s_launch_count": ([], ctypes.c_uint64),
                "tq4_1s_debug_hook": ([ctypes.c_int, I64], ctypes.c_int),
                "tq4_1s_to_fp8": ([W, P, P, P], ctypes.c_int),
                "tq4_1s_linear_fp8_workspace": ([I64, I64, I64], SZ),
                "tq4_1s_linear_fp8": ([P, I64, P, P, I64, I64, I32, P, P, SZ, P], ctypes.c_int),
                "tq4_1s_affine_quantize": ([P, ctypes.POINTER(_AffineWeight), P], ctypes.c_int),
                "tq4_1s_affine_dequantize": ([ctypes.POINTER(_AffineWeight), P, P], ctypes.c_int),
                "tq4_1s_affine_linear_workspace": ([I64, ctypes.POINTER(_AffineWeight)], SZ),
                "tq4_1s_affine_linear": ([P, I64, ctypes.POINTER(_AffineWeight), P, P, SZ, P], ctypes.c_int),
            }
            for name, (args, res) in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _check(rc: int, what: str):
    if rc != TQ_OK:
        raise TQ4Error(rc, what)


# torch's own raw accessor of the current stream (what its generated code
# calls); the public Stream object costs several microseconds per call
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device | None = None):
    if _raw_stream is not None:
        index = device.index if device is not None and device.index is not None else torch.cuda.current_device()
        return _raw_stream(index)
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: torch.Tensor | None):
    return 0 if t is None else t.data_ptr()


@dataclass
class Packed:
    """A packed TQ4_1S tensor (stack): codes [E][n][k/2] uint8, scales [E][n][k/16] fp16 bits."""
    codes: torch.Tensor
    scales: torch.Tensor
    n: int
    k: int
    num_experts: int
    seed: int
    flags: int = 0   # TQ_WEIGHT_STATIC: no unfinished kernel writes the planes (see include/tq4_1s.h)

    def c_struct(self) -> _Weight:
        # built once per (codes, scales) storage; a call only marshals a pointer to it
        key = (self.codes.data_ptr(), self.scales.data_ptr(), self.n, self.k, self.num_experts, self.seed,
               self.flags)
        cached = self.__dict__.get("_c_struct")
        if cached is None or cached[0] != key:
            cached = (key, _Weight(self.n, self.k, self.num_experts, self.flags, self.seed, key[0], key[1]))
            self.__dict__["_c_struct"] = cached
        return cached[1]

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + self.scales.numel() * 2


def tq4_1s_version() -> int:
    return load_library().tq4_1s_version()


def tq4_1s_error_string(code: int) -> str:
    return load_library().tq4_1s_error_string(code).decode()


def tq4_1s_packed_bytes(n: int, k: int, num_experts: int = 1):
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().tq4_1s_packed_bytes(n, k, num_experts, ctypes.byref(c), ctypes.byref(s)), "packed_bytes")
    return c.value, s.value


def tq4_1s_sign_mask(seed: int) -> int:
    m = ctypes.c_uint32()
    _check(load_library().tq4_1s_sign_mask(seed, ctypes.byref(m)), "sign_mask")
    return m.value


def tq4_1s_codebook():
    """(levels[16], thresholds[15]) as float32 CPU tensors, as the kernels use them."""
    lv = torch.zeros(16, dtype=torch.float32)
    th = torch.zeros(15, dtype=torch.float32)
    _check(load_library().tq4_1s_codebook(_ptr(lv), _ptr(th)), "codebook")
    return lv, th


def _empty_packed(n: int, k: int, num_experts: int, seed: int, device) -> Packed:
    cb, sb = tq4_1s_packed_bytes(n, k, num_experts)
    codes = torch.empty(cb, dtype=torch.uint8, device=device).view(num_experts, n, k // 2)
    scales = torch.empty(sb // 2, dtype=torch.int16, device=device).view(num_experts, n, k // 16)
    return Packed(codes, scales, n, k, num_experts, seed)


def tq4_1s_quantize(W: torch.Tensor, seed: int, out: Packed | None = None) -> Packed:
    """Quantize W ([n][k] or [E][n][k], float32 or bfloat16, CUDA) to TQ4_1S."""
    if W.dim() == 2:
        W = W.unsqueeze(0)
    if W.dim() != 3 or not W.is_cuda or W.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("W must be a CUDA float32/bfloat16 tensor of shape [n][k] or [E][n][k]")
    W = W.contiguous()
    E, n, k = W.shape
    if out is None:
        out = _empty_packed(n, k, E, seed, W.device)
    dt = TQ_DTYPE_F32 if W.dtype == torch.float32 else TQ_DTYPE_BF16
    ws = out.c_struct()
    _check(load_library().tq4_1s_quantize(_ptr(W), dt, ctypes.byref(ws), _stream(W.device)), "quantize")
    return out


def tq4_1s_quantize_batched(Ws, seeds, outs=None) -> list:
    """Quantize several tensors (all float32 or all bfloat16, CUDA, [n][k] or
    [E][n][k]) in batched launches; returns their Packed forms."""
    Ws = [W.unsqueeze(0) if W.dim() == 2 else W for W in Ws]
    if not Ws:
        return []
    dt0 = Ws[0].dtype
    for W in Ws:
        if W.dim() != 3 or not W.is_cuda or W.dtype != dt0 or dt0 not in (torch.float32, torch.bfloat16):
            raise ValueError("every W must be a CUDA tensor of one dtype (float32 or bfloat16), [n][k] or [E][n][k]")
    Ws = [W.contiguous() for W in Ws]
    if outs is None:
        outs = [_empty_packed(W.shape[1], W.shape[2], W.shape[0], s, W.device) for W, s in zip(Ws, seeds)]
    structs = (_Weight * len(Ws))(*[o.c_struct() for o in outs])
    ptrs = (ctypes.c_void_p * len(Ws))(*[W.data_ptr() for W in Ws])
    dt = TQ_DTYPE_F32 if dt0 == torch.float32 else TQ_DTYPE_BF16
    _check(load_library().tq4_1s_quantize_batched(ctypes.cast(ptrs, ctypes.c_void_p), dt,
                                                  ctypes.cast(structs, ctypes.c_void_p), len(Ws),
                                                  _stream(Ws[0].device)), "quantize_batched")
    return outs


def tq4_1s_dequantize(w: Packed) -> torch.Tensor:
    out = torch.empty((w.num_experts, w.n, w.k), dtype=torch.float32, device=w.codes.device)
    ws = w.c_struct()
    _check(load_library().tq4_1s_dequantize(ctypes.byref(ws), _ptr(out), _stream(out.device)), "dequantize")
    return out


_ws_cache: dict = {}


SMALL_M = 128   # tq4_1s_linear takes its stream-K path up to this many rows


def _workspace(nbytes: int, device, kind: str) -> torch.Tensor:
    """A cached workspace per (device, kind), grown on demand.

    The library needs no cleared workspace: its tile counters carry each
    launch's epoch, so values left by earlier calls read as zero arrivals.
    The kinds are kept apart only so that a large small-m buffer and a large
    dequantized-weight buffer are not reallocated back and forth."""
    key = (str(device), kind)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def tq4_1s_linear_workspace(m: int, w: Packed) -> int:
    ws = w.c_struct()
    return load_library().tq4_1s_linear_workspace(m, ctypes.byref(ws))


def tq4_1s_linear(x: torch.Tensor, w: Packed, out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = bf16(x @ W_hat^T) for x bfloat16 [m][k] on CUDA."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][k] tensor")
    x = x.contiguous()
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    wst = w.c_struct()
    if workspace is None:   # (a caller's workspace is checked by the library)
        need = load_library().tq4_1s_linear_workspace(m, ctypes.byref(wst))
        workspace = _workspace(need, x.device, "linear_small" if m <= SMALL_M else "linear_large")
    _check(load_library().tq4_1s_linear(_ptr(x), m, ctypes.byref(wst), _ptr(out), _ptr(workspace),
                                        workspace.numel(), _stream(x.device)), "linear")
    return out


def tq4_1s_moe_workspace(m: int, topk: int, up: Packed, down: Packed) -> int:
    u, d = up.c_struct(), down.c_struct()
    return load_library().tq4_1s_moe_workspace(m, topk, ctypes.byref(u), ctypes.byref(d))


def tq4_1s_moe(x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor, up: Packed, down: Packed,
               out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Sync-free MoE: y_t = bf16(sum_j w_tj * down_e(bf16(relu(up_e(x_t))^2)))."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][H] tensor")
    x = x.contiguous()
    topk_ids = topk_ids.to(torch.int32).contiguous()
    topk_w = topk_w.to(torch.float32).contiguous()
    m, topk = topk_ids.shape
    if out is None:
        out = torch.empty((m, up.k), dtype=torch.bfloat16, device=x.device)
    u, d = up.c_struct(), down.c_struct()
    if workspace is None:   # (a caller's workspace is checked by the library)
        need = load_library().tq4_1s_moe_workspace(m, topk, ctypes.byref(u), ctypes.byref(d))
        workspace = _workspace(need, x.device, "moe")
    _check(load_library().tq4_1s_moe(_ptr(x), m, _ptr(topk_ids), _ptr(topk_w), topk, ctypes.byref(u),
                                     ctypes.byref(d), _ptr(out), _ptr(workspace), workspace.numel(),
                                     _stream(x.device)), "moe")
    return out


def tq4_1s_moe_logits(x: torch.Tensor, logits: torch.Tensor, topk: int, up: Packed, down: Packed,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The MoE with the router on the device: logits float32 [m][E] (CUDA)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][H] tensor")
    if logits.dtype != torch.float32 or logits.dim() != 2 or not logits.is_cuda:
        raise ValueError("logits must be a CUDA float32 [m][E] tensor")
    x = x.contiguous()
    logits = logits.contiguous()
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, up.k), dtype=torch.bfloat16, device=x.device)
    u, d = up.c_struct(), down.c_struct()
    if workspace is None:   # (a caller's workspace is checked by the library)
        need = load_library().tq4_1s_moe_workspace(m, topk, ctypes.byref(u), ctypes.byref(d))
        workspace = _workspace(need, x.device, "moe")
    _check(load_library().tq4_1s_moe_logits(_ptr(x), m, _ptr(logits), topk, ctypes.byref(u), ctypes.byref(d),
                                            _ptr(out), _ptr(workspace), workspace.numel(), _stream(x.device)),
           "moe_logits")
    return out


def tq4_1s_router_topk(logits: torch.Tensor, topk: int):
    """(ids int32 [m][topk], weights float32 [m][topk]) from float32 logits [m][E] on CUDA."""
    if logits.dtype != torch.float32 or logits.dim() != 2 or not logits.is_cuda:
        raise ValueError("logits must be a CUDA float32 [m][E] tensor")
    logits = logits.contiguous()
    m, E = logits.shape
    ids = torch.empty((m, topk), dtype=torch.int32, device=logits.device)
    w = torch.empty((m, topk), dtype=torch.float32, device=logits.device)
    _check(load_library().tq4_1s_router_topk(_ptr(logits), m, E, topk, _ptr(ids), _ptr(w), _stream(logits.device)),
           "router_topk")
    return ids, w


def tq4_1s_moe_route(topk_ids: torch.Tensor, num_experts: int):
    """(offsets [E+1], pairs [m*topk]) -- the routing step of tq4_1s_moe."""
    topk_ids = topk_ids.to(torch.int32).contiguous()
    m, topk = topk_ids.shape
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=topk_ids.device)
    pairs = torch.empty(m * topk, dtype=torch.int32, device=topk_ids.device)
    _check(load_library().tq4_1s_moe_route(_ptr(topk_ids), m, topk, num_experts, _ptr(offsets), _ptr(pairs),
                                           _stream(topk_ids.device)), "moe_route")
    return offsets, pairs


def tq4_1s_get_status(device=None) -> int:
    """Synchronize the current stream and read-and-clear the device status word."""
    s = ctypes.c_int32()
    _check(load_library().tq4_1s_get_status(_stream(device), ctypes.byref(s)), "get_status")
    return s.value


def tq4_1s_launch_count() -> int:
    """Kernel launches issued through the library by this process so far."""
    return int(load_library().tq4_1s_launch_count())


def tq4_1s_linear_static(x: torch.Tensor, w: Packed, out: torch.Tensor | None = None) -> torch.Tensor:
    """tq4_1s_linear without a workspace, for callers that cannot allocate.

    Runs the small-m linear path with its scratch held in a fixed device array
    inside the library (m <= 32, k <= 8192, n <= 32768).  Calls that overlap
    on the GPU share that array and race; serialize them.  The first call on a
    device looks up the array's address, so make it outside stream capture.
    """
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][k] tensor")
    x = x.contiguous()
    if out is None:
        out = torch.empty((x.shape[0], w.n), dtype=torch.bfloat16, device=x.device)
    wst = w.c_struct()
    _check(load_library().tq4_1s_linear_static(_ptr(x), x.shape[0], ctypes.byref(wst), _ptr(out),
                                               _stream(x.device)), "linear_static")
    return out


def tq4_1s_debug_hook(what: int, value: int) -> None:
    """Test hooks of the library (fault injection, short device waits); see include/tq4_1s.h."""
    _check(load_library().tq4_1s_debug_hook(what, value), "debug_hook")


@dataclass
class Fp8Weight:
    """The fp8-resident cache of a TQ4_1S weight: E4M3 codes q [rows][k] (uint8)
    and one float32 scale per row; the cached weight is wscale[n] * q[n][k]."""
    q: torch.Tensor
    wscale: torch.Tensor
    n: int
    k: int
    flags: int = 0


def tq4_1s_to_fp8(w: Packed, flags: int = 0) -> Fp8Weight:
    """Convert a packed TQ4_1S weight (stack) to the fp8 cache (rows = n * E)."""
    rows = w.n * w.num_experts
    q = torch.empty((rows, w.k), dtype=torch.uint8, device=w.codes.device)
    sc = torch.empty(rows, dtype=torch.float32, device=w.codes.device)
    ws = w.c_struct()
    _check(load_library().tq4_1s_to_fp8(ctypes.byref(ws), _ptr(q), _ptr(sc), _stream(q.device)), "to_fp8")
    return Fp8Weight(q, sc, rows, w.k, flags)


def tq4_1s_linear_fp8(x: torch.Tensor, w: Fp8Weight, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = bf16(x @ (wscale * q)^T) with the fp8 cache, x bfloat16 [m][k] on CUDA."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][k] tensor")
    x = x.contiguous()
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    lib = load_library()
    if workspace is None:   # (used only when the decode kernel does not take the shape)
        workspace = _workspace(lib.tq4_1s_linear_fp8_workspace(m, w.n, w.k), x.device, "fp8_large")
    wsz = 0 if workspace is None else workspace.numel()
    _check(lib.tq4_1s_linear_fp8(_ptr(x), m, _ptr(w.q), _ptr(w.wscale), w.n, w.k, w.flags, _ptr(out),
                                 _ptr(workspace), wsz, _stream(x.device)), "linear_fp8")
    return out


@dataclass
class AffineWeight:
    """The MLX-style affine format: codes [n][k*bits/8] (bit stream), bf16
    scales and biases [n][k/64] (as int16 bit patterns)."""
    codes: torch.Tensor
    scales: torch.Tensor
    biases: torch.Tensor
    n: int
    k: int
    bits: int

    def c_struct(self) -> _AffineWeight:
        return _AffineWeight(self.n, self.k, self.bits, 0, self.codes.data_ptr(), self.scales.data_ptr(),
                             self.biases.data_ptr())

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + 2 * (self.scales.numel() + self.biases.numel())


def tq4_1s_affine_quantize(W: torch.Tensor, bits: int) -> AffineWeight:
    """Quantize W (float32 [n][k], CUDA, k % 64 == 0) to the affine format."""
    if W.dim() != 2 or W.dtype != torch.float32 or not W.is_cuda:
        raise ValueError("W must be a CUDA float32 [n][k] tensor")
    W = W.contiguous()
    n, k = W.shape
    out = AffineWeight(torch.empty((n, k * bits // 8), dtype=torch.uint8, device=W.device),
                       torch.empty((n, k // 64), dtype=torch.int16, device=W.device),
                       torch.empty((n, k // 64), dtype=torch.int16, device=W.device), n, k, bits)
    st = out.c_struct()
    _check(load_library().tq4_1s_affine_quantize(_ptr(W), ctypes.byref(st), _stream(W.device)), "affine_quantize")
    return out


def tq4_1s_affine_dequantize(w: AffineWeight) -> torch.Tensor:
    out = torch.empty((w.n, w.k), dtype=torch.float32, device=w.codes.device)
    st = w.c_struct()
    _check(load_library().tq4_1s_affine_dequantize(ctypes.byref(st), _ptr(out), _stream(out.device)),
           "affine_dequantize")
    return out


def tq4_1s_affine_linear(x: torch.Tensor, w: AffineWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a CUDA bfloat16 [m][k] tensor")
    x = x.contiguous()
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    st = w.c_struct()
    lib = load_library()
    ws = _workspace(lib.tq4_1s_affine_linear_workspace(m, ctypes.byref(st)), x.device, "affine")
    _check(lib.tq4_1s_affine_linear(_ptr(x), m, ctypes.byref(st), _ptr(out), _ptr(ws), ws.numel(),
                                    _stream(x.device)), "affine_linear")
    return out
