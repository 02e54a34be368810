"""ctypes binding of libvmoba.so (the C ABI in include/vmoba.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  PyTorch tensors are used as device buffers and torch's
current CUDA stream is passed through.  There is no fallback: if the shared
library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvmoba.so")

VMOBA_BF16 = 0
VMOBA_F32 = 1
STATIC_SELECT_SCRATCH_BYTES = 16 << 20   # VMOBA_STATIC_SELECT_SCRATCH_BYTES

STATUS = {
    0: "VMOBA_OK", -1: "VMOBA_ERR_ARG", -2: "VMOBA_ERR_SHAPE", -3: "VMOBA_ERR_DTYPE",
    -4: "VMOBA_ERR_WORKSPACE", -5: "VMOBA_ERR_CUDA", -6: "VMOBA_ERR_TIMEOUT",
    -7: "VMOBA_ERR_NOT_IMPLEMENTED", -8: "VMOBA_ERR_DEVICE",
}


class VmobaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")


class CShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("mode", ctypes.c_int),
                ("bt", ctypes.c_int), ("bh", ctypes.c_int), ("bw", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class TraceEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int), ("ms", ctypes.c_double)]


HEAD_STATS_DTYPE = np.dtype([("n_selected", "<i8"), ("mass", "<f8"), ("cut_score", "<f4"),
                             ("all_selected", "<i4")])


@dataclass(frozen=True)
class LayerShape:
    """One layer's problem: latent grid, heads, partition mode and block box."""
    T: int
    H: int
    W: int
    n_heads: int
    head_dim: int
    mode: int
    bt: int
    bh: int
    bw: int
    dtype: str = "bf16"             # "bf16" or "f32"

    @property
    def s(self) -> int:
        return self.T * self.H * self.W

    def c(self) -> CShape:
        return CShape(self.T, self.H, self.W, self.n_heads, self.head_dim, self.mode,
                      self.bt, self.bh, self.bw,
                      VMOBA_BF16 if self.dtype == "bf16" else VMOBA_F32)


_LIB = None


def lib() -> ctypes.CDLL:
    """Load libvmoba.so once; raise if it is missing (no fallback path exists)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m block_sparse_attention_layer_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.POINTER(CShape)
    I, F, Z = ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "vmoba_mode_for_layer": (I, [I]),
        "vmoba_num_blocks": (I, [S]),
        "vmoba_workspace_size": (Z, [S]),
        "vmoba_workspace_size_bounded": (Z, [S, ctypes.c_double]),
        "vmoba_bwd_workspace_size": (Z, [S]),
        "vmoba_partition": (I, [S, P, P, P, P, P, P]),
        "vmoba_score_select": (I, [S, P, P, F, F, P, P, P, Z, P]),
        "vmoba_score_select_variant": (I, [S, P, P, I, ctypes.c_double, F, P, P, P, Z, P]),
        "vmoba_build_plan": (I, [S, P, P, Z, P]),
        "vmoba_attn_fwd": (I, [S, P, P, P, P, P, Z, F, P, P, P]),
        "vmoba_attn_bwd": (I, [S, P, P, P, P, P, Z, F, P, P, P, P, P, P, Z, P]),
        "vmoba_get_status": (I, [P, ctypes.POINTER(I), P]),
        "vmoba_debug_set_wait": (I, [ctypes.c_longlong, I]),
        "vmoba_status_string": (ctypes.c_char_p, [I]),
        "vmoba_last_cuda_error": (ctypes.c_char_p, []),
        "vmoba_kernel_launches": (ctypes.c_ulonglong, []),
        "vmoba_score_select_static": (I, [S, P, P, F, F, P, P, P]),
        "vmoba_trace_enable": (I, [I]),
        "vmoba_trace_read": (I, [ctypes.POINTER(TraceEntry), I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        err = VmobaError(fn, rc)
        if rc == -5:        # VMOBA_ERR_CUDA: name the CUDA error behind it
            err.args = (f"{err.args[0]} ({lib().vmoba_last_cuda_error().decode()})",)
        raise err


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _torch_dtype(shape: LayerShape):
    import torch
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def _expect(t, shape_tuple, dtype, name):
    if tuple(t.shape) != tuple(shape_tuple):
        raise ValueError(f"{name}: expected shape {tuple(shape_tuple)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")


# ---------------------------------------------------------------- raw ABI

def mode_for_layer(layer: int) -> int:
    return lib().vmoba_mode_for_layer(layer)


def num_blocks(shape: LayerShape) -> int:
    n = lib().vmoba_num_blocks(ctypes.byref(shape.c()))
    if n < 0:
        raise VmobaError("vmoba_num_blocks", n)
    return n


def workspace_size(shape: LayerShape, max_pair_fraction: float | None = None) -> int:
    """Workspace bytes of a layer: for every pair selected, or (with
    max_pair_fraction) for selections keeping at most that share of each
    head's pool -- tau for the method's threshold selection."""
    if max_pair_fraction is None:
        return lib().vmoba_workspace_size(ctypes.byref(shape.c()))
    return lib().vmoba_workspace_size_bounded(ctypes.byref(shape.c()), float(max_pair_fraction))


def bwd_workspace_size(shape: LayerShape) -> int:
    return lib().vmoba_bwd_workspace_size(ctypes.byref(shape.c()))


def sel_words(shape: LayerShape) -> int:
    return (num_blocks(shape) + 31) // 32


def partition(shape, k, v, k_perm, v_perm, blocks, stream=None):
    """Step 1: K', V' in partition order and the fp32 block means B."""
    dt = _torch_dtype(shape)
    s, h, d = shape.s, shape.n_heads, shape.head_dim
    _expect(k, (s, h, d), dt, "k")
    _expect(v, (s, h, d), dt, "v")
    _expect(k_perm, (h, s, d), dt, "k_perm")
    _expect(v_perm, (h, s, d), dt, "v_perm")
    import torch
    _expect(blocks, (h, num_blocks(shape), d), torch.float32, "blocks")
    _check("vmoba_partition", lib().vmoba_partition(
        ctypes.byref(shape.c()), _ptr(k), _ptr(v), _ptr(k_perm), _ptr(v_perm), _ptr(blocks),
        _stream(stream)))


def _check_common(shape, q=None, k_perm=None, v_perm=None, sel_bits=None, ws=None):
    import torch
    dt = _torch_dtype(shape)
    s, h, d = shape.s, shape.n_heads, shape.head_dim
    if q is not None:
        _expect(q, (s, h, d), dt, "q")
    if k_perm is not None:
        _expect(k_perm, (h, s, d), dt, "k_perm")
    if v_perm is not None:
        _expect(v_perm, (h, s, d), dt, "v_perm")
    if sel_bits is not None:
        _expect(sel_bits, (h, s, sel_words(shape)), torch.int32, "sel_bits")
    if ws is not None and ws.numel() * ws.element_size() < workspace_size(shape, 1e-300):
        raise ValueError("workspace smaller than the smallest vmoba_workspace_size_bounded")


def score_select(shape, q, blocks, tau, scale, sel_bits, stats, ws, stream=None):
    """Steps 2-3: scores, global threshold selection -> bitmap + per-head stats."""
    import torch
    _check_common(shape, q=q, sel_bits=sel_bits, ws=ws)
    _expect(blocks, (shape.n_heads, num_blocks(shape), shape.head_dim), torch.float32, "blocks")
    if stats.numel() * stats.element_size() < shape.n_heads * HEAD_STATS_DTYPE.itemsize:
        raise ValueError("stats buffer too small")
    _check("vmoba_score_select", lib().vmoba_score_select(
        ctypes.byref(shape.c()), _ptr(q), _ptr(blocks), float(tau), float(scale),
        _ptr(sel_bits), _ptr(stats), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


# selection variants of the ablation (include/vmoba.h: vmoba_score_select_variant)
SELECT_THRESHOLD_GLOBAL, SELECT_TOPK_GLOBAL, SELECT_THRESHOLD_LOCAL, SELECT_TOPK_LOCAL = 0, 1, 2, 3
SELECT_VARIANTS = {"threshold_global": 0, "topk_global": 1, "threshold_local": 2, "topk_local": 3,
                   "rownorm_global": 4}


def score_select_variant(shape, q, blocks, variant, param, scale, sel_bits, stats, ws,
                         stream=None):
    """Steps 2-3 with one of the ablation's selection rules: variant is a
    SELECT_* code or a SELECT_VARIANTS name; param is tau or k."""
    import torch
    if isinstance(variant, str):
        variant = SELECT_VARIANTS[variant]
    _check_common(shape, q=q, sel_bits=sel_bits, ws=ws)
    _expect(blocks, (shape.n_heads, num_blocks(shape), shape.head_dim), torch.float32, "blocks")
    if stats.numel() * stats.element_size() < shape.n_heads * HEAD_STATS_DTYPE.itemsize:
        raise ValueError("stats buffer too small")
    _check("vmoba_score_select_variant", lib().vmoba_score_select_variant(
        ctypes.byref(shape.c()), _ptr(q), _ptr(blocks), int(variant), float(param), float(scale),
        _ptr(sel_bits), _ptr(stats), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def score_select_static(shape, q, blocks, tau, scale, sel_bits, stats, stream=None):
    """Steps 2-3 with the library's fixed static scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/vmoba.h)."""
    import torch
    _check_common(shape, q=q, sel_bits=sel_bits)
    _expect(blocks, (shape.n_heads, num_blocks(shape), shape.head_dim), torch.float32, "blocks")
    if stats.numel() * stats.element_size() < shape.n_heads * HEAD_STATS_DTYPE.itemsize:
        raise ValueError("stats buffer too small")
    _check("vmoba_score_select_static", lib().vmoba_score_select_static(
        ctypes.byref(shape.c()), _ptr(q), _ptr(blocks), float(tau), float(scale),
        _ptr(sel_bits), _ptr(stats), _stream(stream)))


def build_plan(shape, sel_bits, ws, stream=None):
    _check_common(shape, sel_bits=sel_bits, ws=ws)
    _check("vmoba_build_plan", lib().vmoba_build_plan(
        ctypes.byref(shape.c()), _ptr(sel_bits), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def attn_fwd(shape, q, k_perm, v_perm, sel_bits, ws, scale, out, lse, stream=None):
    import torch
    _check_common(shape, q, k_perm, v_perm, sel_bits, ws)
    _expect(out, (shape.s, shape.n_heads, shape.head_dim), _torch_dtype(shape), "out")
    _expect(lse, (shape.n_heads, shape.s), torch.float32, "lse")
    _check("vmoba_attn_fwd", lib().vmoba_attn_fwd(
        ctypes.byref(shape.c()), _ptr(q), _ptr(k_perm), _ptr(v_perm), _ptr(sel_bits), _ptr(ws),
        ws.numel() * ws.element_size(), float(scale), _ptr(out), _ptr(lse), _stream(stream)))


def attn_bwd(shape, q, k_perm, v_perm, sel_bits, ws, scale, lse, dout, dq, dk, dv, ws_bwd,
             stream=None):
    """Step 4c; ``ws`` must hold the preceding attn_fwd's fp32 output copy."""
    import torch
    _check_common(shape, q, k_perm, v_perm, sel_bits, ws)
    full = (shape.s, shape.n_heads, shape.head_dim)
    for name, t in (("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        _expect(t, full, _torch_dtype(shape), name)
    _expect(lse, (shape.n_heads, shape.s), torch.float32, "lse")
    if ws_bwd.numel() * ws_bwd.element_size() < bwd_workspace_size(shape):
        raise ValueError("backward workspace smaller than vmoba_bwd_workspace_size")
    _check("vmoba_attn_bwd", lib().vmoba_attn_bwd(
        ctypes.byref(shape.c()), _ptr(q), _ptr(k_perm), _ptr(v_perm), _ptr(sel_bits), _ptr(ws),
        ws.numel() * ws.element_size(), float(scale), _ptr(lse), _ptr(dout),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws_bwd), ws_bwd.numel() * ws_bwd.element_size(),
        _stream(stream)))


def debug_set_wait(wait_cycles: int = 0, skip_forward_loads: bool = False) -> None:
    """Diagnostics for tests of the bounded-wait path (vmoba_debug_set_wait):
    a spin budget in SM cycles (0 = the default) and whether the forward's
    key/value producer issues nothing, so that the waits run out."""
    _check("vmoba_debug_set_wait",
           lib().vmoba_debug_set_wait(int(wait_cycles), 1 if skip_forward_loads else 0))


def get_status(ws, stream=None) -> int:
    v = ctypes.c_int(0)
    _check("vmoba_get_status", lib().vmoba_get_status(_ptr(ws), ctypes.byref(v), _stream(stream)))
    return v.value


def trace_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (per-kernel timing)."""
    lib().vmoba_trace_enable(1 if on else 0)


def trace_read() -> dict:
    """{kernel name: (launches, device ms)} since the last read; clears the trace."""
    buf = (TraceEntry * 256)()
    n = lib().vmoba_trace_read(buf, len(buf))
    return {buf[i].name.decode(): (buf[i].launches, buf[i].ms) for i in range(min(n, len(buf)))}


def kernel_launches() -> int:
    """Kernels libvmoba has launched since load (its own host-side counter)."""
    return int(lib().vmoba_kernel_launches())


def decode_stats(stats_tensor) -> np.ndarray:
    """Device vmoba_head_stats[n_heads] (a uint8 tensor) -> numpy structured array."""
    raw = stats_tensor.detach().cpu().numpy().tobytes()
    return np.frombuffer(raw, dtype=HEAD_STATS_DTYPE)


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
