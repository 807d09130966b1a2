"""Thin ctypes binding of libsage (C ABI in include/sage.h).

Argument marshalling only: torch supplies device memory and the current
stream; every step of the attention path runs in the CUDA library.  If the
library is missing or fails to load, every entry point raises -- there is no
fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libsage.so")

SAGE_OK = 0
STATUS_NAMES = {
    0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED_HEADDIM",
    3: "SAGE_ERR_UNSUPPORTED_DTYPE", 4: "SAGE_ERR_UNSUPPORTED_ARCH", 5: "SAGE_ERR_WORKSPACE_TOO_SMALL",
    6: "SAGE_ERR_CUDA", 7: "SAGE_ERR_TIMEOUT", 8: "SAGE_ERR_MISALIGNED",
}
EXPORTED = ("sage_workspace_bytes", "sage_quant_qkv", "sage_attn_fwd_quantized", "sage_attn_fwd",
            "sage_debug_qk_int32", "sage_last_device_error", "sage_debug_bounded_wait",
            "sage_status_string", "sage_attn_fwd_noalloc", "sage_debug_f8_accum_probe",
            "sage_nvfp4_workspace_bytes", "sage_quant_nvfp4", "sage_attn_fwd_nvfp4_quantized",
            "sage_attn_fwd_nvfp4", "sage_debug_qk_nvfp4", "sage_debug_exp2_poly",
            "sage_debug_kv_quant_two_pass", "sage_quant_kernel_count", "sage_quant_nvfp4_kernel_count",
            "sage_attn_fwd_quantized_lse", "sage_attn_fwd_lse", "sage_debug_mma_rate",
            "sage_debug_wait_limit")


class SageError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class SageParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("sm_scale", ctypes.c_float), ("smooth_k", ctypes.c_int32),
                ("smooth_q", ctypes.c_int32), ("bq", ctypes.c_int32), ("bk", ctypes.c_int32),
                ("pv_accum", ctypes.c_int32), ("return_lse", ctypes.c_int32), ("layout", ctypes.c_int32)]


PV_TWO_LEVEL, PV_TMEM_FP32 = 0, 1
LAYOUTS = {"HND": 0, "NHD": 1}


class SageQuantView(ctypes.Structure):
    _fields_ = [("q8", ctypes.c_void_p), ("k8", ctypes.c_void_p), ("v8t", ctypes.c_void_p),
                ("s_q", ctypes.c_void_p), ("s_k", ctypes.c_void_p), ("s_v", ctypes.c_void_p),
                ("km", ctypes.c_void_p), ("qbar", ctypes.c_void_p), ("dS", ctypes.c_void_p),
                ("Np", ctypes.c_int64), ("qkm", ctypes.c_void_p)]


class SageNvfp4View(ctypes.Structure):
    _fields_ = [("q4", ctypes.c_void_p), ("k4", ctypes.c_void_p), ("v4t", ctypes.c_void_p),
                ("sfq", ctypes.c_void_p), ("sfk", ctypes.c_void_p), ("sfv", ctypes.c_void_p),
                ("km", ctypes.c_void_p), ("qbar", ctypes.c_void_p), ("dS", ctypes.c_void_p),
                ("Np", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsage.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libsage.so not built ({LIB_PATH}); run python -m quantized_attention_block_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, V = ctypes.POINTER(SageParams), ctypes.POINTER(SageQuantView)
        vp, i32 = ctypes.c_void_p, ctypes.c_int32
        L.sage_workspace_bytes.argtypes, L.sage_workspace_bytes.restype = [P], ctypes.c_size_t
        L.sage_quant_qkv.argtypes = [vp, vp, vp, P, vp, ctypes.c_size_t, V, vp]
        L.sage_attn_fwd_quantized.argtypes = [V, vp, P, vp]
        L.sage_attn_fwd.argtypes = [vp, vp, vp, vp, P, vp, ctypes.c_size_t, vp]
        L.sage_attn_fwd_quantized_lse.argtypes = [V, vp, vp, P, vp]
        L.sage_attn_fwd_quantized_lse.restype = ctypes.c_int
        L.sage_attn_fwd_lse.argtypes = [vp, vp, vp, vp, vp, P, vp, ctypes.c_size_t, vp]
        L.sage_attn_fwd_lse.restype = ctypes.c_int
        L.sage_debug_qk_int32.argtypes = [V, P, i32, i32, i32, i32, vp, vp]
        L.sage_last_device_error.argtypes = [vp]
        L.sage_debug_bounded_wait.argtypes = [ctypes.c_uint32, vp]
        L.sage_status_string.argtypes, L.sage_status_string.restype = [ctypes.c_int], ctypes.c_char_p
        L.sage_attn_fwd_noalloc.argtypes, L.sage_attn_fwd_noalloc.restype = [vp, vp, vp, vp, P, vp], ctypes.c_int
        L.sage_debug_f8_accum_probe.argtypes, L.sage_debug_f8_accum_probe.restype = [vp, vp], ctypes.c_int
        F = ctypes.POINTER(SageNvfp4View)
        L.sage_nvfp4_workspace_bytes.argtypes, L.sage_nvfp4_workspace_bytes.restype = [P], ctypes.c_size_t
        L.sage_quant_nvfp4.argtypes = [vp, vp, vp, P, vp, ctypes.c_size_t, F, vp]
        L.sage_attn_fwd_nvfp4_quantized.argtypes = [F, vp, P, vp]
        L.sage_attn_fwd_nvfp4.argtypes = [vp, vp, vp, vp, P, vp, ctypes.c_size_t, vp]
        L.sage_debug_qk_nvfp4.argtypes = [F, P, i32, i32, i32, i32, vp, vp]
        L.sage_debug_exp2_poly.argtypes, L.sage_debug_exp2_poly.restype = [vp, vp, i32, vp], ctypes.c_int
        L.sage_debug_kv_quant_two_pass.argtypes, L.sage_debug_kv_quant_two_pass.restype = [i32], ctypes.c_int
        L.sage_debug_mma_rate.argtypes = [i32, i32, i32, i32, ctypes.POINTER(ctypes.c_double), vp]
        L.sage_debug_mma_rate.restype = ctypes.c_int
        L.sage_debug_wait_limit.argtypes, L.sage_debug_wait_limit.restype = [ctypes.c_uint32, vp], ctypes.c_int
        L.sage_quant_kernel_count.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.sage_quant_kernel_count.restype = ctypes.c_int
        L.sage_quant_nvfp4_kernel_count.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.sage_quant_nvfp4_kernel_count.restype = ctypes.c_int
        for n in ("sage_quant_qkv", "sage_attn_fwd_quantized", "sage_attn_fwd", "sage_debug_qk_int32",
                  "sage_last_device_error", "sage_debug_bounded_wait", "sage_quant_nvfp4",
                  "sage_attn_fwd_nvfp4_quantized", "sage_attn_fwd_nvfp4", "sage_debug_qk_nvfp4"):
            getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != SAGE_OK:
        raise SageError(status, what)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_params(q: torch.Tensor, k: torch.Tensor, *, causal: bool = False, sm_scale: Optional[float] = None,
                smooth_k: bool = True, smooth_q: bool = False, bq: int = 128, bk: int = 64,
                pv_accum: int = PV_TWO_LEVEL, return_lse: bool = False, tensor_layout: str = "HND") -> SageParams:
    """Parameters for q [B, Hq, N, d], k [B, Hkv, N, d] (tensor_layout "HND") or
    q [B, N, Hq, d], k [B, N, Hkv, d] ("NHD")."""
    if tensor_layout not in LAYOUTS:
        raise ValueError(f"tensor_layout must be one of {sorted(LAYOUTS)}")
    if tensor_layout == "HND":
        B, Hq, N, d = q.shape
        Hkv = k.shape[1]
    else:
        B, N, Hq, d = q.shape
        Hkv = k.shape[2]
    dt = {torch.bfloat16: 0, torch.float16: 1}.get(q.dtype, -1)
    return SageParams(B, Hq, Hkv, N, d, dt, int(causal), float(sm_scale if sm_scale else 0.0),
                      int(smooth_k), int(smooth_q), bq, bk, int(pv_accum), int(return_lse), LAYOUTS[tensor_layout])


def workspace_bytes(p: SageParams) -> int:
    return int(lib().sage_workspace_bytes(ctypes.byref(p)))


def alloc_workspace(p: SageParams, device=None) -> torch.Tensor:
    n = workspace_bytes(p)
    if n == 0:
        raise SageError(1, "sage_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def sage_quant_qkv(q, k, v, p: SageParams, workspace: torch.Tensor, stream=None) -> SageQuantView:
    view = SageQuantView()
    _check(lib().sage_quant_qkv(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(p), _ptr(workspace),
                                workspace.numel(), ctypes.byref(view), _stream(stream)), "sage_quant_qkv")
    return view


def sage_attn_fwd_quantized(view: SageQuantView, o: torch.Tensor, p: SageParams, stream=None) -> torch.Tensor:
    _check(lib().sage_attn_fwd_quantized(ctypes.byref(view), _ptr(o), ctypes.byref(p), _stream(stream)),
           "sage_attn_fwd_quantized")
    return o


def sage_attn_fwd(q, k, v, *, causal: bool = False, sm_scale: Optional[float] = None, smooth_k: bool = True,
                  smooth_q: bool = False, bq: int = 128, bk: int = 64, pv_accum: int = PV_TWO_LEVEL,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None, tensor_layout: str = "HND") -> torch.Tensor:
    """SageAttention forward: [B,Hq,N,d] x [B,Hkv,N,d] -> [B,Hq,N,d] (input dtype); with
    tensor_layout "NHD" the tensors are [B,N,H,d]."""
    p = make_params(q, k, causal=causal, sm_scale=sm_scale, smooth_k=smooth_k, smooth_q=smooth_q, bq=bq, bk=bk,
                    pv_accum=pv_accum, tensor_layout=tensor_layout)
    if workspace is None:
        workspace = alloc_workspace(p, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sage_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(p), _ptr(workspace),
                               workspace.numel(), _stream(stream)), "sage_attn_fwd")
    return out


def sage_attn_fwd_lse(q, k, v, *, causal: bool = False, sm_scale: Optional[float] = None, smooth_k: bool = True,
                      smooth_q: bool = False, bq: int = 128, bk: int = 64, pv_accum: int = PV_TWO_LEVEL,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None, tensor_layout: str = "HND"):
    """sage_attn_fwd that also returns each row's log-sum-exp of the scores
    (fp32 [B,Hq,N], natural log, for the original keys): (out, lse)."""
    p = make_params(q, k, causal=causal, sm_scale=sm_scale, smooth_k=smooth_k, smooth_q=smooth_q, bq=bq, bk=bk,
                    pv_accum=pv_accum, tensor_layout=tensor_layout)
    if workspace is None:
        workspace = alloc_workspace(p, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((p.B, p.Hq, p.N), dtype=torch.float32, device=q.device)
    _check(lib().sage_attn_fwd_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), ctypes.byref(p),
                                   _ptr(workspace), workspace.numel(), _stream(stream)), "sage_attn_fwd_lse")
    return out, lse


def sage_attn_fwd_quantized_lse(view: SageQuantView, o: torch.Tensor, lse: torch.Tensor, p: SageParams,
                                stream=None) -> None:
    _check(lib().sage_attn_fwd_quantized_lse(ctypes.byref(view), _ptr(o), _ptr(lse), ctypes.byref(p),
                                             _stream(stream)), "sage_attn_fwd_quantized_lse")


def sage_debug_qk_int32(view: SageQuantView, p: SageParams, b: int, h: int, qtile: int, ktile: int,
                        stream=None) -> torch.Tensor:
    out = torch.empty((128, 128), dtype=torch.int32, device="cuda")
    _check(lib().sage_debug_qk_int32(ctypes.byref(view), ctypes.byref(p), b, h, qtile, ktile, _ptr(out),
                                     _stream(stream)), "sage_debug_qk_int32")
    return out


def sage_last_device_error(stream=None) -> int:
    return int(lib().sage_last_device_error(_stream(stream)))


def sage_debug_bounded_wait(timeout_us: int, stream=None) -> int:
    return int(lib().sage_debug_bounded_wait(int(timeout_us), _stream(stream)))


F8_ACCUM_PROBE_EXACT = (1 + 2.0 ** -18, 1 + 2.0 ** -14, 1 + 2.0 ** -12, 256.0, 32.0, 4096 + 2.0 ** -10,
                        1 + 2.0 ** -18, 1 + 2.0 ** -13)


def sage_debug_f8_accum_probe(stream=None) -> torch.Tensor:
    """The 8 probe sums of the FP8 tensor-core accumulator (exact values in F8_ACCUM_PROBE_EXACT)."""
    out = torch.zeros(8, dtype=torch.float32, device="cuda")
    _check(lib().sage_debug_f8_accum_probe(_ptr(out), _stream(stream)), "sage_debug_f8_accum_probe")
    return out


def view_tensors(view: SageQuantView, p: SageParams, workspace: torch.Tensor) -> Dict[str, torch.Tensor]:
    """torch views of the quantised tensors inside the workspace (for inspection)."""
    B, Hq, Hkv, N, d = p.B, p.Hq, p.Hkv, p.N, p.d
    Np = int(view.Np)
    Tm, Tn = -(-N // p.bq), -(-N // p.bk)
    base = workspace.data_ptr()

    def sl(ptr, nbytes, dtype, shape):
        off = ptr - base
        return workspace[off:off + nbytes].view(dtype).view(*shape)

    out = {
        "q8": sl(view.q8, B * Hq * Np * d, torch.int8, (B, Hq, Np, d)),
        "k8": sl(view.k8, B * Hkv * Np * d, torch.int8, (B, Hkv, Np, d)),
        "v8t": sl(view.v8t, B * Hkv * d * Np, torch.uint8, (B, Hkv, d, Np)),
        "s_q": sl(view.s_q, 4 * B * Hq * Tm, torch.float32, (B, Hq, Tm)),
        "s_k": sl(view.s_k, 4 * B * Hkv * Tn, torch.float32, (B, Hkv, Tn)),
        "s_v": sl(view.s_v, 4 * B * Hkv * d, torch.float32, (B, Hkv, d)),
        "km": sl(view.km, 4 * B * Hkv * d, torch.float32, (B, Hkv, d)),
    }
    if view.qkm:
        out["qkm"] = sl(view.qkm, 4 * B * Hq * Np, torch.float32, (B, Hq, Np))
    if view.qbar:
        out["qbar"] = sl(view.qbar, 4 * B * Hq * Tm * d, torch.float32, (B, Hq, Tm, d))
        out["dS"] = sl(view.dS, 4 * B * Hq * Tm * Np, torch.float32, (B, Hq, Tm, Np))
    return out


# ---------------------------------------------------------------- NVFP4 path
def nvfp4_workspace_bytes(p: SageParams) -> int:
    return int(lib().sage_nvfp4_workspace_bytes(ctypes.byref(p)))


def alloc_nvfp4_workspace(p: SageParams, device=None) -> torch.Tensor:
    n = nvfp4_workspace_bytes(p)
    if n == 0:
        raise SageError(1, "sage_nvfp4_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sage_quant_nvfp4(q, k, v, p: SageParams, workspace: torch.Tensor, stream=None) -> SageNvfp4View:
    view = SageNvfp4View()
    _check(lib().sage_quant_nvfp4(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(p), _ptr(workspace),
                                  workspace.numel(), ctypes.byref(view), _stream(stream)), "sage_quant_nvfp4")
    return view


def sage_attn_fwd_nvfp4_quantized(view: SageNvfp4View, o: torch.Tensor, p: SageParams,
                                  stream=None) -> torch.Tensor:
    _check(lib().sage_attn_fwd_nvfp4_quantized(ctypes.byref(view), _ptr(o), ctypes.byref(p), _stream(stream)),
           "sage_attn_fwd_nvfp4_quantized")
    return o


def sage_attn_fwd_nvfp4(q, k, v, *, causal: bool = False, sm_scale: Optional[float] = None,
                        smooth_k: bool = True, smooth_q: bool = True, bq: int = 128,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream=None, tensor_layout: str = "HND") -> torch.Tensor:
    """SageAttention3-style NVFP4 forward: [B,Hq,N,128] x [B,Hkv,N,128] -> [B,Hq,N,128]
    (tensor_layout "NHD": [B,N,H,128])."""
    p = make_params(q, k, causal=causal, sm_scale=sm_scale, smooth_k=smooth_k, smooth_q=smooth_q, bq=bq,
                    tensor_layout=tensor_layout)
    if workspace is None:
        workspace = alloc_nvfp4_workspace(p, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sage_attn_fwd_nvfp4(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(p), _ptr(workspace),
                                     workspace.numel(), _stream(stream)), "sage_attn_fwd_nvfp4")
    return out


def sage_debug_qk_nvfp4(view: SageNvfp4View, p: SageParams, b: int, h: int, qtile: int, ktile: int,
                        stream=None) -> torch.Tensor:
    out = torch.empty((128, 128), dtype=torch.float32, device="cuda")
    _check(lib().sage_debug_qk_nvfp4(ctypes.byref(view), ctypes.byref(p), b, h, qtile, ktile, _ptr(out),
                                     _stream(stream)), "sage_debug_qk_nvfp4")
    return out


def sage_debug_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x of a float32 device tensor through the kernel's FMA-pipe exponential."""
    y = torch.empty_like(x)
    _check(lib().sage_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "sage_debug_exp2_poly")
    return y


MMA_KINDS = {"i8": 0, "f8": 1, "f4": 2}


def sage_debug_mma_rate(kind: str, n: int, iters: int, ctas: int = 0, stream=None) -> float:
    """Enqueue the tensor-core rate probe (one CTA per SM by default) on `stream`
    and return the operation count of that launch; time it with CUDA events."""
    ops = ctypes.c_double(0.0)
    _check(lib().sage_debug_mma_rate(MMA_KINDS[kind], int(n), int(iters), int(ctas), ctypes.byref(ops),
                                     _stream(stream)), "sage_debug_mma_rate")
    return float(ops.value)


def sage_quant_kernel_count(p: SageParams) -> int:
    """Kernels sage_quant_qkv enqueues for p on the current device (memsets not counted)."""
    n = ctypes.c_int32(0)
    _check(lib().sage_quant_kernel_count(ctypes.byref(p), ctypes.byref(n)), "sage_quant_kernel_count")
    return int(n.value)


def sage_quant_nvfp4_kernel_count(p: SageParams) -> int:
    """Kernels sage_quant_nvfp4 enqueues for p on the current device (memsets not counted)."""
    n = ctypes.c_int32(0)
    _check(lib().sage_quant_nvfp4_kernel_count(ctypes.byref(p), ctypes.byref(n)), "sage_quant_nvfp4_kernel_count")
    return int(n.value)


def sage_debug_kv_quant_two_pass(on) -> None:
    """Force (True / 1) or release (False / 0) the two-pass K/V quantisation path in
    this process; 2 forces the one-read path even when a group's tiles may not
    all be resident (a test of its bounded waits)."""
    _check(lib().sage_debug_kv_quant_two_pass(int(on)), "sage_debug_kv_quant_two_pass")


def sage_debug_wait_limit(timeout_us: int, stream=None) -> None:
    """Limit of the in-kernel bounded waits for later launches (0: the default 4 s)."""
    _check(lib().sage_debug_wait_limit(int(timeout_us), _stream(stream)), "sage_debug_wait_limit")


def nvfp4_view_tensors(view: SageNvfp4View, p: SageParams, workspace: torch.Tensor) -> Dict[str, torch.Tensor]:
    """torch views (raw device layouts) of the NVFP4 tensors inside the workspace."""
    B, Hq, Hkv, N, d = p.B, p.Hq, p.Hkv, p.N, p.d
    Np = int(view.Np)
    T, Tm = Np // 128, -(-N // p.bq)
    base = workspace.data_ptr()

    def sl(ptr, nbytes, dtype, shape):
        off = ptr - base
        return workspace[off:off + nbytes].view(dtype).view(*shape)

    out = {
        "q4": sl(view.q4, B * Hq * Np * d // 2, torch.uint8, (B, Hq, Np, d // 2)),
        "k4": sl(view.k4, B * Hkv * Np * d // 2, torch.uint8, (B, Hkv, Np, d // 2)),
        "v4t": sl(view.v4t, B * Hkv * d * Np // 2, torch.uint8, (B, Hkv, d, Np // 2)),
        "sfq": sl(view.sfq, B * Hq * T * 1024, torch.uint8, (B, Hq, T, 1024)),
        "sfk": sl(view.sfk, B * Hkv * T * 1024, torch.uint8, (B, Hkv, T, 1024)),
        "sfv": sl(view.sfv, B * Hkv * T * 1024, torch.uint8, (B, Hkv, T, 1024)),
        "km": sl(view.km, 4 * B * Hkv * d, torch.float32, (B, Hkv, d)),
    }
    if view.qbar:
        out["qbar"] = sl(view.qbar, 4 * B * Hq * Tm * d, torch.float32, (B, Hq, Tm, d))
        out["dS"] = sl(view.dS, 4 * B * Hq * Tm * Np, torch.float32, (B, Hq, Tm, Np))
    return out


def attention_ops(B: int, Hq: int, N: int, d: int, causal: bool) -> float:
    """4 N^2 d per head (two matmuls), halved when causal (the TOPS numerator)."""
    full = 4.0 * B * Hq * N * N * d
    return full / 2 if causal else full
