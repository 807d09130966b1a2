"""Shared helpers for the parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded host inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

# Output tolerance for floating point parity (stated with the method's target):
# element-wise max-abs <= 1e-2 and cosine >= 0.9999 against the oracle.
MAX_ABS = 1e-2
MIN_COS = 0.9999


def to_gpu(*ts):
    return [t.cuda() for t in ts]


def gpu_quant(w: W.Workload, q, k, v, pv_accum: int = sage.PV_TWO_LEVEL):
    p = sage.make_params(q, k, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                         smooth_q=w.smooth_q, bq=w.bq, bk=w.bk, pv_accum=pv_accum)
    ws = sage.alloc_workspace(p)
    qd, kd, vd = to_gpu(q, k, v)
    view = sage.sage_quant_qkv(qd, kd, vd, p, ws)
    torch.cuda.synchronize()
    return p, ws, view, (qd, kd, vd)


def gpu_attention(w: W.Workload, q, k, v, pv_accum: int = sage.PV_TWO_LEVEL):
    p, ws, view, (qd, kd, vd) = gpu_quant(w, q, k, v, pv_accum)
    o = torch.empty_like(qd)
    sage.sage_attn_fwd_quantized(view, o, p)
    torch.cuda.synchronize()
    assert sage.sage_last_device_error() == 0
    return p, ws, view, o


def oracle_quant(w: W.Workload, q, k, v):
    return oracle.quantize_sage(q, k, v, bq=w.bq, bk=w.bk, smooth_k=w.smooth_k, smooth_q=w.smooth_q)


def compare_quant(w: W.Workload, p, ws, view, ref, heads=None):
    """Bit-exact comparison of the quantised tensors and scales; delta_S within fp32 tolerance."""
    g = {k: t.cpu().numpy() for k, t in sage.view_tensors(view, p, ws).items()}
    N = w.N
    bad = {}

    def eq(name, a, b):
        a, b = np.asarray(a), np.asarray(b)
        if a.dtype.kind == "f":
            n = int(np.sum(a.view(np.uint32) != b.view(np.uint32)))
        else:
            n = int(np.sum(a != b))
        if n:
            bad[name] = n

    eq("q8", g["q8"][:, :, :N], ref["q8"])
    eq("q8_pad", g["q8"][:, :, N:], np.zeros_like(g["q8"][:, :, N:]))
    eq("s_q", g["s_q"], ref["s_q"])
    eq("k8", g["k8"][:, :, :N], ref["k8"])
    eq("k8_pad", g["k8"][:, :, N:], np.zeros_like(g["k8"][:, :, N:]))
    eq("s_k", g["s_k"], ref["s_k"])
    eq("km", g["km"], ref["km"])
    eq("v8", np.swapaxes(g["v8t"], 2, 3)[:, :, :N], ref["v8"])
    eq("v8_pad", g["v8t"][:, :, :, N:], np.zeros_like(g["v8t"][:, :, :, N:]))
    eq("s_v", g["s_v"], ref["s_v"])
    if w.smooth_q:
        eq("qbar", g["qbar"], ref["qbar"])
        dS_g = g["dS"][..., :N].astype(np.float64)
        dS_r = ref["dS"].astype(np.float64)
        tol = 1e-5 * np.abs(dS_r).max() + 1e-6
        err = np.abs(dS_g - dS_r).max()
        if err > tol:
            bad["dS"] = float(err)
        if np.any(g["dS"][..., N:] != 0):
            bad["dS_pad"] = 1
    return bad


def oracle_rows(w: W.Workload, quant, b, h, r0, r1):
    return oracle.attention_sage_head(quant, b, h, r0, r1, bq=w.bq, bk=w.bk, causal=w.causal,
                                      sm_scale=w.sm_scale)


def compare_out(ref: np.ndarray, out: np.ndarray):
    m = oracle.metrics(ref, out)
    return m, (m["max_abs"] <= MAX_ABS and m["cos"] >= MIN_COS and np.isfinite(out).all())
