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
    o = torch.full_like(qd, float("nan"))  # a row the kernel does not write stays NaN
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


def accept_boundary_rows(w: W.Workload, out: np.ndarray, refs: np.ndarray, oracle_row, max_frac: float = 0.01):
    """Output rows that miss the bar only because a quantisation decision sits
    on a rounding boundary.  The kernel forms each exponent argument in fp32
    (one ulp is about 1e-6 of it at |t| ~ 8) and takes the exponential on the
    MUFU, so a code of P whose value lies within that distance of a rounding
    midpoint may round the other way than the oracle's.  For the coarse FP4
    grid that moves one element of P by up to a third, and the row's output by
    a few hundredths.  Several results are then correct.  A failing row is
    accepted when the oracle itself, with the score scale moved by at most
    1e-6 of itself, gives a row the GPU's matches within the bar.  At most
    max_frac of the rows may be accepted that way.  oracle_row(b, h, r,
    sm_scale) -> the oracle's row.  Returns (refs with accepted rows replaced,
    the accepted (b, h, r) list, the rows that stay failing)."""
    refs = refs.copy()
    accepted, failing = [], []
    for b in range(out.shape[0]):
        for h in range(out.shape[1]):
            err = np.abs(refs[b, h] - out[b, h]).max(axis=-1)
            for r in np.nonzero(~(err <= MAX_ABS))[0]:
                r = int(r)
                hit = None
                for f in (1e-7, -1e-7, 2e-7, -2e-7, 5e-7, -5e-7, 1e-6, -1e-6):
                    alt = oracle_row(b, h, r, w.sm_scale * (1.0 + f))
                    if np.abs(alt - out[b, h, r]).max() <= MAX_ABS:
                        hit = alt
                        break
                if hit is None:
                    failing.append((b, h, r))
                else:
                    refs[b, h, r] = hit
                    accepted.append((b, h, r))
    n_rows = out.shape[0] * out.shape[1] * out.shape[2]
    if len(accepted) > max_frac * n_rows:
        failing += accepted
    return refs, accepted, failing


# ---------------------------------------------------------------- NVFP4 path
def sf_index(rows: int) -> np.ndarray:
    """Byte offsets, inside one tile's 1 KB scale block, of scale (m, grp) for
    m < 128, grp < 8: two 512-byte blocks (grp // 4), byte 16 (m % 32) +
    4 (m // 32) + grp % 4 -- the device layout written by sage_quant_nvfp4."""
    m = np.arange(rows)[:, None]
    g = np.arange(8)[None, :]
    return (g // 4) * 512 + 16 * (m % 32) + 4 * (m // 32) + g % 4


def unpack_nibbles(raw: np.ndarray) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] E2M1 codes (even element in the low nibble)."""
    out = np.empty(raw.shape[:-1] + (raw.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = raw & 15
    out[..., 1::2] = raw >> 4
    return out


def unpack_sf(raw: np.ndarray) -> np.ndarray:
    """[..., T, 1024] scale blocks -> [..., T*128, 8] scales per row and 16-group."""
    idx = sf_index(128)
    return raw[..., idx].reshape(raw.shape[:-2] + (raw.shape[-2] * 128, 8))


def gpu_quant_nvfp4(w: W.Workload, q, k, v):
    p = sage.make_params(q, k, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                         smooth_q=w.smooth_q, bq=w.bq, bk=w.bk)
    ws = sage.alloc_nvfp4_workspace(p)
    qd, kd, vd = to_gpu(q, k, v)
    view = sage.sage_quant_nvfp4(qd, kd, vd, p, ws)
    torch.cuda.synchronize()
    return p, ws, view, (qd, kd, vd)


def gpu_attention_nvfp4(w: W.Workload, q, k, v):
    p, ws, view, (qd, kd, vd) = gpu_quant_nvfp4(w, q, k, v)
    o = torch.full_like(qd, float("nan"))  # a row the kernel does not write stays NaN
    sage.sage_attn_fwd_nvfp4_quantized(view, o, p)
    torch.cuda.synchronize()
    assert sage.sage_last_device_error() == 0
    return p, ws, view, o


def oracle_quant_nvfp4(w: W.Workload, q, k, v):
    return oracle.quantize_nvfp4(q, k, v, bq=w.bq, smooth_k=w.smooth_k, smooth_q=w.smooth_q)


def gpu_nvfp4_in_oracle_layout(view, p, ws) -> dict:
    """The GPU's NVFP4 tensors rearranged to the oracle's layouts (codes one per
    byte [.., N, d]; Q/K scales [.., N, d/16]; V scales [.., ceil(N/16), d])."""
    t = {k: x.cpu().numpy() for k, x in sage.nvfp4_view_tensors(view, p, ws).items()}
    N = p.N
    Np = int(view.Np)
    v4 = np.swapaxes(unpack_nibbles(t["v4t"]), 2, 3)             # [B,Hkv,Np,d]
    T = Np // 128
    sfv = np.empty(t["sfv"].shape[:2] + (T * 8, p.d), np.uint8)
    idx = sf_index(128)                                            # [channel, grp]
    for tt in range(T):
        sfv[:, :, tt * 8:(tt + 1) * 8, :] = np.swapaxes(t["sfv"][:, :, tt][..., idx], 2, 3)
    out = {
        "q4": unpack_nibbles(t["q4"])[:, :, :N], "q4_pad": unpack_nibbles(t["q4"])[:, :, N:],
        "sfq": unpack_sf(t["sfq"])[:, :, :N], "sfq_pad": unpack_sf(t["sfq"])[:, :, N:],
        "k4": unpack_nibbles(t["k4"])[:, :, :N], "k4_pad": unpack_nibbles(t["k4"])[:, :, N:],
        "sfk": unpack_sf(t["sfk"])[:, :, :N], "sfk_pad": unpack_sf(t["sfk"])[:, :, N:],
        "v4": v4[:, :, :N], "v4_pad": v4[:, :, N:],
        "sfv": sfv[:, :, :-(-N // 16)], "sfv_pad": sfv[:, :, -(-N // 16):],
        "km": t["km"],
    }
    if "qbar" in t:
        out["qbar"] = t["qbar"]
        out["dS"] = t["dS"]
    return out


def compare_quant_nvfp4(w: W.Workload, g: dict, ref: dict) -> dict:
    """Bit-exact comparison (codes, scales, km, qbar); delta_S within fp32 tolerance."""
    bad = {}
    for name in ("q4", "sfq", "k4", "sfk", "v4", "sfv", "km"):
        a, b = np.asarray(g[name]), np.asarray(ref[name])
        n = int(np.sum(a.view(np.uint32) != b.view(np.uint32))) if a.dtype.kind == "f" else int(np.sum(a != b))
        if n:
            bad[name] = n
    for name in ("q4_pad", "sfq_pad", "k4_pad", "sfk_pad", "v4_pad", "sfv_pad"):
        if np.any(g[name] != 0):
            bad[name] = int(np.count_nonzero(g[name]))
    if w.smooth_q:
        if np.any(g["qbar"].view(np.uint32) != ref["qbar"].view(np.uint32)):
            bad["qbar"] = 1
        dS_g = g["dS"][..., :w.N].astype(np.float64)
        dS_r = ref["dS"].astype(np.float64)
        if np.abs(dS_g - dS_r).max() > 1e-5 * np.abs(dS_r).max() + 1e-6:
            bad["dS"] = float(np.abs(dS_g - dS_r).max())
    return bad


def oracle_rows_nvfp4(w: W.Workload, quant, b, h, r0, r1):
    return oracle.attention_nvfp4_head(quant, b, h, r0, r1, bq=w.bq, causal=w.causal, sm_scale=w.sm_scale)
