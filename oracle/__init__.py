"""CPU oracle for the SageAttention quantized attention forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may use this package; the product
path never does.  The arithmetic lives in ``sage_oracle.c`` (plain scalar C,
built with gcc, no FMA contraction); this module only marshals numpy arrays
and fans independent heads out over a thread pool (ctypes releases the GIL).

Every function cites the passage it follows in ``sage_oracle.c``.  What each
oracle function is pinned by is listed in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

TILE = 128  # keys per online-softmax block (the kernel's K tile)


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (IEEE semantics: no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True, cwd=_HERE)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f32, f64, u8 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_uint8
        L.or_e4m3_decode.argtypes, L.or_e4m3_decode.restype = [u8], f32
        L.or_e4m3_encode.argtypes, L.or_e4m3_encode.restype = [f32], u8
        L.or_e2m1_decode.argtypes, L.or_e2m1_decode.restype = [u8], f32
        L.or_e2m1_encode.argtypes, L.or_e2m1_encode.restype = [f32], u8
        L.or_mean_rows.argtypes = [P, i64, i32, P]
        L.or_block_means.argtypes = [P, i64, i32, i32, P]
        L.or_quant_int8.argtypes = [P, i64, i32, i32, P, i32, P, P]
        L.or_quant_fp8_per_channel.argtypes = [P, i64, i32, P, P]
        L.or_delta_s.argtypes = [P, i64, P, P, i64, i32, P]
        L.or_quant_nvfp4_rows.argtypes = [P, i64, i32, i32, P, i32, P, P]
        L.or_quant_nvfp4_cols.argtypes = [P, i64, i32, P, P]
        L.or_attn_core.argtypes = [P, P, P, P, P, P, i32, P, i64, i32, i32, i32, f64, i32, i32, i64, i64, P, P]
        L.or_attn_naive_f64.argtypes = [P, P, P, i64, i32, i32, f64, i64, i64, P]
        for name in ("or_mean_rows", "or_block_means", "or_quant_int8", "or_quant_fp8_per_channel",
                     "or_delta_s", "or_quant_nvfp4_rows", "or_quant_nvfp4_cols", "or_attn_core",
                     "or_attn_naive_f64"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _ok(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def _f32(x) -> np.ndarray:
    """Exact widening of fp16/bf16 host tensors (torch or numpy) to fp32 numpy."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _pool(n_jobs: int, threads: Optional[int]):
    t = threads or os.cpu_count() or 1
    return ThreadPoolExecutor(max_workers=max(1, min(t, n_jobs)))


# ---------------------------------------------------------------- codecs
def e4m3_encode(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.or_e4m3_encode(float(v)) for v in x], dtype=np.uint8)


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    L = lib()
    c = np.asarray(c, dtype=np.uint8).ravel()
    return np.array([L.or_e4m3_decode(int(v)) for v in c], dtype=np.float32)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.or_e2m1_encode(float(v)) for v in x], dtype=np.uint8)


def e2m1_decode(c: np.ndarray) -> np.ndarray:
    L = lib()
    c = np.asarray(c, dtype=np.uint8).ravel()
    return np.array([L.or_e2m1_decode(int(v)) for v in c], dtype=np.float32)


E4M3_TABLE = None
E2M1_TABLE = None


def e4m3_table() -> np.ndarray:
    global E4M3_TABLE
    if E4M3_TABLE is None:
        E4M3_TABLE = e4m3_decode(np.arange(256, dtype=np.uint8))
    return E4M3_TABLE


def e2m1_table() -> np.ndarray:
    global E2M1_TABLE
    if E2M1_TABLE is None:
        E2M1_TABLE = e2m1_decode(np.arange(16, dtype=np.uint8))
    return E2M1_TABLE


# ---------------------------------------------------------------- preprocessing
def mean_rows(X: np.ndarray) -> np.ndarray:
    X = _f32(X)
    out = np.empty(X.shape[1], np.float32)
    _ok(lib().or_mean_rows(_p(X), X.shape[0], X.shape[1], _p(out)), "mean_rows")
    return out


def block_means(X: np.ndarray, blk: int) -> np.ndarray:
    X = _f32(X)
    T = -(-X.shape[0] // blk)
    out = np.empty((T, X.shape[1]), np.float32)
    _ok(lib().or_block_means(_p(X), X.shape[0], X.shape[1], blk, _p(out)), "block_means")
    return out


def quant_int8(X: np.ndarray, blk: int, mean: Optional[np.ndarray] = None, mean_per_block: bool = False):
    X = _f32(X)
    rows, d = X.shape
    T = -(-rows // blk)
    out = np.empty((rows, d), np.int8)
    sc = np.empty(T, np.float32)
    mean = None if mean is None else np.ascontiguousarray(mean, np.float32)
    _ok(lib().or_quant_int8(_p(X), rows, d, blk, _p(mean), int(mean_per_block), _p(out), _p(sc)), "quant_int8")
    return out, sc


def quant_fp8_per_channel(V: np.ndarray):
    V = _f32(V)
    out = np.empty(V.shape, np.uint8)
    sv = np.empty(V.shape[1], np.float32)
    _ok(lib().or_quant_fp8_per_channel(_p(V), V.shape[0], V.shape[1], _p(out), _p(sv)), "quant_fp8")
    return out, sv


def delta_s(qbar: np.ndarray, K: np.ndarray, km: Optional[np.ndarray]) -> np.ndarray:
    qbar = np.ascontiguousarray(qbar, np.float32)
    K = _f32(K)
    km = None if km is None else np.ascontiguousarray(km, np.float32)
    out = np.empty((qbar.shape[0], K.shape[0]), np.float32)
    _ok(lib().or_delta_s(_p(qbar), qbar.shape[0], _p(K), _p(km), K.shape[0], K.shape[1], _p(out)), "delta_s")
    return out


def quant_nvfp4_rows(X: np.ndarray, blk: int, mean: Optional[np.ndarray] = None, mean_per_block: bool = False):
    X = _f32(X)
    rows, d = X.shape
    codes = np.empty((rows, d), np.uint8)
    sf = np.empty((rows, d // 16), np.uint8)
    mean = None if mean is None else np.ascontiguousarray(mean, np.float32)
    _ok(lib().or_quant_nvfp4_rows(_p(X), rows, d, blk, _p(mean), int(mean_per_block), _p(codes), _p(sf)),
        "quant_nvfp4_rows")
    return codes, sf


def quant_nvfp4_cols(V: np.ndarray):
    V = _f32(V)
    rows, d = V.shape
    codes = np.empty((rows, d), np.uint8)
    sf = np.empty((-(-rows // 16), d), np.uint8)
    _ok(lib().or_quant_nvfp4_cols(_p(V), rows, d, _p(codes), _p(sf)), "quant_nvfp4_cols")
    return codes, sf


def quantize_sage(q, k, v, *, bq: int, bk: int, smooth_k: bool = True, smooth_q: bool = False,
                  threads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Preprocessing of SageAttention2 Algorithm 1 for [B, H, N, d] host tensors.

    Returns q8 [B,Hq,N,d] int8, s_q [B,Hq,Tm], k8 [B,Hkv,N,d], s_k [B,Hkv,Tn],
    km [B,Hkv,d], v8 [B,Hkv,N,d] (E4M3 codes, natural layout), s_v [B,Hkv,d],
    and when smooth_q: qbar [B,Hq,Tm,d], dS [B,Hq,Tm,N].
    """
    Q, K, V = _f32(q), _f32(k), _f32(v)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    Tm, Tn = -(-N // bq), -(-N // bk)
    res = {
        "q8": np.empty((B, Hq, N, d), np.int8), "s_q": np.empty((B, Hq, Tm), np.float32),
        "k8": np.empty((B, Hkv, N, d), np.int8), "s_k": np.empty((B, Hkv, Tn), np.float32),
        "km": np.zeros((B, Hkv, d), np.float32),
        "v8": np.empty((B, Hkv, N, d), np.uint8), "s_v": np.empty((B, Hkv, d), np.float32),
    }
    if smooth_q:
        res["qbar"] = np.empty((B, Hq, Tm, d), np.float32)
        res["dS"] = np.empty((B, Hq, Tm, N), np.float32)

    def kv_job(b, g):
        if smooth_k:
            res["km"][b, g] = mean_rows(K[b, g])
        res["k8"][b, g], res["s_k"][b, g] = quant_int8(K[b, g], bk, res["km"][b, g] if smooth_k else None)
        res["v8"][b, g], res["s_v"][b, g] = quant_fp8_per_channel(V[b, g])

    def q_job(b, h):
        g = h // G
        if smooth_q:
            qb = block_means(Q[b, h], bq)
            res["qbar"][b, h] = qb
            res["q8"][b, h], res["s_q"][b, h] = quant_int8(Q[b, h], bq, qb, True)
            res["dS"][b, h] = delta_s(qb, K[b, g], res["km"][b, g] if smooth_k else None)
        else:
            res["q8"][b, h], res["s_q"][b, h] = quant_int8(Q[b, h], bq, None)

    with _pool(B * Hkv, threads) as ex:
        list(ex.map(lambda bg: kv_job(*bg), [(b, g) for b in range(B) for g in range(Hkv)]))
    with _pool(B * Hq, threads) as ex:
        list(ex.map(lambda bh: q_job(*bh), [(b, h) for b in range(B) for h in range(Hq)]))
    return res


# ---------------------------------------------------------------- attention
def _attn_core(Qv, Kv, Vv, row_scale, col_scale, dS, bq, out_scale, N, d, causal, sm_scale,
               p_mode, round32, r0, r1, tile=TILE, with_lse=False):
    out = np.empty((r1 - r0, d), np.float64)
    lse = np.empty(r1 - r0, np.float64) if with_lse else None
    _ok(lib().or_attn_core(_p(Qv), _p(Kv), _p(Vv), _p(row_scale), _p(col_scale), _p(dS), int(bq),
                           _p(out_scale), N, d, tile, int(causal), float(sm_scale), int(p_mode),
                           int(round32), int(r0), int(r1), _p(out), _p(lse)), "attn_core")
    return (out, lse) if with_lse else out


def attention_sage_head(quant: Dict[str, np.ndarray], b: int, h: int, r0: int, r1: int, *,
                        bq: int, bk: int, causal: bool, sm_scale: float, tile: int = TILE,
                        with_lse: bool = False):
    """SageAttention2 Algorithm 1 (INT8 QK^T, E4M3 P~*448, FP8 PV, two-level FP32
    accumulation, final / 448 * delta_V) for rows [r0, r1) of head (b, h).
    with_lse: also the rows' log-sum-exp of the scores the algorithm uses (those
    of the smoothed K; add lse_smooth_k_correction for the unsmoothed keys)."""
    Hq, Hkv = quant["q8"].shape[1], quant["k8"].shape[1]
    g = h // (Hq // Hkv)
    N, d = quant["q8"].shape[2], quant["q8"].shape[3]
    Qv = np.ascontiguousarray(quant["q8"][b, h], np.float64)
    Kv = np.ascontiguousarray(quant["k8"][b, g], np.float64)
    Vv = np.ascontiguousarray(e4m3_table()[quant["v8"][b, g]], np.float64)
    row_scale = np.ascontiguousarray(np.repeat(quant["s_q"][b, h].astype(np.float64), bq)[:N])
    col_scale = np.ascontiguousarray(np.repeat(quant["s_k"][b, g].astype(np.float64), bk)[:N])
    dS = np.ascontiguousarray(quant["dS"][b, h]) if "dS" in quant else None
    out_scale = np.ascontiguousarray(quant["s_v"][b, g], np.float64)
    return _attn_core(Qv, Kv, Vv, row_scale, col_scale, dS, bq, out_scale, N, d, causal, sm_scale,
                      1, 1, r0, r1, tile, with_lse)


def lse_smooth_k_correction(q, quant: Dict[str, np.ndarray], b: int, h: int, r0: int, r1: int, *,
                            sm_scale: float) -> np.ndarray:
    """Smooth K subtracts km from every key, which shifts row i's scores by the
    constant sm_scale (Q_i . km): softmax is unchanged, the log-sum-exp is not.
    Adding this (fp64) to the log-sum-exp of the smoothed scores gives the one
    over the original keys (SageAttention2 note, "Smooth K" and its
    "softmax invariance" remark).  km is zero without smooth K."""
    Hq, Hkv = quant["q8"].shape[1], quant["k8"].shape[1]
    g = h // (Hq // Hkv)
    Q = np.asarray(_f32(q[b, h]), np.float64)[r0:r1]
    return sm_scale * (Q @ quant["km"][b, g].astype(np.float64))


def attention_exact_head(q, k, v, b: int, h: int, r0: int, r1: int, *, causal: bool, sm_scale: float):
    """fp64 softmax(Q K^T * sm_scale) V for rows [r0, r1) of head (b, h) (GQA: kv head h // G)."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = h // (Hq // Hkv)
    Q = np.ascontiguousarray(_f32(q[b, h]), np.float64)
    K = np.ascontiguousarray(_f32(k[b, g]), np.float64)
    V = np.ascontiguousarray(_f32(v[b, g]), np.float64)
    N, d = Q.shape
    out = np.empty((r1 - r0, d), np.float64)
    _ok(lib().or_attn_naive_f64(_p(Q), _p(K), _p(V), N, d, int(causal), float(sm_scale), r0, r1, _p(out)),
        "attn_naive")
    return out


def attention_blocked_f64_head(q, k, v, b: int, h: int, r0: int, r1: int, *, causal: bool,
                               sm_scale: float, tile: int = TILE, with_lse: bool = False):
    """The oracle's blocked online softmax with identity codecs, all in fp64."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = h // (Hq // Hkv)
    Q = np.ascontiguousarray(_f32(q[b, h]), np.float64)
    K = np.ascontiguousarray(_f32(k[b, g]), np.float64)
    V = np.ascontiguousarray(_f32(v[b, g]), np.float64)
    N, d = Q.shape
    return _attn_core(Q, K, V, None, None, None, 1, None, N, d, causal, sm_scale, 0, 0, r0, r1, tile, with_lse)


# ---------------------------------------------------------------- NVFP4 (SageAttention3)
def quantize_nvfp4(q, k, v, *, bq: int, smooth_k: bool = True, smooth_q: bool = True,
                   threads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """SageAttention3-style preprocessing: smooth K (mean), smooth Q per bq-row block
    with delta_S, then E2M1 codes with one E4M3 scale per 16 elements (along d for
    Q/K, along tokens for V).  Codes are one per byte here."""
    Q, K, V = _f32(q), _f32(k), _f32(v)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    Tm = -(-N // bq)
    res = {
        "q4": np.empty((B, Hq, N, d), np.uint8), "sfq": np.empty((B, Hq, N, d // 16), np.uint8),
        "k4": np.empty((B, Hkv, N, d), np.uint8), "sfk": np.empty((B, Hkv, N, d // 16), np.uint8),
        "v4": np.empty((B, Hkv, N, d), np.uint8), "sfv": np.empty((B, Hkv, -(-N // 16), d), np.uint8),
        "km": np.zeros((B, Hkv, d), np.float32),
    }
    if smooth_q:
        res["qbar"] = np.empty((B, Hq, Tm, d), np.float32)
        res["dS"] = np.empty((B, Hq, Tm, N), np.float32)

    def kv_job(b, g):
        if smooth_k:
            res["km"][b, g] = mean_rows(K[b, g])
        res["k4"][b, g], res["sfk"][b, g] = quant_nvfp4_rows(K[b, g], N, res["km"][b, g] if smooth_k else None)
        res["v4"][b, g], res["sfv"][b, g] = quant_nvfp4_cols(V[b, g])

    def q_job(b, h):
        g = h // G
        if smooth_q:
            qb = block_means(Q[b, h], bq)
            res["qbar"][b, h] = qb
            res["q4"][b, h], res["sfq"][b, h] = quant_nvfp4_rows(Q[b, h], bq, qb, True)
            res["dS"][b, h] = delta_s(qb, K[b, g], res["km"][b, g] if smooth_k else None)
        else:
            res["q4"][b, h], res["sfq"][b, h] = quant_nvfp4_rows(Q[b, h], bq, None)

    with _pool(B * Hkv, threads) as ex:
        list(ex.map(lambda bg: kv_job(*bg), [(b, g) for b in range(B) for g in range(Hkv)]))
    with _pool(B * Hq, threads) as ex:
        list(ex.map(lambda bh: q_job(*bh), [(b, h) for b in range(B) for h in range(Hq)]))
    return res


def dequant_nvfp4_rows(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    vals = e2m1_table()[codes].astype(np.float64)
    scales = np.repeat(e4m3_table()[sf].astype(np.float64), 16, axis=-1)
    return vals * scales


def dequant_nvfp4_cols(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    N = codes.shape[-2]
    vals = e2m1_table()[codes].astype(np.float64)
    scales = np.repeat(e4m3_table()[sf].astype(np.float64), 16, axis=-2)[..., :N, :]
    return vals * scales


def attention_nvfp4_head(quant: Dict[str, np.ndarray], b: int, h: int, r0: int, r1: int, *,
                         bq: int, causal: bool, sm_scale: float, tile: int = TILE) -> np.ndarray:
    """SageAttention3-style attention for rows [r0, r1) of head (b, h): FP4 QK^T,
    + delta_S, online softmax, two-level P quantisation (s_P1 = rowmax/2688,
    s_P2 = E4M3(amax16/6)), FP4 PV, two-level FP32 accumulation."""
    Hq, Hkv = quant["q4"].shape[1], quant["k4"].shape[1]
    g = h // (Hq // Hkv)
    N, d = quant["q4"].shape[2], quant["q4"].shape[3]
    Qv = np.ascontiguousarray(dequant_nvfp4_rows(quant["q4"][b, h], quant["sfq"][b, h]))
    Kv = np.ascontiguousarray(dequant_nvfp4_rows(quant["k4"][b, g], quant["sfk"][b, g]))
    Vv = np.ascontiguousarray(dequant_nvfp4_cols(quant["v4"][b, g], quant["sfv"][b, g]))
    dS = np.ascontiguousarray(quant["dS"][b, h]) if "dS" in quant else None
    return _attn_core(Qv, Kv, Vv, None, None, dS, bq, None, N, d, causal, sm_scale, 2, 1, r0, r1, tile)


# ---------------------------------------------------------------- metrics
def metrics(ref: np.ndarray, out: np.ndarray) -> Dict[str, float]:
    """CosSim, relative L1, RMSE and max-abs over the flattened tensors (the
    accuracy metrics named in the SageAttention2 note, Tables 4 and 6)."""
    a = np.asarray(ref, np.float64).ravel()
    b = np.asarray(out, np.float64).ravel()
    cos = float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))
    return {
        "cos": cos,
        "rel_l1": float(np.abs(a - b).sum() / (np.abs(a).sum() + 1e-300)),
        "rmse": float(np.sqrt(np.mean((a - b) ** 2))),
        "max_abs": float(np.abs(a - b).max()) if a.size else 0.0,
    }
