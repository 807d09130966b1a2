"""CPU checks of the C ABI: the library loads without a GPU, exports every
entry point include/sage.h declares, and rejects bad arguments on the host
(no CUDA call is reached)."""
import ctypes
import os
import re

import pytest

from quantized_attention_block_b200 import build as libbuild
from quantized_attention_block_b200 import sage

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return sage.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "sage.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(sage.EXPORTED)


def P(**kw):
    base = dict(B=1, Hq=2, Hkv=2, N=256, d=64, dtype=0, causal=0, sm_scale=0.0, smooth_k=1, smooth_q=0, bq=128, bk=64)
    base.update(kw)
    return sage.SageParams(**base)


def test_workspace_bytes_valid_and_invalid(L):
    p = P()
    n = sage.workspace_bytes(p)
    # at least the three quantised tensors: Q, K (int8) and V (e4m3), padded to 128 rows
    assert n >= 3 * 1 * 2 * 256 * 64
    assert sage.workspace_bytes(P(smooth_q=1)) > n  # + qbar and delta_S
    for bad in (P(d=96), P(Hq=3, Hkv=2), P(N=0), P(bq=16), P(bq=256), P(bk=32), P(bk=256), P(dtype=7),
                P(causal=2), P(return_lse=2), P(layout=2)):
        assert sage.workspace_bytes(bad) == 0
    # one Q scale per 32 rows: INT8/FP8 path only (the NVFP4 smooth-Q block is 64 or 128 rows)
    assert sage.workspace_bytes(P(bq=32)) > 0
    assert sage.nvfp4_workspace_bytes(P(d=128, bq=32)) == 0
    assert sage.nvfp4_workspace_bytes(P(d=128, bq=64)) > 0
    assert sage.workspace_bytes(P(layout=1)) == n  # NHD inputs: the same workspace


def test_entry_points_reject_bad_arguments_on_host(L):
    view = sage.SageQuantView()
    p = P()
    st = L.sage_quant_qkv(None, None, None, ctypes.byref(p), None, 0, ctypes.byref(view), None)
    assert st == 1  # SAGE_ERR_INVALID_ARG
    st = L.sage_quant_qkv(None, None, None, ctypes.byref(P(d=256)), None, 0, ctypes.byref(view), None)
    assert st == 2  # SAGE_ERR_UNSUPPORTED_HEADDIM
    st = L.sage_quant_qkv(None, None, None, ctypes.byref(P(dtype=3)), None, 0, ctypes.byref(view), None)
    assert st == 3  # SAGE_ERR_UNSUPPORTED_DTYPE
    st = L.sage_attn_fwd_quantized(None, None, ctypes.byref(p), None)
    assert st == 1
    st = L.sage_attn_fwd(None, None, None, None, None, None, 0, None)
    assert st == 1
    st = L.sage_debug_qk_int32(None, ctypes.byref(p), 0, 0, 0, 0, None, None)
    assert st == 1
    assert L.sage_status_string(7) == b"SAGE_ERR_TIMEOUT"


def test_noalloc_reports_parameter_errors_like_sage_attn_fwd(L):
    """The no-allocation entry point validates the parameters before it looks at
    the static scratch size, so unsupported parameters get the same status as
    from sage_attn_fwd (checked on the host, no CUDA call is reached)."""
    for bad, want in ((P(d=96), 2), (P(dtype=3), 3), (P(Hq=3, Hkv=2), 1), (P(N=0), 1)):
        st_ws = L.sage_attn_fwd(None, None, None, None, ctypes.byref(bad), None, 0, None)
        st_na = L.sage_attn_fwd_noalloc(None, None, None, None, ctypes.byref(bad), None)
        assert st_na == st_ws == want, (bad.d, bad.dtype, st_na, st_ws)
    assert L.sage_attn_fwd_noalloc(None, None, None, None, None, None) == 1
    # far beyond the 32 MiB static scratch: rejected before any device query
    big = P(B=4, Hq=32, Hkv=32, N=4096, d=128)
    assert L.sage_attn_fwd_noalloc(None, None, None, None, ctypes.byref(big), None) == 5


def test_mma_rate_probe_rejects_bad_shapes_on_host(L):
    ops = ctypes.c_double(0.0)
    for kind, n, iters in ((3, 128, 10), (0, 96, 10), (2, 256, 10), (1, 128, 0), (1, 128, 3_000_000)):
        assert L.sage_debug_mma_rate(kind, n, iters, 0, ctypes.byref(ops), None) == 1, (kind, n, iters)
    assert L.sage_debug_mma_rate(0, 128, 10, 0, None, None) == 1

