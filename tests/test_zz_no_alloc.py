"""sage_attn_fwd_noalloc: the forward for callers that cannot allocate device
memory (they only own their input and output buffers).  It must produce what
the workspace-taking sage_attn_fwd produces, on consecutive calls that reuse
the library's one static scratch array, and reject problems whose scratch
would not fit.  Kept in a file of its own that is collected last."""
import ctypes

import pytest
import torch

from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

from harness import compare_out

pytestmark = pytest.mark.gpu


def _noalloc(qd, kd, vd, w):
    L = sage.lib()
    p = sage.make_params(qd, kd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                         smooth_q=w.smooth_q, bq=w.bq, bk=w.bk)
    o = torch.empty_like(qd)
    st = L.sage_attn_fwd_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), ctypes.byref(p),
                                 torch.cuda.current_stream().cuda_stream)
    return st, o


def _with_workspace(qd, kd, vd, w):
    return sage.sage_attn_fwd(qd, kd, vd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                              smooth_q=w.smooth_q, bq=w.bq, bk=w.bk)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # first call: a larger causal d=128 problem (about 12 MB of scratch);
    # second call: a smaller smooth-Q d=64 problem that reuses the same array
    first = W.get("prefill").with_(name="noalloc_a", B=1, Hq=8, Hkv=8, N=4096)
    second = W.small_variant(W.get("video"), N=600, B=1, Hq=2)
    for w in (first, second):
        q, k, v = W.make_qkv(w)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        st, o = _noalloc(qd, kd, vd, w)
        assert st == 0, sage.STATUS_NAMES.get(st, st)
        ref = _with_workspace(qd, kd, vd, w)
        torch.cuda.synchronize()
        assert sage.sage_last_device_error() == 0
        # same kernels on the same inputs: the outputs must be the same bits (a
        # stale byte left in the shared array by the previous call would show here)
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), w.name
        m, ok = compare_out(ref.float().cpu().numpy(), o.float().cpu().numpy())
        assert ok, (w.name, m)


def test_noalloc_rejects_problems_larger_than_the_static_scratch():
    w = W.get("prefill")  # B4 H32 N4096 d128: ~200 MB of scratch
    q = torch.empty((w.B, w.Hq, w.N, w.d), dtype=w.dtype, device="cuda")
    st, _ = _noalloc(q, q, q, w)
    assert st == 5  # SAGE_ERR_WORKSPACE_TOO_SMALL
