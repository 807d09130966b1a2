"""Failure detection of the one-read K/V quantiser, tested without a GPU fault.

The one-read kernel keeps each K or V tile in shared memory until every tile
of its (head, K|V) group has added its column statistics; the launcher takes
that path only when a group's tiles fit twice in the CTAs resident at once.
Here a test hook forces it on a head of 1024 tiles, more than one B200 holds
at once, with a 20 ms wait limit: the resident tiles' bounded waits run out,
they record SAGE_ERR_TIMEOUT and return without writing codes (every wait
ends, the context stays usable), and the attention kernel, seeing the unread
error, leaves O untouched instead of computing it from stale codes."""
import pytest
import torch

from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_one_read_wait_timeout_is_reported_and_o_left_unwritten():
    N = 131072  # 1024 tiles per (head, K|V) group
    w = W.get("prefill").with_(name="one_read_timeout", B=1, Hq=1, Hkv=1, N=N, causal=False)
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = sage.make_params(qd, kd, causal=False, sm_scale=w.sm_scale, smooth_k=1, smooth_q=0, bq=w.bq, bk=w.bk)
    assert sage.sage_last_device_error() == 0
    o = torch.full_like(qd, float("nan"))
    try:
        sage.sage_debug_kv_quant_two_pass(2)
        sage.sage_debug_wait_limit(20000)
        assert sage.sage_quant_kernel_count(p) == 2  # the one-read path, forced
        sage.sage_attn_fwd(qd, kd, vd, causal=False, sm_scale=w.sm_scale, smooth_k=1, smooth_q=0, bq=w.bq,
                           bk=w.bk, out=o)
        torch.cuda.synchronize()
        err = sage.sage_last_device_error()
    finally:
        sage.sage_debug_kv_quant_two_pass(0)
        sage.sage_debug_wait_limit(0)
    assert err == 7, sage.STATUS_NAMES.get(err, err)  # SAGE_ERR_TIMEOUT, then cleared
    assert torch.isnan(o).all(), "the attention kernel ran on stale codes"
    # the default path on the same inputs: the statistics pass (this head's tiles
    # do not fit for one read), every wait ends, the result is finite
    assert sage.sage_quant_kernel_count(p) == 4
    o2 = sage.sage_attn_fwd(qd[:, :, :4096], kd[:, :, :4096], vd[:, :, :4096], causal=False, sm_scale=w.sm_scale,
                            smooth_k=1, smooth_q=0, bq=w.bq, bk=w.bk)
    torch.cuda.synchronize()
    assert sage.sage_last_device_error() == 0
    assert torch.isfinite(o2).all()
