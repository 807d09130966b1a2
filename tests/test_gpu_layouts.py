"""NHD tensors ([B, N, H, d], the pages' tensor_layout="NHD") against HND on
the same data: the quantised tensors in the workspace are head-major either
way, so outputs and log-sum-exps must be the same bytes.  The HND path is the
one checked against the oracle elsewhere."""
import pytest
import torch

from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    "prefill_causal": W.small_variant(W.get("prefill"), N=300, B=2, Hq=2),
    "video_smoothq_d64": W.small_variant(W.get("video"), N=385, B=1, Hq=2),
    "gqa_bq32_smoothq": W.get("gqa").with_(name="gqa_nhd", B=2, Hq=4, Hkv=2, N=260, bq=32, smooth_q=True,
                                           qk_shared_bias_std=0.0, k_bias_std=3.0),
    "fp16_no_smooth_k": W.get("tiny").with_(name="fp16_nhd", B=1, Hq=2, Hkv=2, N=200, smooth_k=False),
}


def _nhd(*ts):
    return [t.transpose(1, 2).contiguous() for t in ts]


@pytest.mark.parametrize("two_pass", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_nhd_equals_hnd(name, two_pass):
    w = CASES[name]
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kw = dict(causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k, smooth_q=w.smooth_q, bq=w.bq, bk=w.bk)
    sage.sage_debug_kv_quant_two_pass(two_pass)
    try:
        o_h, lse_h = sage.sage_attn_fwd_lse(qd, kd, vd, **kw)
        qn, kn, vn = _nhd(qd, kd, vd)
        o_n, lse_n = sage.sage_attn_fwd_lse(qn, kn, vn, tensor_layout="NHD", **kw)
        torch.cuda.synchronize()
    finally:
        sage.sage_debug_kv_quant_two_pass(False)
    assert sage.sage_last_device_error() == 0
    assert o_n.shape == (w.B, w.N, w.Hq, w.d)
    assert torch.equal(o_n.transpose(1, 2).contiguous().view(torch.int16), o_h.view(torch.int16))
    assert torch.equal(lse_n, lse_h)


@pytest.mark.parametrize("two_pass", [False, True])
def test_nhd_equals_hnd_nvfp4(two_pass):
    w = W.small_variant(W.get("nvfp4"), N=300, B=2, Hq=2)
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kw = dict(causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k, smooth_q=w.smooth_q, bq=w.bq)
    sage.sage_debug_kv_quant_two_pass(two_pass)
    try:
        o_h = sage.sage_attn_fwd_nvfp4(qd, kd, vd, **kw)
        qn, kn, vn = _nhd(qd, kd, vd)
        o_n = sage.sage_attn_fwd_nvfp4(qn, kn, vn, tensor_layout="NHD", **kw)
        torch.cuda.synchronize()
    finally:
        sage.sage_debug_kv_quant_two_pass(False)
    assert sage.sage_last_device_error() == 0
    assert torch.equal(o_n.transpose(1, 2).contiguous().view(torch.int16), o_h.view(torch.int16))


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("pv_accum", [sage.PV_TWO_LEVEL, sage.PV_TMEM_FP32])
def test_output_writes_stay_inside_o(layout, pv_accum):
    """The output tiles leave the kernel by bulk tensor stores whose map clips
    rows past N: with a ragged N (the last Q tile is mostly past N) and O placed
    between sentinel bytes in one buffer, no byte outside O changes, and O is
    the same as in a buffer of its own."""
    w = W.small_variant(W.get("prefill"), N=300, B=2, Hq=3)
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    if layout == "NHD":
        qd, kd, vd = _nhd(qd, kd, vd)
    kw = dict(causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k, smooth_q=w.smooth_q, bq=w.bq, bk=w.bk,
              pv_accum=pv_accum, tensor_layout=layout)
    ref = sage.sage_attn_fwd(qd, kd, vd, **kw)
    n = qd.numel()
    guard = 4096  # elements on each side (16-byte aligned offsets keep O aligned)
    buf = torch.full((n + 2 * guard,), -7.0, dtype=qd.dtype, device=qd.device)
    out = buf[guard:guard + n].view(qd.shape)
    sage.sage_attn_fwd(qd, kd, vd, out=out, **kw)
    torch.cuda.synchronize()
    assert sage.sage_last_device_error() == 0
    sentinel = torch.full((guard,), -7.0, dtype=qd.dtype, device=qd.device)
    assert torch.equal(buf[:guard].view(torch.int16), sentinel.view(torch.int16))
    assert torch.equal(buf[guard + n:].view(torch.int16), sentinel.view(torch.int16))
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
