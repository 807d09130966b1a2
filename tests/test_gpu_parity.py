"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Quantised tensors, scales and INT32 QK^T tiles are
compared bit-exactly; attention outputs element by element within max-abs
1e-2 and cosine >= 0.9999."""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

from harness import compare_out, compare_quant, gpu_attention, gpu_quant, oracle_quant, oracle_rows

pytestmark = pytest.mark.gpu

# Same recipes at sizes the oracle finishes in seconds: several 128-row tiles
# and a ragged tail (N % 128 != 0, N % 64 != 0).
SMALL = {
    "tiny": W.get("tiny"),
    "prefill": W.small_variant(W.get("prefill"), N=600, B=1, Hq=2),
    "video": W.small_variant(W.get("video"), N=600, B=1, Hq=2),
    "gqa": W.small_variant(W.get("gqa"), N=600, B=1, Hq=8, Hkv=2),
}
EDGE = {
    "N1": W.get("tiny").with_(name="N1", N=1, bq=128),
    "N127_causal": W.get("prefill").with_(name="N127_causal", B=1, Hq=1, Hkv=1, N=127),
    "N129_causal_d64": W.get("video").with_(name="N129_causal_d64", B=1, Hq=2, Hkv=2, N=129, causal=True),
    "N200_fp16_bq64_bk128": W.get("tiny").with_(name="N200_fp16", N=200, bq=64, bk=128),
    "N300_no_smooth_k": W.get("prefill").with_(name="N300_nosk", B=2, Hq=2, Hkv=1, N=300, smooth_k=False),
    "N257_smoothq_causal_d128": W.get("gqa").with_(name="N257_sq", B=1, Hq=2, Hkv=2, N=257, smooth_q=True,
                                                   qk_shared_bias_std=2.0, k_bias_std=0.0),
    "N513_bq64_bk64_d64": W.get("video").with_(name="N513", B=1, Hq=1, Hkv=1, N=513, bq=64),
    # one Q scale per 32-row TMEM lane group
    "N300_bq32_causal": W.get("prefill").with_(name="N300_bq32", B=1, Hq=2, Hkv=2, N=300, bq=32),
    "N385_bq32_smoothq_d64": W.get("video").with_(name="N385_bq32", B=1, Hq=2, Hkv=2, N=385, bq=32),
    "N260_bq32_smoothq_gqa_causal": W.get("gqa").with_(name="N260_bq32_sq", B=1, Hq=4, Hkv=2, N=260, bq=32,
                                                        smooth_q=True, qk_shared_bias_std=0.0, k_bias_std=3.0),
    # delta_S cases for the split-row kernel: fp16 at d = 64, non-causal d = 128
    "N333_fp16_smoothq_d64": W.get("video").with_(name="N333_fp16_sq", B=1, Hq=2, Hkv=2, N=333,
                                                  dtype=torch.float16),
    "N450_smoothq_d128": W.get("prefill").with_(name="N450_sq", B=1, Hq=2, Hkv=2, N=450, causal=False,
                                                smooth_q=True, qk_shared_bias_std=2.0),
}


@pytest.mark.parametrize("name", list(SMALL) + list(EDGE))
def test_quant_bit_exact(name):
    w = {**SMALL, **EDGE}[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, _ = gpu_quant(w, q, k, v)
    bad = compare_quant(w, p, ws, view, oracle_quant(w, q, k, v))
    assert not bad, bad


@pytest.mark.parametrize("name", list(SMALL) + list(EDGE))
def test_one_read_kv_quant_equals_two_pass(name):
    """The one-read K/V kernel (each tile waits in shared memory for its head's
    km / s_v) and the two-pass path (statistics kernel first) write the same
    bytes: codes, scales, km, qbar and delta_S."""
    w = {**SMALL, **EDGE}[name]
    q, k, v = W.make_qkv(w)
    p, ws1, view1, _ = gpu_quant(w, q, k, v)
    assert sage.sage_last_device_error() == 0
    sage.sage_debug_kv_quant_two_pass(True)
    try:
        _, ws2, view2, _ = gpu_quant(w, q, k, v)
    finally:
        sage.sage_debug_kv_quant_two_pass(False)
    assert sage.sage_last_device_error() == 0
    t1, t2 = sage.view_tensors(view1, p, ws1), sage.view_tensors(view2, p, ws2)
    assert t1.keys() == t2.keys()
    for key in t1:
        a = t1[key].contiguous().cpu().numpy()
        b = t2[key].contiguous().cpu().numpy()
        assert a.shape == b.shape, key
        np.testing.assert_array_equal(a.reshape(-1).view(np.uint8), b.reshape(-1).view(np.uint8), err_msg=key)


def test_quant_kernel_count_follows_the_path():
    """head_dim 128 takes the one-read K/V kernel (2 kernels + delta_S), head_dim
    64 and the forced two-pass path 4 (+ delta_S)."""
    for name, one_read in (("prefill", True), ("gqa", True), ("video", False)):
        w = W.get(name)
        p = sage.SageParams(w.B, w.Hq, w.Hkv, w.N, w.d, 0, int(w.causal), float(w.sm_scale or 0.0),
                            int(w.smooth_k), int(w.smooth_q), w.bq, w.bk, 0)
        extra = 1 if w.smooth_q else 0
        assert sage.sage_quant_kernel_count(p) == (2 if one_read else 4) + extra, name
        sage.sage_debug_kv_quant_two_pass(True)
        try:
            assert sage.sage_quant_kernel_count(p) == 4 + extra, name
        finally:
            sage.sage_debug_kv_quant_two_pass(False)


@pytest.mark.parametrize("name", ["tiny", "prefill", "video", "gqa"])
def test_qk_int32_tiles_bit_exact(name):
    w = SMALL[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, _ = gpu_quant(w, q, k, v)
    t = sage.view_tensors(view, p, ws)
    q8 = t["q8"].cpu().numpy().astype(np.int64)
    k8 = t["k8"].cpu().numpy().astype(np.int64)
    G = w.Hq // w.Hkv
    ntile = int(view.Np) // 128
    for (b, h, qt, kt) in [(0, 0, 0, 0), (0, w.Hq - 1, ntile - 1, 0), (w.B - 1, w.Hq // 2, 0, ntile - 1),
                           (0, 0, ntile - 1, ntile - 1)]:
        got = sage.sage_debug_qk_int32(view, p, b, h, qt, kt).cpu().numpy()
        ref = q8[b, h, qt * 128:(qt + 1) * 128] @ k8[b, h // G, kt * 128:(kt + 1) * 128].T
        np.testing.assert_array_equal(got, ref.astype(np.int32))


PV_MODES = {"two_level": sage.PV_TWO_LEVEL, "tmem_fp32": sage.PV_TMEM_FP32}


@pytest.mark.parametrize("mode", list(PV_MODES))
@pytest.mark.parametrize("name", list(SMALL) + list(EDGE))
def test_attention_matches_oracle_elementwise(name, mode):
    w = {**SMALL, **EDGE}[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention(w, q, k, v, PV_MODES[mode])
    quant = oracle_quant(w, q, k, v)
    out = o.float().cpu().numpy()
    refs = np.stack([np.stack([oracle_rows(w, quant, b, h, 0, w.N) for h in range(w.Hq)]) for b in range(w.B)])
    m, ok = compare_out(refs, out)
    assert ok, m


LSE_CASES = ["prefill", "video", "gqa", "N127_causal", "N300_no_smooth_k", "N257_smoothq_causal_d128",
             "N260_bq32_smoothq_gqa_causal", "N200_fp16_bq64_bk128"]


@pytest.mark.parametrize("mode", list(PV_MODES))
@pytest.mark.parametrize("name", LSE_CASES)
def test_lse_matches_oracle(name, mode):
    """Each row's log-sum-exp (return_lse) against the oracle's m + ln l of the
    same quantised scores plus the smooth-K correction sm_scale Q.km (fp64):
    within 1e-4 + 1e-5 |lse| (fp32 sums and the approximate exp2 / log2).
    Asking for it leaves the output bit-identical."""
    w = {**SMALL, **EDGE}[name]
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = sage.make_params(qd, kd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k, smooth_q=w.smooth_q,
                         bq=w.bq, bk=w.bk, pv_accum=PV_MODES[mode], return_lse=True)
    ws = sage.alloc_workspace(p)
    view = sage.sage_quant_qkv(qd, kd, vd, p, ws)
    o1, o2 = torch.empty_like(qd), torch.empty_like(qd)
    lse = torch.full((w.B, w.Hq, w.N), float("nan"), dtype=torch.float32, device="cuda")
    sage.sage_attn_fwd_quantized(view, o1, p)
    sage.sage_attn_fwd_quantized_lse(view, o2, lse, p)
    torch.cuda.synchronize()
    assert sage.sage_last_device_error() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    quant = oracle_quant(w, q, k, v)
    got = lse.cpu().numpy().astype(np.float64)
    sm = w.sm_scale if w.sm_scale else 1.0 / np.sqrt(w.d)
    for b in range(w.B):
        for h in range(w.Hq):
            _, l = oracle.attention_sage_head(quant, b, h, 0, w.N, bq=w.bq, bk=w.bk, causal=w.causal,
                                              sm_scale=w.sm_scale, with_lse=True)
            ref = l + oracle.lse_smooth_k_correction(q, quant, b, h, 0, w.N, sm_scale=sm)
            err = np.abs(got[b, h] - ref)
            assert np.all(err <= 1e-4 + 1e-5 * np.abs(ref)), (b, h, float(err.max()), int(np.argmax(err)))
    # the one-call form gives the same bytes
    o3, lse3 = sage.sage_attn_fwd_lse(qd, kd, vd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                                      smooth_q=w.smooth_q, bq=w.bq, bk=w.bk, pv_accum=PV_MODES[mode])
    torch.cuda.synchronize()
    assert torch.equal(o3.view(torch.int16), o2.view(torch.int16)) and torch.equal(lse3, lse)


def test_lse_needs_return_lse_at_quantisation():
    w = SMALL["prefill"]
    q, k, v = W.make_qkv(w)
    p, ws, view, (qd, kd, vd) = gpu_quant(w, q, k, v)
    assert not view.qkm
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    with pytest.raises(sage.SageError):
        sage.sage_attn_fwd_quantized_lse(view, torch.empty_like(qd), lse, p)


def test_pv_accumulation_modes_agree_closely():
    """The TMEM FP32 accumulator and the two-level scheme differ only in FP32
    rounding order (the accumulator keeps full FP32: see the probe test)."""
    w = SMALL["gqa"]
    q, k, v = W.make_qkv(w)
    o0 = gpu_attention(w, q, k, v, sage.PV_TWO_LEVEL)[3].float()
    o1 = gpu_attention(w, q, k, v, sage.PV_TMEM_FP32)[3].float()
    assert (o0 - o1).abs().max().item() <= 1e-2


def test_sage_attn_fwd_one_call_equals_two_step():
    w = SMALL["prefill"]
    q, k, v = W.make_qkv(w)
    _, _, _, o2 = gpu_attention(w, q, k, v)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1 = sage.sage_attn_fwd(qd, kd, vd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                            smooth_q=w.smooth_q, bq=w.bq, bk=w.bk)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_bounded_wait_times_out_and_context_survives():
    """Failure detection without a fault: a wait nobody ends gives up after the
    limit, the status comes back as SAGE_ERR_TIMEOUT, and the context still works."""
    assert sage.sage_last_device_error() == 0
    assert sage.sage_debug_bounded_wait(2000) == 7  # SAGE_ERR_TIMEOUT
    assert sage.sage_last_device_error() == 0       # cleared
    w = SMALL["tiny"]
    q, k, v = W.make_qkv(w)
    gpu_attention(w, q, k, v)


def test_rejects_invalid_arguments():
    w = SMALL["tiny"]
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    with pytest.raises(sage.SageError):
        sage.sage_attn_fwd(qd, kd, vd, bq=96)
    with pytest.raises(sage.SageError):
        sage.sage_attn_fwd(qd[..., :48].contiguous(), kd[..., :48].contiguous(), vd[..., :48].contiguous())


# ---------------------------------------------------------------- full sizes
FULL = ["prefill", "video", "gqa"]


def _sample_tiles(n_tiles, rng, k=3):
    picks = {0, n_tiles - 1}
    while len(picks) < min(n_tiles, k + 2):
        picks.add(int(rng.integers(0, n_tiles)))
    return sorted(picks)


@pytest.mark.parametrize("mode", list(PV_MODES))
@pytest.mark.parametrize("name", FULL)
def test_full_size_quant_bit_exact_and_sampled_attention(name, mode):
    """At the benchmark's sizes and launch configuration: every quantised value
    checked bit-exactly; attention outputs on sampled Q tiles of five sampled
    heads (first, last / ragged tail, random) checked element by element, and
    every output row checked against the convex-combination bound."""
    w = W.get(name)
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention(w, q, k, v, PV_MODES[mode])
    quant = oracle_quant(w, q, k, v)
    bad = compare_quant(w, p, ws, view, quant)
    assert not bad, bad
    rng = np.random.default_rng(123)
    n_tiles = int(view.Np) // 128
    # five (batch, head) pairs (the first, the last, three at random: for GQA
    # they span several KV groups) x four Q tiles (first, last / ragged, two at
    # random): about 20 tiles per workload
    heads = {(0, 0), (w.B - 1, w.Hq - 1)}
    while len(heads) < min(5, w.B * w.Hq):
        heads.add((int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq))))
    heads = sorted(heads)
    from concurrent.futures import ThreadPoolExecutor
    jobs = []
    for (b, h) in heads:
        for t in _sample_tiles(n_tiles, rng, k=2):
            r0, r1 = t * 128, min((t + 1) * 128, w.N)
            jobs.append((b, h, r0, r1))
    with ThreadPoolExecutor() as ex:
        refs = list(ex.map(lambda j: oracle_rows(w, quant, *j), jobs))
    out = o.float().cpu().numpy()
    for (b, h, r0, r1), ref in zip(jobs, refs):
        m, ok = compare_out(ref, out[b, h, r0:r1])
        assert ok, ((b, h, r0, r1), m)
    # Every row at this size, by a property that holds at any size: O is a
    # convex combination of its head's V rows (P >= 0, normalised by l), so each
    # element is finite (the output starts as NaN, so an unwritten row fails)
    # and lies within the range of its V column, widened by the E4M3 rounding of
    # P and of V (2^-4 relative each: (1 + 2^-4)^2 - 1 < 0.13) and bf16 output.
    of = o.float()
    vf = v.to(o.device).float()
    G = w.Hq // w.Hkv
    vmax = vf.amax(dim=2).repeat_interleave(G, dim=1)[:, :, None, :]
    vmin = vf.amin(dim=2).repeat_interleave(G, dim=1)[:, :, None, :]
    slack = 0.15 * torch.maximum(vmax.abs(), vmin.abs()) + 1e-3
    assert bool(torch.isfinite(of).all())
    assert bool((of <= vmax + slack).all()) and bool((of >= vmin - slack).all())


def test_fp8_accumulator_precision_probe():
    """The two-level accumulation of SageAttention2 exists because Ada/Hopper FP8
    MMAs keep about 13 accumulator bits (SA2 note, "5. Numerical
    Considerations").  This runs the tcgen05 kind::f8f6f4 probe: sums that need
    at most 12 mantissa bits must come back exact whatever the accumulator
    width; the others show how many bits it keeps (recorded, not asserted)."""
    got = sage.sage_debug_f8_accum_probe().cpu().numpy().astype(np.float64)
    exact = np.array(sage.F8_ACCUM_PROBE_EXACT)
    assert got[2] == exact[2] and got[3] == 256.0 and got[4] == 32.0, got
    bits = [int(-np.log2(abs(g - round(g)) or 2.0 ** -40)) if g != round(g) else None for g in got]
    print("f8 accumulator probe:", got.tolist(), "exact:", [float(x) == float(y) for x, y in zip(got, exact)], bits)


def test_fma_pipe_exp2_accuracy():
    """The FMA-pipe polynomial exp2 the softmax can take for a share of its
    exponentials (a compile-time option; the shipped kernels use the MUFU for
    all of them): relative error against fp64 exp2 below 1.2e-5 over the range
    the kernel would feed it (scores minus the row max plus log2 448), and a
    tiny non-negative value for masked scores."""
    x = torch.cat([torch.linspace(-125.0, 9.0, 2_000_001), torch.tensor([0.0, 1.0, -1.0, 8.807354922057604])])
    y = sage.sage_debug_exp2_poly(x.cuda()).cpu().double()
    ref = torch.exp2(x.double())
    rel = ((y - ref).abs() / ref).max().item()
    assert rel < 1.2e-5, rel
    masked = sage.sage_debug_exp2_poly(torch.tensor([-float("inf"), -1e30, -500.0]).cuda()).cpu()
    assert torch.all(masked >= 0) and torch.all(masked <= 2.0 ** -125)


def test_mma_rate_probe_runs_every_shape():
    """The tensor-core rate probe bench.py divides by: every (kind, N) launches,
    counts 2 M N K per instruction, and lands in a plausible range for one B200
    (hundreds to a few thousand dense TOPS)."""
    st = torch.cuda.current_stream()
    for kind, n in (("i8", 256), ("i8", 128), ("i8", 64), ("f8", 256), ("f8", 128), ("f8", 64), ("f4", 128)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        ops = sage.sage_debug_mma_rate(kind, n, 20000, 0, st)
        e1.record(st)
        torch.cuda.synchronize()
        assert sage.sage_last_device_error() == 0
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert ops == 2.0 * 128 * n * 128 * 20000 * sms
        tops = ops / (e0.elapsed_time(e1) * 1e-3) / 1e12
        assert 100.0 < tops < 20000.0, (kind, n, tops)

