"""GPU parity of the NVFP4 path (SageAttention3 style) against the CPU oracle on
the same seeded inputs: E2M1 codes, E4M3 block scales, km and qbar bit-exact;
the block-scaled FP4 Q K^T tile within fp32 summation error of the exact dot
products; attention outputs element by element within max-abs 1e-2 and
cosine >= 0.9999."""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

from harness import (accept_boundary_rows, compare_out, compare_quant_nvfp4, gpu_attention_nvfp4,
                     gpu_nvfp4_in_oracle_layout, gpu_quant_nvfp4, oracle_quant_nvfp4, oracle_rows_nvfp4)

pytestmark = pytest.mark.gpu

NV = W.get("nvfp4")
SMALL = {
    "nvfp4_N600": W.small_variant(NV, N=600, B=1, Hq=2),
    "nvfp4_N300_B2": W.small_variant(NV, N=300, B=2, Hq=2),
}
EDGE = {
    "N1": NV.with_(name="N1", B=1, Hq=1, Hkv=1, N=1),
    "N127_causal": NV.with_(name="N127_causal", B=1, Hq=2, Hkv=2, N=127, causal=True),
    "N257_causal_bq64": NV.with_(name="N257_causal_bq64", B=1, Hq=2, Hkv=2, N=257, causal=True, bq=64),
    "N200_fp16_no_smooth_q": NV.with_(name="N200_fp16", B=1, Hq=2, Hkv=2, N=200, dtype=torch.float16,
                                      smooth_q=False),
    "N384_gqa_no_smooth_k": NV.with_(name="N384_gqa", B=1, Hq=4, Hkv=2, N=384, smooth_q=False, smooth_k=False,
                                     qk_shared_bias_std=0.0, k_bias_std=3.0),
    "N513_gqa_causal": NV.with_(name="N513_gqa_causal", B=1, Hq=4, Hkv=1, N=513, causal=True, smooth_q=False,
                                qk_shared_bias_std=0.0, k_bias_std=3.0),
}
ALL = {**SMALL, **EDGE}


@pytest.mark.parametrize("name", list(ALL))
def test_nvfp4_quant_bit_exact(name):
    w = ALL[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, _ = gpu_quant_nvfp4(w, q, k, v)
    bad = compare_quant_nvfp4(w, gpu_nvfp4_in_oracle_layout(view, p, ws), oracle_quant_nvfp4(w, q, k, v))
    assert not bad, bad


@pytest.mark.parametrize("name", list(ALL))
def test_nvfp4_one_read_k_equals_two_pass(name):
    """The one-read K kernel (each tile waits in shared memory for its head's
    column sums) and the statistics-pass path write the same bytes."""
    w = ALL[name]
    q, k, v = W.make_qkv(w)
    p, ws1, view1, _ = gpu_quant_nvfp4(w, q, k, v)
    assert sage.sage_last_device_error() == 0
    sage.sage_debug_kv_quant_two_pass(True)
    try:
        _, ws2, view2, _ = gpu_quant_nvfp4(w, q, k, v)
    finally:
        sage.sage_debug_kv_quant_two_pass(False)
    assert sage.sage_last_device_error() == 0
    t1, t2 = sage.nvfp4_view_tensors(view1, p, ws1), sage.nvfp4_view_tensors(view2, p, ws2)
    assert t1.keys() == t2.keys()
    for key in t1:
        a = t1[key].contiguous().cpu().numpy()
        b = t2[key].contiguous().cpu().numpy()
        np.testing.assert_array_equal(a.reshape(-1).view(np.uint8), b.reshape(-1).view(np.uint8), err_msg=key)


def test_nvfp4_quant_kernel_count_follows_the_path():
    w = NV
    p = sage.SageParams(w.B, w.Hq, w.Hkv, w.N, w.d, 0, int(w.causal), float(w.sm_scale or 0.0),
                        int(w.smooth_k), int(w.smooth_q), w.bq, w.bk, 0)
    extra = 1 if w.smooth_q else 0
    assert sage.sage_quant_nvfp4_kernel_count(p) == 3 + extra
    sage.sage_debug_kv_quant_two_pass(True)
    try:
        assert sage.sage_quant_nvfp4_kernel_count(p) == 4 + extra
    finally:
        sage.sage_debug_kv_quant_two_pass(False)


@pytest.mark.parametrize("name", ["nvfp4_N600", "N384_gqa_no_smooth_k"])
def test_nvfp4_qk_tile_matches_exact_dot_products(name):
    """The block-scaled MMA tile against the exact sums of the exact products
    (E2M1 x E4M3 x E2M1 x E4M3 is exact in fp32): the only error allowed is
    fp32 summation, bounded by 2^-16 of the sum of |products| per element
    (128 terms x 2^-24, rounded up); a wrong nibble order, scale layout or
    swizzle gives errors of the order of the sum itself."""
    w = ALL[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, _ = gpu_quant_nvfp4(w, q, k, v)
    ref = oracle_quant_nvfp4(w, q, k, v)
    G = w.Hq // w.Hkv
    ntile = int(view.Np) // 128
    for (b, h, qt, kt) in [(0, 0, 0, 0), (0, w.Hq - 1, ntile - 1, 0), (w.B - 1, w.Hq // 2, 0, ntile - 1),
                           (0, 0, ntile - 1, ntile - 1)]:
        got = sage.sage_debug_qk_nvfp4(view, p, b, h, qt, kt).cpu().numpy().astype(np.float64)
        Qv = oracle.dequant_nvfp4_rows(ref["q4"][b, h], ref["sfq"][b, h])
        Kv = oracle.dequant_nvfp4_rows(ref["k4"][b, h // G], ref["sfk"][b, h // G])
        r0, r1 = qt * 128, min((qt + 1) * 128, w.N)
        c0, c1 = kt * 128, min((kt + 1) * 128, w.N)
        exact = Qv[r0:r1] @ Kv[c0:c1].T
        bound = np.abs(Qv[r0:r1]) @ np.abs(Kv[c0:c1]).T * 2.0 ** -16 + 1e-30
        err = np.abs(got[:r1 - r0, :c1 - c0] - exact)
        assert np.all(err <= bound), (b, h, qt, kt, float(err.max()), float((err / bound).max()))
        # padded rows / keys hold zero codes: their scores are exactly 0
        assert np.all(got[r1 - r0:, :] == 0) and np.all(got[:, c1 - c0:] == 0)


@pytest.mark.parametrize("name", list(ALL))
def test_nvfp4_attention_matches_oracle_elementwise(name):
    w = ALL[name]
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention_nvfp4(w, q, k, v)
    quant = oracle_quant_nvfp4(w, q, k, v)
    out = o.float().cpu().numpy()
    refs = np.stack([np.stack([oracle_rows_nvfp4(w, quant, b, h, 0, w.N) for h in range(w.Hq)])
                     for b in range(w.B)])
    m, ok = compare_out(refs, out)
    assert ok, m


def test_nvfp4_one_call_equals_two_step():
    w = SMALL["nvfp4_N600"]
    q, k, v = W.make_qkv(w)
    _, _, _, o2 = gpu_attention_nvfp4(w, q, k, v)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1 = sage.sage_attn_fwd_nvfp4(qd, kd, vd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                                  smooth_q=w.smooth_q, bq=w.bq)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_nvfp4_rejects_head_dim_64():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    assert sage.nvfp4_workspace_bytes(sage.make_params(q, q)) == 0
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd_nvfp4(q, q, q, workspace=ws)
    assert e.value.status == 2  # SAGE_ERR_UNSUPPORTED_HEADDIM


def test_nvfp4_full_size_quant_bit_exact_and_sampled_attention():
    """At the benchmark's sizes and launch configuration: every NVFP4 code and
    scale checked bit-exactly; attention on sampled Q tiles (first, last /
    ragged, random) of sampled heads checked element by element."""
    w = NV
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention_nvfp4(w, q, k, v)
    quant = oracle_quant_nvfp4(w, q, k, v)
    bad = compare_quant_nvfp4(w, gpu_nvfp4_in_oracle_layout(view, p, ws), quant)
    assert not bad, bad
    rng = np.random.default_rng(321)
    n_tiles = int(view.Np) // 128
    heads = sorted({(0, 0), (w.B - 1, w.Hq - 1), (int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq)))})
    picks = sorted({0, n_tiles - 1, int(rng.integers(0, n_tiles))})
    jobs = [(b, h, t * 128, min((t + 1) * 128, w.N)) for (b, h) in heads for t in picks]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor() as ex:
        refs = list(ex.map(lambda j: oracle_rows_nvfp4(w, quant, *j), jobs))
    out = o.float().cpu().numpy()
    for (b, h, r0, r1), ref in zip(jobs, refs):
        m, ok = compare_out(ref, out[b, h, r0:r1])
        assert ok, ((b, h, r0, r1), m)


def _random_case(i: int):
    """A seeded random NVFP4 configuration (d = 128): sequence length, batch,
    GQA ratio, causal mask, smooth K / smooth Q, smooth-Q block size, dtype."""
    rng = np.random.default_rng(2000 + i)
    hkv = int(rng.choice([1, 2]))
    g = int(rng.choice([1, 2, 4]))
    smooth_q = bool(rng.random() < 0.5)
    w = NV.with_(
        name=f"nvfp4_rand{i}",
        B=int(rng.choice([1, 2])),
        Hq=hkv * g,
        Hkv=hkv,
        N=int(rng.choice([1, 2, 63, 64, 65, 127, 128, 129]) if rng.random() < 0.3 else rng.integers(2, 700)),
        dtype=torch.float16 if rng.random() < 0.3 else torch.bfloat16,
        causal=bool(rng.random() < 0.5),
        smooth_k=bool(rng.random() < 0.8),
        smooth_q=smooth_q,
        bq=int(rng.choice([64, 128])),
        seed=int(rng.integers(0, 2**31 - 1)),
    )
    if g > 1:
        # (a bias shared by Q and K needs as many K heads as Q heads)
        w = w.with_(qk_shared_bias_std=0.0, k_bias_std=3.0)
    return w


@pytest.mark.parametrize("i", range(32))
def test_nvfp4_random_configuration_matches_oracle(i):
    """Codes and scales bit-exact and every output row element by element on
    seeded random configurations (the output starts as NaN).  A row whose FP4
    code of P sits on a rounding boundary may be matched against the oracle
    with the score scale moved within the kernel's fp32 error
    (harness.accept_boundary_rows, at most 1% of the rows)."""
    w = _random_case(i)
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention_nvfp4(w, q, k, v)
    quant = oracle_quant_nvfp4(w, q, k, v)
    bad = compare_quant_nvfp4(w, gpu_nvfp4_in_oracle_layout(view, p, ws), quant)
    assert not bad, (w, bad)
    out = o.float().cpu().numpy()
    refs = np.stack([np.stack([oracle_rows_nvfp4(w, quant, b, h, 0, w.N) for h in range(w.Hq)])
                     for b in range(w.B)])
    refs, accepted, failing = accept_boundary_rows(
        w, out, refs, lambda b, h, r, sm: oracle.attention_nvfp4_head(quant, b, h, r, r + 1, bq=w.bq,
                                                                        causal=w.causal, sm_scale=sm)[0])
    assert not failing, (w, failing)
    m, ok = compare_out(refs, out)
    assert ok, (w, m, accepted)
