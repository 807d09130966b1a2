"""The parity harness's acceptance of rows on a rounding boundary, checked on
the CPU with the oracle alone: a row equal to the oracle's with the score
scale moved by 5e-7 (a code of P on the other side of an FP4 midpoint, 0.024
away from the plain oracle row) is accepted; a row with a planted error of
0.05 is not; and no more than the allowed share of rows is accepted."""
import numpy as np

import oracle
from quantized_attention_block_b200 import workloads as W

from harness import accept_boundary_rows, oracle_quant_nvfp4

# the seeded NVFP4 case in which a kernel row sat on such a boundary
CASE = W.get("nvfp4").with_(name="nvfp4_boundary", B=2, Hq=8, Hkv=2, N=127, causal=True, smooth_k=True,
                             smooth_q=True, bq=64, seed=1933539867, qk_shared_bias_std=0.0, k_bias_std=3.0)


def _setup():
    w = CASE
    q, k, v = W.make_qkv(w)
    quant = oracle_quant_nvfp4(w, q, k, v)

    def row(b, h, r, sm):
        return oracle.attention_nvfp4_head(quant, b, h, r, r + 1, bq=w.bq, causal=w.causal, sm_scale=sm)[0]

    refs = np.stack([np.stack([oracle.attention_nvfp4_head(quant, b, h, 0, w.N, bq=w.bq, causal=w.causal,
                                                           sm_scale=w.sm_scale) for h in range(w.Hq)])
                     for b in range(w.B)])
    return w, refs, row


def test_boundary_row_is_accepted_and_a_real_error_is_not():
    w, refs, row = _setup()
    b, h, r = 1, 3, 82
    moved = row(b, h, r, w.sm_scale * (1 - 5e-7))
    assert np.abs(moved - refs[b, h, r]).max() > 0.02  # the row really sits on a boundary

    out = refs.copy()
    out[b, h, r] = moved
    new_refs, accepted, failing = accept_boundary_rows(w, out, refs, row)
    assert accepted == [(b, h, r)] and failing == []
    assert np.array_equal(new_refs[b, h, r], moved)

    out2 = refs.copy()
    out2[0, 0, 5] += 0.05
    _, accepted2, failing2 = accept_boundary_rows(w, out2, refs, row)
    assert accepted2 == [] and failing2 == [(0, 0, 5)]


def test_accepted_share_is_bounded():
    w, refs, row = _setup()
    b, h, r = 1, 3, 82
    out = refs.copy()
    out[b, h, r] = row(b, h, r, w.sm_scale * (1 - 5e-7))
    # one accepted row of 2032 is above a 0.01% cap: it then counts as failing
    _, accepted, failing = accept_boundary_rows(w, out, refs, row, max_frac=1e-4)
    assert (b, h, r) in failing
