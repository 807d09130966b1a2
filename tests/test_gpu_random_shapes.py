"""GPU parity on seeded random configurations of the INT8/FP8 path, beyond the
hand-picked edge cases: sequence length (ragged or not, down to 1), batch, GQA
ratio, head dim, causal mask, smooth K / smooth Q, Q and K block sizes, input
dtype and PV accumulation mode all drawn at random.  Each case checks the
quantised tensors bit-exactly and every output row element by element against
the oracle (the output starts as NaN, so an unwritten row fails); a row whose
E4M3 code of P sits on a rounding boundary may be matched with the score scale
moved within the kernel's fp32 error (harness.accept_boundary_rows, at most 1%
of the rows)."""
import numpy as np
import pytest
import torch

from quantized_attention_block_b200 import sage
from quantized_attention_block_b200 import workloads as W

import oracle
from harness import accept_boundary_rows, compare_out, compare_quant, gpu_attention, oracle_quant, oracle_rows

pytestmark = pytest.mark.gpu

N_CASES = 64


def _case(i: int) -> tuple:
    rng = np.random.default_rng(1000 + i)
    d = int(rng.choice([64, 128]))
    smooth_q = bool(rng.random() < 0.4)
    # the recipes' input distributions: K bias + outlier channels, or a bias
    # shared by Q and K (the case smooth Q is for)
    base = W.get("video") if smooth_q else W.get("prefill")
    hkv = int(rng.choice([1, 2]))
    g = int(rng.choice([1, 2, 4]))
    w = base.with_(
        name=f"rand{i}",
        B=int(rng.choice([1, 2])),
        Hq=hkv * g,
        Hkv=hkv,
        N=int(rng.choice([1, 2, 63, 64, 65, 127, 128, 129]) if rng.random() < 0.3 else rng.integers(2, 700)),
        d=d,
        dtype=torch.float16 if rng.random() < 0.3 else torch.bfloat16,
        causal=bool(rng.random() < 0.5),
        smooth_k=bool(rng.random() < 0.8),
        smooth_q=smooth_q,
        bq=int(rng.choice([32, 64, 128])),
        bk=int(rng.choice([64, 128])),
        seed=int(rng.integers(0, 2**31 - 1)),
    )
    if smooth_q and g > 1:
        # (a bias shared by Q and K needs as many K heads as Q heads)
        w = w.with_(qk_shared_bias_std=0.0, k_bias_std=3.0)
    mode = int(rng.choice([sage.PV_TWO_LEVEL, sage.PV_TMEM_FP32]))
    return w, mode


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_configuration_matches_oracle(i):
    w, mode = _case(i)
    q, k, v = W.make_qkv(w)
    p, ws, view, o = gpu_attention(w, q, k, v, mode)
    quant = oracle_quant(w, q, k, v)
    bad = compare_quant(w, p, ws, view, quant)
    assert not bad, (w, bad)
    out = o.float().cpu().numpy()
    refs = np.stack([np.stack([oracle_rows(w, quant, b, h, 0, w.N) for h in range(w.Hq)]) for b in range(w.B)])
    refs, accepted, failing = accept_boundary_rows(
        w, out, refs, lambda b, h, r, sm: oracle.attention_sage_head(quant, b, h, r, r + 1, bq=w.bq, bk=w.bk,
                                                                       causal=w.causal, sm_scale=sm)[0])
    assert not failing, (w, mode, failing)
    m, ok = compare_out(refs, out)
    assert ok, (w, mode, m, accepted)
