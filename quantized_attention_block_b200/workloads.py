"""Seeded synthetic Q/K/V generators for the five attention workloads.

This module holds NO arithmetic of the attention method: it only draws random
numbers, adds the per-channel biases / outlier channels that the workloads
describe, and casts to the input dtype.  Both the CUDA path and the CPU oracle
consume exactly these host tensors.

Workload shapes and distributions follow the SageAttention2 reading note
(zhaifeiyue.github.io/papers/2411.10958/detail: Table 2 models -- Llama3.1,
CogVideoX, HunyuanVideo -- and Figure 5's kernel sweep over N and head_dim)
and the SageAttention3 note (zhaifeiyue.github.io/papers/2505.11594).  The
pages measure on real model activations, which are not available; these
seeded tensors stand in for them:

  * "N(0, s)" means standard deviation s (torch.randn * s).
  * A "per-channel bias shared across tokens" is one vector of shape
    [1, H, 1, d] added to every token of every batch.
  * "4 outlier channels x10": per head, 4 channel indices drawn by the seeded
    generator are multiplied by 10 after the bias is added.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: torch.dtype
    causal: bool
    smooth_k: bool
    smooth_q: bool
    bq: int          # Q quantisation block (rows)
    bk: int          # K quantisation block (rows)
    nvfp4: bool
    seed: int
    # distribution recipe
    k_bias_std: float = 0.0
    qk_shared_bias_std: float = 0.0
    k_outlier_channels: int = 0
    k_outlier_mult: float = 1.0
    # the recipe names the two-level FP32 accumulation of P~V explicitly
    names_two_level: bool = False

    @property
    def sm_scale(self) -> float:
        return self.d ** -0.5

    def ops(self) -> float:
        """Attention op count: 4*N^2*d per head (two matmuls), halved when causal."""
        full = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return full / 2.0 if self.causal else full

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # Tiny non-causal fp16 case: 64x64 quant blocks, K bias N(0,3).
    "tiny_fp16_N256_d64": Workload(
        "tiny_fp16_N256_d64", B=1, Hq=2, Hkv=2, N=256, d=64, dtype=torch.float16,
        causal=False, smooth_k=True, smooth_q=False, bq=64, bk=64, nvfp4=False,
        seed=0, k_bias_std=3.0),
    # LLM prefill, causal: K bias N(0,3) + 4 outlier channels x10.
    "llm_prefill_causal_B4_H32_N4096_d128": Workload(
        "llm_prefill_causal_B4_H32_N4096_d128", B=4, Hq=32, Hkv=32, N=4096, d=128,
        dtype=torch.bfloat16, causal=True, smooth_k=True, smooth_q=False, bq=128, bk=64,
        nvfp4=False, seed=2, k_bias_std=3.0, k_outlier_channels=4, k_outlier_mult=10.0),
    # Video-DiT self-attention (CogVideoX-like token count), smooth_q + delta_S.
    "video_dit_B2_H48_N17776_d64": Workload(
        "video_dit_B2_H48_N17776_d64", B=2, Hq=48, Hkv=48, N=17776, d=64,
        dtype=torch.bfloat16, causal=False, smooth_k=True, smooth_q=True, bq=128, bk=64,
        nvfp4=False, seed=3, qk_shared_bias_std=2.0),
    # Long-context GQA, causal: 32 Q heads share 8 KV heads.
    "long_gqa_causal_B1_Hq32_Hkv8_N32768_d128": Workload(
        "long_gqa_causal_B1_Hq32_Hkv8_N32768_d128", B=1, Hq=32, Hkv=8, N=32768, d=128,
        dtype=torch.bfloat16, causal=True, smooth_k=True, smooth_q=False, bq=128, bk=64,
        nvfp4=False, seed=4, k_bias_std=3.0, names_two_level=True),
    # NVFP4 (SageAttention3-style), non-causal, Q/K mean-smoothed.
    "nvfp4_B2_H24_N8192_d128": Workload(
        "nvfp4_B2_H24_N8192_d128", B=2, Hq=24, Hkv=24, N=8192, d=128,
        dtype=torch.bfloat16, causal=False, smooth_k=True, smooth_q=True, bq=128, bk=64,
        nvfp4=True, seed=5, qk_shared_bias_std=2.0),
}

# Short aliases used by tests and bench.
ALIASES = {
    "tiny": "tiny_fp16_N256_d64",
    "prefill": "llm_prefill_causal_B4_H32_N4096_d128",
    "video": "video_dit_B2_H48_N17776_d64",
    "gqa": "long_gqa_causal_B1_Hq32_Hkv8_N32768_d128",
    "nvfp4": "nvfp4_B2_H24_N8192_d128",
}


def get(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def make_qkv(w: Workload, seed: int | None = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Return host (CPU) Q, K, V in HND layout [B, H, N, d], dtype w.dtype.

    Deterministic for a given (workload shape, seed): the draws happen in a
    fixed order on a CPU torch.Generator.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    if w.qk_shared_bias_std:
        if Hq != Hkv:
            raise ValueError("a shared Q/K bias needs Hq == Hkv")
        bias = torch.randn((1, Hkv, 1, d), generator=g) * w.qk_shared_bias_std
        q += bias
        k += bias
    if w.k_bias_std:
        k += torch.randn((1, Hkv, 1, d), generator=g) * w.k_bias_std
    if w.k_outlier_channels:
        for h in range(Hkv):
            ch = torch.randperm(d, generator=g)[: w.k_outlier_channels]
            k[:, h, :, ch] *= w.k_outlier_mult
    return q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def small_variant(w: Workload, N: int, B: int = 1, Hq: int | None = None, Hkv: int | None = None) -> Workload:
    """Same recipe at a size the oracle finishes in seconds (several tiles + ragged tail)."""
    hq = Hq if Hq is not None else min(w.Hq, 2 * max(1, w.Hq // w.Hkv))
    hkv = Hkv if Hkv is not None else max(1, hq * w.Hkv // w.Hq)
    return w.with_(name=f"{w.name}@B{B}_Hq{hq}_Hkv{hkv}_N{N}", B=B, Hq=hq, Hkv=hkv, N=N)
