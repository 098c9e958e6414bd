"""The five synthetic MoE-layer workloads and their input recipes.

Every workload is a DWDP rank's MoE expert block at one size.  The method is
described in "DWDP: Distributed Weight Data Parallelism for High-Performance
LLM Inference on NVL72" (arXiv 2604.01621, abstract): each GPU stays data
parallel and runs the MoE block on its own tokens, with the expert weights
split between GPUs.  The explainer page "Distributed Weight Data Parallelism
cuts LLM inference stalls" shows four ranks per group (first figure), so a
rank holds a quarter of the routed experts locally (the "local pool") and
pulls the other three quarters from its peers (the "remote pool").

The pages give the model (DeepSeek-R1) but none of the layer's arithmetic, so
the shapes and routing rules below are the DeepSeek-R1 layer shape read
plainly.  No dataset or trained weight is used: every tensor is drawn from a
seeded generator (see ``moe_inputs.gen``).

This module holds sizes and distributions only, none of the method's
arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

SEED = 0


@dataclass(frozen=True)
class MoEConfig:
    cfg_id: int          # small integer, part of every generator key
    name: str
    T: int               # tokens on this rank (per layer)
    H: int               # hidden size
    I: int               # expert intermediate size
    E: int               # routed experts
    k: int               # experts per token
    score: str           # "softmax" (top-k of softmax) or "sigmoid" (group-limited)
    n_group: int         # expert groups (sigmoid routing)
    topk_group: int      # groups kept per token (sigmoid routing)
    routed_scale: float  # multiplier on the routed weights
    renormalize: bool    # renormalise the k selected weights to sum 1
    has_shared: bool     # one always-on shared expert with weight 1
    x_dtype: str         # "f32" or "bf16": the layer input as handed over
    w_dtype: str         # "bf16" or "e4m3" (with fp32 per-128x128-block scales)
    local_count: int     # experts [0, local_count) sit in the local pool
    layers: int          # consecutive MoE layers (pipelined workloads)
    x_sigma: float       # x ~ N(0, x_sigma)
    wg_sigma: float      # router weight W_g ~ N(0, wg_sigma), fp32
    w_sigma: float       # expert weights ~ N(0, w_sigma)
    bias: str            # "none" | "normal" | "zipf": router selection bias
    bias_sigma: float = 0.0
    zipf_s: float = 0.0
    zipf_amp: float = 0.0
    seq_count: int = 1   # sequences concatenated into the T tokens
    seq_cv: float = 0.0  # coefficient of variation of their lengths

    @property
    def A(self) -> int:
        """Routed (token, expert) assignments per layer."""
        return self.T * self.k

    @property
    def remote_count(self) -> int:
        return self.E - self.local_count

    @property
    def rows(self) -> int:
        """Rows of the permuted activation matrix: assignments + shared rows."""
        return self.A + (self.T if self.has_shared else 0)

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


_R1 = dict(H=7168, I=2048, E=256, k=8, score="sigmoid", n_group=8, topk_group=4,
           routed_scale=2.5, renormalize=True, has_shared=True, x_dtype="bf16",
           local_count=64, x_sigma=1.0, wg_sigma=0.02, w_sigma=0.02)

CONFIGS: dict[int, MoEConfig] = {
    # Tiny layer: softmax top-2 over 8 experts, fp32 input, no shared expert.
    1: MoEConfig(cfg_id=1, name="tiny_T64_H256_I128_E8_top2", T=64, H=256, I=128,
                 E=8, k=2, score="softmax", n_group=1, topk_group=1,
                 routed_scale=1.0, renormalize=True, has_shared=False,
                 x_dtype="f32", w_dtype="bf16", local_count=4, layers=1,
                 x_sigma=1.0, wg_sigma=0.1, w_sigma=0.02, bias="none"),
    # DeepSeek-R1-shaped decode step (128 tokens).  W_g sigma is not stated
    # for this workload; the 0.02 of the prefill workloads is used.
    2: MoEConfig(cfg_id=2, name="r1_decode_T128", T=128, w_dtype="bf16", layers=1,
                 bias="normal", bias_sigma=0.01, **_R1),
    # Prefill of one 8K sequence, unbiased router.
    3: MoEConfig(cfg_id=3, name="r1_prefill_T8192", T=8192, w_dtype="bf16", layers=1,
                 bias="none", **_R1),
    # Imbalanced prefill: 4 sequences (length CV 0.5), Zipf(1.2) expert skew,
    # two layers with the next layer's remote experts prefetched.
    4: MoEConfig(cfg_id=4, name="r1_prefill_imbalanced_T16384_2layers", T=16384,
                 w_dtype="bf16", layers=2, bias="zipf", zipf_s=1.2, zipf_amp=1.0,
                 seq_count=4, seq_cv=0.5, **_R1),
    # FP8 pipeline: four layers, e4m3 weights with fp32 128x128 block scales.
    5: MoEConfig(cfg_id=5, name="r1_fp8_pipeline_T4096_4layers", T=4096,
                 w_dtype="e4m3", layers=4, bias="normal", bias_sigma=0.05, **_R1),
}


# Reduced cases of the same kernels for profiler captures, a few GB on the
# device: the decode shape with 32 routed experts (about 4 tokens each, as in
# the 128-token decode step), the prefill shape and the FP8 shape with 32
# experts; and a two-layer decode pipeline for the selective-fetch measurement.
PROFILE_CASES: dict[int, MoEConfig] = {
    21: CONFIGS[2].with_(cfg_id=21, name="r1_decode_shape_E32_T16", T=16, E=32, local_count=8),
    # the 8K-prefill router (T, H, E as in the prefill workload) with small experts
    22: CONFIGS[3].with_(cfg_id=22, name="r1_router_shape_T8192_I128", I=128),
    23: CONFIGS[3].with_(cfg_id=23, name="r1_prefill_shape_E32_T1024", T=1024, E=32,
                         local_count=8),
    25: CONFIGS[5].with_(cfg_id=25, name="r1_fp8_shape_E32_T512", T=512, E=32, local_count=8,
                         layers=1),
    # two decode-sized layers through the prefetch pipeline: 32 tokens touch about
    # 60 % of the routed experts, the case a selective fetch is for
    33: CONFIGS[2].with_(cfg_id=33, name="r1_decode_T32_2layers", T=32, layers=2),
}


def config(cfg: int | str | MoEConfig) -> MoEConfig:
    if isinstance(cfg, MoEConfig):
        return cfg
    if isinstance(cfg, int):
        return CONFIGS[cfg] if cfg in CONFIGS else PROFILE_CASES[cfg]
    for c in list(CONFIGS.values()) + list(PROFILE_CASES.values()):
        if c.name == cfg:
            return c
    raise KeyError(cfg)
