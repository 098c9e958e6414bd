"""Helpers shared by the GPU tests (device workloads + oracle references)."""
from __future__ import annotations

import numpy as np
import torch

from moe_inputs import config, device as mdev

# Floating-point bar: max |gpu - oracle| <= RTOL_BF16 * max |oracle| over the
# compared outputs (bf16 weights and activations, fp32 accumulation; the GPU
# rounds x_perm, h and y_perm to bf16 while the oracle keeps fp64).
RTOL_BF16 = 2e-2
RTOL_FP8 = 6e-2

# Test-only workloads: same recipes, other sizes (own generator keys).
MID_SIGMOID = config(2).with_(cfg_id=11, name="mid_sigmoid_T300_H512_I256_E32", T=300, H=512,
                              I=256, E=32, k=4, n_group=4, topk_group=2, local_count=8)
MID_SOFTMAX = config(1).with_(cfg_id=12, name="mid_softmax_f32_T257_H384_I256_E16", T=257, H=384,
                              I=256, E=16, k=3, local_count=6)
SPARSE_DECODE = config(2).with_(cfg_id=13, name="sparse_decode_T5_H256_I128_E64", T=5, H=256,
                                I=128, E=64, k=8, n_group=8, topk_group=4, local_count=16)
MID_FP8 = config(5).with_(cfg_id=24, name="mid_fp8_T300_H512_I256_E32", T=300, H=512, I=256,
                          E=32, k=4, n_group=4, topk_group=2, local_count=8, layers=1)
DECODE_FP8 = config(5).with_(cfg_id=25, name="decode_fp8_T7_H256_I128_E64", T=7, H=256, I=128,
                             E=64, k=8, n_group=8, topk_group=4, local_count=16, layers=1)
# Mid-size layers (whole-layer, element-by-element against the oracle) that
# reach each token-tile width of the grouped GEMMs with ragged tiles:
#   ~256 tokens per expert -> 256-token tiles (one 512-column TMEM set, 16
#   epilogue warps for bf16 weights, 8 with e4m3 weights);
#   ~125 tokens per expert -> 128-token tiles, double-buffered accumulators,
#   row counts that are not multiples of 16.
MID_BN256 = config(2).with_(cfg_id=27, name="mid_bn256_T2048_H512_I256_E8_k1", T=2048, H=512,
                            I=256, E=8, k=1, n_group=1, topk_group=1, local_count=3)
# the same with H = 384: the down GEMM's 256-row tiles do not divide H, so it
# runs single 128-row tiles
MID_BN256_H384 = config(2).with_(cfg_id=31, name="mid_bn256_T2048_H384_I256_E8_k1", T=2048, H=384,
                                 I=256, E=8, k=1, n_group=1, topk_group=1, local_count=3)
MID_BN256_FP8 = config(5).with_(cfg_id=28, name="mid_bn256_fp8_T2048_H512_I256_E8_k1", T=2048,
                                H=512, I=256, E=8, k=1, n_group=1, topk_group=1, local_count=3,
                                layers=1)
# e4m3 weights with H = 384: the down GEMM runs single 128-row tiles
MID_FP8_H384 = config(5).with_(cfg_id=32, name="mid_fp8_T300_H384_I256_E32", T=300, H=384, I=256,
                               E=32, k=4, n_group=4, topk_group=2, local_count=8, layers=1)
MID_BN128 = config(2).with_(cfg_id=29, name="mid_bn128_T1000_H384_I256_E16_k2", T=1000, H=384,
                            I=256, E=16, k=2, n_group=4, topk_group=2, local_count=5)
# e4m3 weights take 256-token tiles from ~97 tokens per expert on (they are
# converted once per token tile): ~88 tokens per expert keeps 128-token tiles,
# ~125 reaches 256-token tiles holding ragged row counts
MID_BN128_FP8 = config(5).with_(cfg_id=30, name="mid_bn128_fp8_T700_H512_I256_E16_k2", T=700,
                                H=512, I=256, E=16, k=2, n_group=4, topk_group=2, local_count=5,
                                layers=1)
MID_BN256_FP8_K2 = config(5).with_(cfg_id=34, name="mid_bn256_fp8_T1000_H512_I256_E16_k2", T=1000,
                                   H=512, I=256, E=16, k=2, n_group=4, topk_group=2, local_count=5,
                                   layers=1)
# the largest shapes the ABI takes: 1024 experts, k = 32, 32 groups (one per lane)
MAX_EXPERTS = config(2).with_(cfg_id=26, name="max_E1024_k32_G32_T64", T=64, H=256, I=128,
                              E=1024, k=32, n_group=32, topk_group=4, local_count=256)
ONE_TOKEN = config(2).with_(cfg_id=14, name="one_token_H256_I256_E16", T=1, H=256, I=256, E=16,
                            k=2, n_group=4, topk_group=2, local_count=4)


def sync_check():
    from split_weight_b200 import _lib as L
    torch.cuda.synchronize()
    L.check(L.moe_check_device())


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def assert_close_rel(got: np.ndarray, ref: np.ndarray, rtol: float, what: str):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= rtol * scale, f"{what}: max|err| {err:.4g} > {rtol} * max|ref| {scale:.4g}"
    return err / scale


def run_layer(dl: mdev.DeviceLayer):
    dl.layer.forward(dl.x)
    sync_check()
    return dl.layer


def tile_width(cfg) -> int:
    """Token-tile width the grouped GEMM picks for a layer from its mean
    tokens per routed expert (the library's rule, restated to check that a
    test reaches the width it is written for)."""
    mean = -(-cfg.A // cfg.E)
    for bn, top in ((16, 8), (32, 16), (64, 32), (128, 96 if cfg.w_dtype == "e4m3" else 160)):
        if mean <= top:
            return bn
    return 256
