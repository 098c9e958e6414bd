"""Puts a seeded workload on the GPU: the layer input, router weights and the
expert weights written straight into split pools by the GPU generator.

Holds none of the MoE layer's arithmetic: it only places the generator's
values where the library's data structures expect them.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import gen, gpu_gen
from .configs import MoEConfig, config


def default_placement(cfg: MoEConfig):
    """Experts [0, local_count) in the local pool (slot e), the rest in the
    remote pool (slot e - local_count)."""
    e = np.arange(cfg.E)
    pool = (e >= cfg.local_count).astype(np.int64)
    slot = np.where(pool == 0, e, e - cfg.local_count)
    return pool, slot


def random_placement(cfg: MoEConfig, seed: int, n_local: int | None = None):
    """A random split of the experts over the two pools with shuffled slots."""
    rng = np.random.default_rng(seed)
    n_local = int(rng.integers(0, cfg.E + 1)) if n_local is None else n_local
    local = rng.permutation(cfg.E)[:n_local]
    pool = np.ones(cfg.E, dtype=np.int64)
    pool[local] = 0
    slot = np.empty(cfg.E, dtype=np.int64)
    for q in (0, 1):
        members = np.nonzero(pool == q)[0]
        slot[members] = rng.permutation(len(members))
    return pool, slot


def layer_shape(cfg: MoEConfig, act_dtype: str | None = None):
    """The library's LayerShape of a workload.  The grouped GEMMs read bf16
    activations unless act_dtype="e4m3" is asked for (e4m3 weights only):
    the FP8 pipeline states bf16 activations, so e4m3 activations are an
    opt-in narrowing of it."""
    from split_weight_b200 import LayerShape
    return LayerShape(T=cfg.T, H=cfg.H, I=cfg.I, E=cfg.E, k=cfg.k, score=cfg.score,
                      n_group=cfg.n_group, topk_group=cfg.topk_group,
                      routed_scale=cfg.routed_scale, renormalize=cfg.renormalize,
                      has_shared=cfg.has_shared, x_dtype=cfg.x_dtype, w_dtype=cfg.w_dtype,
                      y_dtype="f32" if cfg.x_dtype == "f32" else "bf16",
                      act_dtype=act_dtype or "bf16")


def x_tensor(li: gen.LayerInputs, device) -> torch.Tensor:
    if li.x_bits is not None:
        return torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(li.x).to(device)


def fill_weights(cfg: MoEConfig, layer: int, weights, stream: int | None = None) -> None:
    """Writes every routed expert (and the shared one) into its (pool, slot)."""
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    lay = weights.layout
    for e in range(cfg.E + (1 if cfg.has_shared else 0)):
        base = weights.expert_base(e)
        gsc = base + lay.gu_scale_offset if lay.gu_scale_offset >= 0 else None
        dsc = base + lay.down_scale_offset if lay.down_scale_offset >= 0 else None
        gpu_gen.fill_expert(cfg, layer, e, base + lay.gu_offset, base + lay.down_offset, gsc, dsc, s)


@dataclass
class DeviceLayer:
    cfg: MoEConfig
    layer_index: int
    inputs: gen.LayerInputs
    x: torch.Tensor
    layer: object          # split_weight_b200.MoELayer
    pool: np.ndarray
    slot: np.ndarray


def build_layer(cfg, layer: int = 0, device="cuda", placement=None,
                act_dtype: str | None = None, gather: bool | None = None) -> DeviceLayer:
    from split_weight_b200 import MoELayer, SplitWeights
    cfg = config(cfg)
    li = gen.layer_inputs(cfg, layer)
    pool, slot = placement if placement is not None else default_placement(cfg)
    w = SplitWeights.allocate(cfg.H, cfg.I, cfg.w_dtype, pool, slot, cfg.has_shared, device)
    fill_weights(cfg, layer, w)
    wg = torch.from_numpy(li.wg).to(device)
    bias = torch.from_numpy(li.bias).to(device) if li.bias is not None else None
    ml = MoELayer(layer_shape(cfg, act_dtype), wg, bias, w, device, gather=gather)
    return DeviceLayer(cfg, layer, li, x_tensor(li, device), ml, pool, slot)


def peer_store(cfg: MoEConfig, layer: int, weights, device="cuda") -> torch.Tensor:
    """The remote experts of one layer as a peer would hold them: the remote
    pool's slots, contiguous, in a buffer of their own (the copy source of
    the prefetch)."""
    from split_weight_b200 import SplitWeights
    store = torch.empty(max(weights.n_remote, 1) * weights.stride, dtype=torch.uint8, device=device)
    shadow = SplitWeights(weights.H, weights.I, weights.w_dtype, weights.pool_slot, weights.local,
                          weights.n_local, store, weights.n_remote, weights.shared)
    lay = weights.layout
    s = torch.cuda.current_stream().cuda_stream
    for e in range(cfg.E):
        v = int(np.uint32(weights.pool_slot[e]))
        if v >> 31 == 1:
            base = shadow.slot_base(1, v & 0x7FFFFFFF)
            gsc = base + lay.gu_scale_offset if lay.gu_scale_offset >= 0 else None
            dsc = base + lay.down_scale_offset if lay.down_scale_offset >= 0 else None
            gpu_gen.fill_expert(cfg, layer, e, base + lay.gu_offset, base + lay.down_offset, gsc,
                                dsc, s)
    return store
