"""ORACLE (test infrastructure): the oracle applied to a seeded workload.

Regenerates inputs with the host generators of ``moe_inputs`` and runs the
plain CPU definition of the layer.  Used only by tests, the smoke check and
the benchmark's CPU baseline.
"""
from __future__ import annotations

import numpy as np

from moe_inputs import gen
from moe_inputs.configs import MoEConfig, config

from . import moe as om


class LazyPool:
    """Pool slots generated on first access (host copy of the weights)."""

    def __init__(self, cfg: MoEConfig, layer: int, slot_to_expert: dict[int, int], cache: dict):
        self.cfg, self.layer, self.map, self.cache = cfg, layer, slot_to_expert, cache

    def __getitem__(self, slot: int):
        e = self.map[slot]
        key = (self.layer, e)
        if key not in self.cache:
            self.cache[key] = gen.expert_host(self.cfg, self.layer, e)
        return self.cache[key]


def split_pools(cfg, layer: int, pool: np.ndarray, slot: np.ndarray, cache: dict | None = None):
    cfg = config(cfg)
    cache = {} if cache is None else cache
    maps = ({}, {})
    for e in range(cfg.E):
        maps[int(pool[e])][int(slot[e])] = e
    table = [(int(pool[e]) << 31) | int(slot[e]) for e in range(cfg.E)]
    shared = gen.expert_host(cfg, layer, cfg.E) if cfg.has_shared else None
    return om.SplitPools(table, LazyPool(cfg, layer, maps[0], cache),
                         LazyPool(cfg, layer, maps[1], cache), shared)


def route(cfg, layer: int = 0, inputs: gen.LayerInputs | None = None):
    cfg = config(cfg)
    li = gen.layer_inputs(cfg, layer) if inputs is None else inputs
    return om.route(li.x, li.wg, li.bias, k=cfg.k, score=cfg.score, n_group=cfg.n_group,
                    topk_group=cfg.topk_group, routed_scale=cfg.routed_scale,
                    renormalize=cfg.renormalize)


def layer_full(cfg, layer: int, pool, slot, inputs: gen.LayerInputs | None = None):
    """Whole-layer oracle: (y fp64 [T,H], idx, w, (offsets, perm_src, inv_pos))."""
    cfg = config(cfg)
    li = gen.layer_inputs(cfg, layer) if inputs is None else inputs
    idx, w, _ = route(cfg, layer, li)
    y, perm = om.moe_layer(li.x.astype(np.float64), idx, w, cfg.E,
                           split_pools(cfg, layer, pool, slot))
    return y, idx, w, perm


def layer_tokens(cfg, layer: int, tokens: np.ndarray, idx: np.ndarray, w: np.ndarray, pool, slot,
                 inputs: gen.LayerInputs | None = None, cache: dict | None = None):
    """Oracle output rows for the given tokens only."""
    cfg = config(cfg)
    li = gen.layer_inputs(cfg, layer) if inputs is None else inputs
    pools = split_pools(cfg, layer, pool, slot, cache)
    return om.moe_layer_tokens(li.x[tokens].astype(np.float64), idx[tokens], w[tokens],
                               pools.expert, pools.shared)
