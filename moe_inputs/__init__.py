"""Seeded synthetic workloads for the DWDP MoE block (shared by the oracle
and the GPU path as bytes; holds none of the layer's arithmetic)."""
from .configs import CONFIGS, SEED, MoEConfig, config  # noqa: F401
