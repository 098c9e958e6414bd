"""split_weight_b200: the per-rank MoE block of DWDP (Distributed Weight Data
Parallelism) on one B200.

The C ABI (include/moe.h, libswb_moe.so) holds every step: routing, the
expert permutation, the tcgen05 grouped SwiGLU GEMMs over a split (local +
remote) weight table, the weighted combine and the copy-engine prefetch of
remote experts.  ``_lib`` binds it with ctypes; ``layer`` drives a layer or a
pipeline of layers with torch buffers and streams.
"""
from . import _lib  # noqa: F401  (raises ImportError when the library is missing)
from ._lib import MoEError, check  # noqa: F401
from .layer import (DenseBlock, LayerShape, MoELayer, PeerPools, PrefetchPipeline, Progress,  # noqa: F401
                    ReadyGate, SplitWeights, close_pool, export_pool, import_pool)
