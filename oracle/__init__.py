"""ORACLE: a plain, slow, CPU-only statement of the DWDP per-rank MoE block.

This package is TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke``
and ``bench.py``'s CPU-baseline leg (``cpu_baseline`` / ``--impl reference``)
import it.  The product path (``split_weight_b200``) never imports, links or
runs anything here, and this package uses none of the product's code: the two
share only the seeded input generators of ``moe_inputs``.

Parity pins (tests/test_oracle_*.py) check it against facts the mathematics
fixes: brute-force top-k, closed forms, textbook special cases, exact
invariants (permutation inverse, pool invariance, dense-FFN identity) and a
correctly rounded decimal reference for its exponential.
"""
from .moe import (  # noqa: F401
    POOL_LOCAL, POOL_REMOTE, SplitPools, build, exp64, group_scores, moe_layer,
    moe_layer_tokens, permute, route, router_logits, select_group_limited, sigmoid_f32,
    swiglu_ffn, topk_desc,
)
