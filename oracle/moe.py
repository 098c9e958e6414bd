"""ORACLE of the DWDP per-rank MoE expert block: plain, slow, CPU only.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this module.  It shares no code with the CUDA path.

What it follows.  "DWDP: Distributed Weight Data Parallelism for
High-Performance LLM Inference on NVL72" (arXiv 2604.01621, abstract) keeps
every GPU data parallel: each rank runs the MoE block on its own tokens, with
the MoE weights split over its peers and the missing experts fetched.  The
explainer "Distributed Weight Data Parallelism cuts LLM inference stalls"
adds, in its split-weight figure, that the local and remote expert weights
have to reach the grouped GEMM kernel of the block; where the weights sit
changes nothing in what the block computes.  So the oracle is the plain
definition of one MoE layer, with each expert's weights looked up through a
(pool, slot) table spanning a local and a remote pool.

The pages state none of the layer's arithmetic.  The readings used (DeepSeek-R1
layer shape, read plainly) are:

* router logits in one fixed fp32 order (``router.c``);
* softmax routing: top-k of the logits, weights renormalised over the k;
* sigmoid routing: s = sigmoid(l) (fp64, own exp, rounded to fp32), selection
  key s + bias (fp32), group score = sum of the two largest keys of a group,
  keep topk_group groups, then top-k keys inside them; weights s_j / sum(s)
  times routed_scale in fp32;  ties always go to the lower index;
* permutation: stable counting sort of the assignments a = t*k + j by expert;
* expert FFN: SwiGLU, h = silu(x W_gate^T) * (x W_up^T), y = h W_down^T, in
  fp64 on the exact weight values (bf16, or e4m3 code times its fp32 block
  scale); one shared expert on every token with weight 1;
* combine: y[t] = sum_j w[t,j] y_{e_j}[t] (ascending j) + y_shared[t].
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from decimal import Decimal, getcontext
from typing import Callable

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle_router.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles router.c (plain C, -ffp-contract=off) next to this file."""
    src = os.path.join(_HERE, "router.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(src) > os.path.getmtime(_SO):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _router_lib():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_router_logits.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.oracle_router_logits.restype = None
        _lib = lib
    return _lib


# ---------------------------------------------------------------------------
# router logits
# ---------------------------------------------------------------------------
def router_logits(x: np.ndarray, wg: np.ndarray) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] W_g[e,h] in fp32, in 256-wide fused-multiply-add
    chunks summed in ascending order (order defined in router.c)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    wg = np.ascontiguousarray(wg, dtype=np.float32)
    T, H = x.shape
    E, H2 = wg.shape
    assert H == H2
    out = np.empty((T, E), dtype=np.float32)
    if T and E:
        _router_lib().oracle_router_logits(x.ctypes.data, wg.ctypes.data, T, H, E, out.ctypes.data)
    return out


# ---------------------------------------------------------------------------
# fp64 exponential and sigmoid, written from the mathematics
# ---------------------------------------------------------------------------
def _derive_exp_constants():
    """Cody-Waite argument reduction (W. J. Cody, W. Waite, "Software Manual
    for the Elementary Functions", 1980): ln 2 split as LN2_HI + LN2_LO with
    LN2_HI's low 21 mantissa bits zero, so n * LN2_HI is exact for |n| < 2^21;
    then exp(r) = sum_{i<=13} r^i / i! for |r| <= ln2/2 (truncation below
    2^-55 relative)."""
    getcontext().prec = 60
    ln2 = Decimal(2).ln()
    inv_ln2 = float(1 / ln2)
    hi_bits = np.array([float(ln2)], dtype=np.float64).view(np.uint64)[0] & ~np.uint64((1 << 21) - 1)
    ln2_hi = float(np.array([hi_bits], dtype=np.uint64).view(np.float64)[0])
    ln2_lo = float(ln2 - Decimal(ln2_hi))
    coef = [1 / math.factorial(i) for i in range(14)]  # correctly rounded int division
    return inv_ln2, ln2_hi, ln2_lo, coef


INV_LN2, LN2_HI, LN2_LO, EXP_COEF = _derive_exp_constants()


def exp64(y: np.ndarray) -> np.ndarray:
    """e^y in fp64 for |y| <= 700.  Every step is one IEEE operation (numpy
    evaluates each operator separately, nothing is fused):
    n = rint(y / ln2), r = (y - n LN2_HI) - n LN2_LO, Horner polynomial in r,
    scaled by 2^n exactly."""
    y = np.asarray(y, dtype=np.float64)
    n = np.rint(y * INV_LN2)
    r = (y - n * LN2_HI) - n * LN2_LO
    p = np.full_like(r, EXP_COEF[13])
    for i in range(12, -1, -1):
        p = p * r + EXP_COEF[i]
    return np.ldexp(p, n.astype(np.int64))


def sigmoid_f32(l: np.ndarray) -> np.ndarray:
    """s = fp32( 1 / (1 + e^-x) ), x = l widened to fp64 and clamped to
    [-120, 40].  The clamp changes no fp32 result: sigma(x) rounds to 1.0f for
    x >= 18 and to 0.0f for x <= -104."""
    x = np.clip(np.asarray(l, dtype=np.float32).astype(np.float64), -120.0, 40.0)
    e = exp64(-x)
    return (1.0 / (1.0 + e)).astype(np.float32)


# ---------------------------------------------------------------------------
# scoring and selection
# ---------------------------------------------------------------------------
def topk_desc(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, in descending key order; equal
    keys are taken lower index first (stable sort of -key)."""
    order = np.argsort(-np.asarray(keys, dtype=np.float32), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def group_scores(keys: np.ndarray, n_group: int) -> np.ndarray:
    """Score of each contiguous expert group: fp32 sum of its two largest keys
    (its single key for one-expert groups)."""
    T, E = keys.shape
    gs = E // n_group
    srt = np.sort(keys.reshape(T, n_group, gs), axis=2)
    if gs == 1:
        return srt[:, :, 0].astype(np.float32)
    return (srt[:, :, -1] + srt[:, :, -2]).astype(np.float32)


def select_group_limited(keys: np.ndarray, n_group: int, topk_group: int, k: int) -> np.ndarray:
    """Keep the topk_group best groups (ties to the lower group), then the top-k
    keys among their experts."""
    T, E = keys.shape
    gsel = topk_desc(group_scores(keys, n_group), topk_group)
    mask = np.zeros((T, n_group), dtype=bool)
    mask[np.arange(T)[:, None], gsel] = True
    cand = np.repeat(mask, E // n_group, axis=1)
    masked = np.where(cand, keys, np.float32(-np.inf)).astype(np.float32)
    return topk_desc(masked, k)


def route(x: np.ndarray, wg: np.ndarray, bias: np.ndarray | None, *, k: int, score: str,
          n_group: int = 1, topk_group: int = 1, routed_scale: float = 1.0,
          renormalize: bool = True, logits: np.ndarray | None = None):
    """Router + top-k of one MoE layer.

    Returns (topk_idx int32 [T,k], topk_w float64 [T,k], logits fp32 [T,E]).
    For sigmoid routing topk_w holds the fp32 weights exactly (the arithmetic
    is defined in fp32); for softmax routing it is the fp64 value.
    """
    l = router_logits(x, wg) if logits is None else np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    rows = np.arange(T)[:, None]
    if score == "softmax":
        idx = topk_desc(l, k)
        l64 = l.astype(np.float64)
        lmax = l64[rows, idx[:, :1]]
        num = np.exp(l64[rows, idx] - lmax)
        den = num.sum(axis=1, keepdims=True) if renormalize else \
            np.exp(l64 - lmax).sum(axis=1, keepdims=True)
        return idx, num / den * routed_scale, l
    if score == "sigmoid":
        s = sigmoid_f32(l)
        key = s if bias is None else (s + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)
        idx = select_group_limited(key, n_group, topk_group, k)
        ssel = s[rows, idx]
        if renormalize:
            d = np.zeros(T, dtype=np.float32)
            for j in range(k):
                d = (d + ssel[:, j]).astype(np.float32)
            w = (ssel / d[:, None]).astype(np.float32)
        else:
            w = ssel
        w = (w * np.float32(routed_scale)).astype(np.float32)
        return idx, w.astype(np.float64), l
    raise ValueError(score)


# ---------------------------------------------------------------------------
# permutation
# ---------------------------------------------------------------------------
def permute(topk_idx: np.ndarray, E: int):
    """Stable counting sort of the assignments a = t*k + j by expert.

    Returns offsets [E+1] (offsets[e] = first row of expert e), perm_src [A]
    (token of each permuted row) and inv_pos [T,k] (row of assignment (t,j)).
    """
    T, k = topk_idx.shape
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm_src = (order // k).astype(np.int32)
    inv_pos = np.empty(T * k, dtype=np.int32)
    inv_pos[order] = np.arange(T * k, dtype=np.int32)
    return offsets, perm_src, inv_pos.reshape(T, k)


# ---------------------------------------------------------------------------
# split-weight lookup and the expert FFN
# ---------------------------------------------------------------------------
POOL_LOCAL, POOL_REMOTE = 0, 1


class SplitPools:
    """Expert weights reached through a (pool, slot) table spanning two pools.

    pool_slot[e] = (pool << 31) | slot; pools[pool][slot] is an object with
    gu_f64() -> [2I, H] and down_f64() -> [H, I] (exact values).
    """

    def __init__(self, pool_slot, local, remote, shared=None):
        self.pool_slot = np.asarray(pool_slot, dtype=np.int64)
        self.pools = (local, remote)
        self.shared = shared

    def expert(self, e: int):
        ps = int(self.pool_slot[e])
        return self.pools[(ps >> 31) & 1][ps & 0x7FFFFFFF]


def swiglu_ffn(x64: np.ndarray, gu: np.ndarray, down: np.ndarray) -> np.ndarray:
    """SwiGLU expert in fp64: gate rows [0, I), up rows [I, 2I) of gu."""
    I = gu.shape[0] // 2
    g = x64 @ gu[:I].T
    u = x64 @ gu[I:].T
    with np.errstate(over="ignore"):
        h = g * (1.0 / (1.0 + np.exp(-g))) * u
    return h @ down.T


def moe_layer(x64: np.ndarray, topk_idx: np.ndarray, topk_w: np.ndarray, E: int,
              pools: SplitPools):
    """Full layer output y [T,H] (fp64) from the routing, plus the permutation."""
    T, k = topk_idx.shape
    H = x64.shape[1]
    offsets, perm_src, inv_pos = permute(topk_idx, E)
    y_perm = np.zeros((T * k, H), dtype=np.float64)
    for e in range(E):
        o0, o1 = int(offsets[e]), int(offsets[e + 1])
        if o1 > o0:
            w = pools.expert(e)
            y_perm[o0:o1] = swiglu_ffn(x64[perm_src[o0:o1]], w.gu_f64(), w.down_f64())
    y = np.zeros((T, H), dtype=np.float64)
    for j in range(k):
        y += topk_w[:, j:j + 1] * y_perm[inv_pos[:, j]]
    if pools.shared is not None:
        y += swiglu_ffn(x64, pools.shared.gu_f64(), pools.shared.down_f64())
    return y, (offsets, perm_src, inv_pos)


def moe_layer_tokens(x64_rows: np.ndarray, idx_rows: np.ndarray, w_rows: np.ndarray,
                     expert_weights: Callable[[int], object], shared=None) -> np.ndarray:
    """The same layer output for a subset of tokens only (the block is per
    token): y[t] = sum_j w[t,j] FFN_{e_j}(x_t) + FFN_shared(x_t).
    expert_weights(e) returns an object with gu_f64() / down_f64()."""
    n, k = idx_rows.shape
    y = np.zeros((n, x64_rows.shape[1]), dtype=np.float64)
    contrib = {}
    for e in np.unique(idx_rows):
        w = expert_weights(int(e))
        toks = np.nonzero((idx_rows == e).any(axis=1))[0]
        out = swiglu_ffn(x64_rows[toks], w.gu_f64(), w.down_f64())
        for r, t in enumerate(toks):
            contrib[(int(t), int(e))] = out[r]
    for j in range(k):
        for t in range(n):
            y[t] += w_rows[t, j] * contrib[(t, int(idx_rows[t, j]))]
    if shared is not None:
        y += swiglu_ffn(x64_rows, shared.gu_f64(), shared.down_f64())
    return y
