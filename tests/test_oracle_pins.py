"""Pins of the oracle against facts fixed by the mathematics (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a changed summation order, a wrong
tie rule) fails at least one of them.  None re-types the oracle's formula.
"""
import itertools
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from moe_inputs import config, gen

getcontext().prec = 50


def _ulp_diff64(a, b):
    ai = np.asarray(a, dtype=np.float64).view(np.int64)
    bi = np.asarray(b, dtype=np.float64).view(np.int64)
    return np.abs(ai - bi)


# ---------------------------------------------------------------- exp / sigmoid
def test_exp64_vs_correctly_rounded_decimal():
    rng = np.random.default_rng(5)
    y = np.concatenate([rng.uniform(-40, 120, 4000), rng.uniform(-1, 1, 2000),
                        [0.0, 1.0, -1.0, 0.5 * np.log(2), 709.0, -700.0, 1e-300]])
    ours = oracle.exp64(y)
    ref = np.array([float(Decimal(float(v)).exp()) for v in y])
    d = _ulp_diff64(ours, ref)
    assert d.max() <= 1, d.max()
    assert (d == 0).mean() > 0.85   # plain Horner: faithful, mostly correctly rounded
    assert oracle.exp64(np.array([0.0]))[0] == 1.0


def test_sigmoid_vs_correctly_rounded_decimal():
    rng = np.random.default_rng(6)
    l = np.concatenate([rng.standard_normal(20000) * 4, rng.uniform(-110, 30, 2000)]).astype(np.float32)
    ours = oracle.sigmoid_f32(l)
    ref = np.array([float(np.float32(float(1 / (1 + (-Decimal(float(v))).exp())))) for v in l],
                   dtype=np.float32)
    ui = np.abs(ours.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ui.max() <= 1
    assert (ui == 0).mean() > 0.9999


def test_sigmoid_special_values():
    s = oracle.sigmoid_f32(np.array([0.0, 40.0, 18.0, 1e30, -104.0, -120.0, -1e30, -17.0],
                                    dtype=np.float32))
    assert s[0] == np.float32(0.5)
    assert s[1] == 1.0 and s[2] == 1.0 and s[3] == 1.0
    assert s[4] == 0.0 and s[5] == 0.0 and s[6] == 0.0
    assert 0 < s[7] < 1e-7
    x = np.sort(np.random.default_rng(7).standard_normal(5000).astype(np.float32) * 8)
    assert (np.diff(oracle.sigmoid_f32(x)) >= 0).all()


# ---------------------------------------------------------------- router logits
def test_logits_use_fused_multiply_add():
    # p = -(1+2^-11); then fma((1+2^-12), (1+2^-12), p) = 2^-24 exactly;
    # a separate multiply would round the product to 1+2^-11 and give 0.
    a = np.float32(1 + 2 ** -12)
    x = np.array([[1.0, a]], dtype=np.float32)
    w = np.array([[-(1 + 2 ** -11), a]], dtype=np.float32)
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2 ** -24)


def test_logits_chunked_summation_order():
    # 512 = two 256-wide chunks.  Chunk 0 is 2^24 followed by 255 ones, each
    # lost to round-half-even (P_0 = 2^24); chunk 1 is 256 ones (P_1 = 256).
    # So l = 2^24 + 256.  A single left-to-right chain would give 2^24.
    x = np.ones((1, 512), dtype=np.float32)
    w = np.ones((1, 512), dtype=np.float32)
    w[0, 0] = 2.0 ** 24
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2 ** 24 + 256)
    # chunks are summed in ascending order: (P0 + P1) + P2 with P0 = 2^24,
    # P1 = 1, P2 = 1  ->  2^24 (each add ties to even), not 2^24 + 2
    x = np.zeros((1, 768), dtype=np.float32)
    w = np.zeros((1, 768), dtype=np.float32)
    x[0, 0], w[0, 0] = 1.0, 2.0 ** 24
    x[0, 256], w[0, 256] = 1.0, 1.0
    x[0, 512], w[0, 512] = 1.0, 1.0
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2 ** 24)
    # ragged last chunk (H = 300): same value as the exact sum of small integers
    x = np.arange(300, dtype=np.float32)[None, :] % 7
    w = np.arange(300, dtype=np.float32)[None, :] % 5
    assert oracle.router_logits(x, w)[0, 0] == float((x.astype(np.int64) * w.astype(np.int64)).sum())


def test_logits_exact_for_small_integers_and_transpose():
    rng = np.random.default_rng(8)
    x = rng.integers(-8, 9, (7, 768)).astype(np.float32)
    w = rng.integers(-8, 9, (5, 768)).astype(np.float32)
    ref = x.astype(np.int64) @ w.astype(np.int64).T   # exact, |.| < 2^24
    np.testing.assert_array_equal(oracle.router_logits(x, w), ref.astype(np.float32))


def test_logits_within_rounding_bound_of_fp64():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((16, 7168)).astype(np.float32)
    w = (rng.standard_normal((32, 7168)) * 0.02).astype(np.float32)
    ours = oracle.router_logits(x, w).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    bound = 7168 * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T)
    assert (np.abs(ours - ref) <= bound).all()


# ---------------------------------------------------------------- selection
def _dominates(ka, a, kb, b):
    return ka > kb or (ka == kb and a < b)


def _brute_topset(keys, cand, k):
    """The unique k-subset of cand whose members all dominate every non-member."""
    found = None
    for S in itertools.combinations(cand, k):
        rest = [e for e in cand if e not in S]
        if all(_dominates(keys[a], a, keys[b], b) for a in S for b in rest):
            assert found is None
            found = S
    return set(found)


def _check_order(keys, idx):
    for a, b in zip(idx[:-1], idx[1:]):
        assert _dominates(keys[a], a, keys[b], b)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(10)
    for _ in range(200):
        keys = (rng.integers(0, 5, 8) / 4).astype(np.float32)  # many ties
        idx = oracle.topk_desc(keys[None, :], 2)[0]
        assert set(idx.tolist()) == _brute_topset(keys, list(range(8)), 2)
        _check_order(keys, idx)


def test_group_limited_brute_force():
    rng = np.random.default_rng(11)
    E, G, Gk, k = 16, 4, 2, 3
    gs = E // G
    for _ in range(150):
        keys = (rng.integers(0, 6, E) / 8).astype(np.float32)
        idx = oracle.select_group_limited(keys[None, :], G, Gk, k)[0]
        # group score by brute force over pairs of distinct members
        score = [max(np.float32(keys[a] + keys[b]) for a, b in
                     itertools.combinations(range(g * gs, (g + 1) * gs), 2)) for g in range(G)]
        gsel = _brute_topset(np.array(score, dtype=np.float32), list(range(G)), Gk)
        cand = [e for e in range(E) if e // gs in gsel]
        assert set(idx.tolist()) == _brute_topset(keys, cand, k)
        _check_order(keys, idx)


def test_group_limited_with_all_groups_is_plain_topk():
    rng = np.random.default_rng(12)
    keys = rng.standard_normal((50, 32)).astype(np.float32)
    for row in range(50):
        a = oracle.select_group_limited(keys[row:row + 1], 4, 4, 5)[0]
        assert set(a.tolist()) == _brute_topset(keys[row], list(range(32)), 5)


def test_softmax_weights_closed_form():
    c = config(1)
    li = gen.layer_inputs(c)
    idx, w, l = oracle.route(li.x, li.wg, None, k=2, score="softmax")
    l64 = l.astype(np.float64)
    t = np.arange(c.T)
    d = l64[t, idx[:, 1]] - l64[t, idx[:, 0]]
    np.testing.assert_allclose(w[:, 0], 1 / (1 + np.exp(d)), rtol=1e-14)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
    # unnormalised: full-softmax probabilities of the two chosen experts
    _, w2, _ = oracle.route(li.x, li.wg, None, k=2, score="softmax", renormalize=False)
    p = np.exp(l64 - l64.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(w2, p[t[:, None], idx], rtol=1e-13)


def test_sigmoid_route_structure():
    c = config(2)
    li = gen.layer_inputs(c)
    idx, w, l = oracle.route(li.x, li.wg, li.bias, k=c.k, score="sigmoid", n_group=8,
                             topk_group=4, routed_scale=2.5)
    s = 1 / (1 + np.exp(-l.astype(np.float64)))
    t = np.arange(c.T)[:, None]
    np.testing.assert_allclose(w.sum(1), 2.5, rtol=2e-6)
    np.testing.assert_allclose(w / w[:, :1], s[t, idx] / s[t, idx[:, :1]], rtol=2e-6)
    for r in range(c.T):
        assert len(set(idx[r].tolist())) == c.k
        assert len(set((idx[r] // 32).tolist())) <= 4
    # bias shifts selection only: with bias the keys of chosen experts dominate
    key = (oracle.sigmoid_f32(l) + li.bias[None, :]).astype(np.float32)
    kk = key[t, idx]
    assert (np.diff(kk, axis=1) <= 0).all()


# ---------------------------------------------------------------- permutation
def _perm_by_loops(idx, E):
    T, k = idx.shape
    rows, inv = [], np.full((T, k), -1)
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    inv[t, j] = len(rows)
                    rows.append(t)
    counts = [int((idx == e).sum()) for e in range(E)]
    return np.array(rows), inv, counts


def test_permute_against_loops_and_invariants():
    rng = np.random.default_rng(13)
    for T, k, E in [(1, 1, 1), (7, 2, 8), (40, 3, 5), (0, 2, 4), (33, 8, 256)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]) if T else \
            np.zeros((0, k), dtype=np.int32)
        idx = idx.astype(np.int32)
        off, src, inv = oracle.permute(idx, E)
        rows, inv_ref, counts = _perm_by_loops(idx, E)
        np.testing.assert_array_equal(src, rows.astype(np.int32) if T else src)
        np.testing.assert_array_equal(inv, inv_ref)
        assert off[0] == 0 and off[-1] == T * k and (np.diff(off) == counts).all()
        x = rng.standard_normal((T, 3))
        xp = x[src]
        for j in range(k):
            np.testing.assert_array_equal(xp[inv[:, j]], x)


# ---------------------------------------------------------------- FFN / layer
class _W:
    def __init__(self, gu, down):
        self.gu, self.down = gu, down

    def gu_f64(self):
        return self.gu

    def down_f64(self):
        return self.down


def _dense_swiglu(x, gate, up, down):
    # independent form: silu(g) = g (1 + tanh(g/2)) / 2, explicit einsums
    g = np.einsum("th,ih->ti", x, gate)
    u = np.einsum("th,ih->ti", x, up)
    h = g * (1 + np.tanh(g / 2)) / 2 * u
    return np.einsum("ti,hi->th", h, down)


def _rand_experts(rng, E, H, I):
    return [_W(rng.standard_normal((2 * I, H)) * 0.1, rng.standard_normal((H, I)) * 0.1)
            for _ in range(E)]


def test_dense_identity_single_expert():
    rng = np.random.default_rng(14)
    T, H, I, E = 9, 16, 8, 3
    ws = _rand_experts(rng, E, H, I)
    x = rng.standard_normal((T, H))
    for e in range(E):
        idx = np.full((T, 1), e, dtype=np.int32)
        pools = oracle.SplitPools([(0 << 31) | i for i in range(E)], ws, [])
        y, _ = oracle.moe_layer(x, idx, np.ones((T, 1)), E, pools)
        ref = _dense_swiglu(x, ws[e].gu[:I], ws[e].gu[I:], ws[e].down)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_shared_expert_and_combine_linearity():
    rng = np.random.default_rng(15)
    T, H, I, E, k = 11, 16, 8, 6, 2
    ws = _rand_experts(rng, E, H, I)
    sh = _rand_experts(rng, 1, H, I)[0]
    x = rng.standard_normal((T, H))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1, (T, k))
    table = [(0 << 31) | i for i in range(E)]
    y0, _ = oracle.moe_layer(x, idx, w, E, oracle.SplitPools(table, ws, []))
    y1, _ = oracle.moe_layer(x, idx, w, E, oracle.SplitPools(table, ws, [], shared=sh))
    np.testing.assert_allclose(y1 - y0, _dense_swiglu(x, sh.gu[:I], sh.gu[I:], sh.down),
                               rtol=1e-10, atol=1e-13)
    y2, _ = oracle.moe_layer(x, idx, 2 * w, E, oracle.SplitPools(table, ws, []))
    np.testing.assert_allclose(y2, 2 * y0, rtol=1e-13, atol=1e-15)
    # k = 1, w = 1 is a plain gather of each token's expert output
    idx1 = idx[:, :1]
    y3, _ = oracle.moe_layer(x, idx1, np.ones((T, 1)), E, oracle.SplitPools(table, ws, []))
    for t in range(T):
        e = idx1[t, 0]
        ref = _dense_swiglu(x[t:t + 1], ws[e].gu[:I], ws[e].gu[I:], ws[e].down)[0]
        np.testing.assert_allclose(y3[t], ref, rtol=1e-12, atol=1e-15)


def test_pool_invariance():
    rng = np.random.default_rng(16)
    T, H, I, E, k = 13, 16, 8, 8, 2
    ws = _rand_experts(rng, E, H, I)
    x = rng.standard_normal((T, H))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1, (T, k))
    ref = None
    for trial in range(6):
        if trial == 0:
            local = list(range(E))            # all local
        elif trial == 1:
            local = []                        # all remote
        else:
            local = sorted(rng.choice(E, rng.integers(1, E), replace=False).tolist())
        remote = [e for e in range(E) if e not in local]
        lslots = list(rng.permutation(len(local)))
        rslots = list(rng.permutation(len(remote)))
        lpool, rpool = [None] * len(local), [None] * len(remote)
        table = [0] * E
        for i, e in enumerate(local):
            lpool[lslots[i]] = ws[e]
            table[e] = (0 << 31) | int(lslots[i])
        for i, e in enumerate(remote):
            rpool[rslots[i]] = ws[e]
            table[e] = (1 << 31) | int(rslots[i])
        y, _ = oracle.moe_layer(x, idx, w, E, oracle.SplitPools(table, lpool, rpool))
        if ref is None:
            ref = y
        np.testing.assert_array_equal(y, ref)


def test_sampled_tokens_match_full_layer():
    c = config(1)
    li = gen.layer_inputs(c)
    idx, w, _ = oracle.route(li.x, li.wg, None, k=c.k, score="softmax")
    experts = [gen.expert_host(c, 0, e) for e in range(c.E)]
    table = [(0 << 31) | e if e < 4 else (1 << 31) | (e - 4) for e in range(c.E)]
    pools = oracle.SplitPools(table, experts[:4], experts[4:])
    x64 = li.x.astype(np.float64)
    y, _ = oracle.moe_layer(x64, idx, w, c.E, pools)
    sel = np.array([0, 5, 17, 63])
    ys = oracle.moe_layer_tokens(x64[sel], idx[sel], w[sel], pools.expert)
    np.testing.assert_allclose(ys, y[sel], rtol=1e-12, atol=1e-15)


def test_fp8_weights_reduce_to_bf16_when_scales_are_one():
    # every e4m3 value is exactly a bf16 value; with scale 1 the e4m3 expert
    # and the bf16 expert holding the same values give the same layer
    rng = np.random.default_rng(17)
    H, I = 128, 128
    codes_gu = rng.integers(0, 0x7E, (2 * I, H)).astype(np.uint8) | \
        (rng.integers(0, 2, (2 * I, H)).astype(np.uint8) << 7)
    codes_dn = rng.integers(0, 0x60, (H, I)).astype(np.uint8)
    e8 = gen.ExpertHost(gu=codes_gu, down=codes_dn, gu_scale=np.ones((2, 1), np.float32),
                        down_scale=np.ones((1, 1), np.float32))
    bf = gen.ExpertHost(gu=gen.f32_to_bf16_bits(gen.E4M3_VALUES[codes_gu].astype(np.float32)),
                        down=gen.f32_to_bf16_bits(gen.E4M3_VALUES[codes_dn].astype(np.float32)))
    np.testing.assert_array_equal(e8.gu_f64(), bf.gu_f64())
    x = rng.standard_normal((5, H)) * 0.01
    idx = np.zeros((5, 1), dtype=np.int32)
    a, _ = oracle.moe_layer(x, idx, np.ones((5, 1)), 1, oracle.SplitPools([0], [e8], []))
    b, _ = oracle.moe_layer(x, idx, np.ones((5, 1)), 1, oracle.SplitPools([0], [bf], []))
    np.testing.assert_array_equal(a, b)
    # and a non-unit block scale multiplies exactly
    e8s = gen.ExpertHost(gu=codes_gu, down=codes_dn,
                         gu_scale=np.array([[0.5], [2.0]], np.float32),
                         down_scale=np.ones((1, 1), np.float32))
    np.testing.assert_array_equal(e8s.gu_f64()[:128], 0.5 * e8.gu_f64()[:128])
    np.testing.assert_array_equal(e8s.gu_f64()[128:], 2.0 * e8.gu_f64()[128:])
