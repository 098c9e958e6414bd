"""The C ABI on the host: symbols, layouts and argument checks (no GPU work)."""
import ctypes

import pytest

from split_weight_b200 import _lib as L


def test_library_exports_every_declared_function():
    names = L.header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L._lib, n), f"{n} declared in include/moe.h but not exported"
    assert L.moe_abi_version() == 1


def test_status_strings():
    for code, name in [(0, "MOE_OK"), (1, "MOE_ERR_INVALID_ARG"), (2, "MOE_ERR_UNSUPPORTED"),
                       (3, "MOE_ERR_WORKSPACE"), (4, "MOE_ERR_CUDA"), (5, "MOE_ERR_TIMEOUT"),
                       (6, "MOE_ERR_DEVICE_CHECK")]:
        assert L.status_string(code) == name


def test_expert_layout():
    lay = L.expert_layout(7168, 2048, L.MOE_BF16)
    assert (lay.gu_offset, lay.down_offset) == (0, 2 * 2048 * 7168 * 2)
    assert lay.bytes == 3 * 2048 * 7168 * 2 and lay.gu_scale_offset == -1
    lay = L.expert_layout(7168, 2048, L.MOE_E4M3)
    assert lay.down_offset == 2 * 2048 * 7168
    assert lay.gu_scale_offset == 3 * 2048 * 7168
    assert lay.down_scale_offset == lay.gu_scale_offset + 32 * 56 * 4
    assert lay.bytes % 256 == 0 and lay.bytes >= lay.down_scale_offset + 56 * 16 * 4
    bad = L.moe_expert_layout()
    assert L.moe_expert_layout_get(7168, 100, L.MOE_BF16, ctypes.byref(bad)) == L.MOE_ERR_INVALID_ARG
    assert L.moe_expert_layout_get(256, 128, L.MOE_F32, ctypes.byref(bad)) == L.MOE_ERR_UNSUPPORTED


def _route_cfg(**kw):
    c = dict(T=16, H=256, E=8, k=2, score=L.MOE_SCORE_SOFTMAX, n_group=1, topk_group=1,
             routed_scale=1.0, renormalize=1)
    c.update(kw)
    return L.moe_route_cfg(*[c[f] for f, _ in L.moe_route_cfg._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), L.MOE_ERR_INVALID_ARG),
    (dict(k=9), L.MOE_ERR_INVALID_ARG),
    (dict(E=2000), L.MOE_ERR_INVALID_ARG),
    (dict(H=100), L.MOE_ERR_INVALID_ARG),
    (dict(score=7), L.MOE_ERR_INVALID_ARG),
    (dict(score=L.MOE_SCORE_SIGMOID, n_group=3), L.MOE_ERR_INVALID_ARG),
    (dict(score=L.MOE_SCORE_SIGMOID, n_group=4, topk_group=5), L.MOE_ERR_INVALID_ARG),
    (dict(score=L.MOE_SCORE_SIGMOID, n_group=4, topk_group=1, k=3), L.MOE_ERR_INVALID_ARG),
])
def test_route_rejects_bad_config(kw, code):
    c = _route_cfg(**kw)
    assert L.moe_route(ctypes.byref(c), 16, L.MOE_BF16, 16, None, 16, 16, None, 0, None) == code
    assert L.moe_last_error()


@pytest.mark.parametrize("T,H,planes", [
    (128, 7168, 28),     # decode: small tiles split over the 28 chunks of 256 h
    (3001, 512, 1),      # medium batch: 64x64 tiles, logits written once
    (8192, 7168, 28),    # 8K prefill: 64x128 tiles split over the chunks
    (7700, 384, 2),      # large batch with a short last chunk (256 + 128 h)
])
def test_route_workspace_holds_one_plane_per_split_chunk(T, H, planes):
    """moe_route's workspace is one fp32 [T, E] plane per 256-wide chunk when
    the logits kernel splits the chunks over its grid, else the logits alone
    (host-side query, no GPU)."""
    c = _route_cfg(T=T, H=H, E=256, k=8, score=L.MOE_SCORE_SIGMOID, n_group=8, topk_group=4)
    assert L.moe_route_workspace_size(ctypes.byref(c)) == planes * T * 256 * 4


@pytest.mark.parametrize("w,act,has_shared,want", [
    (L.MOE_BF16, L.MOE_BF16, 1, 256),                 # two tile counters
    (L.MOE_E4M3, L.MOE_BF16, 1, 256),                 # conversion path: the same counters
    (L.MOE_E4M3, L.MOE_E4M3, 1, (2048 // 128) * (4096 * 8 + 4096) * 4),   # h's scales
    (L.MOE_E4M3, L.MOE_E4M3, 0, (2048 // 128) * (4096 * 8) * 4),
])
def test_grouped_ffn_workspace_size(w, act, has_shared, want):
    """bf16 activations: 256 bytes for the dynamic tile schedule's counters;
    e4m3 activations: the fp32 scales of h, [I/128][rows], rounded up to 256
    bytes (host-side query, no GPU)."""
    d = L.moe_ffn_desc(4096, 7168, 2048, 256, 8, w, act, has_shared)
    assert L.moe_grouped_ffn_workspace_size(ctypes.byref(d)) == -(-want // 256) * 256


def test_route_rejects_null_misaligned_and_small_workspace():
    c = _route_cfg()
    assert L.moe_route(ctypes.byref(c), None, L.MOE_BF16, 16, None, 16, 16, None, 0,
                       None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(c), 18, L.MOE_BF16, 16, None, 16, 16, None, 0,
                       None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(c), 16, L.MOE_E4M3, 16, None, 16, 16, None, 0,
                       None) == L.MOE_ERR_UNSUPPORTED
    need = L.moe_route_workspace_size(ctypes.byref(c))
    assert need > 0
    assert L.moe_route(ctypes.byref(c), 16, L.MOE_BF16, 16, None, 16, 16, 16, need - 1,
                       None) == L.MOE_ERR_WORKSPACE
    # bias only exists for sigmoid scoring
    assert L.moe_route(ctypes.byref(c), 16, L.MOE_BF16, 16, 16, 16, 16, 16, need,
                       None) == L.MOE_ERR_INVALID_ARG
    # T = 0 is a legal no-op
    c0 = _route_cfg(T=0)
    assert L.moe_route(ctypes.byref(c0), None, L.MOE_BF16, None, None, None, None, None, 0,
                       None) == L.MOE_OK


def test_permute_rejects_bad_arguments():
    args = dict(T=4, k=2, E=8, H=256)
    p = 16
    ok_ws = L.moe_permute_workspace_size(4, 2, 8)
    assert ok_ws > 0

    def call(T=4, k=2, E=8, H=256, xdt=L.MOE_BF16, pdt=L.MOE_BF16, ws=ok_ws, x=p):
        return L.moe_permute(T, k, E, H, p, x, xdt, pdt, 1, p, p, p, p, None, p, ws, None)
    assert call(k=0) == L.MOE_ERR_INVALID_ARG
    assert call(E=0) == L.MOE_ERR_INVALID_ARG
    assert call(H=200) == L.MOE_ERR_INVALID_ARG
    assert call(xdt=L.MOE_E4M3) == L.MOE_ERR_UNSUPPORTED
    assert call(pdt=L.MOE_F32) == L.MOE_ERR_UNSUPPORTED
    assert call(ws=ok_ws - 4) == L.MOE_ERR_WORKSPACE
    assert call(x=24) == L.MOE_ERR_INVALID_ARG
    # e4m3 gather needs a scale buffer
    assert L.moe_permute(4, 2, 8, 256, p, p, L.MOE_BF16, L.MOE_E4M3, 0, p, p, p, p, None, p, ok_ws,
                         None) == L.MOE_ERR_INVALID_ARG
    del args


def _ffn(**kw):
    d = dict(T=4, H=256, I=128, E=4, k=2, w_dtype=L.MOE_BF16, act_dtype=L.MOE_BF16, has_shared=0)
    d.update(kw)
    return L.moe_ffn_desc(*[d[f] for f, _ in L.moe_ffn_desc._fields_])


def _table(ps, local_count=2, remote_count=2, stride=None, base=1 << 20, shared=None):
    stride = L.expert_layout(256, 128, L.MOE_BF16).bytes if stride is None else stride
    arr = (ctypes.c_int32 * len(ps))(*ps)
    t = L.moe_expert_table(base, local_count, stride, base * 4, remote_count, stride, shared,
                           ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)))
    t._keep = arr
    return t


def test_grouped_ffn_rejects_bad_tables():
    good = [0, 1, (1 << 31) | 0, (1 << 31) | 1]
    p = 1 << 12

    def call(d, t):
        return L.moe_grouped_ffn(ctypes.byref(d), ctypes.byref(t), p, None, p, p, p, None, 0, None)
    assert call(_ffn(H=200), _table(good)) == L.MOE_ERR_INVALID_ARG
    assert call(_ffn(I=100), _table(good)) == L.MOE_ERR_INVALID_ARG
    assert call(_ffn(w_dtype=L.MOE_F32), _table(good)) == L.MOE_ERR_UNSUPPORTED
    bad_slot = [0, 1, (1 << 31) | 0, (1 << 31) | 2]           # remote pool has 2 slots
    assert call(_ffn(), _table(bad_slot)) == L.MOE_ERR_INVALID_ARG
    bad_pool = [0, 2, (1 << 31) | 0, (1 << 31) | 1]           # local pool has 2 slots
    assert call(_ffn(), _table(bad_pool)) == L.MOE_ERR_INVALID_ARG
    assert call(_ffn(), _table(good, stride=256)) == L.MOE_ERR_INVALID_ARG   # stride < image
    assert call(_ffn(), _table(good, base=(1 << 20) + 16)) == L.MOE_ERR_INVALID_ARG
    assert call(_ffn(has_shared=1), _table(good)) == L.MOE_ERR_INVALID_ARG   # no shared image
    null_ps = _table(good)
    null_ps.pool_slot = None
    assert call(_ffn(), null_ps) == L.MOE_ERR_INVALID_ARG
    assert call(_ffn(T=0), _table(good)) == L.MOE_OK


def test_combine_and_prefetch_argument_checks():
    p = 16
    assert L.moe_combine(4, 0, 256, p, p, p, 0, p, L.MOE_BF16, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_combine(4, 2, 100, p, p, p, 0, p, L.MOE_BF16, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_combine(4, 2, 256, p, p, p, 0, p, L.MOE_E4M3, None) == L.MOE_ERR_UNSUPPORTED
    assert L.moe_combine(4, 2, 256, p, None, p, 0, p, L.MOE_BF16, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_combine(0, 2, 256, None, None, None, 0, None, L.MOE_BF16, None) == L.MOE_OK
    assert L.moe_prefetch_layer(None, 1 << 20, 64, 0, None, None, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_prefetch_layer(1 << 20, (1 << 20) + 32, 64, 0, None, None,
                                None) == L.MOE_ERR_INVALID_ARG   # overlapping ranges
    assert L.moe_prefetch_layer(None, None, 0, 0, None, None, None) == L.MOE_OK
    assert L.moe_wait_ready(None, 10) == L.MOE_ERR_INVALID_ARG


def test_injected_cuda_failure_is_reported_and_cleared():
    L.moe_debug_fail_next_cuda_calls(1)
    rc = L.moe_prefetch_layer(1 << 20, 1 << 24, 64, 0, None, None, None)
    assert rc == L.MOE_ERR_CUDA
    assert "injected" in L.moe_last_error()
    L.moe_debug_fail_next_cuda_calls(0)


@pytest.mark.parametrize("n,lead,base,steps", [(24, 2, 100, 24), (24, 0, 0, 24), (6, 2, 100, 4),
                                               (5, 9, 7, 3), (192, 3, 0xFFFFFFF0, 24),
                                               (3, 0, 5, 40)])
def test_pace_threshold_spreads_chunks_over_the_reports(n, lead, base, steps):
    """moe_pace_threshold: the first `lead` chunks need nothing beyond base;
    the others need a share of the reports that never decreases along the
    fetch and stays within base + steps (wrap-around arithmetic)."""
    t = [L.moe_pace_threshold(c, n, lead, base & 0xFFFFFFFF, steps) for c in range(n)]
    rel = [(v - base) & 0xFFFFFFFF for v in t]
    assert all(r == 0 for r in rel[:lead])
    assert all(a <= b for a, b in zip(rel, rel[1:]))
    assert all(0 <= r <= steps for r in rel)
    if lead < n:
        assert rel[-1] == ((n - lead) * (steps + 1)) // (n - lead + 1)


def test_paced_and_selective_calls_check_arguments_first():
    """Argument errors come back before anything is enqueued (no GPU here)."""
    p = 1 << 12
    pr = L.moe_progress(p, p + 4, 0, 8)
    bad_steps = L.moe_progress(p, p + 4, 0, 1)
    odd_word = L.moe_progress(p + 2, p + 4, 0, 8)
    assert L.moe_prefetch_layer_paced(p, 1 << 24, 1 << 20, 1 << 16, None, None, p, 1, None, 0,
                                      None) == L.MOE_ERR_INVALID_ARG            # no pace
    assert L.moe_prefetch_layer_paced(p, 1 << 24, 1 << 20, 1 << 16, None, None, p, 1,
                                      ctypes.byref(odd_word), 0, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_prefetch_layer_paced(p, 1 << 24, 1 << 20, 1 << 16, None, None, p, 1,
                                      ctypes.byref(pr), -1, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_prefetch_layer_paced(p, 1 << 24, 1 << 20, 0, None, None, p, 1,
                                      ctypes.byref(pr), 0, None) == L.MOE_ERR_INVALID_ARG
    d, tbl = _ffn(), _table([0, 1, 1 << 31, (1 << 31) | 1])
    assert L.moe_grouped_ffn_paced(ctypes.byref(d), ctypes.byref(tbl), None, None, p, None, None,
                                   None, p, p, p, None, 0, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_ffn_paced(ctypes.byref(d), ctypes.byref(tbl), None, ctypes.byref(bad_steps),
                                   p, None, None, None, p, p, p, None, 0,
                                   None) == L.MOE_ERR_INVALID_ARG
    slots = (ctypes.c_int32 * 3)(0, 4, 9)
    assert L.moe_prefetch_slots(p, 1 << 24, 256, 9, slots, 3, None, None, p, 1,
                                None) == L.MOE_ERR_INVALID_ARG              # slot 9 of 9
    assert L.moe_prefetch_slots(p, p + 256, 256, 9, slots, 2, None, None, p, 1,
                                None) == L.MOE_ERR_INVALID_ARG              # overlapping pools
    assert L.moe_prefetch_slots(p, 1 << 24, 256, 9, slots, -1, None, None, p, 1,
                                None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_experts_touched(p, 10, 0, p, None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_experts_touched(None, 10, 8, p, None) == L.MOE_ERR_INVALID_ARG
