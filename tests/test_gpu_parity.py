"""GPU parity: every C-ABI call against the CPU oracle on the same seeded inputs.

Routing indices, counts, offsets and the permutation must be bit-exact; the
sigmoid routing weights too (their arithmetic is defined in fp32).  Layer
outputs must satisfy max|err| <= 2e-2 * max|ref| (bf16 path).
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import config, device as mdev, gen
from oracle import workload as ow
from split_weight_b200 import _lib as L

from gpu_util import (DECODE_FP8, MAX_EXPERTS, MID_BN128, MID_BN128_FP8, MID_BN256, MID_BN256_FP8,
                      MID_BN256_FP8_K2, tile_width,
                      MID_BN256_H384, MID_FP8, MID_FP8_H384, MID_SIGMOID, MID_SOFTMAX, ONE_TOKEN,
                      RTOL_BF16, RTOL_FP8,
                      SPARSE_DECODE, assert_close_rel, run_layer, sync_check, to_np)

pytestmark = pytest.mark.gpu

SMALL = [config(1), MID_SIGMOID, MID_SOFTMAX, SPARSE_DECODE, ONE_TOKEN]


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _check_routing(dl, idx_ref, w_ref):
    ml = dl.layer
    T = dl.cfg.T
    idx = ml.topk_idx[:T].cpu().numpy()
    np.testing.assert_array_equal(idx, idx_ref, err_msg="topk_idx differs from the oracle")
    w = ml.topk_w[:T].cpu().numpy()
    if dl.cfg.score == "sigmoid":
        np.testing.assert_array_equal(w, w_ref.astype(np.float32), err_msg="topk_w not bit-exact")
    else:
        np.testing.assert_allclose(w, w_ref, rtol=2e-6, atol=1e-7)


def _check_permutation(dl, idx_ref):
    ml, c = dl.layer, dl.cfg
    off, src, inv = oracle.permute(idx_ref, c.E)
    np.testing.assert_array_equal(ml.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(ml.perm_src[:c.A].cpu().numpy(), src)
    np.testing.assert_array_equal(ml.inv_pos[:c.T].cpu().numpy(), inv)
    if ml.shape.act_dtype != "bf16":
        return   # e4m3 rows: see test_e4m3_gather_quantises_each_128_block
    if ml.gather:
        return   # no x_perm: the grouped GEMM gathers from x (test_gathered_path_full_parity)
    # gathered rows: x (rounded to bf16 when it came as fp32), then the shared rows
    xp = ml.x_perm[:c.rows].view(torch.int16).cpu().numpy().view(np.uint16)
    xb = gen.f32_to_bf16_bits(dl.inputs.x)
    np.testing.assert_array_equal(xp[:c.A], xb[src])
    if c.has_shared:
        np.testing.assert_array_equal(xp[c.A:], xb)


def _rtol(cfg):
    return RTOL_FP8 if cfg.w_dtype == "e4m3" else RTOL_BF16


@pytest.mark.parametrize("cfg", SMALL + [MID_FP8, DECODE_FP8, MAX_EXPERTS], ids=lambda c: c.name)
def test_small_layer_full_parity(cfg):
    """Whole layers, every output element against the oracle.  The e4m3-weight
    workloads run their stated path: bf16 activations, the weights
    dequantised to bf16 in shared memory, the bf16 tensor-core MMA."""
    dl = mdev.build_layer(cfg)
    run_layer(dl)
    y_ref, idx_ref, w_ref, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    _check_routing(dl, idx_ref, w_ref)
    _check_permutation(dl, idx_ref)
    assert_close_rel(to_np(dl.layer.y[:cfg.T]), y_ref, _rtol(cfg), f"{cfg.name} y")


@pytest.mark.parametrize("cfg,bn", [(MID_BN256, 256), (MID_BN256_H384, 256), (MID_BN256_FP8, 256),
                                    (MID_BN256_FP8_K2, 256), (MID_BN128, 128), (MID_BN128_FP8, 128),
                                    (MID_FP8_H384, 128)],
                         ids=lambda c: getattr(c, "name", str(c)))
def test_mid_layer_each_tile_width_full_parity(cfg, bn):
    """Whole mid-size layers whose experts get enough tokens each for the
    grouped GEMMs to run 256-token tiles (one 512-column TMEM accumulator
    set, the wide epilogue; with e4m3 weights the converted-operand ring
    beside three TMA stages) or 128-token tiles with ragged row counts, in
    the two-tile (gate/up, paired down) and single-tile (H = 384) down modes;
    every output element against the oracle."""
    dl = mdev.build_layer(cfg)
    run_layer(dl)
    y_ref, idx_ref, w_ref, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    _check_routing(dl, idx_ref, w_ref)
    _check_permutation(dl, idx_ref)
    counts = np.diff(dl.layer.offsets.cpu().numpy())
    assert tile_width(cfg) == bn, "tile width not reached"
    assert (counts % 16 != 0).any(), "no ragged token tile"
    assert_close_rel(to_np(dl.layer.y[:cfg.T]), y_ref, _rtol(cfg), f"{cfg.name} y")


@pytest.mark.parametrize("cfg", [MID_SIGMOID, MID_BN256, MID_BN128_FP8, MID_BN256_FP8_K2,
                                 SPARSE_DECODE],
                         ids=lambda c: c.name)
def test_gathered_path_full_parity(cfg):
    """The grouped GEMM gathering its token rows itself from x through
    perm_src (moe_grouped_ffn_x, TMA tile::gather4) instead of reading the
    x_perm that moe_permute gathers: every output element against the
    oracle, and bit-identical to the x_perm path."""
    dl = mdev.build_layer(cfg, gather=True)
    assert dl.layer.gather
    run_layer(dl)
    y_ref, idx_ref, w_ref, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    _check_routing(dl, idx_ref, w_ref)
    _check_permutation(dl, idx_ref)
    assert_close_rel(to_np(dl.layer.y[:cfg.T]), y_ref, _rtol(cfg), f"{cfg.name} y (gathered)")
    y_gathered = dl.layer.y.clone()
    x = mdev.build_layer(cfg)
    assert not x.layer.gather
    run_layer(x)
    assert torch.equal(x.layer.y, y_gathered)


@pytest.mark.parametrize("cfg", [MID_FP8, DECODE_FP8, MID_BN128_FP8], ids=lambda c: c.name)
def test_fp8_tensor_core_path_e4m3_activations(cfg):
    """The opt-in fp8 tensor-core path: x_perm and h quantised to e4m3 per
    (row, 128 columns), both GEMMs kind::f8f6f4 with per-block promotion."""
    dl = mdev.build_layer(cfg, act_dtype="e4m3")
    run_layer(dl)
    y_ref, idx_ref, w_ref, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    _check_routing(dl, idx_ref, w_ref)
    _check_permutation(dl, idx_ref)
    assert_close_rel(to_np(dl.layer.y[:cfg.T]), y_ref, RTOL_FP8, f"{cfg.name} y (e4m3 act)")


def test_generator_gpu_matches_host(cuda_device):
    for cfg in (config(2), config(5).with_(H=512, I=256)):
        lay = L.expert_layout(cfg.H, cfg.I, L.MOE_E4M3 if cfg.w_dtype == "e4m3" else L.MOE_BF16)
        buf = torch.empty(lay.bytes, dtype=torch.uint8, device=cuda_device)
        from moe_inputs import gpu_gen
        base = buf.data_ptr()
        gsc = base + lay.gu_scale_offset if lay.gu_scale_offset >= 0 else None
        dsc = base + lay.down_scale_offset if lay.down_scale_offset >= 0 else None
        gpu_gen.fill_expert(cfg, 0, 7, base + lay.gu_offset, base + lay.down_offset, gsc, dsc,
                            torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        host = gen.expert_host(cfg, 0, 7)
        raw = buf.cpu().numpy()
        esz = 2 if cfg.w_dtype == "bf16" else 1
        gu = raw[lay.gu_offset: lay.gu_offset + host.gu.size * esz].view(host.gu.dtype)
        np.testing.assert_array_equal(gu.reshape(host.gu.shape), host.gu)
        dn = raw[lay.down_offset: lay.down_offset + host.down.size * esz].view(host.down.dtype)
        np.testing.assert_array_equal(dn.reshape(host.down.shape), host.down)
        if host.gu_scale is not None:
            s = raw[lay.gu_scale_offset: lay.gu_scale_offset + host.gu_scale.size * 4].view(np.float32)
            np.testing.assert_array_equal(s.reshape(host.gu_scale.shape), host.gu_scale)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_pool_invariance_bit_identical(seed):
    cfg = MID_SIGMOID
    ref_dl = mdev.build_layer(cfg)
    y_ref = run_layer(ref_dl).y.clone()
    del ref_dl
    for n_local in (None, 0, cfg.E):
        pl = mdev.random_placement(cfg, seed, n_local)
        dl = mdev.build_layer(cfg, placement=pl)
        y = run_layer(dl).y
        assert torch.equal(y, y_ref), f"placement {pl} changed the output"


@pytest.mark.parametrize("cfg,act", [(MID_SIGMOID, "bf16"), (MID_BN256, "bf16"),
                                     (MID_BN128_FP8, "bf16"), (MID_BN256_FP8_K2, "bf16")],
                         ids=["bf16", "bf16_bn256", "e4m3_weights", "e4m3_weights_bn256"])
def test_dynamic_and_static_tile_schedules_bit_identical(cfg, act):
    """With a workspace the grouped GEMM's CTAs take tiles from a counter
    (dynamic schedule); without one, a fixed round-robin share.  Every output
    element is computed by one tile in a fixed order, so the bits agree."""
    dl = mdev.build_layer(cfg, act_dtype=act)
    y_dyn = run_layer(dl).y.clone()
    ml, h = dl.layer, torch.cuda.current_stream().cuda_stream
    assert ml.ffn_ws.numel() >= L.moe_grouped_ffn_workspace_size(ctypes.byref(ml._desc)) >= 256
    tbl = ml.weights.table()
    L.check(L.moe_grouped_ffn(ctypes.byref(ml._desc), ctypes.byref(tbl), ml.x_perm.data_ptr(),
                              None, ml.offsets.data_ptr(), ml.h.data_ptr(), ml.y_perm.data_ptr(),
                              None, 0, h))
    ml.combine(h)
    sync_check()
    assert torch.equal(ml.y, y_dyn)


def test_all_tokens_one_expert_is_dense_ffn():
    # a large bias on one expert and k = 1: every token goes to expert 5, the
    # grouped GEMM sees one dense group spanning several token tiles
    cfg = MID_SIGMOID.with_(cfg_id=15, k=1, topk_group=1, has_shared=False)
    dl = mdev.build_layer(cfg)
    b = dl.layer.bias.clone()
    b[5] = 10.0
    dl.layer.bias.copy_(b)
    dl.inputs.bias = b.cpu().numpy()
    run_layer(dl)
    assert (dl.layer.topk_idx[:cfg.T] == 5).all()
    y_ref, idx_ref, w_ref, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    assert (idx_ref == 5).all()
    _check_routing(dl, idx_ref, w_ref)
    assert_close_rel(to_np(dl.layer.y[:cfg.T]), y_ref, RTOL_BF16, "dense y")


def test_empty_batch_is_a_no_op(cuda_device):
    cfg = MID_SIGMOID.with_(cfg_id=16, T=0)
    dl = mdev.build_layer(cfg)
    dl.layer.forward(dl.x)
    sync_check()
    assert dl.layer.offsets.cpu().numpy().tolist() == [0] * (cfg.E + 1)


def test_kernel_launch_counter(cuda_device):
    """moe_kernel_launches counts each accepted kernel launch: one layer of
    300 tokens is the split router (chunk logits, partial sums, selection),
    permute (histogram, scan, scatter, gather), the two grouped GEMM kernels
    and the combine; without the gather kernel when the grouped GEMM gathers
    its rows itself; a 0-token layer launches nothing."""
    dl = mdev.build_layer(MID_SIGMOID)
    sync_check()
    n0 = L.moe_kernel_launches()
    dl.layer.forward(dl.x)
    assert L.moe_kernel_launches() - n0 == 3 + 4 + 2 + 1
    dg = mdev.build_layer(MID_SIGMOID, gather=True)
    sync_check()
    n0 = L.moe_kernel_launches()
    dg.layer.forward(dg.x)
    assert L.moe_kernel_launches() - n0 == 3 + 3 + 2 + 1
    empty = mdev.build_layer(MID_SIGMOID.with_(cfg_id=16, T=0))
    n0 = L.moe_kernel_launches()
    empty.layer.forward(empty.x)
    assert L.moe_kernel_launches() == n0
    sync_check()


def test_out_of_range_expert_index_is_reported(cuda_device):
    """An expert index outside [0, E) is skipped and reported.  The rows it
    leaves unwritten in perm_src hold a value that is not a token (filled
    here before the call): the gather must check it before reading x, zero
    the row and report it; the combine must see inv_pos = -1 and skip it."""
    cfg = SPARSE_DECODE
    dl = mdev.build_layer(cfg)
    ml = dl.layer
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    torch.cuda.synchronize()
    ml.topk_idx[0, 0] = cfg.E + 3   # made on the host side: the kernel checks and skips it
    ml.perm_src.fill_(2**31 - 1)
    ml.x_perm.fill_(1.0)
    ml.permute(dl.x, h)
    torch.cuda.synchronize()
    assert L.moe_check_device() == L.MOE_ERR_DEVICE_CHECK
    assert L.moe_check_device() == L.MOE_OK   # the word was cleared
    off = ml.offsets.cpu().numpy()
    assert off[cfg.E] == cfg.A - 1
    assert int(ml.inv_pos[0, 0]) == -1
    assert int(ml.perm_src[cfg.A - 1]) == 2**31 - 1          # never written
    assert not ml.x_perm[cfg.A - 1].any()                      # zero-filled, not read from x
    ml.grouped_ffn(h, x=dl.x)
    ml.combine(h)
    torch.cuda.synchronize()
    assert L.moe_check_device() == L.MOE_ERR_DEVICE_CHECK     # the combine saw inv_pos = -1
    assert torch.isfinite(ml.y[:cfg.T].float()).all()


def test_gathered_token_rows_check_perm_src(cuda_device):
    """The grouped GEMM that gathers its token rows from x through perm_src
    checks every value against [0, T) before the load: a corrupt entry is
    reported (MOE_ERR_DEVICE_CHECK) and token 0 read in its place."""
    cfg = SPARSE_DECODE
    dl = mdev.build_layer(cfg, gather=True)
    ml = dl.layer
    assert ml.gather
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    ml.permute(dl.x, h)
    torch.cuda.synchronize()
    ml.perm_src[0] = 2**31 - 1
    ml.grouped_ffn(h, x=dl.x)
    ml.combine(h)
    torch.cuda.synchronize()
    assert L.moe_check_device() == L.MOE_ERR_DEVICE_CHECK
    assert L.moe_check_device() == L.MOE_OK
    assert torch.isfinite(ml.y[:cfg.T].float()).all()


# ----------------------------------------------------------------- full size
def _full_size_check(cfg, layer: int, n_sample: int = 12):
    dl = mdev.build_layer(cfg, layer=layer)
    run_layer(dl)
    idx_ref, w_ref, _ = ow.route(cfg, layer, dl.inputs)
    _check_routing(dl, idx_ref, w_ref)
    _check_permutation(dl, idx_ref)
    rng = np.random.default_rng(100 + layer)
    toks = np.sort(rng.choice(cfg.T, size=min(n_sample, cfg.T), replace=False))
    y_ref = ow.layer_tokens(cfg, layer, toks, idx_ref, w_ref, dl.pool, dl.slot, dl.inputs)
    y = to_np(dl.layer.y[torch.from_numpy(toks).cuda()])
    return assert_close_rel(y, y_ref, _rtol(cfg), f"{cfg.name} layer {layer} sampled y")


def test_r1_decode_full_size():
    _full_size_check(config(2), 0, n_sample=16)


def test_r1_prefill_8k_full_size():
    _full_size_check(config(3), 0, n_sample=8)


@pytest.mark.parametrize("layer", [0, 1])
def test_r1_prefill_imbalanced_full_size(layer):
    _full_size_check(config(4), layer, n_sample=6)


@pytest.mark.parametrize("layer", [0, 3])
def test_r1_fp8_pipeline_full_size(layer):
    _full_size_check(config(5), layer, n_sample=6)


def test_e4m3_gather_quantises_each_128_block(cuda_device):
    """moe_permute with an e4m3 destination: the permutation is exact and each
    row's 128-column blocks decode to within e4m3 rounding of x."""
    cfg = MID_SIGMOID
    li = gen.layer_inputs(cfg)
    idx_ref, _, _ = ow.route(cfg, 0, li)
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    rows = T * k + T
    dev = cuda_device
    idx = torch.from_numpy(idx_ref).to(dev)
    x = mdev.x_tensor(li, dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T, k, dtype=torch.int32, device=dev)
    xq = torch.empty(rows, H, dtype=torch.uint8, device=dev)
    sc = torch.empty(H // 128, rows, dtype=torch.float32, device=dev)   # [H/128, rows]
    ws = torch.empty(L.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=dev)
    L.check(L.moe_permute(T, k, E, H, idx.data_ptr(), x.data_ptr(), L.MOE_BF16, L.MOE_E4M3, 1,
                          off.data_ptr(), src.data_ptr(), inv.data_ptr(), xq.data_ptr(),
                          sc.data_ptr(), ws.data_ptr(), ws.numel(),
                          torch.cuda.current_stream().cuda_stream))
    sync_check()
    o_ref, s_ref, _ = oracle.permute(idx_ref, E)
    np.testing.assert_array_equal(src.cpu().numpy(), s_ref)
    xs = np.concatenate([li.x[s_ref], li.x]).astype(np.float64)
    scr = sc.cpu().numpy().T                                  # [rows, H/128]
    dec = gen.e4m3_bits_to_f64(xq.cpu().numpy()) * np.repeat(scr, 128, axis=1)
    blk = np.abs(xs).reshape(rows, H // 128, 128).max(axis=2)
    np.testing.assert_allclose(scr, blk / 448, rtol=1e-6)
    # e4m3 has 3 mantissa bits: |err| <= 2^-4 |v| for normal codes, plus the
    # subnormal step 2^-10 * s
    bound = np.abs(xs) * 2.0 ** -4 + np.repeat(scr, 128, axis=1) * 2.0 ** -10
    assert (np.abs(dec - xs) <= bound * (1 + 1e-6)).all()


# ----------------------------------------------------------------- routing only
BIG_ROUTE_BF16 = config(2).with_(cfg_id=18, name="route_T7700_H512_E256", T=7700, H=512, I=128)
BIG_ROUTE_F32 = config(1).with_(cfg_id=19, name="route_f32_T20000_H256_E8", T=20000)
MED_ROUTE = config(2).with_(cfg_id=22, name="route_T3001_H512_E256", T=3001, H=512, I=128)
SPLIT_ROUTE = config(2).with_(cfg_id=20, name="route_T40_H7168_E256", T=40, I=128)
# large batch with a last chunk of 128 h (H = 384): the chunk-split large tile
BIG_ROUTE_H384 = config(2).with_(cfg_id=35, name="route_T7700_H384_E256", T=7700, H=384, I=128)


@pytest.mark.parametrize("cfg", [BIG_ROUTE_BF16, BIG_ROUTE_F32, BIG_ROUTE_H384, MED_ROUTE,
                                 SPLIT_ROUTE],
                         ids=lambda c: c.name)
def test_routing_bit_exact_all_router_kernels(cfg, cuda_device):
    """The logits kernels (chunk-split small tiles for small batches, 64x64
    tiles for medium ones, chunk-split 64x128 tiles for large ones, ragged
    token counts and a short last chunk) give the oracle's bits; so do the
    selection and the permutation that follow."""
    from moe_inputs.gen import layer_inputs
    from split_weight_b200 import MoELayer, SplitWeights
    li = layer_inputs(cfg)
    shape = mdev.layer_shape(cfg)
    w = SplitWeights.allocate(cfg.H, cfg.I, cfg.w_dtype, *mdev.default_placement(cfg),
                              cfg.has_shared, cuda_device)
    bias = torch.from_numpy(li.bias).to(cuda_device) if li.bias is not None else None
    ml = MoELayer(shape, torch.from_numpy(li.wg).to(cuda_device), bias, w, cuda_device)
    x = mdev.x_tensor(li, cuda_device)
    h = torch.cuda.current_stream().cuda_stream
    ml.route(x, h)
    ml.permute(x, h)
    sync_check()
    idx_ref, w_ref, _ = ow.route(cfg, 0, li)
    np.testing.assert_array_equal(ml.topk_idx[:cfg.T].cpu().numpy(), idx_ref)
    got_w = ml.topk_w[:cfg.T].cpu().numpy()
    if cfg.score == "sigmoid":
        np.testing.assert_array_equal(got_w, w_ref.astype(np.float32))
    else:
        np.testing.assert_allclose(got_w, w_ref, rtol=2e-6, atol=1e-7)
    off, src, inv = oracle.permute(idx_ref, cfg.E)
    np.testing.assert_array_equal(ml.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(ml.perm_src[:cfg.A].cpu().numpy(), src)
    np.testing.assert_array_equal(ml.inv_pos[:cfg.T].cpu().numpy(), inv)
