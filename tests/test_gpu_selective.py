"""Selective prefetch on the GPU: moe_experts_touched, moe_prefetch_slots and
the selective PrefetchPipeline schedule (look-ahead prediction, missed slots
fetched before the grouped GEMM, per-slot readiness flags).
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

from moe_inputs import device as mdev
from oracle import workload as ow
from split_weight_b200 import PrefetchPipeline, _lib as L
from split_weight_b200.layer import remote_slots

from gpu_util import (MID_FP8, MID_SIGMOID, RTOL_BF16, RTOL_FP8, assert_close_rel, sync_check,
                      to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


def test_experts_touched_marks_exactly_the_selected_experts(cuda_device):
    rng = np.random.default_rng(5)
    E, A = 300, 5000
    idx = rng.integers(0, E, A, dtype=np.int32)
    idx[rng.integers(0, A, 40)] = rng.integers(0, 20, 40)     # some experts more often
    d_idx = torch.from_numpy(idx).cuda()
    touched = torch.full((E,), 7, dtype=torch.uint8, device="cuda")
    h = torch.cuda.current_stream().cuda_stream
    L.check(L.moe_experts_touched(d_idx.data_ptr(), A, E, touched.data_ptr(), h))
    sync_check()
    want = np.zeros(E, dtype=np.uint8)
    want[idx] = 1
    assert np.array_equal(touched.cpu().numpy(), want)
    # an entry outside [0, E) is reported and skipped
    bad = idx.copy()
    bad[17] = E + 3
    L.check(L.moe_experts_touched(torch.from_numpy(bad).cuda().data_ptr(), A, E,
                                  touched.data_ptr(), h))
    torch.cuda.synchronize()
    assert L.moe_check_device() == L.MOE_ERR_DEVICE_CHECK
    want2 = np.zeros(E, dtype=np.uint8)
    want2[np.delete(bad, 17)] = 1
    assert np.array_equal(touched.cpu().numpy(), want2)
    # empty routing: all zero
    L.check(L.moe_experts_touched(d_idx.data_ptr(), 0, E, touched.data_ptr(), h))
    sync_check()
    assert not touched.cpu().numpy().any()


def test_prefetch_slots_copies_only_the_listed_slots(cuda_device):
    n_slots, sb = 9, 4096 + 256
    src = torch.randint(0, 256, (n_slots * sb,), dtype=torch.uint8, device="cuda")
    dst = torch.zeros_like(src)
    flags = torch.zeros(n_slots, dtype=torch.int32, device="cuda")
    copy = torch.cuda.Stream()
    copy.wait_stream(torch.cuda.current_stream())
    slots = [6, 2, 3, 4, 8]                       # one run of three, two single slots
    arr = (ctypes.c_int32 * len(slots))(*slots)
    L.check(L.moe_prefetch_slots(src.data_ptr(), dst.data_ptr(), sb, n_slots, arr, len(slots),
                                 copy.cuda_stream, None, flags.data_ptr(), 5, None))
    copy.synchronize()
    s2, d2 = src.view(n_slots, sb), dst.view(n_slots, sb)
    f = flags.cpu().numpy()
    for s in range(n_slots):
        if s in slots:
            assert torch.equal(d2[s], s2[s]) and f[s] == 5, s
        else:
            assert not d2[s].any() and f[s] == 0, s
    # a slot outside the pool is refused before anything is enqueued
    arr2 = (ctypes.c_int32 * 2)(1, n_slots)
    assert L.moe_prefetch_slots(src.data_ptr(), dst.data_ptr(), sb, n_slots, arr2, 2,
                                copy.cuda_stream, None, flags.data_ptr(), 6, None) \
        == L.MOE_ERR_INVALID_ARG
    copy.synchronize()
    assert (flags.cpu().numpy() != 6).all()


@pytest.mark.parametrize("cfg,act", [(MID_SIGMOID, "bf16"), (MID_FP8, "bf16")],
                         ids=["bf16", "e4m3_weights"])
def test_selective_pipeline_equals_resident_layers_and_oracle(cfg, act):
    cfg = cfg.with_(cfg_id=cfg.cfg_id + 150, layers=3)
    dls = [mdev.build_layer(cfg, layer=l, act_dtype=act) for l in range(cfg.layers)]
    ref = []
    for d in dls:
        d.layer.forward(d.x)
        ref.append(d.layer.y.clone())
    sync_check()
    oracle_y = [ow.layer_full(cfg, l, d.pool, d.slot, d.inputs)[0] for l, d in enumerate(dls)]
    stores = [mdev.peer_store(cfg, l, dls[l].layer.weights) for l in range(cfg.layers)]
    w0 = dls[0].layer.weights
    pipe = PrefetchPipeline([d.layer for d in dls], stores, w0.n_remote * w0.stride,
                            split=False, gate_slots=1, select=True)
    for d in dls:
        d.layer.weights.remote.zero_()   # the pipeline must not read them
    pipe.prime()
    for rep in range(2):
        outs = pipe.run([d.x for d in dls])
        sync_check()
        for l in range(cfg.layers):
            assert torch.equal(outs[l], ref[l]), f"pass {rep} layer {l}"
            assert_close_rel(to_np(outs[l][:cfg.T]), oracle_y[l],
                             RTOL_FP8 if cfg.w_dtype == "e4m3" else RTOL_BF16,
                             f"pass {rep} layer {l} against the oracle")
    st = pipe.select_stats
    assert len(st) == 2 * cfg.layers
    assert st[0]["missed"] == st[0]["touched"]   # nothing predicted before the first execution
    for i, s in enumerate(st):
        lay = dls[i % cfg.layers].layer
        want = remote_slots(lay.weights.pool_slot,
                            np.bincount(lay.topk_idx.cpu().numpy().ravel(), minlength=cfg.E))
        assert s["touched"] == len(want) and 0 <= s["missed"] <= s["touched"]
