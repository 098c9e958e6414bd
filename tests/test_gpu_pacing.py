"""A fetch paced by the grouped GEMM's progress (GPU).

moe_grouped_ffn_paced raises a progress word as its tiles' MMAs are issued
and writes base + steps + 1 when the call has ended; moe_prefetch_layer_paced
holds each chunk of a fetch on the copy stream until the word reaches the
chunk's threshold.  The paced call must give the ungated call's bits, the
copy must not run ahead of the reports, and a pipeline paced this way must
equal resident layers and the oracle.
"""
import ctypes
import gc
import time

import numpy as np
import pytest
import torch

from moe_inputs import device as mdev
from oracle import workload as ow
from split_weight_b200 import PrefetchPipeline, Progress, _lib as L

from gpu_util import (MID_BN256, MID_FP8, MID_SIGMOID, RTOL_BF16, RTOL_FP8, assert_close_rel,
                      run_layer, sync_check, to_np)

pytestmark = pytest.mark.gpu

CASES = [(MID_SIGMOID, "bf16", False), (MID_BN256, "bf16", True), (MID_FP8, "bf16", False),
         (MID_FP8, "e4m3", False)]
IDS = ["bf16", "bf16_gathered_bn256", "e4m3_weights", "fp8_tensor_cores"]


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _rtol(cfg):
    return RTOL_FP8 if cfg.w_dtype == "e4m3" else RTOL_BF16


def _u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("cfg,act,gather", CASES, ids=IDS)
def test_paced_call_equals_plain_call_and_reports_every_step(cfg, act, gather):
    dl = mdev.build_layer(cfg, act_dtype=act, gather=gather)
    y_ref = run_layer(dl).y.clone()
    ml = dl.layer
    words = torch.zeros(3, dtype=torch.int32, device="cuda")
    base, steps = 0xFFFFFFF0, 7            # the word wraps around during the call
    words[0] = int(np.array([base], dtype=np.uint32).view(np.int32)[0])
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    ml.permute(dl.x, h)
    ml.grouped_ffn(h, None, None, x=dl.x, progress=Progress(words, base, steps))
    ml.combine(h)
    sync_check()
    assert torch.equal(ml.y, y_ref)
    w = _u32(words)
    assert w[0] == (base + steps + 1) & 0xFFFFFFFF
    assert w[1] > 0 and w[2] > 0          # both launches counted their tiles


def test_paced_fetch_waits_for_the_reports(cuda_device):
    """The compute stream sleeps before the paced call: only the lead chunks
    may land meanwhile; once the call runs, every chunk lands and the flags
    reach the epoch."""
    n_chunks, chunk, lead, steps = 6, 1 << 20, 2, 4
    src = torch.randint(0, 256, (n_chunks * chunk,), dtype=torch.uint8, device="cuda")
    dst = torch.zeros_like(src)
    flags = torch.zeros(n_chunks, dtype=torch.int32, device="cuda")
    words = torch.zeros(3, dtype=torch.int32, device="cuda")
    base = 100
    words[0] = base
    dl = mdev.build_layer(MID_SIGMOID)
    ml = dl.layer
    compute, copy, probe = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    pr = Progress(words, base, steps)
    # the pacing call first (behind a sleep), then the paced copy: the copy
    # stream never waits for work enqueued after it, even on a shared queue
    with torch.cuda.stream(compute):
        torch.cuda._sleep(400_000_000)     # well over 100 ms before the call's first report
        ml.route(dl.x, compute.cuda_stream)
        ml.permute(dl.x, compute.cuda_stream)
    ml.grouped_ffn(compute.cuda_stream, None, None, x=dl.x, progress=pr)
    L.check(L.moe_prefetch_layer_paced(src.data_ptr(), dst.data_ptr(), src.numel(), chunk,
                                       copy.cuda_stream, None, flags.data_ptr(), 9,
                                       ctypes.byref(pr.c_struct()), lead, None))
    time.sleep(0.05)
    seen = torch.empty(n_chunks, dtype=torch.int32, pin_memory=True)
    with torch.cuda.stream(probe):
        seen.copy_(flags, non_blocking=True)
    probe.synchronize()
    early = seen.numpy().copy()
    torch.cuda.synchronize()
    # the lead chunks may already have landed; no other chunk before the reports
    assert set(early[:lead]) <= {0, 9}, early
    assert (early[lead:] == 0).all(), early
    assert (flags.cpu().numpy() == 9).all()
    assert torch.equal(dst, src)
    assert _u32(words)[0] == base + steps + 1
    for c in range(n_chunks):
        t = L.moe_pace_threshold(c, n_chunks, lead, base, steps)
        assert (t == base) == (c < lead) and base <= t <= base + steps


@pytest.mark.parametrize("cfg,act", [(MID_SIGMOID, "bf16"), (MID_FP8, "bf16")],
                         ids=["bf16", "e4m3_weights"])
def test_paced_pipeline_equals_resident_layers_and_oracle(cfg, act):
    cfg = cfg.with_(cfg_id=cfg.cfg_id + 200, layers=3)
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
                            split=False, gate_slots=3, pace_steps=5, pace_lead=1)
    for d in dls:
        d.layer.weights.remote.zero_()   # the pipeline must not read them
    pipe.prime()
    for rep in range(2):
        outs = pipe.run([d.x for d in dls])
        sync_check()
        for l in range(cfg.layers):
            assert torch.equal(outs[l], ref[l]), f"pass {rep} layer {l}"
            assert_close_rel(to_np(outs[l][:cfg.T]), oracle_y[l], _rtol(cfg),
                             f"pass {rep} layer {l} against the oracle")
    # every execution's call ended: the word sits at the next execution's base
    assert _u32(pipe.progress_words)[0] == pipe.progress(pipe.g).base


def test_paced_call_ends_the_word_when_it_has_no_work_or_fails(cuda_device):
    """The call's final write of the progress word comes whatever the call did:
    with no tokens, and after an argument error (here H not a multiple of
    128), so that a fetch paced by it is never left waiting."""
    dl = mdev.build_layer(MID_SIGMOID)
    ml = dl.layer
    words = torch.zeros(3, dtype=torch.int32, device="cuda")
    h = torch.cuda.current_stream().cuda_stream
    tbl = ml.weights.table()
    empty = L.moe_ffn_desc(0, ml._desc.H, ml._desc.I, ml._desc.E, ml._desc.k, ml._desc.w_dtype,
                           ml._desc.act_dtype, ml._desc.has_shared)
    pr = Progress(words, 40, 6).c_struct()
    assert L.moe_grouped_ffn_paced(ctypes.byref(empty), ctypes.byref(tbl), None, ctypes.byref(pr),
                                   None, None, None, None, ml.offsets.data_ptr(), None, None,
                                   None, 0, h) == L.MOE_OK
    sync_check()
    assert _u32(words)[0] == 40 + 6 + 1
    bad = L.moe_ffn_desc(ml._desc.T, 100, ml._desc.I, ml._desc.E, ml._desc.k, ml._desc.w_dtype,
                         ml._desc.act_dtype, ml._desc.has_shared)
    pr = Progress(words, 80, 6).c_struct()
    assert L.moe_grouped_ffn_paced(ctypes.byref(bad), ctypes.byref(tbl), None, ctypes.byref(pr),
                                   ml.x_perm.data_ptr(), None, None, None, ml.offsets.data_ptr(),
                                   ml.h.data_ptr(), ml.y_perm.data_ptr(), None, 0,
                                   h) == L.MOE_ERR_INVALID_ARG
    sync_check()
    assert _u32(words)[0] == 80 + 6 + 1
