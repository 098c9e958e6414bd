"""Per-expert readiness of a fetch in flight (GPU).

The grouped GEMM may start before the fetch of the remote experts has
finished: moe_prefetch_layer_flagged writes one flag per chunk after the
chunk lands, and moe_grouped_ffn_gated waits on the device, before the first
load of a remote expert, for the flag of its chunk.  The results must equal
the ungated call's bit for bit and the oracle within tolerance; a flag that
nothing writes must make the wait run out, report MOE_ERR_TIMEOUT and leave
the library usable.
"""
import gc
import time

import pytest
import torch

from moe_inputs import device as mdev
from oracle import workload as ow
from split_weight_b200 import PrefetchPipeline, ReadyGate, _lib as L

from gpu_util import (MID_FP8, MID_SIGMOID, RTOL_BF16, RTOL_FP8, assert_close_rel, run_layer,
                      sync_check, to_np)

pytestmark = pytest.mark.gpu

CASES = [(MID_SIGMOID, "bf16"), (MID_FP8, "bf16"), (MID_FP8, "e4m3")]
IDS = ["bf16", "e4m3_weights", "fp8_tensor_cores"]


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _rtol(cfg):
    return RTOL_FP8 if cfg.w_dtype == "e4m3" else RTOL_BF16


@pytest.mark.parametrize("cfg,act", CASES, ids=IDS)
def test_gate_with_flags_landed_equals_ungated(cfg, act):
    dl = mdev.build_layer(cfg, act_dtype=act)
    y_ref = run_layer(dl).y.clone()
    ml = dl.layer
    flags = torch.full((5,), 7, dtype=torch.int32, device="cuda")
    gate = ReadyGate(flags, 7, slots_per_flag=(cfg.E - cfg.local_count + 4) // 5)
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    ml.permute(dl.x, h)
    ml.grouped_ffn(h, None, gate, x=dl.x)
    ml.combine(h)
    sync_check()
    assert torch.equal(ml.y, y_ref)


@pytest.mark.parametrize("cfg,act", CASES, ids=IDS)
def test_gated_launch_without_room_for_the_copy_is_refused(cfg, act):
    """A gated call's CTAs wait for a fetch that, between buffers of one GPU,
    runs as a copy kernel on the same SMs.  With the register limit lowered
    through the test hook the gated call is refused before its kernel is
    launched, an ungated call still runs, and with the limit restored the
    gated call gives the ungated bits."""
    dl = mdev.build_layer(cfg, act_dtype=act)
    y_ref = run_layer(dl).y.clone()
    ml = dl.layer
    flags = torch.full((5,), 7, dtype=torch.int32, device="cuda")
    gate = ReadyGate(flags, 7, slots_per_flag=(cfg.E - cfg.local_count + 4) // 5)
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    ml.permute(dl.x, h)
    launches = L.moe_kernel_launches()
    L.moe_debug_gated_regs_per_sm(4096)
    try:
        with pytest.raises(L.MoEError) as err:
            ml.grouped_ffn(h, None, gate, x=dl.x)
        assert err.value.status == L.MOE_ERR_CUDA and "no room" in str(err.value)
        assert L.moe_kernel_launches() == launches
        ml.grouped_ffn(h, None, None, x=dl.x)     # no gate: no limit
    finally:
        L.moe_debug_gated_regs_per_sm(0)
    ml.grouped_ffn(h, None, gate, x=dl.x)
    ml.combine(h)
    sync_check()
    assert torch.equal(ml.y, y_ref)


@pytest.mark.parametrize("cfg,act", CASES, ids=IDS)
@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
def test_flag_gated_pipeline_equals_resident_layers_and_oracle(cfg, act, split):
    """Three layers through the alternate buffers with the compute stream
    never waiting for a fetch: the grouped GEMMs wait per chunk on the device.
    The copies are delayed so that the waits really happen."""
    cfg = cfg.with_(cfg_id=cfg.cfg_id + 100, layers=3)
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
                            split=split, gate_slots=3)
    for d in dls:
        d.layer.weights.remote.zero_()   # the pipeline must not read them
    with torch.cuda.stream(pipe.copy_stream):
        torch.cuda._sleep(200_000_000)   # the first chunks land well after the GEMMs start
    pipe.prime()
    for rep in range(2):
        outs = pipe.run([d.x for d in dls])
        sync_check()
        for l in range(cfg.layers):
            assert torch.equal(outs[l], ref[l]), f"pass {rep} layer {l}"
            assert_close_rel(to_np(outs[l][:cfg.T]), oracle_y[l], _rtol(cfg),
                             f"pass {rep} layer {l} against the oracle")


@pytest.mark.parametrize("cfg,act", CASES, ids=IDS)
def test_flag_never_written_times_out_and_library_stays_usable(cfg, act):
    """No copy ever writes the flags: every wait for a remote expert gives up
    after the gate's 50 ms, the call's kernels stop, moe_check_device reports
    MOE_ERR_TIMEOUT (and clears it), and the next ordinary call is right."""
    dl = mdev.build_layer(cfg, act_dtype=act)
    ml = dl.layer
    flags = torch.zeros(4, dtype=torch.int32, device="cuda")
    gate = ReadyGate(flags, 1, slots_per_flag=(cfg.E - cfg.local_count + 3) // 4,
                     timeout_ns=50_000_000)
    h = torch.cuda.current_stream().cuda_stream
    ml.route(dl.x, h)
    ml.permute(dl.x, h)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ml.grouped_ffn(h, None, gate, x=dl.x)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert L.moe_check_device() == L.MOE_ERR_TIMEOUT
    assert "ran out" in L.moe_last_error()
    assert L.moe_check_device() == L.MOE_OK
    assert 0.04 < waited < 5.0
    run_layer(dl)
    y_ref, _, _, _ = ow.layer_full(cfg, 0, dl.pool, dl.slot, dl.inputs)
    assert_close_rel(to_np(ml.y[:cfg.T]), y_ref, _rtol(cfg), "after the timeout")
