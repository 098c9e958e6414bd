"""The copy-engine prefetch into alternate buffers (GPU)."""
import gc

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import config, device as mdev
from oracle import workload as ow
from split_weight_b200 import PrefetchPipeline, _lib as L

from gpu_util import MID_SIGMOID, RTOL_BF16, assert_close_rel, sync_check, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
def test_pipeline_equals_resident_layers(split):
    """Three layers through two alternate buffers, each filled by
    moe_prefetch_layer from the layer's peer store, give the same bits as
    each layer computed with its own resident remote pool, and every output
    element of every layer, in both passes, matches the CPU oracle."""
    cfg = MID_SIGMOID.with_(cfg_id=17, layers=3)
    dls = [mdev.build_layer(cfg, layer=l) for l in range(cfg.layers)]
    ref = []
    for d in dls:
        d.layer.forward(d.x)
        ref.append(d.layer.y.clone())
    sync_check()
    oracle_y = [ow.layer_full(cfg, l, d.pool, d.slot, d.inputs)[0] for l, d in enumerate(dls)]
    stores = [mdev.peer_store(cfg, l, dls[l].layer.weights) for l in range(cfg.layers)]
    for l in range(cfg.layers):   # the peer store holds exactly the remote pool
        assert torch.equal(stores[l], dls[l].layer.weights.remote)
    w0 = dls[0].layer.weights
    pipe = PrefetchPipeline([d.layer for d in dls], stores, w0.n_remote * w0.stride,
                            chunk_bytes=1 << 20, split=split)
    for d in dls:
        d.layer.weights.remote.zero_()   # the pipeline must not read them
    with torch.cuda.stream(pipe.copy_stream):
        torch.cuda._sleep(300_000_000)   # delay the copies: the consumer must wait for them
    pipe.prime()
    for rep in range(2):   # second pass runs on buffers refilled during the first
        outs = pipe.run([d.x for d in dls])
        sync_check()
        for l in range(cfg.layers):
            assert torch.equal(outs[l], ref[l]), f"pass {rep} layer {l}"
            assert_close_rel(to_np(outs[l][:cfg.T]), oracle_y[l], RTOL_BF16,
                             f"pass {rep} layer {l} against the oracle")


@pytest.mark.parametrize("split", [True], ids=["split"])
def test_imbalanced_prefill_full_size_through_the_pipeline(split, cuda_device):
    """The full-size imbalanced prefill (2 layers x 16384 tokens, Zipf-skewed
    routing) run as the benchmark runs it: remote experts only in the peer
    stores, fetched by moe_prefetch_layer into the two alternate buffers.
    Routing and permutation bit-exact, sampled output rows of both layers in
    both passes against the oracle."""
    cfg = config(4)
    dls = [mdev.build_layer(cfg, layer=l) for l in range(cfg.layers)]
    stores = [mdev.peer_store(cfg, l, dls[l].layer.weights) for l in range(cfg.layers)]
    w0 = dls[0].layer.weights
    rbytes = w0.n_remote * w0.stride
    for d in dls:   # the pipeline's buffers replace the layers' own remote pools
        d.layer.weights.remote = torch.empty(1, dtype=torch.uint8, device=cuda_device)
    gc.collect()
    torch.cuda.empty_cache()
    pipe = PrefetchPipeline([d.layer for d in dls], stores, rbytes, split=split)
    pipe.prime()
    rng = np.random.default_rng(7)
    toks = [np.sort(rng.choice(cfg.T, size=5, replace=False)) for _ in range(cfg.layers)]
    refs, cache = [], {}
    for l, d in enumerate(dls):
        idx_ref, w_ref, _ = ow.route(cfg, l, d.inputs)
        refs.append((idx_ref, w_ref, ow.layer_tokens(cfg, l, toks[l], idx_ref, w_ref, d.pool,
                                                     d.slot, d.inputs, cache)))
        cache.clear()
    for rep in range(2):
        outs = pipe.run([d.x for d in dls])
        sync_check()
        for l, d in enumerate(dls):
            idx_ref, w_ref, y_ref = refs[l]
            np.testing.assert_array_equal(d.layer.topk_idx[:cfg.T].cpu().numpy(), idx_ref)
            off, src, inv = oracle.permute(idx_ref, cfg.E)
            np.testing.assert_array_equal(d.layer.offsets.cpu().numpy(), off)
            np.testing.assert_array_equal(d.layer.inv_pos[:cfg.T].cpu().numpy(), inv)
            y = to_np(outs[l][torch.from_numpy(toks[l]).to(cuda_device)])
            assert_close_rel(y, y_ref, RTOL_BF16, f"pass {rep} layer {l} sampled rows")
    del pipe, stores, dls


def test_wait_ready_times_out_then_completes(cuda_device):
    src = torch.randint(0, 255, (1 << 22,), dtype=torch.uint8, device=cuda_device)
    dst = torch.zeros_like(src)
    copy = torch.cuda.Stream()
    ready = torch.cuda.Event()
    ready.record(copy)                     # torch creates the CUDA event on first record
    assert ready.cuda_event != 0
    with torch.cuda.stream(copy):
        torch.cuda._sleep(1_500_000_000)   # ~0.8 s of a bounded spin on the copy stream
    L.check(L.moe_prefetch_layer(src.data_ptr(), dst.data_ptr(), src.numel(), 0,
                                 copy.cuda_stream, None, ready.cuda_event))
    assert L.moe_wait_ready(ready.cuda_event, 20) == L.MOE_ERR_TIMEOUT
    assert L.moe_wait_ready(ready.cuda_event, 20000) == L.MOE_OK
    torch.cuda.synchronize()
    assert torch.equal(dst, src)


def test_prefetch_waits_for_the_free_event(cuda_device):
    """The copy into a buffer must not start before the consumer released it."""
    buf_src = torch.full((1 << 20,), 7, dtype=torch.uint8, device=cuda_device)
    buf = torch.zeros_like(buf_src)
    seen = torch.empty_like(buf)
    compute, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    free, ready = torch.cuda.Event(), torch.cuda.Event()
    ready.record(copy)
    torch.cuda._sleep(500_000_000)          # the consumer is still busy ...
    seen.copy_(buf)                          # ... and reads the old contents
    free.record(compute)
    L.check(L.moe_prefetch_layer(buf_src.data_ptr(), buf.data_ptr(), buf.numel(), 0,
                                 copy.cuda_stream, free.cuda_event, ready.cuda_event))
    torch.cuda.synchronize()
    assert int(seen.max()) == 0              # read before the copy landed
    assert torch.equal(buf, buf_src)


def test_injected_failure_leaves_library_usable(cuda_device):
    src = torch.ones(4096, dtype=torch.uint8, device=cuda_device)
    dst = torch.zeros_like(src)
    L.moe_debug_fail_next_cuda_calls(1)
    s = torch.cuda.current_stream().cuda_stream
    assert L.moe_prefetch_layer(src.data_ptr(), dst.data_ptr(), 4096, 0, s, None,
                                None) == L.MOE_ERR_CUDA
    L.check(L.moe_prefetch_layer(src.data_ptr(), dst.data_ptr(), 4096, 0, s, None, None))
    torch.cuda.synchronize()
    assert torch.equal(src, dst)
