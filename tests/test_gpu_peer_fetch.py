"""moe_prefetch_peers and the pool export/import on one GPU.

A DWDP group needs one GPU per rank; here the ranks' pools are separate
allocations on one device, which exercises the same copies (the copy engine
reads a pool that is not the destination's) without kernels on several
GPUs.  The IPC path runs between two processes on that device: one exports
its pool, the other maps it and pulls it into its remote buffer.
"""
import gc

import pytest
import torch
import torch.multiprocessing as mp

from split_weight_b200 import PeerPools, _lib as L, close_pool, export_pool, import_pool

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory(cuda_device):
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _pool(rank: int, nbytes: int, dev) -> torch.Tensor:
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    return torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=dev, generator=g)


@pytest.mark.parametrize("slices", [1, 5])
def test_each_rank_receives_the_other_pools_in_rank_order(cuda_device, slices):
    G, nbytes = 4, 3 * (1 << 20) + 768
    pools = [_pool(r, nbytes, cuda_device) for r in range(G)]
    copy = torch.cuda.Stream()
    for r in range(G):
        dst = torch.zeros((G - 1) * nbytes, dtype=torch.uint8, device=cuda_device)
        ready = torch.cuda.Event()
        ready.record(copy)
        peers = PeerPools(G, r, [p.data_ptr() for p in pools], nbytes, slices)
        copy.wait_stream(torch.cuda.current_stream())   # dst and the pools are filled there
        peers.fetch(dst, copy, None, ready)
        assert L.moe_wait_ready(ready.cuda_event, 20000) == L.MOE_OK
        want = torch.cat([pools[s] for s in range(G) if s != r])
        assert torch.equal(dst, want), f"rank {r}"


def _exporter(nbytes, q_out, q_in):
    import torch as t
    from split_weight_b200 import export_pool as ex
    t.cuda.set_device(0)
    pool = _pool(1, nbytes, t.device("cuda", 0))
    t.cuda.synchronize()
    q_out.put(ex(pool))
    q_in.get(timeout=120)        # the importer has closed its mapping
    del pool


def test_pool_exported_by_another_process_is_fetched(cuda_device):
    nbytes = (1 << 22) + 256
    ctx = mp.get_context("spawn")
    q_out, q_in = ctx.Queue(), ctx.Queue()
    p = ctx.Process(target=_exporter, args=(nbytes, q_out, q_in))
    p.start()
    try:
        handle = q_out.get(timeout=120)
        base, mapping = import_pool(handle)
        own = _pool(0, nbytes, cuda_device)
        dst = torch.zeros(nbytes, dtype=torch.uint8, device=cuda_device)
        copy = torch.cuda.Stream()
        copy.wait_stream(torch.cuda.current_stream())   # dst is zero-filled there
        PeerPools(2, 0, [own.data_ptr(), base], nbytes, 4).fetch(dst, copy)
        copy.synchronize()
        assert torch.equal(dst, _pool(1, nbytes, cuda_device))
        close_pool(mapping)
    finally:
        q_in.put("done")
        p.join(120)
    assert p.exitcode == 0
