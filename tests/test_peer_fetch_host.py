"""The DWDP group's peer fetch schedule on the host (no GPU work).

moe_peer_fetch_plan gives each rank the copies that pull the other ranks'
expert pools into its remote buffer.  Time-division slicing across
destinations (the explainer's contention caption) must leave no step in
which two destinations read one source, while every peer pool is copied
exactly once into its place in the remote buffer.  The same is checked with
four gloo ranks, each computing only its own plan.
"""
import ctypes
import itertools
import os
import socket

import pytest
import torch.multiprocessing as mp

from split_weight_b200 import _lib as L


def _coverage(plan, G, rank, nbytes):
    """Per source: sorted (src_offset, dst_offset, bytes) must tile [0, nbytes)
    and land at that source's place in the remote buffer."""
    for s in range(G):
        if s == rank:
            assert all(e.src_rank != s for e in plan)
            continue
        pieces = sorted((e.src_offset, e.dst_offset, e.bytes) for e in plan if e.src_rank == s)
        pos = s if s < rank else s - 1
        at = 0
        for src_off, dst_off, n in pieces:
            assert src_off == at and n > 0
            assert dst_off == pos * nbytes + src_off
            at += n
        assert at == nbytes


@pytest.mark.parametrize("G", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("slices", [1, 3, 8])
@pytest.mark.parametrize("nbytes", [256, 256 * 7, 88_080_384 * 64])
def test_plan_copies_each_peer_pool_once_and_no_source_serves_two(G, slices, nbytes):
    plans = [L.peer_fetch_plan(G, r, nbytes, slices) for r in range(G)]
    for r, plan in enumerate(plans):
        assert [e.step for e in plan] == list(range(len(plan)))
        assert all(e.src_offset % 256 == 0 and e.dst_offset % 256 == 0 for e in plan)
        _coverage(plan, G, r, nbytes)
    n = len(plans[0])
    assert all(len(p) == n for p in plans)
    for j in range(n):
        sources = [plans[r][j].src_rank for r in range(G)]
        assert sorted(sources) == list(range(G)), f"step {j}: sources {sources}"
        assert all(plans[r][j].src_rank != r for r in range(G))


def test_plan_pieces_follow_the_slice_count():
    plan = L.peer_fetch_plan(4, 2, 1000 * 256, 3)
    assert len(plan) == 9
    # step j reads source (r + 1 + j mod 3) mod 4: 3, 0, 1, 3, 0, 1, ...
    assert [e.src_rank for e in plan] == [3, 0, 1] * 3
    assert [e.bytes for e in plan if e.src_rank == 0] == [333 * 256, 333 * 256, 334 * 256]
    # fewer 256-byte units than slices: one piece per unit
    assert len(L.peer_fetch_plan(4, 0, 512, 8)) == 3 * 2


def test_plan_argument_errors():
    n = ctypes.c_int32()
    assert L.moe_peer_fetch_plan(1, 0, 256, 1, None, 0, ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
    assert L.moe_peer_fetch_plan(4, 4, 256, 1, None, 0, ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
    assert L.moe_peer_fetch_plan(4, 0, 100, 1, None, 0, ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
    assert L.moe_peer_fetch_plan(4, 0, 256, 0, None, 0, ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
    small = (L.moe_peer_copy * 2)()
    assert L.moe_peer_fetch_plan(4, 0, 1024, 4, small, 2, ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
    assert n.value == 12
    pools = (ctypes.c_void_p * 4)(1 << 20, None, 3 << 20, 4 << 20)
    # rank 1's pool is not read, but rank 0's own slot may be NULL only for rank 0
    assert L.moe_prefetch_peers(4, 0, pools, 1024, 4, 8 << 20, None, None,
                                None) == L.MOE_ERR_INVALID_ARG
    pools = (ctypes.c_void_p * 4)(None, 2 << 20, 3 << 20, 4 << 20)
    assert L.moe_prefetch_peers(4, 0, pools, 1024, 4, (8 << 20) + 16, None, None,
                                None) == L.MOE_ERR_INVALID_ARG   # dst alignment
    assert L.moe_prefetch_peers(4, 0, pools, 1 << 20, 4, 3 << 20, None, None,
                                None) == L.MOE_ERR_INVALID_ARG   # dst overlaps a pool


def test_unsliced_random_order_pulls_stack_where_the_plan_never_does():
    """Without the schedule, a destination pulls its peers in some order of its
    own.  With the order uniform and independent per rank in a group of 4,
    the three-way stacking the contention caption describes happens in a
    sizeable fraction of cases (enumerated here); the plan's rotation has
    none by construction."""
    G = 4
    orders = {r: list(itertools.permutations([s for s in range(G) if s != r])) for r in range(G)}
    stacked = total = 0
    for combo in itertools.product(*(orders[r] for r in range(G))):
        total += 1
        if any(max([combo[r][ph] for r in range(G)].count(s) for s in range(G)) >= 3
               for ph in range(G - 1)):
            stacked += 1
    frac = stacked / total
    assert total == 6 ** 4
    assert 0.25 < frac < 0.5   # 4/27 per phase, three phases
    plans = [L.peer_fetch_plan(G, r, 1 << 20, 8) for r in range(G)]
    for j in range(len(plans[0])):
        counts = [sum(plans[r][j].src_rank == s for r in range(G)) for s in range(G)]
        assert max(counts) == 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _plan_worker(rank, world, port, nbytes, slices, out):
    import datetime

    import torch
    import torch.distributed as dist
    from split_weight_b200 import _lib as Lw
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        plan = Lw.peer_fetch_plan(world, rank, nbytes, slices)
        mine = torch.tensor([e.src_rank for e in plan], dtype=torch.int64)
        every = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(every, mine)
        steps = torch.stack(every)          # [rank, step] -> source read
        ok = all(sorted(steps[:, j].tolist()) == list(range(world)) for j in range(steps.shape[1]))
        out[rank] = (ok, int(steps.shape[1]))
    finally:
        dist.destroy_process_group()


def test_four_gloo_ranks_read_distinct_sources_at_every_step():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_plan_worker, args=(r, 4, port, 64 * 88_080_384, 8, out))
             for r in range(4)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert all(out[r] == (True, 24) for r in range(4))
