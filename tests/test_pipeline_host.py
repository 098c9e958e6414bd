"""The prefetch schedule of PrefetchPipeline on the host (no GPU work).

Streams, events and the copy call are replaced by fakes that log, in host
order, what each stream is asked to do.  A small replay then runs the two
streams with CUDA's event rule (a wait is for the last record of the event
enqueued before it) and checks that every grouped GEMM reads a buffer fully
refilled with its own layer's remote experts, for both fetch schedules."""
import numpy as np
import pytest
import torch

import split_weight_b200.layer as layer_mod
from split_weight_b200 import _lib as L


class Log:
    ops: list = []


class FakeEvent:
    count = 0
    by_id: dict = {}

    def __init__(self):
        FakeEvent.count += 1
        self.cuda_event = FakeEvent.count
        self.version = 0  # records enqueued so far (host order)
        FakeEvent.by_id[self.cuda_event] = self

    def record(self, stream=None):
        self.version += 1
        Log.ops.append(("record", getattr(stream, "name", "compute"), self, self.version))


class FakeStream:
    def __init__(self, device=None, name="copy"):
        self.name = name
        self.cuda_stream = name

    def wait_event(self, ev):
        Log.ops.append(("wait", self.name, ev, ev.version))

    def wait_stream(self, other):   # ordering against the caller's earlier work
        pass


class Ptr(tuple):
    """A device pointer stand-in: (owner, byte offset)."""

    def __add__(self, k):
        return Ptr((self[0], self[1] + k))


class Buffer:
    def __init__(self, owner):
        self.owner = owner

    def data_ptr(self):
        return Ptr((self.owner, 0))


class FakeLayer:
    def __init__(self, idx):
        self.idx, self.y = idx, None

    def route(self, x, h):
        pass

    def permute(self, x, h):
        pass

    def grouped_ffn(self, h, remote, gate=None, x=None, progress=None):
        if gate is not None:   # the gated kernel reads each chunk once its flag reached the epoch
            Log.ops.append(("gate", "compute", gate.flags.owner, gate.epoch))
        if progress is not None:
            # reports while the GEMMs still read their buffer: logged before the
            # read, so a paced chunk released by them that touched this buffer
            # would show in the snapshot
            for st in range(1, progress.steps + 1):
                Log.ops.append(("progress", "compute", progress.base + st))
        Log.ops.append(("ffn", "compute", self.idx, remote.owner))
        if progress is not None:   # the call's final write
            Log.ops.append(("progress", "compute", progress.base + progress.steps + 1))

    def combine(self, h):
        pass


def fake_prefetch(src, dst, nbytes, chunk, stream, wait, ready):
    if wait is not None:
        ev = FakeEvent.by_id[wait]
        Log.ops.append(("wait", "copy", ev, ev.version))
    assert src[1] == dst[1]
    Log.ops.append(("copy", "copy", src[0], dst[0], src[1], src[1] + nbytes))
    if ready is not None:
        FakeEvent.by_id[ready].record(FakeStream(name="copy"))
    return L.MOE_OK


def fake_prefetch_flagged(src, dst, nbytes, chunk, stream, wait, flags, epoch, ready):
    if wait is not None:
        ev = FakeEvent.by_id[wait]
        Log.ops.append(("wait", "copy", ev, ev.version))
    assert src[1] == dst[1] and src[1] % chunk == 0
    first = src[1] // chunk
    assert flags[1] == 4 * first
    for i, lo in enumerate(range(src[1], src[1] + nbytes, chunk)):
        hi = min(lo + chunk, src[1] + nbytes)
        Log.ops.append(("copy", "copy", src[0], dst[0], lo, hi))
        Log.ops.append(("flag", "copy", flags[0], first + i, epoch))
    if ready is not None:
        FakeEvent.by_id[ready].record(FakeStream(name="copy"))
    return L.MOE_OK


def fake_prefetch_paced(src, dst, nbytes, chunk, stream, wait, flags, epoch, pace, lead, ready):
    if wait is not None:
        ev = FakeEvent.by_id[wait]
        Log.ops.append(("wait", "copy", ev, ev.version))
    assert src[1] == dst[1] and src[1] % chunk == 0
    first = src[1] // chunk
    assert flags[1] == 4 * first
    n = -(-nbytes // chunk)
    for i, lo in enumerate(range(src[1], src[1] + nbytes, chunk)):
        hi = min(lo + chunk, src[1] + nbytes)
        Log.ops.append(("pwait", "copy", L.moe_pace_threshold(i, n, lead, pace.base, pace.steps)))
        Log.ops.append(("copy", "copy", src[0], dst[0], lo, hi))
        Log.ops.append(("flag", "copy", flags[0], first + i, epoch))
    if ready is not None:
        FakeEvent.by_id[ready].record(FakeStream(name="copy"))
    return L.MOE_OK


class FakeProgress:
    def __init__(self, word, tiles, base, steps):
        self.word, self.tiles, self.base, self.steps = word, tiles, base, steps


class FlagBuffer(Buffer):
    def __init__(self, owner, n):
        super().__init__(owner)
        self.n = n

    def numel(self):
        return self.n


def replay(ops, nbytes, n_flags=0, shared=False):
    """Runs both streams in order, honouring waits; returns (layer, buffer
    contents) for every grouped GEMM in execution order.  shared=True runs
    both streams' work as one hardware queue in host order (streams that
    share a queue): a wait then blocks everything enqueued after it."""
    done = {}  # event id -> highest executed record version
    if shared:
        queues = {"all": list(ops)}
    else:
        queues = {s: [o for o in ops if o[1] == s] for s in ("compute", "copy")}
    pos = {s: 0 for s in queues}
    buffers, seen, moved, flags, word = {}, [], True, {}, 0
    while moved:
        moved = False
        for s, q in queues.items():
            while pos[s] < len(q):
                op = q[pos[s]]
                if op[0] == "wait" and done.get(op[2].cuda_event, 0) < op[3]:
                    break
                if op[0] == "gate" and any(flags.get((op[2], c), 0) < op[3] for c in range(n_flags)):
                    break
                if op[0] == "pwait" and ((word - op[2]) & 0xFFFFFFFF) >= 1 << 31:
                    break   # (int32_t)(word - threshold) < 0
                if op[0] == "progress":
                    if ((op[2] - word) & 0xFFFFFFFF) < 1 << 31:
                        word = op[2]
                if op[0] == "flag":
                    flags[(op[2], op[3])] = op[4]
                if op[0] == "record":
                    done[op[2].cuda_event] = max(done.get(op[2].cuda_event, 0), op[3])
                elif op[0] == "copy":
                    _, _, layer, buf, lo, hi = op
                    content = buffers.setdefault(buf, [None] * nbytes)
                    content[lo:hi] = [layer] * (hi - lo)
                elif op[0] == "ffn":
                    seen.append((op[2], list(buffers.get(op[3], [None] * nbytes))))
                pos[s] += 1
                moved = True
    assert all(pos[s] == len(q) for s, q in queues.items()), "the schedule deadlocks"
    return seen


@pytest.mark.parametrize("pace", [(0, 0), (3, 0), (3, 1), (2, 5)],
                         ids=["unpaced", "paced", "paced_lead1", "paced_all_lead"])
@pytest.mark.parametrize("gate_slots", [0, 2], ids=["events", "flags"])
@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
@pytest.mark.parametrize("n_layers", [1, 2, 3, 4])
def test_every_grouped_gemm_reads_its_own_complete_fetch(monkeypatch, split, n_layers, gate_slots,
                                                         pace):
    """Event-gated schedule: the compute stream waits for ready.  Flag-gated
    schedule: the grouped GEMM of execution g waits on the device for every
    chunk flag of its buffer to reach g + 1; each flag must be written only
    after its chunk holds the right layer, and never for a later fetch before
    the grouped GEMM that needs the earlier one has run.  Paced schedule
    (flags, pace_steps > 0): each chunk of execution g + 1's fetch also
    waits on the copy stream for execution g's progress reports.  Every
    schedule must also complete when both streams share one hardware queue,
    i.e. no wait is enqueued ahead of the work that satisfies it."""
    pace_steps, pace_lead = pace
    if pace_steps and not gate_slots:
        pytest.skip("a paced fetch needs readiness flags")
    monkeypatch.setattr(torch.cuda, "Stream", FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(L, "moe_prefetch_layer", fake_prefetch)
    monkeypatch.setattr(L, "moe_prefetch_layer_flagged", fake_prefetch_flagged)
    monkeypatch.setattr(L, "moe_prefetch_layer_paced", fake_prefetch_paced)
    monkeypatch.setattr(L, "moe_progress", FakeProgress)
    monkeypatch.setattr(layer_mod.ctypes, "byref", lambda o: o)
    monkeypatch.setattr(L, "check", lambda status: None)
    Log.ops = []
    # events: an odd size (the halves split at a 256-byte boundary); flags:
    # 5 slots of 256 bytes, 2 per flag (3 flags, the last one short)
    nbytes = 1000 if gate_slots == 0 else 5 * 256

    # the constructor's device allocations replaced by pointer stand-ins
    pipe = layer_mod.PrefetchPipeline.__new__(layer_mod.PrefetchPipeline)
    pipe.layers = [FakeLayer(l) for l in range(n_layers)]
    pipe.peer_stores = [Buffer(("store", l)) for l in range(n_layers)]
    pipe.remote_bytes, pipe.chunk_bytes = nbytes, 0
    pipe.split, pipe.pending = split, None
    pipe.gate_slots, pipe.window_block, pipe.gate_timeout_ns = gate_slots, None, 0
    n_flags = 0
    if gate_slots:
        pipe.stride, n_flags = 256, 3
        pipe.n_flags = n_flags
        pipe.flags = [FlagBuffer(("flags", 0), n_flags), FlagBuffer(("flags", 1), n_flags)]
    pipe.bufs = [Buffer(("buf", 0)), Buffer(("buf", 1))]
    pipe.copy_stream = FakeStream(name="copy")
    pipe.ready = [FakeEvent() for _ in range(2)]
    pipe.free = [FakeEvent() for _ in range(2)]
    for ev in pipe.ready + pipe.free:
        ev.record(pipe.copy_stream)
    pipe.g = 0
    pipe.pace_steps, pipe.pace_lead, pipe.g_pace0 = pace_steps, pace_lead, 0
    pipe.progress_words = Buffer(("progress", 0))
    pipe.select = False
    pipe.device = None

    compute = FakeStream(name="compute")
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: compute)
    pipe.prime()
    n_exec = 3 * n_layers + 1
    for i in range(n_exec):
        pipe.run_layer(i % n_layers, None, compute, prefetch=True, wrap=True)

    for shared in (False, True):   # independent queues, then one shared queue
        seen = replay(Log.ops, nbytes, n_flags, shared)
        assert len(seen) == n_exec
        for i, (lidx, content) in enumerate(seen):
            assert lidx == i % n_layers
            assert all(c == ("store", lidx) for c in content), (
                f"execution {i} (layer {lidx}) read {sorted(set(map(str, content)))}")


def test_split_halves_cover_the_buffer_once(monkeypatch):
    """fetch_half(0) and fetch_half(1) copy [0, cut) and [cut, n) with cut a
    256-byte multiple; only the second records ready."""
    calls = []
    monkeypatch.setattr(L, "moe_prefetch_layer",
                        lambda s, d, n, c, st, w, r: calls.append((s[1], n, r)) or L.MOE_OK)
    monkeypatch.setattr(L, "check", lambda status: None)
    pipe = layer_mod.PrefetchPipeline.__new__(layer_mod.PrefetchPipeline)
    pipe.peer_stores = [Buffer("store")]
    pipe.bufs = [Buffer("buf0"), Buffer("buf1")]
    pipe.remote_bytes, pipe.chunk_bytes = 16_911_433_728, 0
    pipe.gate_slots, pipe.g = 0, 0
    pipe.copy_stream = FakeStream(name="copy")
    pipe.ready = [FakeEvent(), FakeEvent()]
    free = FakeEvent()
    pipe.fetch_half(0, 1, 0, free)
    pipe.fetch_half(0, 1, 1, free)
    (lo0, n0, r0), (lo1, n1, r1) = calls
    assert lo0 == 0 and lo1 == n0 and n0 + n1 == pipe.remote_bytes and n0 % 256 == 0
    assert r0 is None and r1 == pipe.ready[1].cuda_event


# --------------------------------------------------------------------------
# selective schedule (per-slot flags, look-ahead prediction, missed slots)
# --------------------------------------------------------------------------
class SelLayer(FakeLayer):
    """A layer whose routing touches a fixed set of remote slots."""

    def __init__(self, idx, pool_slot, touched_experts, T=4, k=2, E=8):
        super().__init__(idx)
        self.shape = type("S", (), {"T": T, "k": k, "E": E, "x_dtype": "bf16"})()
        self.weights = type("W", (), {"pool_slot": pool_slot})()
        self.touched_experts = touched_experts
        self.topk_idx = Buffer(("topk", idx))
        self._cfg = ("cfg", idx)
        self.w_gate, self.bias = Buffer(("wg", idx)), None

    def grouped_ffn(self, h, remote, gate=None, x=None, progress=None):
        slots = sorted(layer_mod.remote_slots(self.weights.pool_slot, self.touched_vector()))
        Log.ops.append(("gate_slots", "compute", gate.flags.owner, gate.epoch, tuple(slots)))
        Log.ops.append(("ffn_slots", "compute", self.idx, remote.owner, tuple(slots)))

    def touched_vector(self):
        v = np.zeros(self.shape.E, dtype=np.uint8)
        v[list(self.touched_experts)] = 1
        return v


class HostRows:
    """The pinned (2, E) touched bytes: row 0 the routing, row 1 the prediction."""

    def __init__(self, E):
        self.rows = [torch.zeros(E, dtype=torch.uint8), torch.zeros(E, dtype=torch.uint8)]
        self.pending = [None, None]

    def __getitem__(self, i):
        return self.rows[i]

    def copy_(self, src, non_blocking=False):
        for i in range(2):
            if self.pending[i] is not None:
                self.rows[i].copy_(torch.from_numpy(self.pending[i]))


def replay_slots(ops, shared=False):
    """replay() for the selective ops: copies and flags per slot, and each
    grouped GEMM waits for the flags of the slots it touches."""
    done = {}
    queues = ({"all": list(ops)} if shared else
              {s: [o for o in ops if o[1] == s] for s in ("compute", "copy")})
    pos = {s: 0 for s in queues}
    buffers, flags, seen, moved = {}, {}, [], True
    while moved:
        moved = False
        for s, q in queues.items():
            while pos[s] < len(q):
                op = q[pos[s]]
                if op[0] == "wait" and done.get(op[2].cuda_event, 0) < op[3]:
                    break
                if op[0] == "gate_slots" and any(flags.get((op[2], c), 0) < op[3] for c in op[4]):
                    break
                if op[0] == "record":
                    done[op[2].cuda_event] = max(done.get(op[2].cuda_event, 0), op[3])
                elif op[0] == "slot_copy":
                    buffers.setdefault(op[3], {})[op[4]] = op[2]
                elif op[0] == "flag":
                    flags[(op[2], op[3])] = op[4]
                elif op[0] == "ffn_slots":
                    seen.append((op[2], {c: buffers.get(op[3], {}).get(c) for c in op[4]}))
                pos[s] += 1
                moved = True
    assert all(pos[s] == len(q) for s, q in queues.items()), "the schedule deadlocks"
    return seen


@pytest.mark.parametrize("predict", ["exact", "partial", "none"])
@pytest.mark.parametrize("n_layers", [1, 2, 3])
def test_selective_fetch_covers_every_touched_slot(monkeypatch, n_layers, predict):
    """Every grouped GEMM of the selective schedule must find, at each remote
    slot its routing touches, that slot of its own layer, fetched either as
    predicted by the previous execution or as a miss before it; the
    prediction may be exact, partial or empty, and the schedule must also
    complete as one shared queue."""
    np_ = np
    E = 8
    # experts 0-1 local (slots 0-1), 2-7 remote (slots 5, 0, 3, 1, 4, 2)
    pool_slot = np_.array([0, 1] + [(1 << 31) | s for s in (5, 0, 3, 1, 4, 2)],
                          dtype=np_.uint32).view(np_.int32)
    touched = [{0, 2, 5}, {3, 4, 7, 1}, {2, 6}]
    layers = [SelLayer(l, pool_slot, touched[l]) for l in range(n_layers)]
    pred_of = {"exact": lambda nxt: touched[nxt], "partial": lambda nxt: set(list(touched[nxt])[:1]),
               "none": lambda nxt: set()}[predict]

    host = HostRows(E)
    state = {}

    def fake_touched(idx_ptr, A, E_, out_ptr, h):
        if idx_ptr[0][0] == "topk":          # a layer's own routing
            host.pending[0] = layers[idx_ptr[0][1]].touched_vector()
        else:                                 # the look-ahead prediction
            v = np_.zeros(E, dtype=np_.uint8)
            v[list(pred_of(state["next"]))] = 1
            host.pending[1] = v
        return L.MOE_OK

    def fake_route(cfg, x, dt, wg, bias, idx, w, ws, wsn, h):
        state["next"] = cfg._obj[1] if hasattr(cfg, "_obj") else cfg[1]
        return L.MOE_OK

    def fake_slots(src, dst, slot_bytes, n_slots, arr, n, stream, wait, flags, epoch, ready):
        if wait is not None:
            ev = FakeEvent.by_id[wait]
            Log.ops.append(("wait", "copy", ev, ev.version))
        for i in range(n):
            assert 0 <= arr[i] < n_slots
            Log.ops.append(("slot_copy", "copy", src[0], dst[0], arr[i]))
            Log.ops.append(("flag", "copy", flags[0], arr[i], epoch))
        return L.MOE_OK

    class Ev(FakeEvent):
        def synchronize(self):
            pass

    monkeypatch.setattr(torch.cuda, "Stream", FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: __import__("contextlib").nullcontext())
    monkeypatch.setattr(L, "moe_experts_touched", fake_touched)
    monkeypatch.setattr(L, "moe_route", fake_route)
    monkeypatch.setattr(L, "moe_prefetch_slots", fake_slots)
    monkeypatch.setattr(layer_mod.ctypes, "byref", lambda o: o)
    monkeypatch.setattr(L, "check", lambda status: None)
    Log.ops = []

    pipe = layer_mod.PrefetchPipeline.__new__(layer_mod.PrefetchPipeline)
    pipe.layers = layers
    pipe.peer_stores = [Buffer(("store", l)) for l in range(n_layers)]
    pipe.stride, pipe.remote_bytes, pipe.chunk_bytes = 256, 6 * 256, 0
    pipe.split, pipe.pending, pipe.window_block, pipe.gate_timeout_ns = False, None, None, 0
    pipe.gate_slots, pipe.n_flags = 1, 6
    pipe.flags = [FlagBuffer(("flags", 0), 6), FlagBuffer(("flags", 1), 6)]
    pipe.bufs = [Buffer(("buf", 0)), Buffer(("buf", 1))]
    pipe.copy_stream = FakeStream(name="copy")
    pipe.ready = [FakeEvent() for _ in range(2)]
    pipe.free = [FakeEvent() for _ in range(2)]
    for ev in pipe.ready + pipe.free:
        ev.record(pipe.copy_stream)
    pipe.g, pipe.device = 0, None
    pipe.pace_steps, pipe.pace_lead, pipe.g_pace0 = 0, 0, 0
    pipe.select, pipe.fetched, pipe.select_stats = True, [set(), set()], []
    pipe._pred = {"idx": Buffer(("pred", 0)), "w": Buffer(("predw", 0)),
                  "ws": type("WS", (), {"data_ptr": lambda self: 0, "numel": lambda self: 16})(),
                  "touched": [Buffer(("touched", 0)), Buffer(("touched", 1))], "host": host,
                  "ev": Ev()}
    for lay in layers:
        lay._cfg = ("cfg", lay.idx)

    compute = FakeStream(name="compute")
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: compute)
    pipe.prime()
    n_exec = 3 * n_layers + 1
    for i in range(n_exec):
        pipe.run_layer(i % n_layers, Buffer(("x", i % n_layers)), compute, prefetch=True,
                       wrap=True)

    for shared in (False, True):
        seen = replay_slots(Log.ops, shared)
        assert len(seen) == n_exec
        for i, (lidx, content) in enumerate(seen):
            assert lidx == i % n_layers
            assert all(v == ("store", lidx) for v in content.values()), (i, lidx, content)
    # fetched = predicted + missed, and nothing touched is left out
    for i, st in enumerate(pipe.select_stats):
        assert st["touched"] == len(layer_mod.remote_slots(pool_slot, layers[i % n_layers].touched_vector()))
    if predict == "exact" and n_layers > 1:
        assert all(st["missed"] == 0 for st in pipe.select_stats[1:])
