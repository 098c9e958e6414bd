"""Layer-level driver of the C ABI: one DWDP rank's MoE block.

``MoELayer.forward`` enqueues moe_route -> moe_permute -> moe_grouped_ffn ->
moe_combine on one stream.  torch provides device memory, streams and events
only; every step of the block runs in libswb_moe.so.

``SplitWeights`` holds one layer's expert weights in two pools that have
nothing to do with each other in memory - the rank's own experts (local)
and the buffer the remote experts were fetched into - plus the per-expert
(pool, slot) table through which the grouped GEMM finds each expert (the
split-weight figure of the explainer "Distributed Weight Data Parallelism
cuts LLM inference stalls": no merge into one contiguous buffer).
``PrefetchPipeline`` runs several layers with the next layers' remote
experts copied into alternate buffers on a copy-engine stream (the
explainer's prefetch figure).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib as L

POOL_LOCAL, POOL_REMOTE = 0, 1
_DT = {"f32": L.MOE_F32, "bf16": L.MOE_BF16, "e4m3": L.MOE_E4M3}


@dataclass(frozen=True)
class LayerShape:
    T: int
    H: int
    I: int
    E: int
    k: int
    score: str = "sigmoid"       # "softmax" | "sigmoid"
    n_group: int = 1
    topk_group: int = 1
    routed_scale: float = 1.0
    renormalize: bool = True
    has_shared: bool = False
    x_dtype: str = "bf16"        # "f32" | "bf16"
    w_dtype: str = "bf16"        # "bf16" | "e4m3"
    y_dtype: str = "bf16"        # "f32" | "bf16"
    # activations the grouped GEMMs read: "bf16", or "e4m3" (with e4m3 weights:
    # both GEMMs on the fp8 tensor cores, x_perm and h e4m3 with 1x128 scales)
    act_dtype: str = "bf16"

    @property
    def A(self) -> int:
        return self.T * self.k

    @property
    def rows(self) -> int:
        return self.A + (self.T if self.has_shared else 0)

    def route_cfg(self) -> L.moe_route_cfg:
        return L.moe_route_cfg(self.T, self.H, self.E, self.k,
                               L.MOE_SCORE_SIGMOID if self.score == "sigmoid" else L.MOE_SCORE_SOFTMAX,
                               self.n_group, self.topk_group, self.routed_scale,
                               1 if self.renormalize else 0)

    def ffn_desc(self) -> L.moe_ffn_desc:
        return L.moe_ffn_desc(self.T, self.H, self.I, self.E, self.k, _DT[self.w_dtype],
                              _DT[self.act_dtype], 1 if self.has_shared else 0)


def _stream_handle(stream: torch.cuda.Stream | None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


class SplitWeights:
    """Expert weights of one layer split over a local and a remote pool."""

    def __init__(self, H: int, I: int, w_dtype: str, pool_slot: np.ndarray, local: torch.Tensor,
                 n_local: int, remote: torch.Tensor, n_remote: int, shared: torch.Tensor | None):
        self.H, self.I, self.w_dtype = H, I, w_dtype
        self.layout = L.expert_layout(H, I, _DT[w_dtype])
        self.stride = int(self.layout.bytes)
        self.pool_slot = np.ascontiguousarray(pool_slot, dtype=np.int32)
        self.local, self.n_local = local, n_local
        self.remote, self.n_remote = remote, n_remote
        self.shared = shared

    @staticmethod
    def image_bytes(H: int, I: int, w_dtype: str) -> int:
        return int(L.expert_layout(H, I, _DT[w_dtype]).bytes)

    @classmethod
    def allocate(cls, H, I, w_dtype, pool_of, slot_of, has_shared, device) -> "SplitWeights":
        """Empty pools sized for the given assignment of experts to (pool, slot)."""
        pool_of = np.asarray(pool_of)
        slot_of = np.asarray(slot_of)
        n_local = int((pool_of == POOL_LOCAL).sum())
        n_remote = int((pool_of == POOL_REMOTE).sum())
        b = cls.image_bytes(H, I, w_dtype)
        local = torch.empty(max(n_local, 1) * b, dtype=torch.uint8, device=device)
        remote = torch.empty(max(n_remote, 1) * b, dtype=torch.uint8, device=device)
        shared = torch.empty(b, dtype=torch.uint8, device=device) if has_shared else None
        ps = (pool_of.astype(np.int64) << 31 | slot_of.astype(np.int64)).astype(np.uint32).view(np.int32)
        return cls(H, I, w_dtype, ps, local, n_local, remote, n_remote, shared)

    def slot_base(self, pool: int, slot: int) -> int:
        t = self.local if pool == POOL_LOCAL else self.remote
        return t.data_ptr() + slot * self.stride

    def expert_base(self, e: int) -> int:
        """Device address of expert e's image (e == E: the shared expert)."""
        if e == len(self.pool_slot):
            return self.shared.data_ptr()
        v = int(np.uint32(self.pool_slot[e]))
        return self.slot_base(v >> 31, v & 0x7FFFFFFF)

    def table(self, remote: torch.Tensor | None = None) -> L.moe_expert_table:
        """C table; `remote` overrides the remote pool (an alternate buffer)."""
        rem = self.remote if remote is None else remote
        self._ps_c = self.pool_slot.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        return L.moe_expert_table(self.local.data_ptr(), self.n_local, self.stride,
                                  rem.data_ptr(), self.n_remote, self.stride,
                                  _ptr(self.shared), self._ps_c)


@dataclass
class ReadyGate:
    """Per-chunk readiness flags of a remote buffer (moe_ready_gate): flag c
    covers remote slots [c*slots_per_flag, (c+1)*slots_per_flag) and reaches
    `epoch` once the copy stream has landed that chunk."""
    flags: torch.Tensor          # int32 [n_flags] on the device (read as uint32)
    epoch: int
    slots_per_flag: int
    timeout_ns: int = 0          # 0: the library default (2 s)

    def c_struct(self) -> L.moe_ready_gate:
        return L.moe_ready_gate(self.flags.data_ptr(), self.epoch & 0xFFFFFFFF,
                                self.slots_per_flag, self.flags.numel(), self.timeout_ns)


@dataclass
class Progress:
    """Progress reports of a grouped-GEMM call (moe_progress): words[0] is
    the progress word, words[1:3] the call's tile counters."""
    words: torch.Tensor          # int32 [3] on the device (read as uint32)
    base: int
    steps: int

    def c_struct(self) -> L.moe_progress:
        w = self.words.data_ptr()
        return L.moe_progress(w, w + 4, self.base & 0xFFFFFFFF, self.steps)


class MoELayer:
    """One MoE layer with preallocated device buffers.

    By default moe_permute gathers x_perm (bf16, from bf16 or fp32 x, or e4m3
    with scales) and the grouped GEMM reads it.  With gather=True (bf16 x and
    activations only) the grouped GEMM reads its token rows from x through
    perm_src instead (moe_grouped_ffn_x) and no x_perm is written; it gives
    the same bits, and is slower at large batches, where its four-row TMA
    gathers cannot feed the tensor cores."""

    def __init__(self, shape: LayerShape, w_gate: torch.Tensor, bias: torch.Tensor | None,
                 weights: SplitWeights, device: torch.device | str = "cuda",
                 gather: bool | None = None):
        s = shape
        self.shape, self.w_gate, self.bias, self.weights = s, w_gate, bias, weights
        dev = torch.device(device)
        can_gather = s.x_dtype == "bf16" and s.act_dtype == "bf16"
        self.gather = bool(gather)
        assert can_gather or not self.gather, "gathered token tiles need bf16 x and activations"
        self._cfg = s.route_cfg()
        self._desc = s.ffn_desc()
        i32 = torch.int32
        self.route_ws = torch.empty(max(L.moe_route_workspace_size(ctypes.byref(self._cfg)), 16),
                                    dtype=torch.uint8, device=dev)
        self.perm_ws = torch.empty(max(L.moe_permute_workspace_size(s.T, s.k, s.E), 16),
                                   dtype=torch.uint8, device=dev)
        self.topk_idx = torch.empty(max(s.T, 1), s.k, dtype=i32, device=dev)
        self.topk_w = torch.empty(max(s.T, 1), s.k, dtype=torch.float32, device=dev)
        self.offsets = torch.empty(s.E + 1, dtype=i32, device=dev)
        self.perm_src = torch.empty(max(s.A, 1), dtype=i32, device=dev)
        self.inv_pos = torch.empty(max(s.T, 1), s.k, dtype=i32, device=dev)
        rows = max(s.rows, 1)
        a8 = s.act_dtype == "e4m3"
        adt = torch.uint8 if a8 else torch.bfloat16
        # with gather x_perm is never written: a one-row placeholder
        self.x_perm = torch.empty(1 if self.gather else rows, s.H, dtype=adt, device=dev)
        self.x_scales = torch.empty(s.H // 128, rows, dtype=torch.float32, device=dev) if a8 else None
        self.h = torch.empty(rows, s.I, dtype=adt, device=dev)
        self.ffn_ws = torch.empty(max(L.moe_grouped_ffn_workspace_size(ctypes.byref(self._desc)), 16),
                                  dtype=torch.uint8, device=dev)
        self.y_perm = torch.empty(rows, s.H, dtype=torch.bfloat16, device=dev)
        ydt = torch.float32 if s.y_dtype == "f32" else torch.bfloat16
        self.y = torch.empty(max(s.T, 1), s.H, dtype=ydt, device=dev)

    # -- the four steps, each one C-ABI call ---------------------------------
    def route(self, x: torch.Tensor, stream: int) -> None:
        L.check(L.moe_route(ctypes.byref(self._cfg), x.data_ptr(), _DT[self.shape.x_dtype],
                            self.w_gate.data_ptr(), _ptr(self.bias), self.topk_idx.data_ptr(),
                            self.topk_w.data_ptr(), self.route_ws.data_ptr(),
                            self.route_ws.numel(), stream))

    def permute(self, x: torch.Tensor, stream: int) -> None:
        s = self.shape
        L.check(L.moe_permute(s.T, s.k, s.E, s.H, self.topk_idx.data_ptr(), x.data_ptr(),
                              _DT[s.x_dtype], _DT[s.act_dtype], 1 if s.has_shared else 0,
                              self.offsets.data_ptr(), self.perm_src.data_ptr(),
                              self.inv_pos.data_ptr(),
                              None if self.gather else self.x_perm.data_ptr(),
                              _ptr(self.x_scales),
                              self.perm_ws.data_ptr(), self.perm_ws.numel(), stream))

    def grouped_ffn(self, stream: int, remote: torch.Tensor | None = None,
                    gate: "ReadyGate | None" = None, x: torch.Tensor | None = None,
                    progress: Progress | None = None) -> None:
        """The grouped GEMMs; with a gate, remote experts are read only once
        their chunk of a fetch still in flight has landed.  x: the layer
        input, needed when the token rows are gathered from it.  progress:
        reports that pace a fetch (moe_grouped_ffn_paced)."""
        tbl = self.weights.table(remote)
        g = gate.c_struct() if gate is not None else None
        gp = ctypes.byref(g) if g is not None else None
        if progress is not None:
            pr = progress.c_struct()
            xp = x.data_ptr() if self.gather else None
            ps = self.perm_src.data_ptr() if self.gather else None
            L.check(L.moe_grouped_ffn_paced(ctypes.byref(self._desc), ctypes.byref(tbl), gp,
                                            ctypes.byref(pr), _ptr(self.x_perm), _ptr(self.x_scales),
                                            xp, ps, self.offsets.data_ptr(), self.h.data_ptr(),
                                            self.y_perm.data_ptr(), self.ffn_ws.data_ptr(),
                                            self.ffn_ws.numel(), stream))
            return
        if self.gather:
            assert x is not None, "the gathered grouped GEMM reads the layer input x"
            L.check(L.moe_grouped_ffn_x(ctypes.byref(self._desc), ctypes.byref(tbl), gp,
                                        x.data_ptr(), self.perm_src.data_ptr(),
                                        self.offsets.data_ptr(), self.h.data_ptr(),
                                        self.y_perm.data_ptr(), self.ffn_ws.data_ptr(),
                                        self.ffn_ws.numel(), stream))
            return
        L.check(L.moe_grouped_ffn_gated(ctypes.byref(self._desc), ctypes.byref(tbl), gp,
                                        self.x_perm.data_ptr(), _ptr(self.x_scales),
                                        self.offsets.data_ptr(), self.h.data_ptr(),
                                        self.y_perm.data_ptr(), self.ffn_ws.data_ptr(),
                                        self.ffn_ws.numel(), stream))

    def combine(self, stream: int) -> None:
        s = self.shape
        L.check(L.moe_combine(s.T, s.k, s.H, self.y_perm.data_ptr(), self.inv_pos.data_ptr(),
                              self.topk_w.data_ptr(), 1 if s.has_shared else 0, self.y.data_ptr(),
                              _DT[s.y_dtype], stream))

    def forward(self, x: torch.Tensor, stream: torch.cuda.Stream | None = None,
                remote: torch.Tensor | None = None) -> torch.Tensor:
        """Enqueues the whole block on `stream`; returns the output buffer."""
        h = _stream_handle(stream)
        self.route(x, h)
        self.permute(x, h)
        self.grouped_ffn(h, remote, x=x)
        self.combine(h)
        return self.y


def remote_slots(pool_slot: np.ndarray, touched: np.ndarray) -> set[int]:
    """Remote-pool slots of the experts marked in `touched` [E] (the
    moe_experts_touched bytes), from the (pool << 31) | slot table."""
    ps = np.asarray(pool_slot, dtype=np.int32).view(np.uint32)
    sel = (np.asarray(touched[:len(ps)]) != 0) & ((ps >> 31) == 1)
    return set(int(v) for v in (ps[sel] & 0x7FFFFFFF))


class PrefetchPipeline:
    """Consecutive MoE layers whose remote experts are fetched ahead into two
    alternate buffers by moe_prefetch_layer on a copy-engine stream.

    Layer executions are numbered g = 0, 1, 2, ... across passes; execution g
    computes from bufs[g % 2].  As soon as its grouped GEMMs are enqueued,
    the compute stream records free[g % 2] and the copy stream, after waiting
    for it, fetches the layer of execution g + 2 into the same buffer and
    records ready[g % 2], which execution g + 2 waits for before its grouped
    GEMM.  With wrap=True the fetches issued by the last layers of a pass are
    those of the next pass's first layers, as in a steady stream of forward
    passes.

    With split=True each fetch is issued in two halves: the first after
    execution g's grouped GEMMs, the second after execution g + 1's, and
    ready is recorded after the second.  Each half then starts in the window
    of routing, permutation and combine between two grouped GEMMs instead of
    the whole fetch running beside the next grouped GEMM.

    With gate_slots > 0 the compute stream does not wait for ready: the fetch
    writes a readiness flag per chunk of gate_slots remote slots
    (moe_prefetch_layer_flagged, epoch g + 1 for execution g) and the grouped
    GEMM of execution g starts at once, running local experts first and
    waiting on the device, per chunk, for the remote experts it reaches
    (moe_grouped_ffn_gated).

    window_block(l, x, stream), if given, is enqueued before layer l's MoE
    block: compute that the fetch also hides behind (the explainer's
    attention block between two MoE blocks).

    With pace_steps > 0 (and gate_slots > 0) the fetch is paced by compute:
    right after enqueuing its grouped GEMM call, which reports its progress
    in pace_steps steps (moe_grouped_ffn_paced, base g' (pace_steps + 1) for
    the g'-th paced execution), execution g enqueues the fetch of execution
    g + 1; its first pace_lead chunks go at once, the others wait on the copy
    stream for an even share of those reports (moe_prefetch_layer_paced).
    The copy then runs spread over the grouped GEMMs instead of as one burst
    beside them, and never waits for work enqueued after it.

    With select=True (per-slot flags: gate_slots = 1) the fetch is selective:
    execution g routes the next layer's tokens ahead of time with that
    layer's router on its own input x (a look-ahead prediction), and right
    after its grouped GEMM enqueues fetches only the remote slots so
    predicted (moe_prefetch_slots); when execution g + 1 has routed for
    real, the slots the prediction missed are fetched before its grouped
    GEMM, which waits per slot.  Each execution costs one host
    synchronisation (the touched-expert bytes of its routing and of the
    prediction), and fetches (predicted ∪ missed) slots instead of all.
    select_stats records, per execution, the touched, predicted and missed
    slot counts.
    """

    def __init__(self, layers: list[MoELayer], peer_stores: list[torch.Tensor],
                 remote_bytes: int, device: torch.device | str = "cuda", chunk_bytes: int = 0,
                 split: bool = True, gate_slots: int = 0, window_block=None,
                 gate_timeout_ns: int = 0, pace_steps: int = 0, pace_lead: int = 0,
                 select: bool = False):
        self.layers, self.peer_stores = layers, peer_stores
        self.remote_bytes, self.chunk_bytes = remote_bytes, chunk_bytes
        self.split, self.pending = split, None
        self.gate_slots, self.window_block, self.gate_timeout_ns = gate_slots, window_block, gate_timeout_ns
        dev = self.device = torch.device(device)
        self.bufs = [torch.empty(max(remote_bytes, 1), dtype=torch.uint8, device=dev)
                     for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.ready = [torch.cuda.Event() for _ in range(2)]
        self.free = [torch.cuda.Event() for _ in range(2)]
        for ev in self.ready + self.free:   # torch creates CUDA events on first record
            ev.record(self.copy_stream)
        self.g = 0
        self.stride = layers[0].weights.stride
        self.flags = None
        self.pace_steps, self.pace_lead, self.g_pace0 = 0, 0, 0
        self.progress_words = torch.zeros(3, dtype=torch.int32, device=dev)
        self.select, self._pred = False, None
        self.fetched = [set(), set()]
        self.select_stats: list[dict] = []
        self.configure(gate_slots=gate_slots, pace_steps=pace_steps, pace_lead=pace_lead,
                       select=select)

    def configure(self, split: bool | None = None, gate_slots: int | None = None,
                  window_block=False, pace_steps: int | None = None,
                  pace_lead: int | None = None, select: bool | None = None) -> None:
        """Switches the schedule between runs (after a synchronisation: no
        fetch may be in flight).  window_block=False leaves it as it is."""
        if split is not None:
            self.split = split
        if select is not None:
            self.select = select
            self.fetched = [set(), set()]
            if select and self._pred is None:
                l0, dev = self.layers[0], self.device
                T, k, E = l0.shape.T, l0.shape.k, l0.shape.E
                self._pred = {
                    "idx": torch.empty(max(T, 1), k, dtype=torch.int32, device=dev),
                    "w": torch.empty(max(T, 1), k, dtype=torch.float32, device=dev),
                    "ws": torch.empty_like(l0.route_ws),
                    "touched": torch.zeros(2, E, dtype=torch.uint8, device=dev),
                    "host": torch.zeros(2, E, dtype=torch.uint8).pin_memory(),
                    "ev": torch.cuda.Event(),
                }
        if pace_lead is not None:
            self.pace_lead = pace_lead
        if pace_steps is not None:
            self.pace_steps = pace_steps
            self.g_pace0 = self.g
            self.progress_words.zero_()   # the base of execution g_pace0
        if window_block is not False:
            self.window_block = window_block
        if gate_slots is not None:
            self.gate_slots = gate_slots
            if gate_slots > 0:
                assert self.remote_bytes % self.stride == 0
                n_slots = self.remote_bytes // self.stride
                self.n_flags = max(1, -(-n_slots // gate_slots))
                dev = self.bufs[0].device
                # flags only grow: fresh zeros are below every epoch still to come
                self.flags = [torch.zeros(self.n_flags, dtype=torch.int32, device=dev)
                              for _ in range(2)]
        if self.pace_steps > 0:
            assert self.gate_slots > 0 and self.pace_steps >= 2, \
                "a paced fetch needs readiness flags and at least 2 steps"
        if self.select:
            assert self.gate_slots == 1 and self.pace_steps == 0, \
                "a selective fetch needs per-slot flags (gate_slots=1) and no pacing"
        self.pending = None

    def progress(self, execution: int) -> Progress:
        """The progress reports of a paced execution's grouped GEMM call."""
        return Progress(self.progress_words, (execution - self.g_pace0) * (self.pace_steps + 1),
                        self.pace_steps)

    # -- copies -------------------------------------------------------------
    def _copy(self, layer: int, buf: int, lo: int, hi: int, wait_free, ready, epoch: int,
              pace: Progress | None = None) -> None:
        src = self.peer_stores[layer].data_ptr() + lo
        dst = self.bufs[buf].data_ptr() + lo
        wf = wait_free.cuda_event if wait_free is not None else None
        rd = ready.cuda_event if ready is not None else None
        if pace is not None:
            chunk = self.gate_slots * self.stride
            pr = pace.c_struct()
            L.check(L.moe_prefetch_layer_paced(src, dst, hi - lo, chunk,
                                               self.copy_stream.cuda_stream, wf,
                                               self.flags[buf].data_ptr() + 4 * (lo // chunk),
                                               epoch & 0xFFFFFFFF, ctypes.byref(pr),
                                               self.pace_lead, rd))
        elif self.gate_slots > 0:
            chunk = self.gate_slots * self.stride
            assert lo % chunk == 0
            L.check(L.moe_prefetch_layer_flagged(src, dst, hi - lo, chunk,
                                                 self.copy_stream.cuda_stream, wf,
                                                 self.flags[buf].data_ptr() + 4 * (lo // chunk),
                                                 epoch & 0xFFFFFFFF, rd))
        else:
            L.check(L.moe_prefetch_layer(src, dst, hi - lo, self.chunk_bytes,
                                         self.copy_stream.cuda_stream, wf, rd))

    def _fetch_slots(self, layer: int, buf: int, slots: list[int], wait_free, epoch: int) -> None:
        """Selective fetch of the given remote slots of `layer` into bufs[buf]."""
        n_slots = self.remote_bytes // self.stride
        arr = (ctypes.c_int32 * max(len(slots), 1))(*slots)
        wf = wait_free.cuda_event if wait_free is not None else None
        L.check(L.moe_prefetch_slots(self.peer_stores[layer].data_ptr(), self.bufs[buf].data_ptr(),
                                     self.stride, n_slots, arr, len(slots),
                                     self.copy_stream.cuda_stream, wf, self.flags[buf].data_ptr(),
                                     epoch & 0xFFFFFFFF, None))

    def _cut(self) -> int:
        if self.gate_slots > 0:
            chunk = self.gate_slots * self.stride
            return (self.n_flags // 2) * chunk
        return (self.remote_bytes // 2) // 256 * 256

    def prefetch(self, layer: int, buf: int, wait_free: torch.cuda.Event | None,
                 execution: int | None = None) -> None:
        """The whole fetch of `layer` into bufs[buf] for the given execution."""
        assert self.ready[buf].cuda_event != 0 and (wait_free is None or wait_free.cuda_event != 0)
        ex = self.g if execution is None else execution
        self._copy(layer, buf, 0, self.remote_bytes, wait_free, self.ready[buf], ex + 1)

    def fetch_half(self, layer: int, buf: int, half: int, wait_free: torch.cuda.Event,
                   execution: int | None = None) -> None:
        """One half of a fetch; the second half records ready[buf]."""
        cut = self._cut()
        lo, hi = (0, cut) if half == 0 else (cut, self.remote_bytes)
        assert wait_free.cuda_event != 0 and self.ready[buf].cuda_event != 0
        ex = self.g if execution is None else execution
        self._copy(layer, buf, lo, hi, wait_free, self.ready[buf] if half == 1 else None, ex + 1)

    def prime(self) -> None:
        """Enqueues the fetches of the next two executions (before a run);
        paced, of the next one (each execution enqueues its successor's).
        The copy stream first waits for the current stream: the flags and
        progress words that configure() zero-filled there, and the peer
        stores, must be in place before a fetch writes or reads them."""
        n = len(self.layers)
        self.copy_stream.wait_stream(torch.cuda.current_stream(self.device))
        self.pending = None
        if self.select:   # nothing predicted yet: the first execution fetches what it misses
            self.fetched = [set(), set()]
            return
        for i in range(1 if self.pace_steps > 0 else 2):
            self.prefetch((self.g + i) % n, (self.g + i) % 2, None, self.g + i)

    # -- compute ------------------------------------------------------------
    def run_layer(self, l: int, x: torch.Tensor, stream: torch.cuda.Stream,
                  prefetch: bool = True, wrap: bool = True, ffn_events=None) -> torch.Tensor:
        """One layer execution; ffn_events = (start, end) events around its
        grouped GEMMs, if given."""
        n = len(self.layers)
        layer, h, b, g = self.layers[l], stream.cuda_stream, self.g % 2, self.g
        if self.window_block is not None:
            self.window_block(l, x, stream)
        layer.route(x, h)
        layer.permute(x, h)
        if prefetch and self.select:
            self._run_selective(l, x, stream, ffn_events, wrap)
            layer.combine(h)
            self.g += 1
            return layer.y
        gate = None
        if prefetch and self.gate_slots > 0:
            gate = ReadyGate(self.flags[b], g + 1, self.gate_slots, self.gate_timeout_ns)
        elif prefetch:
            stream.wait_event(self.ready[b])
        progress = self.progress(g) if prefetch and self.pace_steps > 0 else None
        if ffn_events is not None:
            ffn_events[0].record(stream)
        layer.grouped_ffn(h, self.bufs[b], gate, x=x, progress=progress)
        if ffn_events is not None:
            ffn_events[1].record(stream)
        if progress is not None:
            self.free[b].record(stream)
            # execution g + 1's fetch, paced by the call just enqueued: the
            # call goes first, so that the copy stream never waits for work
            # queued behind it (streams may share a hardware queue)
            if l + 1 < n or wrap:
                nb = (g + 1) % 2
                self._copy((l + 1) % n, nb, 0, self.remote_bytes, self.free[nb], self.ready[nb],
                           g + 2, pace=progress)
        elif prefetch and self.split:
            self.free[b].record(stream)
            if self.pending is not None:  # second half of execution g + 1's fetch
                self.fetch_half(*self.pending, 1, self.free[b], g + 1)
                self.pending = None
            if l + 2 < n or wrap:        # first half of execution g + 2's
                self.fetch_half((l + 2) % n, b, 0, self.free[b], g + 2)
                self.pending = ((l + 2) % n, b)
        elif prefetch and (l + 2 < n or wrap):
            self.free[b].record(stream)
            self.prefetch((l + 2) % n, b, self.free[b], g + 2)
        layer.combine(h)
        self.g += 1
        return layer.y

    def _run_selective(self, l: int, x: torch.Tensor, stream: torch.cuda.Stream, ffn_events,
                       wrap: bool) -> None:
        """Execution g of the selective schedule, after its routing and
        permutation: the look-ahead prediction of the next layer, one host
        synchronisation, the missed slots, the grouped GEMM, then the
        predicted fetch of execution g + 1."""
        n = len(self.layers)
        layer, h, b, g = self.layers[l], stream.cuda_stream, self.g % 2, self.g
        s, pr = layer.shape, self._pred
        L.check(L.moe_experts_touched(layer.topk_idx.data_ptr(), s.T * s.k, s.E,
                                      pr["touched"][0].data_ptr(), h))
        nxt = (l + 1) % n
        ahead = l + 1 < n or wrap
        if ahead:   # the next layer's router on this layer's input
            nl = self.layers[nxt]
            L.check(L.moe_route(ctypes.byref(nl._cfg), x.data_ptr(), _DT[nl.shape.x_dtype],
                                nl.w_gate.data_ptr(), _ptr(nl.bias), pr["idx"].data_ptr(),
                                pr["w"].data_ptr(), pr["ws"].data_ptr(), pr["ws"].numel(), h))
            L.check(L.moe_experts_touched(pr["idx"].data_ptr(), s.T * s.k, s.E,
                                          pr["touched"][1].data_ptr(), h))
        with torch.cuda.stream(stream):
            pr["host"].copy_(pr["touched"], non_blocking=True)
        pr["ev"].record(stream)
        pr["ev"].synchronize()
        touched = remote_slots(layer.weights.pool_slot, pr["host"][0].numpy())
        missed = sorted(touched - self.fetched[b])
        if missed:   # after the predicted fetch of this buffer on the copy stream
            self._fetch_slots(l, b, missed, self.free[b], g + 1)
            self.fetched[b] |= set(missed)
        stats = {"touched": len(touched), "missed": len(missed)}
        gate = ReadyGate(self.flags[b], g + 1, 1, self.gate_timeout_ns)
        if ffn_events is not None:
            ffn_events[0].record(stream)
        layer.grouped_ffn(h, self.bufs[b], gate, x=x)
        if ffn_events is not None:
            ffn_events[1].record(stream)
        self.free[b].record(stream)
        if ahead:
            nb = (g + 1) % 2
            pred = sorted(remote_slots(self.layers[nxt].weights.pool_slot, pr["host"][1].numpy()))
            self._fetch_slots(nxt, nb, pred, self.free[nb], g + 2)
            self.fetched[nb] = set(pred)
            stats["predicted_next"] = len(pred)
        self.select_stats.append(stats)

    def run(self, xs: list[torch.Tensor], stream: torch.cuda.Stream | None = None,
            prefetch: bool = True, wrap: bool = True) -> list[torch.Tensor]:
        """Runs all layers once.  With prefetch=False nothing is copied and
        the buffers are used as they are; prime() must have run once before
        the first pass with prefetch."""
        stream = stream if stream is not None else torch.cuda.current_stream()
        return [self.run_layer(l, xs[l], stream, prefetch, wrap) for l in range(len(self.layers))]


class DenseBlock:
    """A dense SwiGLU block on all of a layer's tokens, run through the same
    grouped GEMM (one expert that every token uses): compute between two MoE
    blocks for the prefetch to hide behind.  It stands in for the attention
    block of the explainer's prefetch caption, which this library does not
    implement; inter = 12288 at H = 7168 gives 6*H*inter = 528 MFLOP per
    token, about DeepSeek-R1's attention projections plus causal attention
    over 4K-token sequences.  Its output is not used."""

    def __init__(self, T: int, H: int, inter: int, device, seed: int = 0):
        self.T, self.H, self.inter = T, H, inter
        dev = torch.device(device)
        self.weights = SplitWeights.allocate(H, inter, "bf16", np.zeros(1, dtype=np.int64),
                                             np.zeros(1, dtype=np.int64), False, dev)
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        w = self.weights.local.view(torch.bfloat16)
        w.copy_((torch.randn(w.numel(), device=dev, generator=g) * 0.02).to(torch.bfloat16))
        self.shape = LayerShape(T=T, H=H, I=inter, E=1, k=1, has_shared=False)
        self._desc = self.shape.ffn_desc()
        self.offsets = torch.tensor([0, T], dtype=torch.int32, device=dev)
        self.h = torch.empty(max(T, 1), inter, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(max(T, 1), H, dtype=torch.bfloat16, device=dev)

    def __call__(self, l: int, x: torch.Tensor, stream: torch.cuda.Stream) -> None:
        assert x.dtype == torch.bfloat16 and x.shape[0] == self.T
        tbl = self.weights.table()
        L.check(L.moe_grouped_ffn(ctypes.byref(self._desc), ctypes.byref(tbl), x.data_ptr(), None,
                                  self.offsets.data_ptr(), self.h.data_ptr(), self.y.data_ptr(),
                                  None, 0, stream.cuda_stream))


class PeerPools:
    """The expert pools of a DWDP group as this rank addresses them, and the
    time-division sliced fetch of the ones it lacks (moe_prefetch_peers).

    ``pools[q]`` is the device address of rank q's pool (``bytes_per_rank``
    bytes): this rank's own tensor, a peer's through peer access, or a pool
    mapped with ``import_pool``.  The remote buffer receives the other ranks'
    pools in rank order, skipping this rank."""

    def __init__(self, group_size: int, rank: int, pools: list[int], bytes_per_rank: int,
                 slices: int = 8):
        assert len(pools) == group_size
        self.G, self.rank, self.bytes_per_rank, self.slices = group_size, rank, bytes_per_rank, slices
        self._pools = (ctypes.c_void_p * group_size)(*[p or None for p in pools])

    def fetch(self, dst: torch.Tensor, copy_stream: torch.cuda.Stream,
              wait_free: torch.cuda.Event | None = None,
              ready: torch.cuda.Event | None = None) -> None:
        assert dst.numel() * dst.element_size() >= (self.G - 1) * self.bytes_per_rank
        L.check(L.moe_prefetch_peers(self.G, self.rank, self._pools, self.bytes_per_rank,
                                     self.slices, dst.data_ptr(), copy_stream.cuda_stream,
                                     wait_free.cuda_event if wait_free is not None else None,
                                     ready.cuda_event if ready is not None else None))


def export_pool(t: torch.Tensor) -> bytes:
    """IPC handle (bytes) of the pool held by tensor t, for another process."""
    h = L.moe_pool_handle()
    L.check(L.moe_pool_export(t.data_ptr(), ctypes.byref(h)))
    return ctypes.string_at(ctypes.addressof(h), ctypes.sizeof(h))


def import_pool(handle: bytes) -> tuple[int, int]:
    """Maps a pool exported by another process: (pool address, mapping); pass
    the mapping to close_pool when no copy reads the pool any more."""
    h = L.moe_pool_handle.from_buffer_copy(handle)
    base, mapping = ctypes.c_void_p(), ctypes.c_void_p()
    L.check(L.moe_pool_import(ctypes.byref(h), ctypes.byref(base), ctypes.byref(mapping)))
    return base.value, mapping.value


def close_pool(mapping: int) -> None:
    L.check(L.moe_pool_close(mapping))
