"""ctypes binding of libswb_moe.so (include/moe.h), argument marshalling only.

Every function has the C entry point's name and arguments: device pointers
and streams are plain integers (``tensor.data_ptr()``,
``torch.cuda.Stream.cuda_stream``).  Each returns the moe_status code;
``check`` turns a non-zero code into ``MoEError`` with the library's message.
There is no fallback: if the shared library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswb_moe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK = 4, 5, 6
MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1

i32, i64, f32, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class moe_route_cfg(ctypes.Structure):
    _fields_ = [("T", i32), ("H", i32), ("E", i32), ("k", i32), ("score", i32),
                ("n_group", i32), ("topk_group", i32), ("routed_scale", f32),
                ("renormalize", i32)]


class moe_expert_layout(ctypes.Structure):
    _fields_ = [("gu_offset", i64), ("down_offset", i64), ("gu_scale_offset", i64),
                ("down_scale_offset", i64), ("bytes", i64)]


class moe_expert_table(ctypes.Structure):
    _fields_ = [("local_base", vp), ("local_count", i32), ("local_stride", i64),
                ("remote_base", vp), ("remote_count", i32), ("remote_stride", i64),
                ("shared", vp), ("pool_slot", ctypes.POINTER(i32))]


class moe_ffn_desc(ctypes.Structure):
    _fields_ = [("T", i32), ("H", i32), ("I", i32), ("E", i32), ("k", i32), ("w_dtype", i32),
                ("act_dtype", i32), ("has_shared", i32)]


class moe_peer_copy(ctypes.Structure):
    _fields_ = [("step", i32), ("src_rank", i32), ("src_offset", i64), ("dst_offset", i64),
                ("bytes", i64)]


class moe_pool_handle(ctypes.Structure):
    _fields_ = [("ipc", ctypes.c_char * 64), ("offset", i64)]


class moe_ready_gate(ctypes.Structure):
    _fields_ = [("flags", vp), ("epoch", ctypes.c_uint32), ("slots_per_flag", i32),
                ("n_flags", i32), ("timeout_ns", i64)]


class moe_progress(ctypes.Structure):
    _fields_ = [("word", vp), ("tiles", vp), ("base", ctypes.c_uint32), ("steps", i32)]


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: run python split_weight_b200/build.py "
                      "(the CUDA library is required; there is no CPU fallback)")
_lib = ctypes.CDLL(LIB_PATH)

_SIGS = {
    "moe_status_string": ([i32], ctypes.c_char_p),
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_abi_version": ([], i32),
    "moe_kernel_launches": ([], ctypes.c_uint64),
    "moe_route_workspace_size": ([ctypes.POINTER(moe_route_cfg)], sz),
    "moe_route": ([ctypes.POINTER(moe_route_cfg), vp, i32, vp, vp, vp, vp, vp, sz, vp], i32),
    "moe_permute_workspace_size": ([i32, i32, i32], sz),
    "moe_permute": ([i32, i32, i32, i32, vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp],
                    i32),
    "moe_permute_noalloc": ([i32, i32, i32, i32, vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp],
                           i32),
    "moe_expert_layout_get": ([i32, i32, i32, ctypes.POINTER(moe_expert_layout)], i32),
    "moe_grouped_ffn_workspace_size": ([ctypes.POINTER(moe_ffn_desc)], sz),
    "moe_grouped_ffn": ([ctypes.POINTER(moe_ffn_desc), ctypes.POINTER(moe_expert_table), vp, vp,
                         vp, vp, vp, vp, sz, vp], i32),
    "moe_grouped_ffn_gated": ([ctypes.POINTER(moe_ffn_desc), ctypes.POINTER(moe_expert_table),
                               ctypes.POINTER(moe_ready_gate), vp, vp, vp, vp, vp, vp, sz, vp], i32),
    "moe_prefetch_layer_flagged": ([vp, vp, sz, sz, vp, vp, vp, ctypes.c_uint32, vp], i32),
    "moe_grouped_ffn_x": ([ctypes.POINTER(moe_ffn_desc), ctypes.POINTER(moe_expert_table),
                           ctypes.POINTER(moe_ready_gate), vp, vp, vp, vp, vp, vp, sz, vp], i32),
    "moe_grouped_ffn_paced": ([ctypes.POINTER(moe_ffn_desc), ctypes.POINTER(moe_expert_table),
                               ctypes.POINTER(moe_ready_gate), ctypes.POINTER(moe_progress), vp,
                               vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
    "moe_prefetch_layer_paced": ([vp, vp, sz, sz, vp, vp, vp, ctypes.c_uint32,
                                  ctypes.POINTER(moe_progress), i32, vp], i32),
    "moe_pace_threshold": ([i64, i64, i32, ctypes.c_uint32, i32], ctypes.c_uint32),
    "moe_prefetch_slots": ([vp, vp, sz, i32, ctypes.POINTER(i32), i32, vp, vp, vp,
                            ctypes.c_uint32, vp], i32),
    "moe_experts_touched": ([vp, i64, i32, vp, vp], i32),
    "moe_combine": ([i32, i32, i32, vp, vp, vp, i32, vp, i32, vp], i32),
    "moe_prefetch_layer": ([vp, vp, sz, sz, vp, vp, vp], i32),
    "moe_peer_fetch_plan": ([i32, i32, i64, i32, ctypes.POINTER(moe_peer_copy), i32,
                             ctypes.POINTER(i32)], i32),
    "moe_prefetch_peers": ([i32, i32, ctypes.POINTER(vp), i64, i32, vp, vp, vp, vp], i32),
    "moe_enable_peer_access": ([i32], i32),
    "moe_pool_export": ([vp, ctypes.POINTER(moe_pool_handle)], i32),
    "moe_pool_import": ([ctypes.POINTER(moe_pool_handle), ctypes.POINTER(vp), ctypes.POINTER(vp)],
                        i32),
    "moe_pool_close": ([vp], i32),
    "moe_wait_ready": ([vp, i32], i32),
    "moe_check_device": ([], i32),
    "moe_debug_fail_next_cuda_calls": ([i32], None),
    "moe_debug_gated_regs_per_sm": ([i64], None),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def header_functions() -> list[str]:
    """Names of the functions include/moe.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[^(]*?\b(moe_\w+)\s*\(", text, re.M)))


def status_string(s: int) -> str:
    return _lib.moe_status_string(s).decode()


def moe_last_error() -> str:
    return _lib.moe_last_error().decode()


def check(status: int) -> None:
    if status != MOE_OK:
        raise MoEError(status, moe_last_error())


moe_abi_version = _lib.moe_abi_version
moe_kernel_launches = _lib.moe_kernel_launches
moe_route_workspace_size = _lib.moe_route_workspace_size
moe_route = _lib.moe_route
moe_permute_workspace_size = _lib.moe_permute_workspace_size
moe_permute = _lib.moe_permute
moe_permute_noalloc = _lib.moe_permute_noalloc
moe_expert_layout_get = _lib.moe_expert_layout_get
moe_grouped_ffn_workspace_size = _lib.moe_grouped_ffn_workspace_size
moe_grouped_ffn = _lib.moe_grouped_ffn
moe_grouped_ffn_gated = _lib.moe_grouped_ffn_gated
moe_grouped_ffn_x = _lib.moe_grouped_ffn_x
moe_prefetch_layer_flagged = _lib.moe_prefetch_layer_flagged
moe_grouped_ffn_paced = _lib.moe_grouped_ffn_paced
moe_prefetch_layer_paced = _lib.moe_prefetch_layer_paced
moe_pace_threshold = _lib.moe_pace_threshold
moe_prefetch_slots = _lib.moe_prefetch_slots
moe_experts_touched = _lib.moe_experts_touched
moe_combine = _lib.moe_combine
moe_prefetch_layer = _lib.moe_prefetch_layer
moe_peer_fetch_plan = _lib.moe_peer_fetch_plan
moe_prefetch_peers = _lib.moe_prefetch_peers
moe_enable_peer_access = _lib.moe_enable_peer_access
moe_pool_export = _lib.moe_pool_export
moe_pool_import = _lib.moe_pool_import
moe_pool_close = _lib.moe_pool_close
moe_wait_ready = _lib.moe_wait_ready
moe_check_device = _lib.moe_check_device
moe_debug_fail_next_cuda_calls = _lib.moe_debug_fail_next_cuda_calls
moe_debug_gated_regs_per_sm = _lib.moe_debug_gated_regs_per_sm


def expert_layout(H: int, I: int, w_dtype: int) -> moe_expert_layout:
    out = moe_expert_layout()
    check(moe_expert_layout_get(H, I, w_dtype, ctypes.byref(out)))
    return out


def peer_fetch_plan(group_size: int, rank: int, bytes_per_rank: int, slices: int):
    """The rank's time-division fetch schedule as a list of moe_peer_copy."""
    n = i32(0)
    check(moe_peer_fetch_plan(group_size, rank, bytes_per_rank, slices, None, 0, ctypes.byref(n)))
    arr = (moe_peer_copy * max(n.value, 1))()
    check(moe_peer_fetch_plan(group_size, rank, bytes_per_rank, slices, arr, n.value,
                              ctypes.byref(n)))
    return list(arr[:n.value])
