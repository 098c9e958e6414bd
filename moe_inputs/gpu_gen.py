"""GPU-side fill of expert weights (same bits as the host generator)."""
from __future__ import annotations

import ctypes

from . import build as _b
from .configs import MoEConfig, config
from .gen import TENSOR_DOWN, TENSOR_GU, weight_key

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        l = ctypes.CDLL(_b.build_gpu())
        i64, u32, dbl, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_double, ctypes.c_void_p
        l.moegen_gpu_philox4x32_10.argtypes = [vp, u32, u32, vp, vp]
        l.moegen_gpu_normal_f32.argtypes = [vp, i64, u32, u32, dbl, vp]
        l.moegen_gpu_normal_bf16.argtypes = [vp, i64, u32, u32, dbl, vp]
        l.moegen_gpu_e4m3_blocks.argtypes = [vp, vp, i64, i64, u32, u32, dbl, vp]
        for f in (l.moegen_gpu_philox4x32_10, l.moegen_gpu_normal_f32, l.moegen_gpu_normal_bf16,
                  l.moegen_gpu_e4m3_blocks):
            f.restype = ctypes.c_int
        _lib = l
    return _lib


def _chk(rc: int) -> None:
    if rc != 0:
        raise RuntimeError("GPU generator launch failed: cudaError %d" % rc)


def fill_tensor(cfg: MoEConfig, layer: int, expert: int, tensor: int, rows: int, cols: int,
                ptr: int, scale_ptr: int | None, stream: int) -> None:
    """Writes one expert tensor (row-major [rows, cols]) at device address ptr;
    for e4m3 weights the 128x128 block scales go to scale_ptr."""
    k0, k1 = weight_key(cfg, layer, expert, tensor)
    if cfg.w_dtype == "bf16":
        _chk(lib().moegen_gpu_normal_bf16(ptr, rows * cols, k0, k1, float(cfg.w_sigma), stream))
    elif cfg.w_dtype == "e4m3":
        _chk(lib().moegen_gpu_e4m3_blocks(ptr, scale_ptr, rows, cols, k0, k1, float(cfg.w_sigma),
                                          stream))
    else:
        raise ValueError(cfg.w_dtype)


def fill_expert(cfg, layer: int, expert: int, gu_ptr: int, down_ptr: int,
                gu_scale_ptr: int | None, down_scale_ptr: int | None, stream: int) -> None:
    cfg = config(cfg)
    fill_tensor(cfg, layer, expert, TENSOR_GU, 2 * cfg.I, cfg.H, gu_ptr, gu_scale_ptr, stream)
    fill_tensor(cfg, layer, expert, TENSOR_DOWN, cfg.H, cfg.I, down_ptr, down_scale_ptr, stream)
