"""Seeded synthetic inputs for the MoE-layer workloads.

Two kinds of generator, both keyed by (seed, workload, layer, tensor, expert):

* Small per-layer tensors (the layer input x, the router weight W_g and the
  router selection bias) come from numpy's PCG64 stream, true normals, on the
  host.  Both the oracle and the GPU path receive the same bytes.
* Expert weights (tens of GB at the DeepSeek-R1 shape) come from a
  counter-based generator (Philox4x32-10 with an Irwin-Hall-8 bell shape)
  implemented twice, in ``csrc/philox_cpu.c`` for the host and in
  ``csrc/philox_gpu.cu`` for the GPU, so that the GPU fills its weight pools
  in place while the oracle regenerates just the experts it needs, with the
  same bits.

Holds none of the MoE layer's arithmetic.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from .configs import SEED, MoEConfig, config

_HERE = os.path.dirname(os.path.abspath(__file__))

TID_X, TID_WG, TID_BIAS, TID_SEQ, TID_ZIPF = 0, 1, 2, 3, 4
TENSOR_GU, TENSOR_DOWN = 0, 1


# --------------------------------------------------------------------------
# bf16 / e4m3 bit helpers (format definitions, no layer arithmetic)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even; returns the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (b & 0x7FFFFFFF) > 0x7F800000
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((b[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _e4m3_table() -> np.ndarray:
    """Value of every e4m3 (fn variant) byte: sign, 4-bit exponent (bias 7),
    3-bit mantissa; exponent 0 is subnormal (m * 2^-9); 0x7F/0xFF are NaN."""
    t = np.zeros(256, dtype=np.float64)
    for b in range(256):
        s = -1.0 if b & 0x80 else 1.0
        e = (b >> 3) & 0xF
        m = b & 7
        if e == 0xF and m == 7:
            t[b] = np.nan
        elif e == 0:
            t[b] = s * m * 2.0 ** -9
        else:
            t[b] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3_VALUES = _e4m3_table()


def e4m3_bits_to_f64(q: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(q, dtype=np.uint8)]


# --------------------------------------------------------------------------
# host generator library
# --------------------------------------------------------------------------
_cpu_lib = None


def cpu_lib() -> ctypes.CDLL:
    global _cpu_lib
    if _cpu_lib is None:
        from . import build as _b
        path = _b.build_cpu()
        lib = ctypes.CDLL(path)
        i64, u32, dbl, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_double, ctypes.c_void_p
        lib.moegen_philox4x32_10.argtypes = [vp, u32, u32, vp]
        lib.moegen_normal_f32.argtypes = [vp, i64, u32, u32, dbl]
        lib.moegen_normal_bf16.argtypes = [vp, i64, u32, u32, dbl]
        lib.moegen_e4m3_blocks.argtypes = [vp, vp, i64, i64, u32, u32, dbl]
        lib.moegen_f32_to_e4m3.argtypes = [vp, vp, i64]
        lib.moegen_f32_to_bf16.argtypes = [vp, vp, i64]
        for f in (lib.moegen_philox4x32_10, lib.moegen_normal_f32, lib.moegen_normal_bf16,
                  lib.moegen_e4m3_blocks, lib.moegen_f32_to_e4m3, lib.moegen_f32_to_bf16):
            f.restype = None
        _cpu_lib = lib
    return _cpu_lib


def philox4x32_10(ctr, key) -> tuple[int, int, int, int]:
    """One Philox4x32-10 block on the host (for known-answer tests)."""
    cin = (ctypes.c_uint32 * 4)(*[int(c) & 0xFFFFFFFF for c in ctr])
    cout = (ctypes.c_uint32 * 4)()
    cpu_lib().moegen_philox4x32_10(cin, int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF, cout)
    return tuple(int(v) for v in cout)


def f32_to_e4m3_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    cpu_lib().moegen_f32_to_e4m3(a.ctypes.data, out.ctypes.data, a.size)
    return out


# --------------------------------------------------------------------------
# keys
# --------------------------------------------------------------------------
def weight_key(cfg: MoEConfig, layer: int, expert: int, tensor: int) -> tuple[int, int]:
    """Philox key of one expert tensor.  expert == cfg.E is the shared expert."""
    assert 0 <= cfg.cfg_id < 256 and 0 <= layer < 16 and 0 <= tensor < 16
    assert 0 <= expert < 65536
    return SEED & 0xFFFFFFFF, (cfg.cfg_id << 24) | (layer << 20) | (tensor << 16) | expert


def _rng(cfg: MoEConfig, layer: int, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([SEED, cfg.cfg_id, layer, tid])))


# --------------------------------------------------------------------------
# per-layer small tensors (numpy PCG64)
# --------------------------------------------------------------------------
@dataclass
class LayerInputs:
    x: np.ndarray            # [T, H] float32 values (exactly bf16 values when x_dtype == "bf16")
    x_bits: np.ndarray | None  # [T, H] uint16 bf16 bits, or None for fp32 input
    wg: np.ndarray           # [E, H] float32
    bias: np.ndarray | None  # [E] float32 or None


def gen_x(cfg, layer: int = 0, rows: slice | None = None):
    """Layer input x ~ N(0, x_sigma), drawn as fp32 and rounded to bf16 (RNE)
    for bf16 workloads.  Returns (values_f32, bf16_bits_or_None)."""
    cfg = config(cfg)
    x = _rng(cfg, layer, TID_X).standard_normal((cfg.T, cfg.H), dtype=np.float32)
    if cfg.x_sigma != 1.0:
        x = (x * np.float32(cfg.x_sigma)).astype(np.float32)
    if rows is not None:
        x = np.ascontiguousarray(x[rows])
    if cfg.x_dtype == "bf16":
        bits = f32_to_bf16_bits(x)
        return bf16_bits_to_f32(bits), bits
    return x, None


def gen_wg(cfg, layer: int = 0) -> np.ndarray:
    cfg = config(cfg)
    w = _rng(cfg, layer, TID_WG).standard_normal((cfg.E, cfg.H), dtype=np.float32)
    return (w * np.float32(cfg.wg_sigma)).astype(np.float32)


def gen_bias(cfg, layer: int = 0) -> np.ndarray | None:
    """Router selection bias.  "zipf": b_e = amp * r_e^(-s), r_e the 1-based
    rank of expert e in a seeded permutation, so the hot experts land in both
    pools."""
    cfg = config(cfg)
    if cfg.bias == "none":
        return None
    if cfg.bias == "normal":
        b = _rng(cfg, layer, TID_BIAS).standard_normal(cfg.E, dtype=np.float32)
        return (b * np.float32(cfg.bias_sigma)).astype(np.float32)
    if cfg.bias == "zipf":
        perm = _rng(cfg, 0, TID_ZIPF).permutation(cfg.E)
        rank = np.empty(cfg.E, dtype=np.float64)
        rank[perm] = np.arange(1, cfg.E + 1, dtype=np.float64)
        return (cfg.zipf_amp * rank ** (-cfg.zipf_s)).astype(np.float32)
    raise ValueError(cfg.bias)


def seq_lengths(cfg) -> list[int]:
    """Sequence lengths whose coefficient of variation is seq_cv and whose sum
    is T: L_i = (T/n)(1 + cv z_i), z standardised seeded normals.  The MoE
    block is per token, so the split is metadata: the tokens are concatenated."""
    cfg = config(cfg)
    n = cfg.seq_count
    if n <= 1:
        return [cfg.T]
    z = _rng(cfg, 0, TID_SEQ).standard_normal(n)
    z = (z - z.mean()) / z.std()
    L = np.rint(cfg.T / n * (1.0 + cfg.seq_cv * z)).astype(np.int64)
    L[-1] = cfg.T - L[:-1].sum()
    assert (L > 0).all()
    return [int(v) for v in L]


def layer_inputs(cfg, layer: int = 0) -> LayerInputs:
    cfg = config(cfg)
    x, bits = gen_x(cfg, layer)
    return LayerInputs(x=x, x_bits=bits, wg=gen_wg(cfg, layer), bias=gen_bias(cfg, layer))


# --------------------------------------------------------------------------
# expert weights (counter-based; host copy for the oracle)
# --------------------------------------------------------------------------
@dataclass
class ExpertHost:
    """One expert's weights on the host.

    bf16:  gu [2I, H] uint16 bits (gate rows first), down [H, I] uint16 bits.
    e4m3:  gu / down uint8 codes plus fp32 scales per 128x128 block
           (gu_scale [2I/128, H/128], down_scale [H/128, I/128]).
    """
    gu: np.ndarray
    down: np.ndarray
    gu_scale: np.ndarray | None = None
    down_scale: np.ndarray | None = None

    def gu_f64(self) -> np.ndarray:
        return _dequant(self.gu, self.gu_scale)

    def down_f64(self) -> np.ndarray:
        return _dequant(self.down, self.down_scale)


def _dequant(q: np.ndarray, s: np.ndarray | None) -> np.ndarray:
    if s is None:
        return bf16_bits_to_f32(q).astype(np.float64)
    v = e4m3_bits_to_f64(q)
    rows, cols = q.shape
    full = np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)[:rows, :cols]
    return v * full


def _host_tensor(cfg: MoEConfig, layer: int, expert: int, tensor: int, rows: int, cols: int):
    k0, k1 = weight_key(cfg, layer, expert, tensor)
    lib = cpu_lib()
    if cfg.w_dtype == "bf16":
        out = np.empty((rows, cols), dtype=np.uint16)
        lib.moegen_normal_bf16(out.ctypes.data, out.size, k0, k1, float(cfg.w_sigma))
        return out, None
    if cfg.w_dtype == "e4m3":
        q = np.empty((rows, cols), dtype=np.uint8)
        s = np.empty(((rows + 127) // 128, (cols + 127) // 128), dtype=np.float32)
        lib.moegen_e4m3_blocks(q.ctypes.data, s.ctypes.data, rows, cols, k0, k1, float(cfg.w_sigma))
        return q, s
    raise ValueError(cfg.w_dtype)


def expert_host(cfg, layer: int, expert: int) -> ExpertHost:
    """Weights of routed expert `expert` (or the shared one when expert == E)."""
    cfg = config(cfg)
    gu, gus = _host_tensor(cfg, layer, expert, TENSOR_GU, 2 * cfg.I, cfg.H)
    dn, dns = _host_tensor(cfg, layer, expert, TENSOR_DOWN, cfg.H, cfg.I)
    return ExpertHost(gu=gu, down=dn, gu_scale=gus, down_scale=dns)
