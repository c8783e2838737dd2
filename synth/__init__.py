"""Seeded synthetic inputs for the FP8 ViT attention path.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the method's arithmetic: it builds BF16 activation tensors with
the shapes and value distribution of the workloads (N(0,1) with 1% of the
channels scaled x8), int32 ``cu_seqlens`` offsets, and the workload recipes.
The draws come from the counter-based generator in ``synth.c`` so that any
consumer (CPU oracle or GPU) sees the same bytes for the same seed.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-pthread",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64] * 3
        lib.synth_splitmix64.restype = ctypes.c_uint64
        lib.synth_splitmix64.argtypes = [ctypes.c_uint64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_double_to_bf16.restype = ctypes.c_uint16
        lib.synth_double_to_bf16.argtypes = [ctypes.c_double]
        lib.synth_outlier_columns.restype = ctypes.c_int
        lib.synth_outlier_columns.argtypes = [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_void_p]
        lib.synth_fill_bf16.restype = ctypes.c_int
        lib.synth_fill_bf16.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int32, ctypes.c_double, ctypes.c_int32,
                                        ctypes.c_void_p]
        _lib = lib
    return _lib


def splitmix64(x: int) -> int:
    return int(_load().synth_splitmix64(x & 0xFFFFFFFFFFFFFFFF))


def stream_key(seed: int, slot: int, tensor: int) -> int:
    """Key of the stream for (seed, slot = forward or layer index, tensor id)."""
    return int(_load().synth_key(seed, slot, tensor))


def normal(key: int, i: int) -> float:
    return float(_load().synth_normal(key, i))


def outlier_count(ncols: int, frac: float = 0.01) -> int:
    """Number of outlier channels: 1% of the columns, rounded to nearest."""
    return int(math.floor(frac * ncols + 0.5))


def outlier_columns(key: int, ncols: int, n_out: int) -> np.ndarray:
    cols = np.zeros(max(n_out, 1), dtype=np.int32)
    rc = _load().synth_outlier_columns(key, ncols, n_out, cols.ctypes.data)
    if rc != 0:
        raise ValueError(f"synth_outlier_columns failed ({rc})")
    return cols[:n_out]


def bf16_tensor(key: int, rows: int, ncols: int, n_out: int | None = None, factor: float = 8.0,
                threads: int | None = None) -> np.ndarray:
    """BF16 bits (uint16) of shape [rows, ncols] drawn from stream ``key``."""
    if n_out is None:
        n_out = outlier_count(ncols)
    out = np.empty((rows, ncols), dtype=np.uint16)
    if threads is None:
        threads = min(os.cpu_count() or 1, 64)
    rc = _load().synth_fill_bf16(key, rows, ncols, n_out, factor, threads, out.ctypes.data)
    if rc != 0:
        raise ValueError(f"synth_fill_bf16 failed ({rc})")
    return out


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def cu_seqlens(lengths) -> np.ndarray:
    """int32 prefix offsets [B+1] of the packed segments."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


@dataclass(frozen=True)
class Workload:
    """One workload recipe: packed segment lengths, heads, head_dim, seeds."""
    name: str
    seg_lens: tuple
    heads: int
    head_dim: int
    mode: str                      # "static" or "dynamic"
    seeds: tuple                   # one seed per forward / layer
    fp8_out: bool = False
    group_quant: bool = False
    margin: float = 1.5
    per_layer_rings: bool = False  # the seeds are layers of one forward, each with its own ring
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return int(sum(self.seg_lens))

    @property
    def hd(self) -> int:
        return self.heads * self.head_dim

    @property
    def softmax_scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    def attn_flops(self) -> float:
        """Counted FLOPs of one attention call: sum_i 4 * S_i^2 * D * H."""
        return float(sum(4.0 * s * s * self.head_dim * self.heads for s in self.seg_lens))

    def qkv(self, slot: int, threads: int | None = None):
        """(q, k, v) BF16 bit arrays [T, H*D] for forward/layer ``slot``."""
        seed = self.seeds[slot % len(self.seeds)]
        return tuple(bf16_tensor(stream_key(seed, slot, t), self.tokens, self.hd, threads=threads)
                     for t in (TENSOR_Q, TENSOR_K, TENSOR_V))


# The five workloads (vLLM "FP8 ViT Encoder Attention": Usage, Performance
# tables; image sizes at 16x16 patches: 1440x2560 -> 14400 tokens,
# 2160x3840 -> 32400 tokens).
WORKLOADS = {
    "1x1024_d72": Workload("1x1024 tokens, 16 heads, head_dim 72, static scales",
                   (1024,), 16, 72, "static", (1,)),
    "1x8192_d128": Workload("1x8192 tokens, 16 heads, head_dim 128, dynamic ring over 20 forwards",
                   (8192,), 16, 128, "dynamic", tuple(range(100, 120)), group_quant=True),
    "1x2304_d72": Workload("1x2304 tokens, 16 heads, head_dim 72, dynamic",
                        (2304,), 16, 72, "dynamic", (300,)),
    "1x4096_d72": Workload("1x4096 tokens, 16 heads, head_dim 72, dynamic",
                        (4096,), 16, 72, "dynamic", (301,)),
    "1x8192_d72": Workload("1x8192 tokens, 16 heads, head_dim 72, dynamic",
                        (8192,), 16, 72, "dynamic", (302,)),
    "1x16384_d72": Workload("1x16384 tokens, 16 heads, head_dim 72, dynamic",
                         (16384,), 16, 72, "dynamic", (303,)),
    "3x14400_d72": Workload("3x14400 tokens, 16 heads, head_dim 72, static scales, fp8 output",
                   (14400, 14400, 14400), 16, 72, "static", (400,), fp8_out=True),
    "3x32400_d72": Workload("3x32400 tokens, 16 heads, head_dim 72, 27 layers, dynamic, group quant",
                   (32400, 32400, 32400), 16, 72, "dynamic", tuple(range(500, 527)),
                   group_quant=True, per_layer_rings=True),
}
