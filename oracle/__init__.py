"""CPU oracle for the FP8 ViT attention path -- TEST INFRASTRUCTURE ONLY.

The oracle is the plain, slow, single-threaded statement of what the path
computes (``oracle.c``): the e4m3 codec, the amax / ring-buffer / scale rules,
the per-tensor and per-token-group quantizers, fp64 softmax attention over
the dequantised FP8 tensors, and the same attention over BF16 tensors (the
BF16 comparator's reference).  Only the tests, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import it.  It shares no code with the
CUDA library and never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

RING_SLOTS = 16

_P = ctypes.c_void_p
_I32, _I64, _F32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load_signatures(lib):
    sig = {
        "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
        "orc_e4m3_encode": (ctypes.c_uint8, [_F32]),
        "orc_e4m3_encode_array": (None, [_P, _I64, _P]),
        "orc_e4m3_decode_array": (None, [_P, _I64, _P]),
        "orc_bf16_to_float": (_F32, [ctypes.c_uint16]),
        "orc_double_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
        "orc_amax_bf16": (_F32, [_P, _I64]),
        "orc_descale_from_amax": (_F32, [_F32]),
        "orc_ring_update": (None, [_P, _P, _P, _P]),
        "orc_quantize_per_tensor": (None, [_P, _I64, _F32, _P]),
        "orc_group_quant": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _P]),
        "orc_attn_pairs": (ctypes.c_int, [_P, _P, _P, _F32, _F32, _F32, _P, _I32, _I32, _I32,
                                          _F32, _P, _P, _I64, _P, _P]),
        "orc_attn_full": (ctypes.c_int, [_P, _P, _P, _F32, _F32, _F32, _P, _I32, _I32, _I32,
                                         _F32, _P]),
        "orc_fp8_output": (None, [_P, _I64, _F32, _P]),
        "orc_attn_pairs_bf16": (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _F32, _P, _P,
                                               _I64, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        _load_signatures(lib)
        _lib = lib
    return _lib


class use_library:
    """Context manager: route the wrappers below to another build of the
    oracle (used by the tests that plant mistakes in a copy of oracle.c to
    show the pins catch them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        lib = ctypes.CDLL(self.path)
        _load_signatures(lib)
        _lib = lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


# --- e4m3 codec -------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    codes, p = _c(codes, np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().orc_e4m3_decode_array(p, codes.size, out.ctypes.data)
    return out


def e4m3_encode(x) -> np.ndarray:
    x, p = _c(x, np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(p, x.size, out.ctypes.data)
    return out


def double_to_bf16(d: float) -> int:
    return int(_load().orc_double_to_bf16(float(d)))


# --- amax, ring, scales ----------------------------------------------------------

def amax_bf16(x_bits) -> float:
    x, p = _c(x_bits, np.uint16)
    return float(np.float32(_load().orc_amax_bf16(p, x.size)))


def descale_from_amax(v: float) -> float:
    return float(np.float32(_load().orc_descale_from_amax(float(np.float32(v)))))


class Ring:
    """Dynamic-scaling state: float hist[3][16] (q, k, v rows) and a shared
    write position.  ``update`` runs one forward's rule and returns the three
    descales."""

    def __init__(self):
        self.hist = np.zeros((3, RING_SLOTS), dtype=np.float32)
        self.pos = np.zeros(1, dtype=np.int32)

    def update(self, amax3) -> np.ndarray:
        a = np.ascontiguousarray(amax3, dtype=np.float32)
        out = np.empty(3, dtype=np.float32)
        _load().orc_ring_update(self.hist.ctypes.data, self.pos.ctypes.data, a.ctypes.data,
                                out.ctypes.data)
        return out


def quantize_per_tensor(x_bits, descale: float) -> np.ndarray:
    x, p = _c(x_bits, np.uint16)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_quantize_per_tensor(p, x.size, float(np.float32(descale)), out.ctypes.data)
    return out


def group_quant(x_bits, group: int = 128):
    """Per-token-group quantizer; returns (codes [m, n], scales [m, n/group])."""
    x, p = _c(x_bits, np.uint16)
    m, n = x.shape
    xq = np.empty((m, n), dtype=np.uint8)
    sc = np.empty((m, n // group), dtype=np.float32)
    rc = _load().orc_group_quant(p, m, n, group, xq.ctypes.data, sc.ctypes.data)
    if rc != 0:
        raise ValueError("n must be a multiple of group")
    return xq, sc


# --- attention -------------------------------------------------------------

def attn_pairs(q8, k8, v8, dq, dk, dv, cu_seqlens, heads: int, head_dim: int, sm_scale: float,
               tokens, head_ids, want_psum: bool = False):
    """fp64 attention for the (token, head) pairs; returns out [n, D] (and the
    probability sums if ``want_psum``)."""
    q8, pq = _c(q8, np.uint8)
    k8, pk = _c(k8, np.uint8)
    v8, pv = _c(v8, np.uint8)
    cu, pc = _c(cu_seqlens, np.int32)
    toks, pt = _c(tokens, np.int64)
    hs, ph = _c(head_ids, np.int32)
    n = toks.size
    out = np.empty((n, head_dim), dtype=np.float64)
    psum = np.empty(n, dtype=np.float64) if want_psum else None
    rc = _load().orc_attn_pairs(pq, pk, pv, float(dq), float(dk), float(dv), pc, cu.size - 1,
                                heads, head_dim, float(sm_scale), pt, ph, n, out.ctypes.data,
                                psum.ctypes.data if want_psum else None)
    if rc != 0:
        raise ValueError(f"orc_attn_pairs failed ({rc})")
    return (out, psum) if want_psum else out


def attn_full(q8, k8, v8, dq, dk, dv, cu_seqlens, heads: int, head_dim: int,
              sm_scale: float) -> np.ndarray:
    """fp64 attention over every token and head; returns [T, H, D]."""
    q8, pq = _c(q8, np.uint8)
    k8, pk = _c(k8, np.uint8)
    v8, pv = _c(v8, np.uint8)
    cu, pc = _c(cu_seqlens, np.int32)
    T = int(cu[-1])
    out = np.zeros((T, heads, head_dim), dtype=np.float64)
    rc = _load().orc_attn_full(pq, pk, pv, float(dq), float(dk), float(dv), pc, cu.size - 1,
                               heads, head_dim, float(sm_scale), out.ctypes.data)
    if rc != 0:
        raise ValueError(f"orc_attn_full failed ({rc})")
    return out


def attn_pairs_bf16(q, k, v, cu_seqlens, heads: int, head_dim: int, sm_scale: float, tokens,
                    head_ids, want_psum: bool = False):
    """fp64 attention over BF16 inputs (bit patterns, [T, H*D] or [T, H, D])
    for the (token, head) pairs; returns out [n, D] (and the probability sums)."""
    q, pq = _c(q, np.uint16)
    k, pk = _c(k, np.uint16)
    v, pv = _c(v, np.uint16)
    cu, pc = _c(cu_seqlens, np.int32)
    toks, pt = _c(tokens, np.int64)
    hs, ph = _c(head_ids, np.int32)
    n = toks.size
    out = np.empty((n, head_dim), dtype=np.float64)
    psum = np.empty(n, dtype=np.float64) if want_psum else None
    rc = _load().orc_attn_pairs_bf16(pq, pk, pv, pc, cu.size - 1, heads, head_dim,
                                     float(sm_scale), pt, ph, n, out.ctypes.data,
                                     psum.ctypes.data if want_psum else None)
    if rc != 0:
        raise ValueError(f"orc_attn_pairs_bf16 failed ({rc})")
    return (out, psum) if want_psum else out


def attn_full_bf16(q, k, v, cu_seqlens, heads: int, head_dim: int, sm_scale: float) -> np.ndarray:
    """fp64 attention over BF16 inputs for every token and head; returns [T, H, D]."""
    cu = np.asarray(cu_seqlens, dtype=np.int32)
    T = int(cu[-1])
    toks = np.repeat(np.arange(int(cu[0]), T, dtype=np.int64), heads)
    hs = np.tile(np.arange(heads, dtype=np.int32), T - int(cu[0]))
    out = np.zeros((T, heads, head_dim), dtype=np.float64)
    if toks.size:
        out[int(cu[0]):] = attn_pairs_bf16(q, k, v, cu, heads, head_dim, sm_scale, toks,
                                           hs).reshape(T - int(cu[0]), heads, head_dim)
    return out


def fp8_output(o, output_scale: float) -> np.ndarray:
    o, p = _c(o, np.float64)
    out = np.empty(o.shape, dtype=np.uint8)
    _load().orc_fp8_output(p, o.size, float(np.float32(output_scale)), out.ctypes.data)
    return out
