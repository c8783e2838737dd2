"""Python binding of libfp8vit.so -- the B200 FP8 vision-encoder attention path.

Argument marshalling only: every step of the path runs in the CUDA kernels
behind the C ABI (``include/fp8vit.h``); PyTorch supplies device memory and
the current CUDA stream.  The library must be built (``__graft_entry__.build``
or ``python -m fp8_quantized_vit_b200._build``); there is no fallback.

Entry points (same names as the C ABI):
  fp8_amax_ring_update, fp8_amax_ring_update_noalloc, fp8_amax3, fp8_ring_push,
  fp8_quantize_qkv_per_tensor,
  fp8_varlen_attn_fwd, fp8_varlen_attn_fwd_bf16_group_quant (with new_tile_counters),
  per_token_group_quant_fp8, fp8_static_scales_load,
  fp8_static_scales_save, fp8_descale_from_amax, fp8_ring_read_amax, ring_init
and ``FP8EncoderAttention``, which chains them for one attention layer
(dynamic ring or static scales, BF16 or FP8 output; with a process group, the
images of one batch split across GPUs, see ``sharding``).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8vit.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, EIO, EPARSE, ENOTFOUND, ETIMEOUT = range(8)
RING_BYTES = 256
E4M3_MAX = 448.0

_P, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float

_SIGNATURES = {
    "fp8vit_create": (_I32, [_I32, ctypes.POINTER(_P)]),
    "fp8vit_destroy": (_I32, [_P]),
    "fp8vit_check": (_I32, [_P, _P, ctypes.POINTER(_I32)]),
    "fp8vit_status_string": (ctypes.c_char_p, [_I32]),
    "fp8vit_set_attn_p_terms": (_I32, [_P, _I32]),
    "fp8vit_tmap_cache_stats": (_I32, [_P, ctypes.POINTER(ctypes.c_uint64),
                                       ctypes.POINTER(ctypes.c_uint64)]),
    "fp8vit_inject_lost_arrival": (_I32, [_P, _P]),
    "fp8vit_inject_attn_timeout": (_I32, [_P, _P]),
    "fp8vit_version": (_I32, []),
    "fp8vit_ring_init": (_I32, [_P, _P]),
    "fp8_amax_ring_update": (_I32, [_P, _P, _P, _P, _I64, _P, _P, _P]),
    "fp8_amax_ring_update_noalloc": (_I32, [_P, _P, _P, _I64, _P, _P, _P]),
    "fp8_ring_read_amax": (_I32, [_P, _P, _P]),
    "fp8_amax3": (_I32, [_P, _P, _P, _P, _I64, _P, _P]),
    "fp8_ring_push": (_I32, [_P, _P, _P, _P]),
    "fp8_quantize_qkv_per_tensor": (_I32, [_P, _P, _P, _P, _I64, _P, _P, _P, _P, _P]),
    "fp8_amax_ring_quantize_qkv": (_I32, [_P, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _P]),
    "fp8_varlen_attn_fwd": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I64, _I32, _I32,
                                   _F32, _P, _I32, _P, _P]),
    "bf16_varlen_attn_fwd": (_I32, [_P, _P, _P, _P, _P, _I32, _I32, _I64, _I32, _I32, _F32, _P,
                                    _P]),
    "fp8_varlen_attn_fwd_qbf16": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I64, _I32,
                                         _I32, _F32, _P, _I32, _P, _P]),
    "fp8_varlen_attn_fwd_group_quant": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I64,
                                               _I32, _I32, _F32, _P, _P, _P]),
    "fp8_varlen_attn_fwd_bf16_group_quant": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32,
                                                    _I64, _I32, _I32, _F32, _P, _P, _P, _P,
                                                    _P]),
    "per_token_group_quant_fp8": (_I32, [_P, _P, _I64, _I64, _I32, _P, _P, _P]),
    "fp8_static_scales_load": (_I32, [ctypes.c_char_p, ctypes.c_char_p, _P]),
    "fp8_static_scales_save": (_I32, [ctypes.c_char_p, _I32, ctypes.POINTER(ctypes.c_char_p),
                                      _P, _F32]),
    "fp8_descale_from_amax": (_F32, [_F32]),
    "fp8_descale_from_amax_margin": (_F32, [_F32, _F32]),
}

_lib = None
_lock = threading.RLock()  # library loading and the per-device default contexts


class FP8VitError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def lib():
    """The loaded libfp8vit.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                       "`python -m fp8_quantized_vit_b200._build`")
                handle = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().fp8vit_status_string(status).decode()


def _check(status: int, what: str):
    if status != OK:
        raise FP8VitError(status, what)


# The current stream's raw handle: torch's direct accessor where it exists
# (a tenth of the cost of building a torch.cuda.Stream object per call).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream=None) -> int:
    if stream is None:
        if _raw_stream is not None and _cur_device is not None:
            return _raw_stream(_cur_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: torch.Tensor | None, dtype=None, name: str = "tensor") -> int | None:
    """Device address of a contiguous CUDA tensor of one of the dtypes in
    ``dtype`` (a dtype or a tuple of them); ValueError otherwise.  The common
    case costs one combined test; the message is built only on failure."""
    if t is None:
        return None
    if t.is_cuda and t.is_contiguous() and (
            dtype is None or (t.dtype in dtype if type(dtype) is tuple else t.dtype is dtype)):
        return t.data_ptr()
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


_FP8 = (torch.uint8, torch.float8_e4m3fn)


class Context:
    """A library context on one device (status word + amax scratch)."""

    def __init__(self, device: int | None = None):
        if device is None:
            device = torch.cuda.current_device()
        h = _P()
        _check(lib().fp8vit_create(device, ctypes.byref(h)), "fp8vit_create")
        self.handle = h.value
        self.device = device

    def check(self, stream=None) -> tuple[int, int]:
        """Synchronize and return (status, site) of the first device fault."""
        site = _I32(0)
        st = lib().fp8vit_check(self.handle, _stream(stream), ctypes.byref(site))
        return st, site.value

    def tmap_cache_stats(self) -> tuple[int, int]:
        """(hits, misses) of the context's tensor-map cache."""
        h, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
        _check(lib().fp8vit_tmap_cache_stats(self.handle, ctypes.byref(h), ctypes.byref(m)),
               "fp8vit_tmap_cache_stats")
        return h.value, m.value

    def set_attn_p_terms(self, terms: int):
        """P of the attention's PV product as 2 e4m3 terms (hi + lo, the
        default, meets the attention tolerance) or 1 (faster, ~3 significant
        bits of P)."""
        _check(lib().fp8vit_set_attn_p_terms(self.handle, terms), "fp8vit_set_attn_p_terms")

    def close(self):
        if getattr(self, "handle", None):
            lib().fp8vit_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_default_ctx: dict[int, Context] = {}


def default_context() -> Context:
    """The shared context of the current device (created on first use)."""
    dev = torch.cuda.current_device()
    with _lock:
        if dev not in _default_ctx:
            _default_ctx[dev] = Context(dev)
        return _default_ctx[dev]


def _ctx(ctx):
    return (ctx or default_context()).handle


# ---- ring ------------------------------------------------------------------------

def new_ring(device=None) -> torch.Tensor:
    """A zeroed ring state (64 x float32 = 256 bytes) on the device."""
    r = torch.empty(RING_BYTES // 4, dtype=torch.float32, device=device or "cuda")
    ring_init(r)
    return r


def ring_init(ring: torch.Tensor, stream=None):
    _check(lib().fp8vit_ring_init(_ptr(ring, torch.float32, "ring"), _stream(stream)),
           "fp8vit_ring_init")


def fp8_amax_ring_update(q, k, v, ring, descale3, ctx=None, stream=None):
    n = q.numel()
    if k.numel() != n or v.numel() != n:
        raise ValueError("q, k, v must have the same number of elements")
    _check(lib().fp8_amax_ring_update(
        _ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), n, _ptr(ring, torch.float32, "ring"),
        _ptr(descale3, torch.float32, "descale3"), _stream(stream)), "fp8_amax_ring_update")
    return descale3


def fp8_amax_ring_update_noalloc(q, k, v, ring, descale3, stream=None):
    """fp8_amax_ring_update without a context: the reduction scratch is a
    fixed array inside the library, shared by every call on the device, so
    calls that overlap on the GPU must not use it (order them, or use a
    context).  The first call on a device must come before any stream
    capture on it."""
    n = q.numel()
    if k.numel() != n or v.numel() != n:
        raise ValueError("q, k, v must have the same number of elements")
    _check(lib().fp8_amax_ring_update_noalloc(
        _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
        n, _ptr(ring, torch.float32, "ring"), _ptr(descale3, torch.float32, "descale3"),
        _stream(stream)), "fp8_amax_ring_update_noalloc")
    return descale3


def fp8_amax3(q, k, v, amax3, ctx=None, stream=None):
    """amax3[t] = max |x_t| of q, k, v (no ring update)."""
    n = q.numel()
    if k.numel() != n or v.numel() != n:
        raise ValueError("q, k, v must have the same number of elements")
    _check(lib().fp8_amax3(_ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                           _ptr(v, torch.bfloat16, "v"), n, _ptr(amax3, torch.float32, "amax3"),
                           _stream(stream)), "fp8_amax3")
    return amax3


def fp8_ring_push(amax3, ring, descale3, stream=None):
    """One forward of the ring rule for the device amax values amax3."""
    _check(lib().fp8_ring_push(_ptr(amax3, torch.float32, "amax3"),
                               _ptr(ring, torch.float32, "ring"),
                               _ptr(descale3, torch.float32, "descale3"), _stream(stream)),
           "fp8_ring_push")
    return descale3


def fp8_ring_read_amax(ring, stream=None) -> list[float]:
    out = (ctypes.c_float * 3)()
    _check(lib().fp8_ring_read_amax(_ptr(ring, torch.float32, "ring"), out, _stream(stream)),
           "fp8_ring_read_amax")
    return [float(x) for x in out]


# ---- quantizers ----------------------------------------------------------------------

def fp8_quantize_qkv_per_tensor(q, k, v, descale3, q8, k8, v8, ctx=None, stream=None):
    """Per-tensor e4m3 codes of q, k, v with the device descales; q8=None
    leaves Q to fp8_varlen_attn_fwd_qbf16, which quantizes it itself."""
    n = q.numel()
    for t in (k, v, k8, v8) + ((q8,) if q8 is not None else ()):
        if t.numel() != n:
            raise ValueError("all tensors must have the same number of elements")
    _check(lib().fp8_quantize_qkv_per_tensor(
        _ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), n, _ptr(descale3, torch.float32, "descale3"),
        _ptr(q8, _FP8, "q8"), _ptr(k8, _FP8, "k8"), _ptr(v8, _FP8, "v8"), _stream(stream)),
        "fp8_quantize_qkv_per_tensor")
    return q8, k8, v8


def fp8_amax_ring_quantize_qkv(q, k, v, ring, descale3, q8, k8, v8, ctx=None, stream=None):
    """fp8_amax_ring_update followed by fp8_quantize_qkv_per_tensor in one
    cooperative launch (same ring state, descales and codes); q8=None leaves
    Q's codes to fp8_varlen_attn_fwd_qbf16 (the amax still covers Q)."""
    n = q.numel()
    for t in (k, v, k8, v8) + ((q8,) if q8 is not None else ()):
        if t.numel() != n:
            raise ValueError("all tensors must have the same number of elements")
    _check(lib().fp8_amax_ring_quantize_qkv(
        _ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), n, _ptr(ring, torch.float32, "ring"),
        _ptr(descale3, torch.float32, "descale3"), _ptr(q8, _FP8, "q8"), _ptr(k8, _FP8, "k8"),
        _ptr(v8, _FP8, "v8"), _stream(stream)), "fp8_amax_ring_quantize_qkv")
    return q8, k8, v8


def per_token_group_quant_fp8(x, group, xq, scales, ctx=None, stream=None):
    if x.dim() != 2:
        raise ValueError("x must be [m, n]")
    m, n = x.shape
    if xq.numel() != m * n or scales.numel() != (m * (n // group) if group > 0 else -1):
        raise ValueError("output sizes do not match [m, n] and [m, n/group]")
    _check(lib().per_token_group_quant_fp8(
        _ctx(ctx), _ptr(x, torch.bfloat16, "x"), m, n, group, _ptr(xq, _FP8, "xq"),
        _ptr(scales, torch.float32, "scales"), _stream(stream)), "per_token_group_quant_fp8")
    return xq, scales


# ---- attention ----------------------------------------------------------------------

def fp8_varlen_attn_fwd(q8, k8, v8, q_descale, k_descale, v_descale, cu_seqlens, max_seqlen,
                        softmax_scale, out, output_scale=None, ctx=None, stream=None):
    """q8/k8/v8: e4m3 [T, H, D]; out: BF16 [T, H, D], or e4m3 with output_scale."""
    if q8.dim() != 3:
        raise ValueError("q8 must be [T, H, D]")
    T, H, D = q8.shape
    if k8.shape != q8.shape or v8.shape != q8.shape or out.shape != q8.shape:
        raise ValueError("q8, k8, v8 and out must have the same [T, H, D] shape")
    fp8_out = output_scale is not None
    _check(lib().fp8_varlen_attn_fwd(
        _ctx(ctx), _ptr(q8, _FP8, "q8"), _ptr(k8, _FP8, "k8"), _ptr(v8, _FP8, "v8"),
        _ptr(q_descale, torch.float32, "q_descale"), _ptr(k_descale, torch.float32, "k_descale"),
        _ptr(v_descale, torch.float32, "v_descale"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, float(softmax_scale),
        _ptr(out, _FP8 if fp8_out else torch.bfloat16, "out"), 1 if fp8_out else 0,
        _ptr(output_scale, torch.float32, "output_scale"), _stream(stream)),
        "fp8_varlen_attn_fwd")
    return out


def fp8_varlen_attn_fwd_qbf16(q, k8, v8, q_descale, k_descale, v_descale, cu_seqlens,
                              max_seqlen, softmax_scale, out, output_scale=None, ctx=None,
                              stream=None):
    """fp8_varlen_attn_fwd with Q given in BF16 [T, H, D]: the kernel divides
    it by q_descale and rounds it to e4m3 in its prologue (the same bytes the
    per-tensor quantizer writes), so Q's codes never go through memory."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, D]")
    T, H, D = q.shape
    if k8.shape != q.shape or v8.shape != q.shape or out.shape != q.shape:
        raise ValueError("q, k8, v8 and out must have the same [T, H, D] shape")
    fp8_out = output_scale is not None
    _check(lib().fp8_varlen_attn_fwd_qbf16(
        _ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k8, _FP8, "k8"), _ptr(v8, _FP8, "v8"),
        _ptr(q_descale, torch.float32, "q_descale"), _ptr(k_descale, torch.float32, "k_descale"),
        _ptr(v_descale, torch.float32, "v_descale"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, float(softmax_scale),
        _ptr(out, _FP8 if fp8_out else torch.bfloat16, "out"), 1 if fp8_out else 0,
        _ptr(output_scale, torch.float32, "output_scale"), _stream(stream)),
        "fp8_varlen_attn_fwd_qbf16")
    return out


def bf16_varlen_attn_fwd(q, k, v, cu_seqlens, max_seqlen, softmax_scale, out, ctx=None,
                         stream=None):
    """BF16 attention on the same kernel skeleton (the comparator of the FP8
    path): q, k, v, out BF16 [T, H, D]."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, D]")
    T, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or out.shape != q.shape:
        raise ValueError("q, k, v and out must have the same [T, H, D] shape")
    _check(lib().bf16_varlen_attn_fwd(
        _ctx(ctx), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, float(softmax_scale),
        _ptr(out, torch.bfloat16, "out"), _stream(stream)), "bf16_varlen_attn_fwd")
    return out


def fp8_varlen_attn_fwd_group_quant(q8, k8, v8, q_descale, k_descale, v_descale, cu_seqlens,
                                    max_seqlen, softmax_scale, xq, scales, ctx=None, stream=None):
    """Attention with the group-128 quantizer fused into the epilogue
    (head_dim 128): xq e4m3 [T, H * 128], scales fp32 [T, H]; the same bytes as
    fp8_varlen_attn_fwd (bf16 out) followed by per_token_group_quant_fp8."""
    if q8.dim() != 3:
        raise ValueError("q8 must be [T, H, D]")
    T, H, D = q8.shape
    if k8.shape != q8.shape or v8.shape != q8.shape:
        raise ValueError("q8, k8 and v8 must have the same [T, H, D] shape")
    if xq.numel() != T * H * D or scales.numel() != T * H * D // 128:
        raise ValueError("xq must hold T * H * D codes and scales T * H * D / 128 floats")
    _check(lib().fp8_varlen_attn_fwd_group_quant(
        _ctx(ctx), _ptr(q8, _FP8, "q8"), _ptr(k8, _FP8, "k8"), _ptr(v8, _FP8, "v8"),
        _ptr(q_descale, torch.float32, "q_descale"), _ptr(k_descale, torch.float32, "k_descale"),
        _ptr(v_descale, torch.float32, "v_descale"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, float(softmax_scale),
        _ptr(xq, _FP8, "xq"), _ptr(scales, torch.float32, "scales"), _stream(stream)),
        "fp8_varlen_attn_fwd_group_quant")
    return xq, scales


def tile_counters_size(total_tokens: int, num_seqs: int, row_elems: int) -> int:
    """Entries of the arrival counters (one per query tile and 128-column
    group of a [total_tokens, row_elems] output) that
    fp8_varlen_attn_fwd_bf16_group_quant needs."""
    return ((int(total_tokens) + 127) // 128 + int(num_seqs)) * (int(row_elems) // 128)


def new_tile_counters(total_tokens: int, num_seqs: int, row_elems: int,
                      device=None) -> torch.Tensor:
    """Zeroed counters (uint32 bits held in an int32 tensor); a completed call
    leaves them zero, so one buffer serves every later call of at most this
    size on the same stream."""
    return torch.zeros(tile_counters_size(total_tokens, num_seqs, row_elems),
                       dtype=torch.int32, device=device or "cuda")


def fp8_varlen_attn_fwd_bf16_group_quant(q8, k8, v8, q_descale, k_descale, v_descale,
                                         cu_seqlens, max_seqlen, softmax_scale, out, xq, scales,
                                         tile_counters, ctx=None, stream=None):
    """Attention with BF16 output ``out`` [T, H, D] and, in the same launch,
    its per-token groups of 128 quantized: xq e4m3 [T, H * D], scales fp32
    [T, H * D / 128] (head_dim 72 or 128, H * D a multiple of 128); the same
    bytes as fp8_varlen_attn_fwd followed by per_token_group_quant_fp8.
    ``tile_counters``: see new_tile_counters."""
    if q8.dim() != 3:
        raise ValueError("q8 must be [T, H, D]")
    T, H, D = q8.shape
    if k8.shape != q8.shape or v8.shape != q8.shape or out.shape != q8.shape:
        raise ValueError("q8, k8, v8 and out must have the same [T, H, D] shape")
    if xq.numel() != T * H * D or scales.numel() != T * H * D // 128:
        raise ValueError("xq must hold T * H * D codes and scales T * H * D / 128 floats")
    if tile_counters.numel() < tile_counters_size(T, cu_seqlens.numel() - 1, H * D):
        raise ValueError("tile_counters is too small (see tile_counters_size)")
    _check(lib().fp8_varlen_attn_fwd_bf16_group_quant(
        _ctx(ctx), _ptr(q8, _FP8, "q8"), _ptr(k8, _FP8, "k8"), _ptr(v8, _FP8, "v8"),
        _ptr(q_descale, torch.float32, "q_descale"), _ptr(k_descale, torch.float32, "k_descale"),
        _ptr(v_descale, torch.float32, "v_descale"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, float(softmax_scale),
        _ptr(out, torch.bfloat16, "out"), _ptr(xq, _FP8, "xq"),
        _ptr(scales, torch.float32, "scales"), _ptr(tile_counters, torch.int32, "tile_counters"),
        _stream(stream)), "fp8_varlen_attn_fwd_bf16_group_quant")
    return out, xq, scales


# ---- static scales ------------------------------------------------------------------

def fp8_static_scales_load(path: str, layer: str) -> tuple[float, float, float]:
    out = (ctypes.c_float * 3)()
    _check(lib().fp8_static_scales_load(path.encode(), layer.encode(), out),
           f"fp8_static_scales_load({layer})")
    return float(out[0]), float(out[1]), float(out[2])


def fp8_static_scales_save(path: str, layers, qkv_amax, margin: float = 1.5):
    import numpy as np
    names = (ctypes.c_char_p * len(layers))(*[s.encode() for s in layers])
    vals = np.ascontiguousarray(np.asarray(qkv_amax, dtype=np.float32).reshape(len(layers), 3))
    _check(lib().fp8_static_scales_save(path.encode(), len(layers), names, vals.ctypes.data,
                                        float(margin)), "fp8_static_scales_save")


def fp8_descale_from_amax(v: float) -> float:
    return float(lib().fp8_descale_from_amax(float(v)))


def fp8_descale_from_amax_margin(amax: float, margin: float) -> float:
    return float(lib().fp8_descale_from_amax_margin(float(amax), float(margin)))


# ---- one attention layer ---------------------------------------------------------------

class FP8EncoderAttention:
    """One ViT-encoder attention layer on the FP8 path.

    Holds the layer's scale state (a device ring for dynamic scaling, or
    static descales), and runs
        [amax ring update] -> per-tensor quantize -> varlen FP8 attention
    (the first two as one cooperative launch on one GPU)
        [-> per-token-group quantize of the output: fused at head_dim 128,
            the attention launch's tail at head_dim 72 with group_tail]
    on the current stream.  The intermediate FP8 buffers and the output are the
    layer's own: they grow to the largest token count seen and are reused, so
    a call allocates nothing once that size has been met, and the tensors a
    call returns are overwritten by the layer's next call (pass ``out`` to
    keep an output).
    """

    def __init__(self, num_heads: int, head_dim: int, softmax_scale: float | None = None,
                 static_amax=None, margin: float = 1.5, device=None, ctx: Context | None = None,
                 process_group=None, fold_q: bool = False, group_tail: bool = False):
        self.H, self.D = num_heads, head_dim
        # group_tail: where a 128-column group spans heads (head_dim 72), the
        # group quantizer runs as the attention launch's tail
        # (fp8_varlen_attn_fwd_bf16_group_quant) instead of a separate launch
        self.group_tail = group_tail
        # fold_q: the attention kernel quantizes Q in its prologue
        # (fp8_varlen_attn_fwd_qbf16); the quantizer writes only K and V codes
        self.fold_q = fold_q
        self.softmax_scale = (float(torch.tensor(head_dim ** -0.5, dtype=torch.float32))
                              if softmax_scale is None else softmax_scale)
        self.device = torch.device(device or "cuda")
        self.ctx = ctx or default_context()
        self.descale = torch.zeros(3, dtype=torch.float32, device=self.device)
        self._dq, self._dk, self._dv = self.descale[0:1], self.descale[1:2], self.descale[2:3]
        self.process_group = process_group
        self._amax3 = torch.zeros(3, dtype=torch.float32, device=self.device)
        self.ring = None
        if static_amax is None:
            self.ring = new_ring(self.device)
        else:
            self.set_static_amax(static_amax, margin=None)
        self._bufs = {}

    @classmethod
    def from_scale_file(cls, path: str, layer: str, num_heads: int, head_dim: int, **kw):
        vals = fp8_static_scales_load(path, layer)
        obj = cls(num_heads, head_dim, static_amax=vals, **kw)
        return obj

    def set_static_amax(self, values, margin: float | None = None):
        """Use static scales.  ``values`` are in the amax domain (already
        including the save margin, as stored in a scale file); pass ``margin``
        to apply one here instead."""
        if margin is None:
            d = [fp8_descale_from_amax(float(x)) for x in values]
        else:
            d = [fp8_descale_from_amax_margin(float(x), float(margin)) for x in values]
        self.descale.copy_(torch.tensor(d, dtype=torch.float32))
        self.ring = None

    def _buffers(self, T: int, fp8_out: bool, group_quant: bool = False) -> dict:
        """Views of the first T tokens of the layer's buffers (one set per
        output type, reallocated only when T exceeds the capacity held)."""
        st = self._bufs.get(fp8_out)
        if st is None or st["cap"] < T:
            shape = (T, self.H, self.D)
            mk = lambda dt: torch.empty(shape, dtype=dt, device=self.device)
            st = dict(cap=T, q8=mk(torch.uint8), k8=mk(torch.uint8), v8=mk(torch.uint8),
                      out=mk(torch.uint8 if fp8_out else torch.bfloat16))
            self._bufs[fp8_out] = st
        if group_quant and "xq" not in st:
            hd = self.H * self.D
            st["xq"] = torch.empty((st["cap"], hd), dtype=torch.uint8, device=self.device)
            st["xs"] = torch.empty((st["cap"], hd // 128), dtype=torch.float32,
                                   device=self.device)
        return {k: v[:T] for k, v in st.items() if k != "cap"}

    def _counters(self, T: int, num_seqs: int) -> torch.Tensor:
        hd = self.H * self.D
        need = tile_counters_size(T, num_seqs, hd)
        c = self._bufs.get("tile_counters")
        if c is None or c.numel() < need:
            c = new_tile_counters(T, num_seqs, hd, self.device)
            self._bufs["tile_counters"] = c
        return c

    def forward(self, q, k, v, cu_seqlens, max_seqlen: int, output_scale=None, out=None,
                group_quant: bool = False):
        """q, k, v: BF16 [T, H, D] on the device; cu_seqlens: int32 [B+1].
        Returns the attention output (BF16, or e4m3 codes if output_scale), or
        with ``group_quant`` the o-proj input: (e4m3 codes [T, H*D], fp32
        scales [T, H*D/128]) of the BF16 output's per-token groups of 128 --
        fused into the attention epilogue at head_dim 128, a separate
        per_token_group_quant_fp8 call otherwise."""
        if group_quant and output_scale is not None:
            raise ValueError("group_quant and output_scale are exclusive")
        T = q.shape[0]
        if group_quant and (self.H * self.D) % 128 != 0:
            raise ValueError("group_quant needs num_heads * head_dim to be a multiple of 128")
        b = self._buffers(T, output_scale is not None, group_quant)
        fold = self.fold_q and not (group_quant and (self.D == 128 or self.group_tail))
        q8 = None if fold else b["q8"]
        if self.ring is not None and self.process_group is not None:
            # this rank holds some of the batch's images: agree on the
            # per-tensor amax with the other ranks before the ring update
            from .sharding import allreduce_amax3
            fp8_amax3(q, k, v, self._amax3, ctx=self.ctx)
            allreduce_amax3(self._amax3, self.process_group)
            fp8_ring_push(self._amax3, self.ring, self.descale)
        if self.ring is not None and self.process_group is None:
            # amax, ring rule and quantization in one cooperative launch
            fp8_amax_ring_quantize_qkv(q, k, v, self.ring, self.descale, q8, b["k8"],
                                       b["v8"], ctx=self.ctx)
        else:
            fp8_quantize_qkv_per_tensor(q, k, v, self.descale, q8, b["k8"], b["v8"],
                                        ctx=self.ctx)
        attn = fp8_varlen_attn_fwd_qbf16 if fold else fp8_varlen_attn_fwd
        qa = q if fold else b["q8"]
        if group_quant:
            hd = self.H * self.D
            xq, xs = b["xq"], b["xs"]
            if self.D != 128 and self.group_tail and not fold:
                fp8_varlen_attn_fwd_bf16_group_quant(
                    b["q8"], b["k8"], b["v8"], self._dq, self._dk,
                    self._dv, cu_seqlens, max_seqlen, self.softmax_scale, b["out"], xq,
                    xs, self._counters(T, cu_seqlens.numel() - 1), ctx=self.ctx)
            elif self.D == 128:
                fp8_varlen_attn_fwd_group_quant(b["q8"], b["k8"], b["v8"], self._dq,
                                                self._dk, self._dv, cu_seqlens,
                                                max_seqlen, self.softmax_scale, xq, xs,
                                                ctx=self.ctx)
            else:
                o = b["out"]
                attn(qa, b["k8"], b["v8"], self._dq, self._dk,
                     self._dv, cu_seqlens, max_seqlen, self.softmax_scale, o,
                     ctx=self.ctx)
                per_token_group_quant_fp8(o.view(T, hd), 128, xq, xs, ctx=self.ctx)
            return xq, xs
        o = b["out"] if out is None else out
        attn(qa, b["k8"], b["v8"], self._dq, self._dk, self._dv,
             cu_seqlens, max_seqlen, self.softmax_scale, o, output_scale=output_scale,
             ctx=self.ctx)
        return o

    __call__ = forward
