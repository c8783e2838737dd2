"""The allocation-free amax/ring entry point (fp8_amax_ring_update_noalloc).

Callers that cannot allocate device memory (a pool that already holds the
free HBM, no room for cudaMalloc's device-wide synchronisation, no place to
keep a context) use this variant, whose scratch is a fixed array inside the
library.  It must give the same descales and ring contents as the context
entry point, bit for bit, on consecutive calls that reuse the shared array.
This file is collected last so that a failure here leaves every other test
already run."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

fv = pytest.importorskip("fp8_quantized_vit_b200")


def _noalloc_fn():
    fn = fv.lib().fp8_amax_ring_update_noalloc
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p]
    return fn


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def test_noalloc_matches_context_entry_point_on_consecutive_calls():
    assert torch.cuda.is_available()
    fn = _noalloc_fn()
    ctx = fv.Context()
    rows, cols = 3000, 1152  # 3.46 M elements per tensor, plus an odd tail below
    ring_ctx, ring_na = fv.new_ring(), fv.new_ring()
    d_ctx = torch.zeros(3, dtype=torch.float32, device="cuda")
    d_na = torch.zeros(3, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        x = [synth.bf16_tensor(synth.stream_key(900 + call, call, t), rows, cols).ravel()
             for t in range(3)]
        n = x[0].size - 5  # a ragged element count exercises the tail path
        dev = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in x]
        fv.lib().fp8_amax_ring_update(ctx.handle, dev[0].data_ptr(), dev[1].data_ptr(),
                                      dev[2].data_ptr(), n, ring_ctx.data_ptr(),
                                      d_ctx.data_ptr(), stream)
        if call == 0:
            st = fn(dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(), n,
                    ring_na.data_ptr(), d_na.data_ptr(), stream)
            assert st == fv.OK, fv.status_string(st)
        else:
            # the second call goes through the Python wrapper (argument checks,
            # default stream), on flat views of the first n elements
            fv.fp8_amax_ring_update_noalloc(dev[0][:n], dev[1][:n], dev[2][:n], ring_na, d_na)
        torch.cuda.synchronize()
        assert (_bits(d_na) == _bits(d_ctx)).all(), (call, d_na, d_ctx)
        assert (_bits(ring_na) == _bits(ring_ctx)).all(), call
    st, site = ctx.check()
    assert st == fv.OK


def test_noalloc_rejects_bad_arguments():
    fn = _noalloc_fn()
    buf = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = buf.data_ptr()
    assert fn(None, p, p, 8, p, p, None) == fv.EINVAL
    assert fn(p, p, p, -1, p, p, None) == fv.EINVAL
    assert fn(p + 2, p, p, 8, p, p, None) == fv.EINVAL
