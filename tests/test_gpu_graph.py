"""The layer forward (amax ring update -> per-tensor quantize -> varlen FP8
attention -> per-token-group quantize) captured once in a CUDA graph and
replayed: every replay must give the eager path's bytes exactly (ring state,
descales, attention output, group codes and scales), and the eager path must
match the oracle.  Nothing on the path synchronizes with the host, and the
dynamic scale lives in a device ring, so the whole forward is capturable."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_attn_close, bf16_bits_to_f64

pytestmark = pytest.mark.gpu

fv = pytest.importorskip("fp8_quantized_vit_b200")


def _inputs(f, T, H, D):
    return [synth.bf16_tensor(synth.stream_key(901, f, t), T, H * D) for t in range(3)]


def _dev_bf16(bits, T, H, D):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16) \
        .reshape(T, H, D).cuda()


@pytest.mark.parametrize("lens,H,D", [((300, 190), 4, 72), ((640,), 2, 128)])
def test_graph_replay_matches_eager_and_oracle(lens, H, D):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    cu_d = torch.from_numpy(cu).cuda()
    ctx = fv.Context()
    eager = fv.FP8EncoderAttention(H, D, ctx=ctx)
    graphed = fv.FP8EncoderAttention(H, D, ctx=ctx)
    group = 128 if (H * D) % 128 == 0 else 32
    n_groups = H * D // group
    # static input / output buffers of the graph
    sq, sk, sv = (torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    g_xq = torch.empty((T, H * D), dtype=torch.uint8, device="cuda")
    g_xs = torch.empty((T, n_groups), dtype=torch.float32, device="cuda")

    def forward(layer, q, k, v, xq, xs):
        o = layer(q, k, v, cu_d, max(lens))
        fv.per_token_group_quant_fp8(o.view(T, H * D), group, xq, xs, ctx=ctx)
        return o

    # forward 0 eagerly on both layers (allocates the layers' buffers, sets
    # the kernel attributes) so that capture sees a steady state
    x0 = [_dev_bf16(b, T, H, D) for b in _inputs(0, T, H, D)]
    e_xq, e_xs = torch.empty_like(g_xq), torch.empty_like(g_xs)
    forward(eager, *x0, e_xq, e_xs)
    for s, x in zip((sq, sk, sv), x0):
        s.copy_(x)
    forward(graphed, sq, sk, sv, g_xq, g_xs)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            g_out = forward(graphed, sq, sk, sv, g_xq, g_xs)
    torch.cuda.current_stream().wait_stream(cap)
    # capture recorded the forward without running it: restore the ring to
    # the eager layer's state after forward 0 before the first replay
    graphed.ring.copy_(eager.ring)
    graphed.descale.copy_(eager.descale)

    ring_o = oracle.Ring()
    ring_o.update([oracle.amax_bf16(b) for b in _inputs(0, T, H, D)])
    sm = np.float32(1.0 / math.sqrt(D))
    for f in range(1, 20):  # the ring wraps after 16 forwards
        bits = _inputs(f, T, H, D)
        x = [_dev_bf16(b, T, H, D) for b in bits]
        e_out = forward(eager, *x, e_xq, e_xs)
        for s, xx in zip((sq, sk, sv), x):
            s.copy_(xx)
        graph.replay()
        torch.cuda.synchronize()
        st, site = ctx.check()
        assert st == fv.OK, (fv.status_string(st), site)
        assert torch.equal(graphed.ring, eager.ring), f
        assert torch.equal(graphed.descale, eager.descale), f
        assert torch.equal(g_out.view(torch.int16), e_out.view(torch.int16)), f
        assert torch.equal(g_xq, e_xq), f
        assert torch.equal(g_xs.view(torch.int32), e_xs.view(torch.int32)), f
        desc = ring_o.update([oracle.amax_bf16(b) for b in bits])
        assert (np.asarray(desc, np.float32).view(np.uint32) ==
                eager.descale.cpu().numpy().view(np.uint32)).all(), f
        if f in (1, 17):
            codes = [oracle.quantize_per_tensor(b, d).reshape(T, H, D) for b, d in zip(bits, desc)]
            ref = oracle.attn_full(*codes, *desc, cu, H, D, sm)
            got = bf16_bits_to_f64(e_out.view(torch.int16).cpu().numpy().view(np.uint16))
            assert_attn_close(got, ref, ("graph forward", f))
    del graph
    ctx.close()
