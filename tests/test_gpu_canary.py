"""Canary bytes after every output buffer: each kernel writes exactly its
outputs and nothing past them.  Outputs are views at the front of larger
device buffers whose tail holds a known pattern; after the launch the tail
must be unchanged.  Ragged sizes put the last vector of each output at its
end.  (compute-sanitizer is not available on the GPUs these run on; this
and the oracle comparisons stand in for it.)"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

fv = pytest.importorskip("fp8_quantized_vit_b200")

CANARY = 4096  # bytes of pattern after each output


@pytest.fixture(scope="module")
def ctx():
    assert torch.cuda.is_available()
    return fv.Context()


def _guarded(nbytes: int):
    """A uint8 buffer of nbytes + CANARY; the tail is filled with 0xA5."""
    buf = torch.full((nbytes + CANARY,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf


def _tail_ok(buf, nbytes):
    return bool((buf[nbytes:] == 0xA5).all().item())


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("lens,H,D", [((300, 1, 77), 2, 72), ((129, 64), 2, 128)])
def test_attention_outputs_stay_inside(ctx, lens, H, D):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    x = [synth.bf16_tensor(synth.stream_key(T, D, t), T, H * D) for t in range(3)]
    desc = [oracle.descale_from_amax(np.float32(1.5) * np.float32(oracle.amax_bf16(a))) for a in x]
    codes = [torch.from_numpy(oracle.quantize_per_tensor(a, d).reshape(T, H, D)).cuda()
             for a, d in zip(x, desc)]
    d = [torch.tensor([v], dtype=torch.float32, device="cuda") for v in desc]
    cu_d = torch.from_numpy(cu).cuda()
    sm = float(np.float32(1.0 / math.sqrt(D)))
    n = T * H * D
    # bf16 output
    buf = _guarded(2 * n)
    out = buf[:2 * n].view(torch.bfloat16).view(T, H, D)
    fv.fp8_varlen_attn_fwd(*codes, *d, cu_d, max(lens), sm, out, ctx=ctx)
    assert ctx.check()[0] == fv.OK and _tail_ok(buf, 2 * n)
    # e4m3 output
    buf = _guarded(n)
    os_d = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    fv.fp8_varlen_attn_fwd(*codes, *d, cu_d, max(lens), sm, buf[:n].view(T, H, D),
                           output_scale=os_d, ctx=ctx)
    assert ctx.check()[0] == fv.OK and _tail_ok(buf, n)
    # BF16 kernel on the BF16 inputs
    buf = _guarded(2 * n)
    out = buf[:2 * n].view(torch.bfloat16).view(T, H, D)
    fv.bf16_varlen_attn_fwd(*(_bf16_dev(a).view(T, H, D) for a in x), cu_d, max(lens), sm, out,
                            ctx=ctx)
    assert ctx.check()[0] == fv.OK and _tail_ok(buf, 2 * n)
    if D == 128:
        # fused group quantizer: codes and scales
        qb, sb = _guarded(n), _guarded(4 * T * H)
        fv.fp8_varlen_attn_fwd_group_quant(*codes, *d, cu_d, max(lens), sm,
                                           qb[:n].view(T, H * D),
                                           sb[:4 * T * H].view(torch.float32).view(T, H), ctx=ctx)
        assert ctx.check()[0] == fv.OK and _tail_ok(qb, n) and _tail_ok(sb, 4 * T * H)


@pytest.mark.parametrize("n", [8 * 1000 + 5, 3 * (1 << 20) + 7])
def test_quantizer_outputs_stay_inside(ctx, n):
    x = [_bf16_dev(synth.bf16_tensor(synth.stream_key(n, 3, t), 1, n)[0]) for t in range(3)]
    desc = torch.zeros(3, dtype=torch.float32, device="cuda")
    ring = fv.new_ring()
    bufs = [_guarded(n) for _ in range(3)]
    fv.fp8_amax_ring_quantize_qkv(*x, ring, desc, *(b[:n] for b in bufs), ctx=ctx)
    assert ctx.check()[0] == fv.OK and all(_tail_ok(b, n) for b in bufs)
    bufs = [_guarded(n) for _ in range(3)]
    fv.fp8_quantize_qkv_per_tensor(*x, desc, *(b[:n] for b in bufs), ctx=ctx)
    assert ctx.check()[0] == fv.OK and all(_tail_ok(b, n) for b in bufs)


@pytest.mark.parametrize("m,n,group", [(7, 1152, 128), (4192, 7168, 128), (33, 256, 16)])
def test_group_quant_outputs_stay_inside(ctx, m, n, group):
    x = _bf16_dev(synth.bf16_tensor(synth.stream_key(m, n, 9), m, n)).view(m, n)
    qb, sb = _guarded(m * n), _guarded(4 * m * (n // group))
    fv.per_token_group_quant_fp8(x, group, qb[:m * n].view(m, n),
                                 sb[:4 * m * (n // group)].view(torch.float32).view(m, n // group),
                                 ctx=ctx)
    assert ctx.check()[0] == fv.OK
    assert _tail_ok(qb, m * n) and _tail_ok(sb, 4 * m * (n // group))
