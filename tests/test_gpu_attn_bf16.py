"""GPU parity of the BF16 attention kernel (the FP8 path's comparator on the
same skeleton) against the fp64 oracle over the same BF16 inputs: every
output on small shapes (ragged tails, empty and single-token images, odd and
even heads, head_dim 72 and 128), sampled rows on the workload shapes.  Gate
as for the FP8 kernel: max-abs 3e-2 as excess over the bf16 rounding of the
exact result, mean-abs 3e-3, cosine >= 0.999."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_attn_close, bf16_bits_to_f64, sample_pairs

pytestmark = pytest.mark.gpu

fv = pytest.importorskip("fp8_quantized_vit_b200")


@pytest.fixture(scope="module")
def ctx():
    assert torch.cuda.is_available()
    return fv.Context()


def _run(ctx, x, cu, H, D, max_seqlen, sm):
    T = x[0].shape[0]
    dev = [torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
           .reshape(T, H, D).cuda() for a in x]
    out = torch.full((T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    fv.bf16_varlen_attn_fwd(*dev, torch.from_numpy(cu).cuda(), max_seqlen, sm, out, ctx=ctx)
    st, site = ctx.check()
    assert st == fv.OK, (fv.status_string(st), site)
    return bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))


SMALL = [((1,), 2, 72), ((2,), 2, 128), ((129,), 4, 72), ((300, 1, 77), 2, 72),
         ((256, 129), 2, 128), ((5, 0, 200), 2, 72), ((513,), 2, 128), ((96, 192, 97), 2, 72),
         ((64, 65, 191), 2, 128)]


@pytest.mark.parametrize("lens,H,D", SMALL)
def test_bf16_small_shapes_full_oracle(ctx, lens, H, D):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    x = [synth.bf16_tensor(synth.stream_key(sum(lens) + D + 3, 0, t), T, H * D) for t in range(3)]
    sm = np.float32(1.0 / math.sqrt(D))
    ref = oracle.attn_full_bf16(*x, cu, H, D, sm)
    got = _run(ctx, x, cu, H, D, max(lens), sm)
    assert not np.isnan(got).any()
    assert_attn_close(got, ref, (lens, H, D))


@pytest.mark.parametrize("name", ["1x1024_d72", "1x8192_d128", "1x16384_d72", "3x32400_d72"])
def test_bf16_workload_sampled_rows(ctx, name):
    w = synth.WORKLOADS[name]
    x = w.qkv(0)
    cu = synth.cu_seqlens(w.seg_lens)
    toks, hs = sample_pairs(cu, w.heads, per_seg=24, seed=len(name) + 1)
    ref = oracle.attn_pairs_bf16(*x, cu, w.heads, w.head_dim, w.softmax_scale, toks, hs)
    got = _run(ctx, x, cu, w.heads, w.head_dim, max(w.seg_lens), w.softmax_scale)
    e = assert_attn_close(got[toks, hs], ref, name)
    print(name, "bf16 errors", e)
    assert not np.isnan(got).any()
