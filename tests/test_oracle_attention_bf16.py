"""Pins for the oracle's fp64 attention over BF16 inputs (the BF16 side of
the pages' BF16-vs-FP8 attention comparison).

A cross-pin to the e4m3 oracle (BF16 tensors whose values are e4m3 grid
points, with unit descales, give the same fp64 result bit for bit: the two
functions then perform the same operations in the same order), torch's fp64
softmax attention on the same values, and the invariants: probabilities sum
to one, constant V, identical keys, a single-key segment, key permutation,
no leak across segments.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _bf16_of(x: np.ndarray) -> np.ndarray:
    """float64 values (exactly representable in bf16) -> bf16 bit patterns."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f64_of(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(seed, lens, H, D):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    x = [synth.bf16_tensor(synth.stream_key(seed, 0, t), T, H * D).reshape(T, H, D)
         for t in range(3)]
    return cu, x


def _torch_ref(x, cu, H, D, sm):
    q, k, v = (torch.from_numpy(_f64_of(a)) for a in x)
    outs = []
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        if b == a:
            continue
        qi, ki, vi = (t[a:b].permute(1, 0, 2) for t in (q, k, v))
        p = torch.softmax(float(sm) * qi @ ki.transpose(1, 2), dim=-1)
        outs.append((p @ vi).permute(1, 0, 2))
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("lens,H,D", [((7,), 2, 72), ((33, 0, 5), 3, 128), ((64, 17), 2, 72)])
def test_matches_torch_fp64(lens, H, D):
    cu, x = _case(sum(lens) + D, lens, H, D)
    sm = np.float32(1.0 / np.sqrt(D))
    got = oracle.attn_full_bf16(*x, cu, H, D, sm)
    want = _torch_ref(x, cu, H, D, sm)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_equals_e4m3_oracle_on_grid_values():
    """Codes decoded to bf16 (every finite e4m3 value is a bf16 value) with
    descales 1: both oracles compute the same sums in the same order."""
    rng = np.random.default_rng(3)
    lens, H, D = (40, 9), 2, 72
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    codes = [(rng.integers(0x20, 0x50, size=(T, H, D)) |
              np.where(rng.random((T, H, D)) < 0.5, 0x80, 0)).astype(np.uint8) for _ in range(3)]
    bf = [_bf16_of(oracle.e4m3_decode(c)) for c in codes]
    sm = np.float32(0.125)
    a = oracle.attn_full(*codes, 1.0, 1.0, 1.0, cu, H, D, sm)
    b = oracle.attn_full_bf16(*bf, cu, H, D, sm)
    assert np.array_equal(a, b)


def test_invariants():
    lens, H, D = (50, 1, 20), 2, 128
    cu, x = _case(11, lens, H, D)
    sm = np.float32(1.0 / np.sqrt(D))
    T = int(cu[-1])
    toks = np.arange(T, dtype=np.int64)
    hs = (toks % H).astype(np.int32)
    _, psum = oracle.attn_pairs_bf16(*x, cu, H, D, sm, toks, hs, want_psum=True)
    assert np.abs(psum - 1.0).max() < 1e-12
    # constant V -> o = V
    q, k, v = x
    vc = np.broadcast_to(v[:1], v.shape).copy()
    o = oracle.attn_full_bf16(q, k, vc, cu, H, D, sm)
    assert np.allclose(o, np.broadcast_to(_f64_of(v[:1]), o.shape), rtol=1e-14, atol=0)
    # identical keys -> mean of V over the segment
    kc = np.broadcast_to(k[:1], k.shape).copy()
    o = oracle.attn_full_bf16(q, kc, v, cu, H, D, sm)
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        assert np.allclose(o[a:b], _f64_of(v[a:b]).mean(axis=0, keepdims=True), atol=1e-12)
    # the single-key segment returns its value row
    o = oracle.attn_full_bf16(q, k, v, cu, H, D, sm)
    a = int(cu[1])
    assert np.array_equal(o[a], _f64_of(v[a]))
    # permuting the keys (and values) of a segment leaves o unchanged
    perm = np.arange(T)
    perm[:50] = np.random.default_rng(5).permutation(50)
    o2 = oracle.attn_full_bf16(q, k[perm], v[perm], cu, H, D, sm)
    assert np.allclose(o2, o, rtol=1e-12, atol=1e-13)
    # packed segments equal separate runs (no cross-segment leak)
    sep = oracle.attn_full_bf16(q[51:], k[51:], v[51:], synth.cu_seqlens((20,)), H, D, sm)
    assert np.array_equal(o[51:], sep)
