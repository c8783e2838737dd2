"""Pins for the oracle's fp64 varlen attention.

Invariants (probabilities sum to one, constant V, identical keys, single-key
segments, key permutation, no cross-segment leak), a closed form for two
keys (the logistic form of a two-way softmax), and torch's fp64 softmax
attention on the dequantised tensors as a library cross-check.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _random_codes(rng, shape, lo=0x20, hi=0x50):
    """Random finite e4m3 codes with both signs (magnitudes ~2^-3 .. 2^3)."""
    c = rng.integers(lo, hi, size=shape).astype(np.uint8)
    return c | np.where(rng.random(shape) < 0.5, 0x80, 0).astype(np.uint8)


def _case(rng, lens, H, D):
    T = int(sum(lens))
    q8 = _random_codes(rng, (T, H, D))
    k8 = _random_codes(rng, (T, H, D))
    v8 = _random_codes(rng, (T, H, D))
    return q8, k8, v8, synth.cu_seqlens(lens)


def _torch_attention(q8, k8, v8, dq, dk, dv, cu, H, D, sm_scale):
    dec = torch.from_numpy(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    q = dec[torch.from_numpy(q8.astype(np.int64))] * dq
    k = dec[torch.from_numpy(k8.astype(np.int64))] * dk
    v = dec[torch.from_numpy(v8.astype(np.int64))] * dv
    outs = []
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        qi = q[a:b].permute(1, 0, 2)  # [H, S, D]
        ki = k[a:b].permute(1, 0, 2)
        vi = v[a:b].permute(1, 0, 2)
        s = torch.matmul(qi, ki.transpose(1, 2)) * float(sm_scale)
        p = torch.softmax(s, dim=-1)
        outs.append(torch.matmul(p, vi).permute(1, 0, 2))
    return torch.cat(outs, 0).numpy()


@pytest.mark.parametrize("lens,H,D", [((7,), 2, 8), ((5, 1, 9), 3, 72), ((33,), 1, 128)])
def test_matches_torch_fp64(lens, H, D):
    rng = np.random.default_rng(sum(lens) * 31 + D)
    q8, k8, v8, cu = _case(rng, lens, H, D)
    dq, dk, dv = np.float32(0.37), np.float32(1.9), np.float32(0.011)
    sm = np.float32(1.0 / math.sqrt(D))
    got = oracle.attn_full(q8, k8, v8, dq, dk, dv, cu, H, D, sm)
    ref = _torch_attention(q8, k8, v8, float(dq), float(dk), float(dv), cu, H, D, float(sm))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_probabilities_sum_to_one():
    rng = np.random.default_rng(5)
    q8, k8, v8, cu = _case(rng, (40, 13), 2, 16)
    toks = np.arange(53)
    _, ps = oracle.attn_pairs(q8, k8, v8, 1.0, 1.0, 1.0, cu, 2, 16, 0.25, toks,
                              np.zeros(53, np.int32), want_psum=True)
    assert np.abs(ps - 1.0).max() < 1e-12


def test_constant_v_gives_v():
    rng = np.random.default_rng(6)
    q8, k8, v8, cu = _case(rng, (31,), 2, 8)
    v8[:] = 0x3A  # 1.25
    out = oracle.attn_full(q8, k8, v8, 1.0, 1.0, 0.5, cu, 2, 8, 0.3)
    assert np.abs(out - 0.625).max() < 1e-13


def test_identical_keys_give_mean_of_v():
    rng = np.random.default_rng(8)
    q8, k8, v8, cu = _case(rng, (17,), 1, 8)
    k8[:] = k8[0]
    out = oracle.attn_full(q8, k8, v8, 1.0, 1.0, 1.0, cu, 1, 8, 0.5)
    vals = oracle.e4m3_decode(v8)
    np.testing.assert_allclose(out, np.broadcast_to(vals.mean(axis=0), out.shape), rtol=1e-13,
                               atol=1e-15)


def test_single_key_segment_is_exact():
    rng = np.random.default_rng(9)
    q8, k8, v8, cu = _case(rng, (4, 1, 3), 2, 8)
    out = oracle.attn_full(q8, k8, v8, 1.0, 1.0, 0.75, cu, 2, 8, 0.5)
    assert (out[4] == oracle.e4m3_decode(v8[4]) * np.float64(np.float32(0.75))).all()


def test_key_permutation_invariance():
    rng = np.random.default_rng(10)
    q8, k8, v8, cu = _case(rng, (23,), 2, 16)
    perm = rng.permutation(23)
    a = oracle.attn_full(q8, k8, v8, 1.0, 1.0, 1.0, cu, 2, 16, 0.25)
    b = oracle.attn_full(q8, k8[perm], v8[perm], 1.0, 1.0, 1.0, cu, 2, 16, 0.25)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_packed_equals_separate_segments():
    rng = np.random.default_rng(11)
    lens = (9, 14, 5)
    q8, k8, v8, cu = _case(rng, lens, 2, 8)
    packed = oracle.attn_full(q8, k8, v8, 0.5, 2.0, 1.0, cu, 2, 8, 0.4)
    for i, L in enumerate(lens):
        a, b = int(cu[i]), int(cu[i + 1])
        alone = oracle.attn_full(q8[a:b], k8[a:b], v8[a:b], 0.5, 2.0, 1.0, synth.cu_seqlens([L]),
                                 2, 8, 0.4)
        assert (alone == packed[a:b]).all()


def test_two_key_closed_form():
    # With two keys the softmax weight of key 1 is the logistic function of
    # the score difference: o = v2 + (v1 - v2) / (1 + exp(s2 - s1)).
    dec = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    q8 = np.array([[[0x40]], [[0x38]]], dtype=np.uint8)      # 2.0 | 1.0
    k8 = np.array([[[0x38]], [[0xB0]]], dtype=np.uint8)      # 1.0 | -0.5
    v8 = np.array([[[0x48]], [[0xC4]]], dtype=np.uint8)      # 4.0 | -3.0
    cu = synth.cu_seqlens([2])
    sm = 0.75
    out = oracle.attn_full(q8, k8, v8, 1.0, 1.0, 1.0, cu, 1, 1, sm)
    for t in range(2):
        qv = dec[q8[t, 0, 0]]
        s1, s2 = sm * qv * dec[k8[0, 0, 0]], sm * qv * dec[k8[1, 0, 0]]
        v1, v2 = dec[v8[0, 0, 0]], dec[v8[1, 0, 0]]
        want = v2 + (v1 - v2) / (1.0 + math.exp(s2 - s1))
        assert abs(out[t, 0, 0] - want) < 1e-14


def test_fp8_output_reference():
    o = np.array([0.0, 1.0, -2.5, 1000.0, 1e-9], dtype=np.float64)
    got = oracle.fp8_output(o, 0.5)
    assert list(got) == [0x00, 0x40, 0xCA, 0x7E, 0x00]


def test_rejects_bad_pairs():
    rng = np.random.default_rng(12)
    q8, k8, v8, cu = _case(rng, (4,), 1, 8)
    with pytest.raises(ValueError):
        oracle.attn_pairs(q8, k8, v8, 1, 1, 1, cu, 1, 8, 1.0, [5], [0])
    with pytest.raises(ValueError):
        oracle.attn_pairs(q8, k8, v8, 1, 1, 1, cu, 1, 8, 1.0, [1], [1])
