"""Pins for the oracle's amax, ring, scale and quantizer rules.

* amax: brute force over the bf16 values.
* ring: hand-derived sequences (tests/golden/ring_sequences.txt).
* per-tensor quantizer and group quantizer: an independent torch-CPU
  restatement of the rule (torch's fp32 division, clamp and float8 cast).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ring_sequences.txt")


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def test_amax_brute_force():
    x = synth.bf16_tensor(synth.stream_key(9, 0, 0), 257, 72, n_out=1)
    want = float(np.max(np.abs(synth.bf16_to_float(x))))
    assert oracle.amax_bf16(x) == want
    # order does not matter
    assert oracle.amax_bf16(x[::-1].copy()) == want
    assert oracle.amax_bf16(np.zeros(5, np.uint16)) == 0.0
    # a negative extreme counts by magnitude
    y = np.array([0x3F80, 0xC100, 0x4000], dtype=np.uint16)  # 1, -8, 2
    assert oracle.amax_bf16(y) == 8.0


def test_descale_hand_values():
    assert oracle.descale_from_amax(224.0) == 0.5
    assert oracle.descale_from_amax(448.0) == 1.0
    assert oracle.descale_from_amax(0.0) == float(np.float32(1e-10))
    assert oracle.descale_from_amax(198.0) == float(np.float32(198.0) / np.float32(448.0))


def _ring_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, seq, maxes = [p.strip() for p in line.split("|")]
        seq = [float(v) for v in seq.split()]
        maxes = [float(v) for v in maxes.split()]
        assert len(seq) == len(maxes), name
        rows.append((name, seq, maxes))
    return rows


@pytest.mark.parametrize("row", _ring_rows(), ids=lambda r: r[0])
def test_ring_hand_sequences(row):
    name, seq, maxes = row
    ring = oracle.Ring()
    for f, (a, m) in enumerate(zip(seq, maxes)):
        # q follows the sequence; k and v follow scaled copies of it
        d = ring.update([a, 2 * a, a / 4])
        assert d[0] == oracle.descale_from_amax(m), (name, f)
        assert d[1] == oracle.descale_from_amax(2 * m), (name, f)
        assert d[2] == oracle.descale_from_amax(m / 4), (name, f)
    assert ring.pos[0] == len(seq) % 16


def test_ring_wraps_every_16():
    ring = oracle.Ring()
    for f in range(40):
        ring.update([1.0, 1.0, 1.0])
        assert ring.pos[0] == (f + 1) % 16


def _torch_per_tensor(bits, descale):
    x = _bf16(bits).float()
    y = (x / torch.tensor(descale, dtype=torch.float32)).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_per_tensor_quant_matches_torch_restatement(seed):
    w = synth.Workload("t", (333,), 4, 72, "static", (seed,))
    q, k, v = w.qkv(0)
    for x in (q, k, v):
        amax = oracle.amax_bf16(x)
        descale = oracle.descale_from_amax(np.float32(1.5) * np.float32(amax))
        got = oracle.quantize_per_tensor(x, descale)
        assert (got == _torch_per_tensor(x, descale)).all()
        # the exact amax (no margin) reaches exactly +-448
        tight = oracle.quantize_per_tensor(x, oracle.descale_from_amax(amax))
        assert (tight & 0x7F).max() == 0x7E


def _torch_group_quant(bits, group):
    x = _bf16(bits).float()
    m, n = x.shape
    g = x.reshape(m, n // group, group)
    amax = g.abs().amax(dim=-1)
    scale = torch.clamp(amax / 448.0, min=1e-10)
    y = (g / scale.unsqueeze(-1)).clamp(-448.0, 448.0)
    return y.reshape(m, n).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), scale.numpy()


@pytest.mark.parametrize("m,n", [(1, 2048), (37, 2048), (5, 7168), (97, 1152), (3, 128)])
def test_group_quant_matches_torch_restatement(m, n):
    x = synth.bf16_tensor(synth.stream_key(77, m, n), m, n)
    xq, sc = oracle.group_quant(x, 128)
    rq, rs = _torch_group_quant(x, 128)
    assert (xq == rq).all()
    assert (sc.view(np.uint32) == rs.view(np.uint32)).all()


def test_group_quant_zero_group_and_clamp():
    x = np.zeros((2, 256), dtype=np.uint16)
    x[1, 128:] = 0x4000  # 2.0 everywhere in the second group of row 1
    xq, sc = oracle.group_quant(x, 128)
    assert (xq[0] == 0).all() and (xq[1, :128] == 0).all()
    assert sc[0, 0] == np.float32(1e-10) and sc[1, 0] == np.float32(1e-10)
    assert sc[1, 1] == np.float32(2.0) / np.float32(448.0)
    assert (xq[1, 128:] == 0x7E).all()   # x / (amax/448) lands on +448


def test_group_quant_rejects_ragged_n():
    with pytest.raises(ValueError):
        oracle.group_quant(np.zeros((1, 200), np.uint16), 128)
