"""Pins for the oracle's amax, ring, scale and quantizer rules.

* amax: brute force over the bf16 values.
* ring: hand-derived sequences (tests/golden/ring_sequences.txt).
* per-tensor quantizer and group quantizer: an independent torch-CPU
  restatement of the rule (torch's fp32 division, clamp and float8 cast),
  and hand values: scales of exactly 1 and 2 map grid values to the golden
  e4m3 codes, saturation, ties to the even code.
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


def _golden_grid():
    """(code, value) of every finite, non-negative-zero row of the golden e4m3
    table (tests/golden/e4m3_codes.txt, from the OCP format definition)."""
    path = os.path.join(os.path.dirname(__file__), "golden", "e4m3_codes.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        v = float(val)
        if np.isfinite(v) and not (v == 0.0 and np.signbit(v)):
            rows.append((int(code, 16), v))
    return rows


def _bf16_bits(values) -> np.ndarray:
    """BF16 bit patterns of values that BF16 holds exactly (every e4m3 value
    and its doubles do: 3 mantissa bits against BF16's 7)."""
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert (bits & 0xFFFF == 0).all()
    return (bits >> 16).astype(np.uint16)


def test_per_tensor_quant_hand_values():
    """With descale 1 (amax-domain value 448) a value on the e4m3 grid maps to
    its own code; with descale 1/2 (amax 224) twice that value does; beyond
    ±448 the code saturates; a tie between two codes goes to the even one."""
    grid = _golden_grid()
    codes = np.array([c for c, _ in grid], dtype=np.uint8)
    vals = [v for _, v in grid]
    d1 = oracle.descale_from_amax(448.0)
    d_half = oracle.descale_from_amax(224.0)
    assert d1 == 1.0 and d_half == 0.5
    assert (oracle.quantize_per_tensor(_bf16_bits(vals), d1) == codes).all()
    assert (oracle.quantize_per_tensor(_bf16_bits([v / 2 for v in vals]), d_half) == codes).all()
    sat = oracle.quantize_per_tensor(_bf16_bits([512.0, -1024.0, 464.0]), d1)
    assert list(sat) == [0x7E, 0xFE, 0x7E]
    # 1.0625 lies halfway between 1.0 (0x38, mantissa 000) and 1.125 (0x39):
    # the even code wins; 1.1875 between 1.125 and 1.25 (0x3A) goes up to 0x3A
    ties = oracle.quantize_per_tensor(_bf16_bits([1.0625, 1.1875, -1.0625]), d1)
    assert list(ties) == [0x38, 0x3A, 0xB8]


def test_group_quant_hand_values():
    """A group whose amax is 448 has scale 448/448 = 1, so its codes are the
    grid values' own codes; a group with amax 896 has scale 2 and the codes of
    half its values; the scales are stored as amax/448 (not its inverse)."""
    grid = _golden_grid()
    codes = np.array([c for c, _ in grid], dtype=np.uint8)
    vals = [v for _, v in grid]
    k = len(vals)
    assert 448.0 in vals and k < 128
    pad = [0.0] * (128 - k)
    row = vals + pad + [2 * v for v in vals] + pad
    x = _bf16_bits(row).reshape(1, 256)
    xq, sc = oracle.group_quant(x, 128)
    assert sc[0, 0] == np.float32(1.0) and sc[0, 1] == np.float32(2.0)
    assert (xq[0, :k] == codes).all() and (xq[0, 128:128 + k] == codes).all()
    assert (xq[0, k:128] == 0).all() and (xq[0, 128 + k:] == 0).all()
