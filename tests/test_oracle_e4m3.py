"""Pins for the oracle's e4m3 codec: the format definition (golden codes),
a library routine (torch's float8_e4m3fn), exhaustive round trips, every
rounding midpoint, saturation, and a brute-force nearest-grid search."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_codes.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        rows.append((int(code, 16), float(val)))
    return rows


def test_decode_golden_codes():
    rows = _golden()
    assert len(rows) >= 20
    for code, val in rows:
        got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        if math.isnan(val):
            assert math.isnan(got), hex(code)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()
    assert (np.signbit(ours[~nan]) == np.signbit(ref[~nan])).all()
    assert nan.sum() == 2  # 0x7F and 0xFF only


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    back = oracle.e4m3_encode(vals)
    assert (back == codes).all()


def _positive_grid():
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E
    return codes, oracle.e4m3_decode(codes)


def test_midpoints_round_to_even_code():
    codes, vals = _positive_grid()
    mids = (vals[:-1] + vals[1:]) / 2.0  # exact in fp64, and representable in fp32
    assert (mids.astype(np.float32).astype(np.float64) == mids).all()
    got = oracle.e4m3_encode(mids.astype(np.float32))
    lo, hi = codes[:-1], codes[1:]
    want = np.where(lo % 2 == 0, lo, hi)
    assert (got == want).all()
    # negative side mirrors with the sign bit
    gotn = oracle.e4m3_encode(-mids.astype(np.float32))
    assert (gotn == (want | 0x80)).all()
    # one fp32 ulp either side of a midpoint goes to the nearer code
    up = np.nextafter(mids.astype(np.float32), np.float32(np.inf))
    dn = np.nextafter(mids.astype(np.float32), np.float32(0))
    assert (oracle.e4m3_encode(up) == hi).all()
    assert (oracle.e4m3_encode(dn) == lo).all()


def test_saturation_and_specials():
    x = np.array([448.0, 448.0001, 463.9, 464.0, 480.0, 1e6, 3e38, np.inf,
                  -448.0, -500.0, -np.inf, 0.0, -0.0, 1e-30, -1e-30, np.nan],
                 dtype=np.float32)
    got = oracle.e4m3_encode(x)
    want = [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E,
            0xFE, 0xFE, 0xFE, 0x00, 0x80, 0x00, 0x80, 0x7F]
    assert list(got) == want


def _random_floats(rng, n):
    mag = np.exp2(rng.uniform(-14.0, 9.5, n))
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    return (sign * mag).astype(np.float32)


def test_brute_force_nearest_grid_point():
    rng = np.random.default_rng(12345)
    codes, vals = _positive_grid()
    for _ in range(10):
        x = _random_floats(rng, 100_000)
        a = np.minimum(np.abs(x.astype(np.float64)), 448.0)
        dist = np.abs(a[:, None] - vals[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # ties: the even code among the (at most two) nearest
        idx_even = np.where(cand & (codes[None, :] % 2 == 0), codes[None, :], 255).min(axis=1)
        idx_any = np.where(cand, codes[None, :], 255).min(axis=1)
        want = np.where(idx_even != 255, idx_even, idx_any).astype(np.uint8)
        want = want | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
        assert (oracle.e4m3_encode(x) == want).all()


def test_matches_torch_cast_within_range():
    rng = np.random.default_rng(7)
    x = _random_floats(rng, 1_000_000)
    x = np.clip(x, -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (oracle.e4m3_encode(x) == ref).all()


def test_bf16_rounding_matches_torch():
    # fp32-representable inputs: torch's float -> bfloat16 cast is then a
    # single round-to-nearest-even step, like ours.
    rng = np.random.default_rng(3)
    d = (rng.standard_normal(20000) * np.exp2(rng.uniform(-20, 20, 20000))).astype(np.float32)
    d = d.astype(np.float64)
    ref = torch.from_numpy(d).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.double_to_bf16(v) for v in d], dtype=np.uint16)
    assert (got == ref).all()
