"""Shared test helpers: error metrics, row sampling, device transfers."""
from __future__ import annotations

import numpy as np

import synth


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_to_float(np.ascontiguousarray(bits)).astype(np.float64)


def bf16_half_ulp(ref: np.ndarray) -> np.ndarray:
    """Half the bfloat16 spacing at |ref| (the rounding error bound of a
    correctly rounded bf16 result)."""
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.exp2(e - 7)
    return np.where(a > 0, 0.5 * ulp, 0.0)


def attn_errors(got: np.ndarray, ref: np.ndarray) -> dict:
    """max-abs, mean-abs, excess over bf16 output rounding, cosine."""
    got = got.astype(np.float64).ravel()
    ref = ref.astype(np.float64).ravel()
    d = np.abs(got - ref)
    excess = np.maximum(0.0, d - bf16_half_ulp(ref))
    cos = float(np.dot(got, ref) / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    return dict(max_abs=float(d.max()), mean_abs=float(d.mean()), max_excess=float(excess.max()),
                cos=cos)


# The attention gate: max-abs 3e-2 (measured as excess over the bf16 rounding
# of the exact result), mean-abs 3e-3, cosine >= 0.999.
ATTN_MAX_EXCESS = 3e-2
ATTN_MEAN_ABS = 3e-3
ATTN_COS = 0.999


def assert_attn_close(got, ref, what=""):
    e = attn_errors(got, ref)
    assert e["max_excess"] <= ATTN_MAX_EXCESS, (what, e)
    assert e["mean_abs"] <= ATTN_MEAN_ABS, (what, e)
    assert e["cos"] >= ATTN_COS, (what, e)
    return e


def sample_pairs(cu: np.ndarray, heads: int, per_seg: int, seed: int, tile: int = 128):
    """(token, head) pairs per segment: its first, middle and last rows, both
    rows on every `tile`-row query-tile edge, and seeded random rows up to
    per_seg; the heads cycle through all of them (each segment starts at a
    different head), so every head and every tile edge is covered."""
    rng = np.random.default_rng(seed)
    toks, hs = [], []
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        L = b - a
        if L <= 0:
            continue
        fixed = {0, L - 1, L // 2, max(0, L - 129)}
        for k in range(1, (L - 1) // tile + 1):
            fixed |= {k * tile - 1, k * tile}
        fixed = sorted(r for r in fixed if r < L)
        rows = fixed + [int(r) for r in rng.integers(0, L, size=max(0, per_seg - len(fixed)))]
        for n, r in enumerate(rows):
            toks.append(a + int(r))
            hs.append(int((n + i) % heads))
    return np.array(toks, dtype=np.int64), np.array(hs, dtype=np.int32)


def complete_tile_pairs(cu: np.ndarray, heads: int, seed: int, tile: int = 128):
    """Every (token, head) pair of one full `tile`-row query tile per segment
    (a seeded choice among the segment's full tiles)."""
    rng = np.random.default_rng(seed)
    toks, hs = [], []
    for i in range(len(cu) - 1):
        a, L = int(cu[i]), int(cu[i + 1] - cu[i])
        if L < tile:
            continue
        t0 = int(rng.integers(0, L // tile)) * tile
        rows = np.arange(a + t0, a + t0 + tile, dtype=np.int64)
        toks.append(np.repeat(rows, heads))
        hs.append(np.tile(np.arange(heads, dtype=np.int32), tile))
    return np.concatenate(toks), np.concatenate(hs)


def oracle_pairs_threaded(fn, args, toks, hs, threads: int = 0):
    """Runs the oracle's per-pair attention (fn(*args, toks, hs)) over chunks
    of the pairs on several host threads (the C call releases the GIL) and
    concatenates the rows in order."""
    import concurrent.futures as cf
    import os
    n = len(toks)
    threads = threads or max(1, min(32, len(os.sched_getaffinity(0))))
    bounds = np.linspace(0, n, threads + 1).astype(int)
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(lambda k: fn(*args, toks[bounds[k]:bounds[k + 1]],
                                         hs[bounds[k]:bounds[k + 1]]), range(threads)))
    return np.concatenate(parts, axis=0)


def e4m3_half_step(y: np.ndarray) -> np.ndarray:
    """Half the e4m3 grid spacing at |y| (y already divided by the scale)."""
    a = np.minimum(np.abs(y), 448.0)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    step = np.where(a >= 2.0 ** -6, np.exp2(e - 3), 2.0 ** -9)
    return 0.5 * step


def fp8_output_errors(got_codes: np.ndarray, ref: np.ndarray, scale: float, decode) -> dict:
    """FP8-output errors in value space: |deq(got) - o| beyond half an e4m3
    step at o (the output format's own rounding; saturation at +-448*scale
    counts as exact), the e4m3 grid distance to the oracle's codes, cosine."""
    deq = decode(got_codes).astype(np.float64).ravel() * scale
    o = ref.astype(np.float64).ravel()
    oc = np.clip(o, -448.0 * scale, 448.0 * scale)
    excess = np.maximum(0.0, np.abs(deq - oc) - e4m3_half_step(o / scale) * scale)
    cos = float(np.dot(deq, o) / (np.linalg.norm(deq) * np.linalg.norm(o) + 1e-300))
    return dict(max_excess=float(excess.max()), mean_excess=float(excess.mean()), cos=cos)


def code_step_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in e4m3 grid steps between codes (sign-magnitude order)."""
    def ordinal(c):
        c = c.astype(np.int32)
        mag = c & 0x7F
        return np.where(c & 0x80, -mag, mag)
    return np.abs(ordinal(a) - ordinal(b))


def assert_fp8_out_close(got_codes, ref, scale, decode, what=""):
    e = fp8_output_errors(got_codes, ref, scale, decode)
    assert e["max_excess"] <= ATTN_MAX_EXCESS, (what, e)
    assert e["mean_excess"] <= ATTN_MEAN_ABS, (what, e)
    assert e["cos"] >= ATTN_COS, (what, e)
    return e
