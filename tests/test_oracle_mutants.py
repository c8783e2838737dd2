"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (a wrong rounding, a
dropped term, a wrong index or sign, a swapped operand), builds it, and runs
the compact pins below against it: at least one pin must fail for every
mutant, and all pins must pass for the unmodified source."""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import synth

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("rounding toward zero", "double mant = rint((s - 1.0) * 8.0);",
     "double mant = floor((s - 1.0) * 8.0);"),
    ("saturation at 480", "if (a >= ORC_E4M3_MAX) return", "if (a >= 480.0) return"),
    ("exponent bias 8", "v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("subnormal step 2^-8", "double k = rint(a * 512.0);", "double k = rint(a * 256.0);"),
    ("sign dropped", "return (uint8_t)(sign | (uint8_t)(((ex + 7) << 3) | (int)mant));",
     "return (uint8_t)((uint8_t)(((ex + 7) << 3) | (int)mant));"),
    ("ring wraps at 15", "*pos = (p + 1) % ORC_RING_SLOTS;", "*pos = (p + 1) % 15;"),
    ("ring max over 15 slots", "for (int j = 0; j < ORC_RING_SLOTS; ++j) {",
     "for (int j = 1; j < ORC_RING_SLOTS; ++j) {"),
    ("descale by reciprocal", "float d = v / 448.0f;", "float d = v * (1.0f / 447.0f);"),
    ("no scale floor", "return d > ORC_SCALE_FLOOR ? d : ORC_SCALE_FLOOR;", "return d;"),
    ("group amax over half the group", "for (int32_t i = 0; i < group; ++i) {\n                float a = fabsf",
     "for (int32_t i = 0; i < group / 2; ++i) {\n                float a = fabsf"),
    ("group scale not divided by 448", "float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    ("group scale floor dropped", "if (s < ORC_SCALE_FLOOR) s = ORC_SCALE_FLOOR;", ""),
    ("group amax of signed values", "float a = fabsf(orc_bf16_to_float(xs[i]));",
     "float a = orc_bf16_to_float(xs[i]);"),
    ("group quantize multiplies by the scale", "float y = orc_bf16_to_float(xs[i]) / s;",
     "float y = orc_bf16_to_float(xs[i]) * s;"),
    ("per-tensor quantize multiplies by the descale", "orc_bf16_to_float(x[i]) / descale);",
     "orc_bf16_to_float(x[i]) * descale);"),
    ("softmax scale dropped", "s[j - a] = (double)sm_scale * acc;", "s[j - a] = acc;"),
    ("key of head 0", "const uint8_t* kj = k8 + j * row + (int64_t)h * D;",
     "const uint8_t* kj = k8 + j * row;"),
    ("v descale dropped", "o[d] += p * (table[vj[d]] * (double)dv);", "o[d] += p * table[vj[d]];"),
    ("key row off by one", "const uint8_t* kj = k8 + j * row + (int64_t)h * D;",
     "const uint8_t* kj = k8 + (j > a ? j - 1 : j) * row + (int64_t)h * D;"),
    ("v read with the k pointer", "const uint8_t* vj = v8 + j * row", "const uint8_t* vj = k8 + j * row"),
    # the BF16 attention (the comparator's reference)
    ("bf16: key of head 0", "const uint16_t* kj = k + j * row + (int64_t)h * D;",
     "const uint16_t* kj = k + j * row;"),
    ("bf16: v read with the k pointer", "const uint16_t* vj = v + j * row",
     "const uint16_t* vj = k + j * row"),
    ("bf16: query of head 0", "qv[d] = (double)orc_bf16_to_float(q[t * row + (int64_t)h * D + d]);",
     "qv[d] = (double)orc_bf16_to_float(q[t * row + d]);"),
    ("bf16: score without the softmax scale",
     "for (int32_t d = 0; d < D; ++d) acc += qv[d] * (double)orc_bf16_to_float(kj[d]);\n            s[j - a] = (double)sm_scale * acc;",
     "for (int32_t d = 0; d < D; ++d) acc += qv[d] * (double)orc_bf16_to_float(kj[d]);\n            s[j - a] = acc;"),
]


def _build(tmp_path, text, name):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           str(src), "-o", str(lib), "-lm"])
    return str(lib)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _pins():
    """Compact pins (each returns True when it holds)."""
    out = {}
    # e4m3: golden values from the format definition, torch decode / cast
    golden = {0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x7E: 448.0, 0xB8: -1.0, 0x70: 128.0}
    dec = oracle.e4m3_decode(np.array(list(golden), dtype=np.uint8))
    out["golden decode"] = bool(np.all(dec == np.array(list(golden.values()))))
    rng = np.random.default_rng(1)
    x = (np.where(rng.random(20000) < 0.5, -1, 1) *
         np.exp2(rng.uniform(-12, 9.2, 20000))).astype(np.float32)
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    out["torch cast"] = bool(np.all(oracle.e4m3_encode(x) == ref))
    out["saturation"] = list(oracle.e4m3_encode(np.array([460.0, 470.0, -1e9], np.float32))) == [0x7E, 0x7E, 0xFE]
    # descale hand values and the floor
    out["descale"] = (oracle.descale_from_amax(224.0) == 0.5 and
                      oracle.descale_from_amax(0.0) == float(np.float32(1e-10)))
    # ring: falling sequence keeps 20 for 16 forwards, then 19, 18
    ring = oracle.Ring()
    got = [float(ring.update([a, a, a])[0]) for a in range(20, 0, -1)]
    want = [oracle.descale_from_amax(m) for m in [20.0] * 16 + [19.0, 18.0, 17.0, 16.0]]
    out["ring"] = got == want and int(ring.pos[0]) == 4
    # per-tensor quantize vs a torch restatement, and two hand values
    xp = synth.bf16_tensor(synth.stream_key(4, 1, 1), 5, 256)
    d = np.float32(1.5) * np.float32(oracle.amax_bf16(xp)) / np.float32(448.0)
    rp = (_bf16(xp).float() / torch.tensor(d)).clamp(-448, 448).to(torch.float8_e4m3fn)
    out["per-tensor quant"] = bool(
        (oracle.quantize_per_tensor(xp, float(d)).reshape(-1) ==
         rp.view(torch.uint8).numpy().reshape(-1)).all() and
        list(oracle.quantize_per_tensor(np.array([0x4000, 0xC080], np.uint16), 0.5)) == [0x48, 0xD0])
    # group quant vs a torch restatement (row 0's first group all zeros)
    xg = synth.bf16_tensor(synth.stream_key(3, 1, 1), 7, 512)
    xg[0, :128] = 0
    xq, sc = oracle.group_quant(xg, 128)
    t = _bf16(xg).float().reshape(7, 4, 128)
    s = torch.clamp(t.abs().amax(-1) / 448.0, min=1e-10)
    rq = (t / s.unsqueeze(-1)).clamp(-448, 448).reshape(7, 512).to(torch.float8_e4m3fn)
    out["group quant"] = bool((xq == rq.view(torch.uint8).numpy()).all() and
                              (sc == s.numpy()).all())
    # attention vs torch fp64 on two segments, two heads
    lens, H, D = (9, 6), 2, 8
    cu = synth.cu_seqlens(lens)
    c = rng.integers(0x28, 0x48, size=(3, 15, H, D)).astype(np.uint8)
    c |= np.where(rng.random(c.shape) < 0.5, 0x80, 0).astype(np.uint8)
    dq, dk, dv, sm = 0.5, 1.25, 0.75, float(np.float32(0.3))
    got = oracle.attn_full(c[0], c[1], c[2], dq, dk, dv, cu, H, D, sm)
    # decode with torch's float8 table (independent of the oracle's decoder)
    tab = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    q, k, v = (tab[torch.from_numpy(c[i].astype(np.int64))] * f
               for i, f in enumerate((dq, dk, dv)))
    ok = True
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        sc_ = torch.einsum("shd,thd->hst", q[a:b], k[a:b]) * sm
        o = torch.einsum("hst,thd->shd", torch.softmax(sc_, -1), v[a:b]).numpy()
        ok &= np.allclose(got[a:b], o, rtol=1e-12, atol=1e-14)
    out["attention"] = bool(ok)
    # BF16 attention vs torch fp64 on the same values
    xb = [synth.bf16_tensor(synth.stream_key(5, 2, t), 15, H * D) for t in range(3)]
    got = oracle.attn_full_bf16(*xb, cu, H, D, sm)
    qb, kb, vb = (_bf16(x).to(torch.float64).reshape(15, H, D) for x in xb)
    ok = True
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        sc_ = torch.einsum("shd,thd->hst", qb[a:b], kb[a:b]) * sm
        o = torch.einsum("hst,thd->shd", torch.softmax(sc_, -1), vb[a:b]).numpy()
        ok &= np.allclose(got[a:b], o, rtol=1e-12, atol=1e-14)
    out["bf16 attention"] = bool(ok)
    return out


def test_pins_hold_for_the_oracle():
    res = _pins()
    assert all(res.values()), res


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_each_planted_mistake_is_caught(tmp_path, name, orig, bad):
    text = open(SRC).read()
    assert orig in text, f"mutation anchor not found: {name}"
    lib = _build(tmp_path, text.replace(orig, bad, 1), "m" + str(abs(hash(name)) % 10 ** 8))
    with oracle.use_library(lib):
        res = _pins()
    assert not all(res.values()), f"no pin caught: {name}"
