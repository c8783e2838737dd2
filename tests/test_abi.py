"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-only entry points (status strings, descale rule,
scale-file reader/writer, argument checks) behave as documented.  No CUDA
compute is launched here."""
import ctypes
import json
import os
import re

import numpy as np
import pytest
import torch

import fp8_quantized_vit_b200 as fv
from fp8_quantized_vit_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8vit.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "scale_file_example.json")


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    yield


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["fp8_amax_ring_update", "fp8_quantize_qkv_per_tensor", "fp8_varlen_attn_fwd",
              "per_token_group_quant_fp8", "fp8_static_scales_load", "fp8_static_scales_save",
              "fp8_descale_from_amax", "fp8vit_create", "fp8vit_check"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fv.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(fv, "_lib", None)
    monkeypatch.setattr(fv, "LIB_PATH", os.path.join(ROOT, "does-not-exist.so"))
    with pytest.raises(RuntimeError):
        fv.lib()


def test_version_and_status_strings():
    assert fv.lib().fp8vit_version() >= 100
    for s in range(8):
        assert fv.status_string(s)
    assert fv.status_string(fv.ETIMEOUT).startswith("bounded wait")


def test_descale_from_amax():
    assert fv.fp8_descale_from_amax(224.0) == 0.5
    assert fv.fp8_descale_from_amax(0.0) == float(np.float32(1e-10))
    assert fv.fp8_descale_from_amax(198.0) == float(np.float32(198.0) / np.float32(448.0))


def test_scale_file_golden_example():
    # vLLM "FP8 ViT Encoder Attention", Scale File Format: the printed example.
    assert fv.fp8_static_scales_load(GOLDEN, "visual.blocks.0.attn.attn") == (224.0, 198.0, 210.0)
    assert fv.fp8_static_scales_load(GOLDEN, "visual.blocks.1.attn.attn") == (218.0, 195.0, 207.0)
    d = [fv.fp8_descale_from_amax(x) for x in (224.0, 198.0, 210.0)]
    assert d[0] == 0.5


def test_scale_file_aliases_and_errors(tmp_path):
    p = tmp_path / "s.json"
    p.write_text(json.dumps({"a": {"q_scale": 1.5, "k_scale": 2.0, "v_scale": 3.25},
                             "b": {"q": 1, "k": 2, "v": 3, "extra": [1, {"x": None}]}}))
    assert fv.fp8_static_scales_load(str(p), "a") == (1.5, 2.0, 3.25)
    assert fv.fp8_static_scales_load(str(p), "b") == (1.0, 2.0, 3.0)
    with pytest.raises(fv.FP8VitError) as e:
        fv.fp8_static_scales_load(str(p), "missing")
    assert e.value.status == fv.ENOTFOUND
    with pytest.raises(fv.FP8VitError) as e:
        fv.fp8_static_scales_load(str(tmp_path / "nope.json"), "a")
    assert e.value.status == fv.EIO
    bad = tmp_path / "bad.json"
    for text in ['{"a": {"q": 1, "k": 2}}',                      # v missing
                 '{"a": {"q": 1, "q_scale": 2, "k": 1, "v": 1}}',  # conflicting alias
                 '{"a": {"q": 1, "k": 2, "v": 3}',                 # truncated
                 '{"a": {"q": "x", "k": 2, "v": 3}}',              # not a number
                 '{"a": {"q": 1, "k": 2, "v": 3}} trailing',
                 '{"a": {"q": -1, "k": 2, "v": 3}}',               # an amax is not negative
                 '{"a": {"q": 1, "k": 1e39, "v": 3}}',             # beyond fp32
                 '{"a": {"q": 1, "k": 2, "v": 1e99999}}']:         # beyond fp64
        bad.write_text(text)
        with pytest.raises(fv.FP8VitError) as e:
            fv.fp8_static_scales_load(str(bad), "a")
        assert e.value.status == fv.EPARSE, text
    # both spellings with the same value are accepted
    bad.write_text('{"a": {"q": 1, "q_scale": 1.0, "k": 2, "v": 3}}')
    assert fv.fp8_static_scales_load(str(bad), "a") == (1.0, 2.0, 3.0)


def test_scale_file_round_trip_with_margin(tmp_path):
    rng = np.random.default_rng(1)
    amax = (rng.random((3, 3)) * 40).astype(np.float32)
    layers = [f"visual.blocks.{i}.attn.attn" for i in range(3)]
    p = str(tmp_path / "cal.json")
    fv.fp8_static_scales_save(p, layers, amax, margin=1.5)
    json.load(open(p))  # valid JSON
    for i, name in enumerate(layers):
        got = fv.fp8_static_scales_load(p, name)
        want = tuple(float(np.float32(1.5) * a) for a in amax[i])
        assert got == want


def test_descale_with_margin_equals_a_saved_and_reloaded_file(tmp_path):
    """The margin applied in C (fp8_descale_from_amax_margin) gives the same
    descales as saving the amax with that margin and loading the file back."""
    rng = np.random.default_rng(2)
    amax = (rng.random((4, 3)) * 60).astype(np.float32)
    amax[0, 0] = 0.0
    layers = [f"l{i}" for i in range(4)]
    p = str(tmp_path / "m.json")
    for margin in (1.5, 1.25, 2.0):
        fv.fp8_static_scales_save(p, layers, amax, margin=margin)
        for i, name in enumerate(layers):
            via_file = [fv.fp8_descale_from_amax(x) for x in fv.fp8_static_scales_load(p, name)]
            direct = [fv.fp8_descale_from_amax_margin(float(a), margin) for a in amax[i]]
            assert direct == via_file, (margin, i)


def test_attn_p_terms_setting_is_checked_on_the_host():
    lib = fv.lib()
    fake_ctx = ctypes.create_string_buffer(64)  # host-only call: the struct is never on the GPU
    assert lib.fp8vit_set_attn_p_terms(None, 2) == fv.EINVAL
    for bad in (0, 3, -1):
        assert lib.fp8vit_set_attn_p_terms(fake_ctx, bad) == fv.EINVAL
    assert lib.fp8vit_set_attn_p_terms(fake_ctx, 1) == fv.OK
    assert lib.fp8vit_set_attn_p_terms(fake_ctx, 2) == fv.OK


def test_new_entry_points_check_arguments_on_the_host():
    lib = fv.lib()
    fake_ctx = ctypes.create_string_buffer(64)
    dummy = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10001)
    # BF16 attention: head_dim outside {72, 128}, misaligned input, null output
    assert lib.bf16_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, 1, 8, 8, 2, 64, 0.1,
                                    dummy, None) == fv.EUNSUPPORTED
    assert lib.bf16_varlen_attn_fwd(fake_ctx, odd, dummy, dummy, dummy, 1, 8, 8, 2, 72, 0.1,
                                    dummy, None) == fv.EINVAL
    assert lib.bf16_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, 1, 8, 8, 2, 72, 0.1,
                                    None, None) == fv.EINVAL
    assert lib.bf16_varlen_attn_fwd(None, dummy, dummy, dummy, dummy, 1, 8, 8, 2, 72, 0.1,
                                    dummy, None) == fv.EINVAL
    # failure-injection hooks need a context
    assert lib.fp8vit_inject_lost_arrival(None, None) == fv.EINVAL
    assert lib.fp8vit_inject_attn_timeout(None, None) == fv.EINVAL
    # the dynamic-path entry point: negative size
    assert lib.fp8_amax_ring_quantize_qkv(fake_ctx, dummy, dummy, dummy, -1, dummy, dummy, dummy,
                                          dummy, dummy, None) == fv.EINVAL


def test_host_argument_checks_need_no_gpu():
    lib = fv.lib()
    fake_ctx = ctypes.create_string_buffer(64)
    dummy = ctypes.c_void_p(0x10000)  # never dereferenced: the checks return first
    # null context / pointers
    assert lib.fp8_varlen_attn_fwd(None, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1, 8,
                                   8, 2, 72, 0.1, dummy, 0, None, None) == fv.EINVAL
    # head_dim outside {72, 128}
    assert lib.fp8_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 2, 64, 0.1, dummy, 0, None, None) == fv.EUNSUPPORTED
    # odd head count at head_dim 72: a token row is not a multiple of 16 bytes
    assert lib.fp8_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 3, 72, 0.1, dummy, 0, None, None) == fv.EUNSUPPORTED
    # FP8 output needs an output scale and BF16 output must not get one
    assert lib.fp8_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 2, 72, 0.1, dummy, 1, None, None) == fv.EINVAL
    assert lib.fp8_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 2, 72, 0.1, dummy, 0, dummy, None) == fv.EINVAL
    # non-positive softmax scale
    assert lib.fp8_varlen_attn_fwd(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 2, 72, 0.0, dummy, 0, None, None) == fv.EINVAL
    # misaligned q8
    odd = ctypes.c_void_p(0x10001)
    assert lib.fp8_varlen_attn_fwd(fake_ctx, odd, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                   8, 8, 2, 72, 0.1, dummy, 0, None, None) == fv.EINVAL
    # fused attention + group quant: head_dim 72 (groups straddle heads), null outputs
    assert lib.fp8_varlen_attn_fwd_group_quant(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy,
                                               dummy, 1, 8, 8, 2, 72, 0.1, dummy, dummy,
                                               None) == fv.EUNSUPPORTED
    assert lib.fp8_varlen_attn_fwd_group_quant(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy,
                                               dummy, 1, 8, 8, 2, 128, 0.1, None, dummy,
                                               None) == fv.EINVAL
    assert lib.fp8_varlen_attn_fwd_group_quant(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy,
                                               dummy, 1, 8, 8, 2, 128, 0.1, dummy, odd,
                                               None) == fv.EINVAL
    # attention + group tail: head_dim outside {72, 128}, H * D not a multiple of
    # 128, null counters, misaligned output
    gt = lib.fp8_varlen_attn_fwd_bf16_group_quant
    args = lambda H, D, out=dummy, cnt=dummy: (fake_ctx, dummy, dummy, dummy, dummy, dummy,
                                               dummy, dummy, 1, 8, 8, H, D, 0.1, out, dummy,
                                               dummy, cnt, None)
    assert gt(*args(16, 64)) == fv.EUNSUPPORTED
    assert gt(*args(2, 72)) == fv.EINVAL
    assert gt(*args(16, 72, cnt=None)) == fv.EINVAL
    assert gt(*args(16, 72, out=odd)) == fv.EINVAL
    # an empty batch passes every check and returns before any launch
    assert gt(fake_ctx, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1, 8, 0, 160, 128, 0.1,
              dummy, dummy, dummy, dummy, None) == fv.OK
    # group quant: n not a multiple of group, unsupported group
    assert lib.per_token_group_quant_fp8(fake_ctx, dummy, 4, 200, 128, dummy, dummy,
                                         None) == fv.EINVAL
    assert lib.per_token_group_quant_fp8(None, dummy, 4, 256, 128, dummy, dummy,
                                         None) == fv.EINVAL
    # quantizers: negative size, misaligned input
    assert lib.fp8_quantize_qkv_per_tensor(fake_ctx, dummy, dummy, dummy, -1, dummy, dummy,
                                           dummy, dummy, None) == fv.EINVAL
    assert lib.fp8_amax_ring_update(fake_ctx, odd, dummy, dummy, 8, dummy, dummy,
                                    None) == fv.EINVAL
    # fused amax + ring + quantize: null K output (a null Q output is allowed:
    # fp8_varlen_attn_fwd_qbf16 quantizes Q itself), misaligned ring
    assert lib.fp8_amax_ring_quantize_qkv(fake_ctx, dummy, dummy, dummy, 8, dummy, dummy, dummy,
                                          None, dummy, None) == fv.EINVAL
    assert lib.fp8_amax_ring_quantize_qkv(fake_ctx, dummy, dummy, dummy, 8, odd, dummy, dummy,
                                          dummy, dummy, None) == fv.EINVAL


def test_layer_buffers_grow_to_the_largest_token_count_and_are_reused():
    """The layer keeps one set of buffers per output type, sized for the
    largest token count seen; a smaller call gets views of their first rows
    (contiguous, no new allocation), a larger one replaces them."""
    layer = object.__new__(fv.FP8EncoderAttention)
    layer.H, layer.D, layer.device, layer._bufs = 16, 72, torch.device("cpu"), {}
    b = layer._buffers(300, False)
    assert b["q8"].shape == (300, 16, 72) and b["out"].dtype == torch.bfloat16
    base = b["q8"].data_ptr()
    s = layer._buffers(129, False, group_quant=True)
    assert s["q8"].data_ptr() == base and s["q8"].shape == (129, 16, 72)
    assert all(t.is_contiguous() for t in s.values())
    assert s["xq"].shape == (129, 1152) and s["xs"].shape == (129, 9)
    assert s["out"].view(129, 1152).shape == (129, 1152)
    assert layer._buffers(300, False)["q8"].data_ptr() == base
    f = layer._buffers(200, True)
    assert f["out"].dtype == torch.uint8 and f["q8"].data_ptr() != base
    g = layer._buffers(301, False)
    assert g["q8"].shape == (301, 16, 72) and len(layer._bufs) == 2
    assert layer._bufs[False]["cap"] == 301


def test_scale_file_loader_survives_damaged_files(tmp_path):
    """Every prefix of a valid scale file, and files with seeded byte damage,
    load or fail with a status (no crash, no read past the text); a file the
    loader accepts gives finite values.  Run in a child process, so that a
    crash in the C++ reader fails this test instead of the whole session."""
    import subprocess
    import sys
    script = r'''
import os, random, sys
sys.path.insert(0, sys.argv[1])
import fp8_quantized_vit_b200 as fv
text = open(sys.argv[2], "rb").read()
p = os.path.join(sys.argv[3], "d.json")
rng = random.Random(7)
cases = [text[:i] for i in range(len(text) + 1)]
for _ in range(400):
    b = bytearray(text)
    for _ in range(rng.randint(1, 4)):
        b[rng.randrange(len(b))] = rng.choice(b'{}[]":,.-+eE0123456789 \\\x00\xff')
    cases.append(bytes(b))
cases += [b"", b"{", b'{"a":', b'{"a": {"q": 1e99999, "k": 1, "v": 1}}', b"[" * 5000,
          b'{"a": {"q": -1, "k": 1, "v": 1}}', b'"' + b"x" * 100000]
ok = bad = 0
for c in cases:
    open(p, "wb").write(c)
    try:
        vals = fv.fp8_static_scales_load(p, "visual.blocks.0.attn.attn")
        assert all(v == v and abs(v) != float("inf") for v in vals), vals
        ok += 1
    except fv.FP8VitError as e:
        assert e.status in (fv.EPARSE, fv.ENOTFOUND, fv.EIO), e.status
        bad += 1
print(ok, bad)
'''
    r = subprocess.run([sys.executable, "-c", script, ROOT, GOLDEN, str(tmp_path)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    ok, bad = map(int, r.stdout.split())
    assert ok >= 1 and bad >= 100


def test_boundary_is_usable_from_plain_c(tmp_path):
    """A C11 program that includes only include/fp8vit.h, compiled with
    warnings as errors and linked against libfp8vit.so, runs the calls that
    need no GPU (tests/abi_from_c.c)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_from_c"
    libdir = os.path.dirname(fv.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "abi_from_c.c"), "-L", libdir, "-lfp8vit",
                           f"-Wl,-rpath,{libdir}", "-lm", "-o", str(exe)])
    r = subprocess.run([str(exe), GOLDEN, str(tmp_path / "s.json")], capture_output=True,
                       text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stderr)


def test_noalloc_entry_point_is_bound_and_checks_on_the_host():
    lib = fv.lib()
    dummy = ctypes.c_void_p(0x10000)  # never dereferenced: the checks return first
    f = lib.fp8_amax_ring_update_noalloc
    assert f.argtypes is not None and len(f.argtypes) == 7
    assert f(None, dummy, dummy, 8, dummy, dummy, None) == fv.EINVAL
    assert f(dummy, dummy, dummy, -1, dummy, dummy, None) == fv.EINVAL
    assert f(ctypes.c_void_p(0x10002), dummy, dummy, 8, dummy, dummy, None) == fv.EINVAL
    assert callable(fv.fp8_amax_ring_update_noalloc)


def test_pointer_checks_refuse_host_tensors_without_a_gpu():
    """The binding's argument check refuses a host tensor (and, on the same
    path, reports non-contiguous tensors and wrong dtypes) before any call
    into the library; the current-stream accessor it uses exists in torch."""
    t = torch.zeros(4, 4, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fv._ptr(t, fv._FP8, "x")
    with pytest.raises(ValueError, match="CUDA tensor"):
        fv._ptr(t.t(), torch.uint8, "x")
    assert fv._ptr(None, torch.float32) is None
    assert fv._raw_stream is not None and fv._cur_device is not None


def test_layer_constructor_runs_without_a_gpu(monkeypatch):
    """FP8EncoderAttention's constructor on host memory with a stand-in
    context: the descale views alias the descale vector (a static-scale
    update through copy_ reaches them), a dynamic layer gets a ring, and the
    default softmax scale is the fp32 rounding of head_dim ** -0.5."""
    import types
    ctx = types.SimpleNamespace(handle=None)
    layer = fv.FP8EncoderAttention(16, 72, device="cpu", ctx=ctx, static_amax=[448.0, 896.0, 1.5])
    assert layer.ring is None and layer.group_tail is False and layer.fold_q is False
    for view, i in zip((layer._dq, layer._dk, layer._dv), range(3)):
        assert view.data_ptr() == layer.descale[i:i + 1].data_ptr()
    assert float(layer._dq) == 1.0 and float(layer._dk) == 2.0
    assert layer.softmax_scale == float(np.float32(72 ** -0.5))
    # a dynamic layer asks for a device ring (ring_init refuses host memory)
    monkeypatch.setattr(fv, "new_ring", lambda device=None: torch.zeros(fv.RING_BYTES // 4))
    dyn = fv.FP8EncoderAttention(4, 128, device="cpu", ctx=ctx, group_tail=True)
    assert dyn.ring is not None and dyn.ring.numel() * dyn.ring.element_size() == fv.RING_BYTES
    assert dyn.group_tail and float(dyn.descale.abs().sum()) == 0.0


def test_tile_counter_workspace_covers_every_counter_index():
    """The counter workspace the binding sizes for the group tail holds every
    counter the kernel indexes: the kernel counts (query tile, group) pairs at
    (seg_start / 128 + tile + segment) * groups + group, distinct for distinct
    pairs because cu_seqlens is a cumulative sum.  Random ragged layouts,
    empty images and single tokens included."""
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 12))
        lens = rng.integers(0, 700, size=n)
        lens[rng.random(n) < 0.2] = int(rng.integers(0, 3))
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        T = int(cu[-1])
        groups = int(rng.choice([9, 16, 18]))
        size = fv.tile_counters_size(T, n, groups * 128)
        seen = set()
        for seg in range(n):
            for qt in range((int(lens[seg]) + 127) // 128):
                for g in range(groups):
                    idx = ((int(cu[seg]) >> 7) + qt + seg) * groups + g
                    assert 0 <= idx < size, (trial, seg, qt, g, idx, size)
                    assert idx not in seen
                    seen.add(idx)
