"""CPU checks of the benchmark's host logic: the traffic record is used only
for the kernel source it was captured on, the workload description names
the shape, the roofline denominators come from the measured peaks, the
group-quantizer table holds the benchmark page's 19 shapes, and the CPU
leg's full-size parity check of forward 0 passes exact outputs and catches
wrong ones."""
import hashlib
import json
import os

import pytest

import bench
import synth


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// one version\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (prof / "traffic.json").write_text(json.dumps(
        {"wl": {"source_sha": sha, "dram_bytes_per_launch": 1234}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic(str(src), "wl") == 1234.0
    assert bench._traffic(str(src), "other") is None
    src.write_text("// another version\n")  # the kernel changed since the capture
    assert bench._traffic(str(src), "wl") is None


def test_committed_traffic_record_is_plausible():
    """When the record was taken on the current attention source, its DRAM
    bytes are those of reading Q, K and V once (50.3 MB) plus the writes that
    leave L2 during the launch; after a kernel change the bench reports null
    until the next capture, and this check has nothing to look at."""
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))[bench.WORKLOAD]
    src = os.path.join(bench.ROOT, "fp8_quantized_vit_b200", "csrc", "attn.cu")
    if rec["source_sha"] != bench._source_sha(src):
        pytest.skip("the attention source changed since the last capture")
    assert 50e6 < rec["dram_bytes_per_launch"] < 60e6


def test_config_names_the_workload_by_its_shape():
    w = synth.WORKLOADS[bench.WORKLOAD]
    c = bench._config(w)
    assert c["workload"].startswith("1x8192 tokens, 16 heads, head_dim 128")
    assert c["seq_lens"] == [8192] and c["heads"] == 16 and c["head_dim"] == 128
    assert c["forwards"] == 20
    assert w.attn_flops() == 4 * 8192 ** 2 * 128 * 16


def test_peaks_come_from_the_measured_file():
    p = bench._peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = json.load(open(path))
        assert p["hbm"] == m["hbm_gbs"] and p["bf16"] == m["bf16_tflops"]
    else:
        pytest.skip("no measured peaks on this machine")


def test_group_quant_table_is_the_pages_table():
    t = bench.GROUP_QUANT_TABLE
    assert len(t) == 19
    assert sum(1 for m, n, _, _ in t if n == 2048) == 10
    assert sum(1 for m, n, _, _ in t if n == 7168) == 9
    # the pages' speed-of-light column is bytes / a constant ~5.3 TB/s
    for m, n, t_sol, _ in t:
        if t_sol > 0:
            rate = (3 * m * n + 4 * m * n // 128) / (t_sol * 1e-6) / 1e12
            assert 5.0 < rate < 5.6, (m, n, rate)


def test_layered_workload_keeps_one_ring_per_layer():
    """The 3 x 32400 workload is 27 encoder layers, each with its own amax ring;
    the 8192-token workload is one layer over 20 forwards, one ring."""
    w = synth.WORKLOADS["3x32400_d72"]
    assert w.per_layer_rings and len(w.seeds) == 27
    assert bench._config(w)["rings"] == "one amax ring per layer (27 layers)"
    assert w.attn_flops() == 3 * 4 * 32400 ** 2 * 72 * 16
    w2 = synth.WORKLOADS[bench.WORKLOAD]
    assert not w2.per_layer_rings
    assert bench._config(w2)["rings"] == "one amax ring over the rotation"


def test_forward0_parity_check_on_the_host():
    """The CPU-baseline leg's full-size parity check: exact descales and codes
    with the oracle's rows rounded to BF16 pass; a wrong row, a wrong code or a
    descale one ulp off fail."""
    import numpy as np
    import torch

    import oracle
    w = synth.Workload("2 images, 300 + 77 tokens, 2 heads, head_dim 72", (300, 77), 2, 72,
                       "dynamic", (5,))
    codes, desc = bench._oracle_inputs(w)
    cu = synth.cu_seqlens(w.seg_lens)
    ref = oracle.attn_full(*codes, *desc, cu, w.heads, w.head_dim, w.softmax_scale)
    bits = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    good = bench._parity_from_outputs(w, codes, desc, np.asarray(desc, np.float32), codes, bits)
    assert good["within_gate"] and good["descales_bit_exact"] and good["codes_bit_exact"]
    assert good["max_excess_over_bf16_rounding"] < 1e-6 and good["cos"] > 0.99999
    assert good["rows"] == 2 * 32

    toks, hs = bench._sample_rows(cu, w.heads, 32, 11)
    assert ((toks >= 0) & (toks < 377)).all() and set(hs.tolist()) == {0, 1}
    assert {0, 127, 128, 299, 300, 376} <= set(toks.tolist())
    bad = bits.copy()
    bad[toks[3], hs[3]] ^= 0x0400  # one output off by many BF16 steps
    assert not bench._parity_from_outputs(w, codes, desc, desc, codes, bad)["within_gate"]
    wrong_codes = [c.copy() for c in codes]
    wrong_codes[1].reshape(-1)[7] ^= 1
    e = bench._parity_from_outputs(w, codes, desc, desc, wrong_codes, bits)
    assert not e["codes_bit_exact"] and not e["within_gate"]
    off = np.asarray(desc, np.float32).copy()
    off.view(np.uint32)[2] += 1
    e = bench._parity_from_outputs(w, codes, desc, off, codes, bits)
    assert not e["descales_bit_exact"] and not e["within_gate"]


def test_forward0_capture_marshals_the_kernels_outputs():
    """The bench's forward-0 capture, with the library's calls replaced by
    host stand-ins that write known bytes: it returns the descales, the three
    code tensors and the BF16 output bits as host arrays of the right shapes."""
    import types

    import numpy as np
    import torch

    T, H, D = 40, 2, 72
    w = synth.Workload("1 image, 40 tokens", (T,), H, D, "dynamic", (1,))
    calls = []

    import inspect

    import fp8_quantized_vit_b200 as fv

    def quant(q, k, v, ring, desc, q8, k8, v8, ctx=None):
        inspect.signature(fv.fp8_amax_ring_quantize_qkv).bind(q, k, v, ring, desc, q8, k8, v8,
                                                              ctx=ctx)
        calls.append("quant")
        desc.copy_(torch.tensor([0.5, 0.25, 0.125]))
        for i, t in enumerate((q8, k8, v8)):
            t.fill_(i + 1)

    def attn(q8, k8, v8, dq, dk, dv, cu, max_s, sm, out, ctx=None):
        inspect.signature(fv.fp8_varlen_attn_fwd).bind(q8, k8, v8, dq, dk, dv, cu, max_s, sm, out,
                                                       ctx=ctx)
        calls.append(("attn", float(dq[0]), float(dv[0]), max_s))
        out.fill_(1.5)

    fake = types.SimpleNamespace(
        new_ring=lambda dev: torch.zeros(64), OK=0, status_string=str,
        fp8_amax_ring_quantize_qkv=quant, fp8_varlen_attn_fwd=attn)
    ctx = types.SimpleNamespace(check=lambda: (0, 0))
    qkv0 = [torch.zeros((T, H, D), dtype=torch.bfloat16) for _ in range(3)]
    q8, k8, v8 = (torch.zeros((T, H, D), dtype=torch.uint8) for _ in range(3))
    out = torch.zeros((T, H, D), dtype=torch.bfloat16)
    desc, codes, bits = bench._forward0_outputs(fake, ctx, w, qkv0, torch.zeros(2), T, q8, k8, v8,
                                                out, "cpu")
    assert calls == ["quant", ("attn", 0.5, 0.125, T)]
    assert desc.dtype == np.float32 and list(desc) == [0.5, 0.25, 0.125]
    assert [c.shape for c in codes] == [(T, H, D)] * 3 and [int(c[0, 0, 0]) for c in codes] == [1, 2, 3]
    assert bits.dtype == np.uint16 and bits.shape == (T, H, D) and (bits == 0x3FC0).all()


def test_parity_field_reports_a_failed_check():
    assert bench._parity_field(None, None, None, RuntimeError("fault"))["error"].startswith(
        "RuntimeError")
    assert "error" in bench._parity_field(None, None, None, (None, None, None))


def test_bench_line_carries_every_contract_key():
    """The JSON line built by the GPU arm names every key of the benchmark
    contract (read from the source: the arm itself needs a GPU)."""
    import ast
    src = open(bench.__file__).read()
    tree = ast.parse(src)
    run = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "run_ours")
    keys = set()
    for node in ast.walk(run):
        if isinstance(node, ast.Dict):
            keys |= {k.value for k in node.keys if isinstance(k, ast.Constant)}
        if isinstance(node, ast.Subscript) and isinstance(node.slice, ast.Constant):
            keys.add(node.slice.value)
    need = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
            "bound", "achieved", "peak", "frac", "traffic", "e2e", "h2d_bytes_per_step",
            "d2h_bytes_per_step", "gpu_launches", "clocks", "cpu_baseline", "cores", "kind",
            "sample", "parity_of_forward0"}
    assert need <= keys, need - keys


def test_reference_arm_prints_its_line(capsys):
    """`--impl reference` (the oracle on the host cores) prints one line with
    the contract keys, its own e2e and cpu_baseline, and impl = reference."""
    import types
    args = types.SimpleNamespace(workload="1x1024_d72", steps=1, warmup=0, ref_step_seconds=0.2)
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("1x1024 tokens")


def test_reference_arm_runs_on_rank_0_only(capsys, monkeypatch):
    """Under torchrun with N > 1 only rank 0 runs the oracle and prints; the
    other ranks exit 0 without work."""
    import types
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = types.SimpleNamespace(workload="1x1024_d72", steps=1, warmup=0, ref_step_seconds=0.2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out.strip() == ""


def test_output_modes_leg_calls_the_binding_as_declared(monkeypatch):
    """The optional output-mode timing leg, run on the CPU with stand-ins for
    the library calls and the CUDA events: every call binds to the real
    binding's signature, each mode runs, and the result has one entry per mode
    (three at head_dim 128)."""
    import inspect
    import types

    import numpy as np
    import torch

    import fp8_quantized_vit_b200 as fv

    seen = []

    def stand_in(name, effect=None):
        sig = inspect.signature(getattr(fv, name))

        def f(*a, **k):
            sig.bind(*a, **k)
            seen.append(name)
            if effect:
                effect(*a, **k)
        return f

    def amax3(q, k, v, out, ctx=None):
        out.copy_(torch.tensor([3.0, 4.0, 5.0]))

    def attn(*a, **k):
        a[9].fill_(1 if a[9].dtype == torch.uint8 else 2.0)

    fake = types.SimpleNamespace(
        OK=0, status_string=str,
        fp8_amax3=stand_in("fp8_amax3", amax3),
        fp8_descale_from_amax=lambda v: float(np.float32(v) / np.float32(448.0)),
        fp8_quantize_qkv_per_tensor=stand_in("fp8_quantize_qkv_per_tensor"),
        fp8_varlen_attn_fwd=stand_in("fp8_varlen_attn_fwd", attn),
        fp8_varlen_attn_fwd_group_quant=stand_in("fp8_varlen_attn_fwd_group_quant"))
    ctx = types.SimpleNamespace(check=lambda: (0, 0))

    class Ev:
        def __init__(self, enable_timing=False):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 1.0

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    for D in (72, 128):
        w = synth.Workload("1 image, 64 tokens", (64,), 2, D, "static", (1,))
        inputs = [[torch.zeros((64, 2, D), dtype=torch.bfloat16) for _ in range(3)]]
        seen.clear()
        res = bench._output_modes(fake, ctx, w, inputs, "cpu", reps=2, rounds=1)
        want = {"bf16", "fp8_output_scale"} | ({"fused_group_quant"} if D == 128 else set())
        assert set(res) == want
        assert all(r["ms"] == 0.5 and r["tflops"] > 0 for r in res.values())
        assert seen[:2] == ["fp8_amax3", "fp8_quantize_qkv_per_tensor"]
        assert ("fp8_varlen_attn_fwd_group_quant" in seen) == (D == 128)


def test_gpus_flag_launches_one_rank_per_gpu(monkeypatch):
    """`bench.py --gpus N` started without torch.distributed.run re-runs
    itself under it with N ranks on 127.0.0.1 (it never times one GPU and
    reports N); under a launcher whose WORLD_SIZE disagrees with --gpus it
    exits non-zero."""
    import sys as _sys
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    monkeypatch.setattr(_sys, "argv", ["bench.py", "--gpus", "4", "--steps", "3"])
    assert bench.main() == 0
    cmd = calls[0]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(_sys, "argv", ["bench.py", "--gpus", "4"])
    assert bench.main() == 2


def test_workload_paths_run_each_configurations_own_step(monkeypatch):
    """bench._Path, run on the CPU with stand-ins for the library calls:
    a static workload with FP8 output calibrates its descales from the exact
    amax with the margin and forms output_scale on the device (amax of the BF16
    output, then the ring rule) before any step, then each step quantizes with
    the static descales and runs the FP8-output attention with that scale; a
    27-layer dynamic workload gives each layer its own ring and adds the group
    quantizer."""
    import inspect
    import types

    import numpy as np
    import torch

    import fp8_quantized_vit_b200 as fv

    seen = []

    def stand_in(name, effect=None):
        sig = inspect.signature(getattr(fv, name))

        def f(*a, **k):
            sig.bind(*a, **k)
            seen.append((name, a, k))
            if effect:
                effect(*a, **k)
        return f

    def amax3(q, k, v, out, ctx=None):
        out.copy_(torch.tensor([3.0, 4.0, 5.0]))

    def push(amax3, ring, desc3, stream=None):
        desc3.copy_(amax3 / 448.0)

    fake = types.SimpleNamespace(
        OK=0, status_string=str,
        fp8_amax3=stand_in("fp8_amax3", amax3),
        fp8_descale_from_amax_margin=lambda a, m: float(np.float32(np.float32(m) * np.float32(a))
                                                        / np.float32(448.0)),
        fp8_ring_push=stand_in("fp8_ring_push", push),
        new_ring=lambda dev=None: torch.zeros(64),
        ring_init=stand_in("ring_init"),
        fp8_quantize_qkv_per_tensor=stand_in("fp8_quantize_qkv_per_tensor"),
        fp8_amax_ring_quantize_qkv=stand_in("fp8_amax_ring_quantize_qkv"),
        fp8_varlen_attn_fwd=stand_in("fp8_varlen_attn_fwd"),
        per_token_group_quant_fp8=stand_in("per_token_group_quant_fp8"),
        fp8_varlen_attn_fwd_bf16_group_quant=stand_in("fp8_varlen_attn_fwd_bf16_group_quant"),
        new_tile_counters=lambda t, n, hd, dev=None: torch.zeros(
            fv.tile_counters_size(t, n, hd), dtype=torch.int32))
    ctx = types.SimpleNamespace(check=lambda: (0, 0))
    T, H, D = 40, 2, 72
    w = synth.Workload("3 tiny images", (10, 10, 20), H, D, "static", (1,), fp8_out=True)
    inputs = [[torch.zeros((T, H, D), dtype=torch.bfloat16) for _ in range(3)]]
    path = bench._Path(fake, ctx, w, inputs, "cpu")
    names = [s[0] for s in seen]
    assert names == ["fp8_amax3", "fp8_quantize_qkv_per_tensor", "fp8_varlen_attn_fwd",
                     "fp8_amax3", "fp8_ring_push"]
    assert torch.equal(path.desc, torch.tensor([1.5 * 3, 1.5 * 4, 1.5 * 5]) / 448.0)
    assert abs(float(path.oscale) - 3.0 / 448.0) < 1e-9
    seen.clear()
    path.step(0)
    assert [s[0] for s in seen] == ["fp8_quantize_qkv_per_tensor", "fp8_varlen_attn_fwd"]
    attn = seen[1]
    assert attn[1][9].dtype == torch.uint8 and attn[2]["output_scale"] is path.oscale
    assert bench._launches_per_step(w, 126 << 20) == 2

    w27 = synth.WORKLOADS["3x32400_d72"]
    small = synth.Workload("27 tiny layers", (10, 10, 20), H, D, "dynamic", w27.seeds,
                           group_quant=True, per_layer_rings=True)
    inputs = [[torch.zeros((T, H, D), dtype=torch.bfloat16) for _ in range(3)] for _ in range(27)]
    seen.clear()
    path = bench._Path(fake, ctx, small, inputs, "cpu")
    assert len(path.rings) == 27 and seen == []
    for i in range(3):
        path.step(i)
    quant = [s for s in seen if s[0] == "fp8_amax_ring_quantize_qkv"]
    assert [q[1][3] is path.rings[i] for i, q in enumerate(quant)] == [True] * 3
    assert [s[0] for s in seen].count("per_token_group_quant_fp8") == 3
    assert bench._launches_per_step(w27, 126 << 20) == 4  # two quantizer kernels above 2 x L2
    # the same workload with the group quantizer as the attention launch's tail
    seen.clear()
    path = bench._Path(fake, ctx, small, inputs, "cpu", group_tail=True)
    path.step(0)
    assert [s[0] for s in seen] == ["fp8_amax_ring_quantize_qkv",
                                    "fp8_varlen_attn_fwd_bf16_group_quant"]
    assert seen[1][1][12] is path.counters
    assert path.counters.numel() == ((T + 127) // 128 + 3) * (H * D // 128)
