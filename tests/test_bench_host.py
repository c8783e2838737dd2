"""CPU checks of the benchmark's host logic: the traffic record is used only
for the kernel source it was captured on, the workload description names
the shape, the roofline denominators come from the measured peaks, and the
group-quantizer table holds the benchmark page's 19 shapes."""
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
