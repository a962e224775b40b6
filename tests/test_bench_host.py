"""Host-side arithmetic of bench.py on CPU: the algorithmic bytes behind every GB/s
and roofline figure, the step statistics, and the rule that ncu traffic counters apply only to the kernel
sources they were taken on."""
import json

import bench
import synth

H, E, I, Is = 7168, 896, 1024, 2048


def test_batch_1_step_bytes_written_out():
    # router E x H + shared gate/up/down 3 x Is x H + 16 experts x 3 x I x H (bf16),
    # gamma H (bf16), x and y one row each (bf16)
    router = E * H * 2
    shared = 3 * Is * H * 2
    experts = 16 * 3 * I * H * 2
    gamma = H * 2
    rows = 2 * 1 * H * 2
    assert (router, shared, experts) == (12_845_056, 88_080_384, 704_643_072)
    assert bench.step_bytes(synth.WORKLOADS[1], [16]) == router + shared + experts + gamma + rows == 805_611_520


def test_step_bytes_counts_each_unique_expert_once_and_rows_per_batch():
    wl = synth.WORKLOADS[2]  # batch 8, uniform router
    one_expert = 3 * I * H * 2
    assert bench.step_bytes(wl, [121]) - bench.step_bytes(wl, [120]) == one_expert
    # two more token rows add their x and y rows only
    assert bench.step_bytes(wl, [120], batch=10) - bench.step_bytes(wl, [120]) == 2 * 2 * H * 2


def test_step_bytes_includes_the_router_bias_and_every_layer():
    zipf = synth.WORKLOADS[3]
    uniform = synth.WORKLOADS[2]
    batch_rows = lambda wl: 2 * wl.B * H * 2
    assert (bench.step_bytes(zipf, [44]) - batch_rows(zipf)) - (bench.step_bytes(uniform, [44]) - batch_rows(uniform)) == 4 * E
    verify = synth.WORKLOADS[4]  # two layers, each with its own unique-expert count
    assert bench.step_bytes(verify, [80, 90]) == bench.step_bytes(verify, [80]) + bench.step_bytes(verify, [90])


def test_traffic_applies_only_to_the_captured_sources(tmp_path, monkeypatch):
    t = {"w": {"bytes_per_launch": 123, "kernel_sources_sha256": "abc"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(t))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.traffic_per_launch("w") == 123
    assert bench.traffic_per_launch("other") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "changed")
    assert bench.traffic_per_launch("w") is None


def test_ingest_traffic_matches_each_captured_launch_to_its_own_step(tmp_path, monkeypatch):
    """Captured launches (after -s skipped ones) are set beside the algorithmic bytes of
    the step they ran; a launch that runs a whole layer stack is set beside all of that
    step's layers."""
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "h")
    head = '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'

    def csv_of(kernel, vals):
        out = head
        for i, (r, w) in enumerate(vals):
            out += f'"{i}","{kernel}","dram__bytes_read.sum","byte","{r:,}"\n'
            out += f'"{i}","{kernel}","dram__bytes_write.sum","byte","{w}"\n'
        return out

    # one layer: steps 0..4, U differs per step; launches 3 and 4 captured
    wl = synth.WORKLOADS[2]
    log = [{"workload": wl.name, "step": s, "layer": 0, "timed": s >= 3, "unique_experts": 100 + s,
            "algorithmic_bytes": bench.step_bytes(wl, [100 + s])} for s in range(5)]
    (tmp_path / "log.json").write_text(json.dumps(log))
    (tmp_path / "a.csv").write_text(csv_of("moe_decode_layer_kernel<false,true>", [(5_000_000_000, 1000),
                                                                                    (5_100_000_000, 2000)]))
    t = bench.ingest_traffic(str(tmp_path / "a.csv"), str(tmp_path / "log.json"), wl.name, "ncu -s 3 -c 2 x")
    assert [l["step"] for l in t["launches"]] == [3, 4]
    assert t["launches"][0]["algorithmic_bytes"] == bench.step_bytes(wl, [103])
    assert t["launches"][1]["traffic"] == 5_100_002_000
    assert t["bytes_per_launch"] == round((5_000_001_000 + 5_100_002_000) / 2)
    assert bench.traffic_per_launch(wl.name) == t["bytes_per_launch"]
    # a two-layer stack in one launch per step: both layers' bytes of the step
    v = synth.WORKLOADS[4]
    log = [{"workload": v.name, "step": s, "layer": l, "timed": s >= 1, "unique_experts": 80 + l,
            "algorithmic_bytes": bench.step_bytes(v, [80 + l])} for s in range(3) for l in range(2)]
    (tmp_path / "log2.json").write_text(json.dumps(log))
    (tmp_path / "b.csv").write_text(csv_of("moe_decode_fused_kernel<false>", [(7_000_000_000, 0)]))
    t = bench.ingest_traffic(str(tmp_path / "b.csv"), str(tmp_path / "log2.json"), v.name, "ncu -s 1 -c 1 x")
    assert t["launches"][0]["step"] == 1
    assert t["launches"][0]["algorithmic_bytes"] == bench.step_bytes(v, [80, 81])


def test_step_stats_mean_is_the_back_to_back_figure_and_quantiles_the_per_step_times():
    per_step_ms = [0.170, 0.150, 0.152, 0.151, 0.153]
    s = bench.step_stats(per_step_ms, total_ms=0.745)  # 5 back-to-back steps: 149 us each
    assert s["us_per_step"] == 149.0
    assert s["us_per_step_median"] == 152.0
    assert s["us_per_step_max"] == 170.0 and s["slowest_step"] == 0
    assert bench.step_stats(per_step_ms)["us_per_step"] == 155.2  # no total: the per-step mean
