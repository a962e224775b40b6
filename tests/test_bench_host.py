"""Host-side arithmetic of bench.py on CPU: the algorithmic bytes behind every GB/s
and roofline figure, and the rule that ncu traffic counters apply only to the kernel
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
