"""bench.py host logic on the CPU: the roofline arithmetic and the recorded-traffic lookup."""
import json

import bench
from seeded_inputs import workload

PEAKS = {"bf16_tflops": 1653.3, "bf16_tflops_sustained": 1396.4, "hbm_gbs": 6544.0}


def test_roofline_tensor_bound():
    w = workload("yolo_highres_80x80_b16")
    t = w.flops / 800e12  # a launch that reaches 800 TFLOP/s
    r = bench.roofline(w, t, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 800.0) < 0.01 and abs(r["frac"] - 800.0 / 1653.3) < 1e-4
    rs = bench.roofline(w, t, PEAKS, sustained=True)
    assert abs(rs["frac"] - 800.0 / 1396.4) < 1e-4


def test_roofline_hbm_bound_below_the_ridge_point():
    w = workload("yolo_c2psa_20x20")  # 200 FLOP per byte, ridge point 253
    assert w.flops / w.bytes < 1653.3e12 / 6544e9
    t = w.bytes / 1000e9
    r = bench.roofline(w, t, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 1000.0) < 0.1


def test_recorded_traffic_only_for_current_sources(tmp_path, monkeypatch):
    path = tmp_path / "traffic.json"
    doc = {"kernel": "k", "kernel_source_sha": bench.kernel_source_sha(),
           "workloads": {"yolo_neck_40x40_b16": {"dram_bytes_per_launch": 123.0}}}
    path.write_text(json.dumps(doc))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("yolo_neck_40x40_b16") == 123.0
    assert bench.recorded_traffic("long_context_32k") is None
    doc["kernel_source_sha"] = "0" * 16  # counters taken on other sources
    path.write_text(json.dumps(doc))
    assert bench.recorded_traffic("yolo_neck_40x40_b16") is None


def test_both_arms_print_the_same_config(capsys, monkeypatch):
    """The reference arm's config dict is the GPU arm's, key for key."""
    import argparse
    w = workload("yolo_c2psa_20x20")
    monkeypatch.setenv("RANK", "0")
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    args = argparse.Namespace(gpus=1, steps=1, warmup=0)
    monkeypatch.setattr(bench, "time_oracle_sample",
                        lambda *a, **k: (w.flops / (w.B * w.H), 0.5, 1))
    bench.run_reference(args, w)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.bench_config(w, 1)


def test_percentiles():
    st = bench.percentiles([float(x) for x in range(1, 101)])
    assert st["median"] == 50.5 and abs(st["p10"] - 10.9) < 1e-9 and abs(st["p90"] - 90.1) < 1e-9


def test_fp8_configs_fit_the_entry_point():
    """The FP8 leg's shapes meet attn_fwd_fp8's rules (d = 128 is implied; Nk a multiple of 16),
    the long-context one matches the bf16 long-context workload, and --part fp8 finds a config
    for every workload name."""
    for name, B, H, N, causal, qk in bench.FP8_CONFIGS:
        assert N % 16 == 0 and B >= 1 and H >= 1
    w = workload("long_context_32k")
    _, B, H, N, causal, qk = bench.fp8_config("long_context_32k")
    assert (B, H, N, causal, qk) == (w.B, w.H, w.Nq, w.causal, w.qk_scale) and w.d == 128
    assert bench.fp8_config("yolo_highres_80x80_b16_d128")[2:4] == (2, 6400)
