"""Host-side helpers of bench.py (no GPU): the planted-key recall count."""

import numpy as np

import bench


def test_plant_recall_counts_listed_blocks():
    # 1 batch, 2 q heads, 4 query blocks of 128 tokens: rows are (head, query block)
    Hq, nqb = 2, 4
    lists = {0: [0], 1: [0, 1], 2: [1, 2], 3: [0, 3], 4: [0], 5: [1], 6: [0, 2], 7: [3]}
    rp = np.zeros(Hq * nqb + 1, dtype=np.int64)
    ci = []
    for row in range(Hq * nqb):
        ci += lists[row]
        rp[row + 1] = len(ci)
    ci = np.array(ci, dtype=np.int32)
    # plants: (b, kv head, key block, key pos, q head, query token)
    plants = [(0, 0, 2, 300, 0, 2 * 128 + 5),   # row 2 lists block 2: hit
              (0, 0, 1, 200, 1, 3 * 128 + 1),   # row 7 lists only block 3: miss
              (0, 0, 0, 10, 1, 2 * 128 + 64),   # row 6 lists block 0: hit
              (0, 0, 2, 290, 0, 3 * 128 + 9)]   # row 3 lists blocks 0, 3: miss
    assert bench._plant_recall(rp, ci, plants, Hq, nqb) == 0.5
    assert bench._plant_recall(rp, ci, [], Hq, nqb) == 0.0


def test_radius_quintile_share_is_a_distribution():
    import torch
    g = torch.Generator().manual_seed(5)
    Q = torch.randn(1, 512, 2, 128, generator=g)
    K = torch.randn(1, 512, 1, 128, generator=g)
    R = torch.rand(1, 1, 8, generator=g)
    share = bench.radius_quintile_share(Q, K, R, 64)
    assert len(share) == 5
    assert abs(sum(share) - 1.0) < 1e-3
    assert all(0.0 <= x <= 1.0 for x in share)


def test_reference_arm_line():
    # the oracle arm on a short prompt of the same workload: one JSON-ready
    # line with the contract's keys, its own cpu_baseline and e2e, and a
    # sampling time bounded by the total budget
    import argparse
    import json
    import time
    args = argparse.Namespace(steps=2, warmup=3, ref_step_budget=3.0, ref_total_budget=2.5, seq_len=4096)
    t0 = time.perf_counter()
    line = bench.run_reference(args)
    took = time.perf_counter() - t0
    json.dumps(line)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["steps"] == 2 and line["warmup"] == 3
    assert line["config"]["seq_len"] == 4096
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert took < 60


def test_attention_traffic_only_for_the_captured_build(tmp_path, monkeypatch):
    # the DRAM traffic figure is reported only for the 128K workload and only
    # while the attention sources hash to the build it was captured on
    import os
    import shutil
    assert bench.attn_traffic(32768) is None
    full = bench.WORKLOADS[bench.WORKLOAD].seqlen
    now = bench.attn_traffic(full)
    assert now in (bench.ATTN_TRAFFIC_BYTES, None)
    for f in bench.ATTN_TRAFFIC_SOURCES:
        os.makedirs(tmp_path / os.path.dirname(f), exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, f), tmp_path / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.attn_traffic(full) == now
    with open(tmp_path / bench.ATTN_TRAFFIC_SOURCES[0], "a") as fh:
        fh.write("\n// edited\n")
    assert bench.attn_traffic(full) is None


def test_reference_arm_reports_the_measured_sample_time():
    # ms_per_step is the time a step's sample took (so steps x ms_per_step
    # fits in the run); the whole-step time extrapolated from it has its own key
    import argparse
    import time
    args = argparse.Namespace(steps=2, warmup=3, ref_step_budget=3.0, ref_total_budget=2.5, seq_len=4096)
    t0 = time.perf_counter()
    line = bench.run_reference(args)
    took_ms = (time.perf_counter() - t0) * 1e3
    assert line["ms_per_step"] * (args.steps + args.warmup) <= took_ms
    assert line["extrapolated_ms_per_full_step"] >= line["ms_per_step"]


def test_roofline_entry_uses_the_burst_peak():
    peaks = {"bf16_tflops": 1700.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6400.0, "source": "measured"}
    r = bench.roofline_entry(850.0, peaks, 2.5e9)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["peak"] == 1700.0 and r["frac"] == 0.5
    assert r["peak_sustained"] == 1400.0 and abs(r["frac_of_sustained"] - 850.0 / 1400.0) < 1e-4
    assert r["traffic"] == 2.5e9 and "burst" in r["peak_kind"]


def test_ttft_ratios():
    r = bench.ttft_ratios(final_ms=0.25, reencode_ms=0.03, full_ms=10.0, final_pairs=1040, full_pairs=33930)
    assert r["time_ratio"] == 0.025
    assert r["time_ratio_with_reencode"] == 0.028
    assert abs(r["flops_ratio"] - 1040 / 33930) < 1e-5


def test_clock_sampler_leaves_no_file_in_the_repo(monkeypatch, tmp_path):
    # without a log directory the samples go to a temporary file that is
    # removed afterwards; nvidia-smi missing gives a labelled empty record
    import subprocess

    def no_smi(*a, **k):
        raise OSError("no nvidia-smi")
    monkeypatch.setattr(subprocess, "Popen", no_smi)
    c = bench.ClockSampler(0)
    assert not c.path.startswith(bench.ROOT)
    c.start()
    rec = c.stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvidia-smi unavailable"]
    import os
    assert not os.path.exists(c.path)
    kept = bench.ClockSampler(0, str(tmp_path))
    kept.start()
    kept.stop()
    assert os.path.exists(kept.path)
