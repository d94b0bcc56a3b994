"""Host-side logic of bench.py (no GPU): the algorithmic work the roofline
fields divide by, which peak a stage is measured against, and the committed
DRAM-traffic records."""
import json
import os
import re

import pytest

import bench
from workloads import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1666.4, "bf16_tflops_sustained": 1363.8}


def test_sustained_peak_for_long_or_power_capped_regions():
    assert bench.sustained_region(1500.0, {})
    assert bench.sustained_region(200.0, {"reasons": ["sw_power_cap"]})
    assert not bench.sustained_region(200.0, {"reasons": []})
    assert not bench.sustained_region(999.0, {})


def test_workload_counts_1m_closed_forms():
    cfg = synth.get_config("1m")
    c = bench.workload_counts(cfg)
    # 2048 documents x 512 tokens; per token K and V (8 heads x 128 x bf16) and Kr (8 x 128 x bf16)
    assert cfg.ntok == 2048 * 512 and cfg.C == 2048 * 8
    assert c["pool_bytes"] == cfg.ntok * 6144 + cfg.C * 6144 + cfg.C * 8 * 4
    assert c["route_bytes"] == 16384 * 8 * 128 * 2
    assert c["route_flops"] == 2 * 512 * 8 * 128 * 16384
    # every query token i sees all Mmax memory rows and local rows 0..Lloc-Tq+i
    Tq, L, M = cfg.Tq, cfg.Lloc, cfg.Mmax
    pairs = Tq * (M + L - Tq) + Tq * (Tq + 1) // 2
    assert c["attn_flops"] == 4 * 128 * 32 * pairs


@pytest.mark.parametrize("name,stage,bound,unit", [
    ("100m", "route_topk", "hbm", "GB/s"),          # 64 query rows: 64 flop per byte, under the ridge
    ("decode16m", "route_topk", "hbm", "GB/s"),
    ("stack10m", "route_topk", "tensor", "TFLOP/s"),  # 4096 rows: above the ridge
    ("decode16m", "sparse_attn", "hbm", "GB/s"),
    ("stack10m", "sparse_attn", "tensor", "TFLOP/s"),
    ("1m", "pool", "hbm", "GB/s"),
])
def test_stage_roofline_bound_and_peak(name, stage, bound, unit):
    cfg = synth.get_config(name)
    counts = bench.workload_counts(cfg)
    for long_region in (False, True):
        r = bench.stage_roofline(stage, 1.0, cfg, counts, PEAKS, "measured", long_region)
        assert r["bound"] == bound and r["unit"] == unit
        if bound == "hbm":
            assert r["peak"] == PEAKS["hbm_gbs"]
        else:
            assert r["peak"] == PEAKS["bf16_tflops_sustained" if long_region else "bf16_tflops"]
        # achieved = algorithmic work / time (1 ms here)
        work = r.get("alg_bytes_per_launch", r.get("alg_flops_per_launch"))
        assert r["achieved"] == pytest.approx(work / (1e6 if unit == "GB/s" else 1e9))


@pytest.mark.parametrize("name,bound,key", [
    ("100m", "hbm", "route_bytes"),
    ("stack10m", "tensor", "route_flops"),
])
def test_interleave_roofline_counts_every_rounds_scan(name, bound, key):
    cfg = synth.get_config(name)
    counts = bench.workload_counts(cfg)
    for rounds in (1, 3):
        r = bench.interleave_roofline(cfg, counts, rounds, 2.0, PEAKS, "measured", False)
        work = r.get("alg_bytes_per_launch", r.get("alg_flops_per_launch"))
        assert r["bound"] == bound and work == counts[key] * rounds
        # achieved = all rounds' scan work / the whole call's time (2 ms here)
        assert r["achieved"] == pytest.approx(work / 2.0 / (1e6 if bound == "hbm" else 1e9), rel=1e-3)
        assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
        assert r["avg_launch_ms"] == 2.0 and r["traffic"] is None


def test_traffic_records_are_well_formed():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, r in rec.items():
        if key.startswith("_"):
            continue
        kernel_file, workload = key.split(":")
        assert os.path.exists(os.path.join(ROOT, "routed_sparse_attention_chunk_b200", "csrc", kernel_file))
        assert workload in synth.CONFIGS
        assert re.fullmatch(r"[0-9a-f]{16}", r["source_sha256_16"])
        assert r["dram_bytes_per_launch"] > 0 and r["command"].startswith("ncu ")
        # the bench reports a record only while the kernel source still matches it
        got = bench.traffic_record(kernel_file, workload)
        assert got is None or got["dram_bytes_per_launch"] == r["dram_bytes_per_launch"]
    assert bench.traffic_record("pool.cu", "no-such-workload") is None


def test_reference_arm_prints_the_contract_line():
    # the oracle arm on a bounded sample of the 1M workload: one JSON line with the
    # same metric and unit as the GPU arm, tagged impl=reference, e2e without copies
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "1m",
                          "--steps", "1", "--warmup", "0", "--ref-budget", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["metric"] == bench.METRIC and r["unit"] == bench.UNIT
    assert r["higher_is_better"] is True and r["steps"] == 1 and r["value"] > 0
    assert r["config"]["workload"].startswith("1m")
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == r["value"] and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
