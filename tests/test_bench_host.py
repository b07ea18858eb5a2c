"""Host-side logic of bench.py (no GPU): accounting, clock parsing, the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_per_token_accounting():
    algo, issued = bench._flops_per_token(64, 128, 256)
    assert algo / 64 == 2 * 128 * 257 + 4 * 128 * 128 == 131328
    # scores once per head (full d_v per CTA); a 256-block multiplies 192 keys per row on average
    assert issued / 64 == 2 * 192 * 128 + 2 * 192 * 128 + 4 * 128 * 128
    assert bench._bytes_per_token(64, 128) == 81920


def test_clock_summary_parses_nvidia_smi_csv():
    c = bench.ClockSampler(0)
    c.text = ("0, 1965, 1965, 600.5, 98, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
              "0, 1800, 1965, 700.0, 99, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
              "0, 345, 1965, 100.0, 0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active\n")
    s = c.summary()
    assert s["sm_mhz"] == (1965 + 1800) / 2  # median over the loaded samples only
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


@pytest.mark.parametrize("workload", ["prefill_8k", "backward_8k", "tiny_f32"])
def test_reference_arm_prints_one_json_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", workload], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_is_dropped_when_kernel_source_changes(tmp_path, monkeypatch):
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for wl, entry in t.items():
        if wl.startswith("_"):
            continue
        kind = next((k for k in ("decode", "backward") if wl.startswith(k)), "prefill")
        got = bench._traffic(wl)
        assert got == (entry["bytes_per_launch"] if entry["kernel_source_hash"] == bench.kernel_source_hash(kind)
                       else None)


def test_backward_accounting():
    w = bench.synth.WORKLOADS["backward_128k"]
    assert w.kind == "backward" and w.T == 131072 and w.seed == 1007
    # the kernel-source hash of the backward covers the prefill kernel its passes run on
    assert "la_prefill_pair.cu" in bench.KERNEL_SOURCES["backward"]
    assert "la_backward.cu" in bench.KERNEL_SOURCES["backward"]


def test_secondary_configs_are_bench_workloads():
    """The default line's extra keys: each a workload the bench can build a case for."""
    assert set(bench.SECONDARY_STEPS) == {"decode_256", "varlen_16", "prefill_8k", "tiny_f32"}
    for name, steps in bench.SECONDARY_STEPS.items():
        w = bench.synth.WORKLOADS[name]
        assert steps >= 10
        assert w.kind in ("prefill", "varlen", "decode")
    assert bench.synth.WORKLOADS["tiny_f32"].dtype == "f32"
