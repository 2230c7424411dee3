"""bench.py's host logic on CPU: the roofline's byte count, the profile digest and the
verify step's reference arm (the fp64 oracle on host cores)."""
import json
import os
import subprocess
import sys

import pytest

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_closed_form():
    w = synth.WORKLOADS["decode_t9_h4096_e128"]
    # per hit expert: gate, up and down, each H*I elements at 4 bits + one scale byte per 32
    per_expert = 3 * 4096 * 1536 * (0.5 + 1 / 32)
    router = 128 * 4096 * 4          # fp32 router weights
    xy = 2 * 9 * 4096 * 2            # bf16 x in, y out
    assert bench.algorithmic_bytes(w, 9, 57) == pytest.approx(57 * per_expert + router + xy)
    assert bench.algorithmic_bytes(w, 9, 0) == pytest.approx(router + xy)


def test_committed_profile_matches_the_engine_sources():
    """The decode profile's digest names the current engine sources, so the bench line
    carries its DRAM traffic; any edit of those sources must come with a new capture."""
    assert bench.profile_traffic() is not None
    assert bench.profile_traffic() > bench.algorithmic_bytes(synth.WORKLOADS["decode_t9_h4096_e128"], 9, 50)


def test_traffic_only_for_the_profiled_launch():
    """The capture is of the decode workload at its own token count: another token count
    (another kernel instance, other bytes) or another workload reports no traffic."""
    assert bench.traffic_for("decode_t9_h4096_e128", 9) == bench.profile_traffic()
    assert bench.traffic_for("decode_t9_h4096_e128", 72) is None
    assert bench.traffic_for("decode_t9_h4096_e128", 384) is None
    assert bench.traffic_for("batched_t144_h6144_e256", 144) is None
    assert bench.traffic_for("sweep_h7168_e256", 9) is None


def test_verify_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "verify_tiny_v1000_g8", "--steps", "3", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "blocks/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "verify_tiny_v1000_g8"


def test_moe_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_h256_e8", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["config"]["workload"] == "tiny_h256_e8"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_roofline_bound_follows_the_intensity():
    """Tensor roofline where the tile stream's intensity exceeds its kind's ridge (the sweep at
    T = 4608), HBM below it (T = 576) and on the verify-block path."""
    w = synth.WORKLOADS["sweep_h7168_e256"]
    by = lambda T: bench.algorithmic_bytes(w, T, 256)
    r = bench.roofline(w.with_tokens(4608), 4608, by(4608), 13.0, "mxf4", None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 6.0 * 4608 * 8 * 7168 * 2048 + 2.0 * 4608 * 7168 * 256
    assert r["algorithmic_flop_per_launch"] == pytest.approx(flops)
    assert r["achieved"] == pytest.approx(flops / 13.0e-3 / 1e12)
    bf16, _ = bench.measured_bf16_tflops()
    assert r["peak"] == pytest.approx(4.0 * bf16)
    assert bench.roofline(w.with_tokens(576), 576, by(576), 2.3, "mxf4", None)["bound"] == "hbm"
    d = synth.WORKLOADS["decode_t9_h4096_e128"]
    r = bench.roofline(d, 9, bench.algorithmic_bytes(d, 9, 57), 0.11, "mxf4", 1.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 1.0


def test_ishard_groups_keep_slices_on_the_engine_tiling():
    assert bench.ishard_groups(1536, 1) == (1, 1)
    assert bench.ishard_groups(1536, 2) == (2, 1)
    assert bench.ishard_groups(1536, 4) == (4, 1)
    assert bench.ishard_groups(1536, 8) == (4, 2)   # 1536 / 8 = 192 is not a multiple of 128
    assert bench.ishard_groups(2048, 8) == (8, 1)
    for inter in (1536, 2048):
        for world in (1, 2, 3, 4, 6, 8):
            g, groups = bench.ishard_groups(inter, world)
            assert g * groups == world and (inter // g) % 128 == 0 and inter % g == 0
