"""Host-side pieces of bench.py that need no GPU: the sampler's arithmetic
ceiling (the denominator beside the HBM fraction) and the reading of the
committed per-launch DRAM traffic, which must go to None for a kernel whose
source changed after the counters were taken."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_sampler_alu_ceiling_arithmetic():
    # 148 SMs x 4 sub-partitions; per warp-item of 256 bf16 logits (512 B)
    # 36 IMAD.WIDE x 4 + 16 packed fp32 x 2 = 176 heavy-pipe cycles
    c = bench._sampler_alu_ceiling(1000.0, 1965.0)
    expect = 592 * 1965e6 / 176 * 512 / 1e9
    assert c["heavy_cycles_per_256_logits"] == 176
    assert c["peak"] == pytest.approx(expect, rel=1e-12)
    assert c["frac"] == pytest.approx(1000.0 / expect, rel=1e-12)
    assert bench._sampler_alu_ceiling(1000.0, None) is None


def test_profile_traffic_tracks_the_source(tmp_path, monkeypatch):
    src = tmp_path / "block_discrete_diffusion_dd_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel source\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench._source_sha("k.cu")
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# comment line\n"
        f"good 123456 k.cu {sha}\n"
        "stale 999 k.cu 0000000000000000\n")
    t = bench._profile_traffic()
    assert t["good"] == 123456.0
    assert t["stale"] is None


def test_committed_traffic_entries_parse():
    t = bench._profile_traffic()
    for k in ("sampler@ragged_b8", "attention@ragged_b8", "sampler@b1_L4096"):
        assert k in t


def test_oracle_sample_plan_keeps_every_core_busy():
    import workloads
    for name, w in workloads.WORKLOADS.items():
        for cores in (1, 8, 16, 64):
            npos, nrows = bench.oracle_sample_plan(w, cores)
            assert 1 <= npos <= w.canvas and 1 <= nrows <= w.rows
            assert nrows == w.rows or nrows >= max(16, 2 * cores)
            assert npos == w.canvas or npos * w.batch * w.heads_q >= 2 * cores


def test_reference_arm_runs_the_oracle_on_the_shared_sample():
    """The --impl reference arm on the small fp32 workload: the oracle on the
    host cores, on the same sample plan as our line's cpu_baseline."""
    import types
    import workloads
    w = workloads.WORKLOADS["tiny_fp32"]
    args = types.SimpleNamespace(steps=2, warmup=1)
    r = bench.run_reference(args, w, None, 0, 1)
    assert r["impl"] == "reference" and r["extrapolated"] is True
    assert r["value"] > 0 and r["unit"] == bench.UNIT and r["gpu_launches"] == 0
    npos, nrows = bench.oracle_sample_plan(w, r["cpu_baseline"]["cores"])
    assert f"{npos}/{w.canvas}" in r["cpu_baseline"]["sample"]
    assert f"{nrows}/{w.rows}" in r["cpu_baseline"]["sample"]
    assert r["e2e"]["value"] == r["value"]
    assert bench.run_reference(args, w, None, 1, 2) is None      # other ranks: no work
