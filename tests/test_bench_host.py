"""Host-side pieces of bench.py (no GPU): the reference arm's JSON line on
the small workload, and the DRAM-traffic lookup, which reports a captured
figure only while the kernel sources it was taken from are unchanged."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.strip().splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["config"]["workload"] == "tiny"


def test_traffic_lookup_follows_the_kernel_sources(tmp_path, monkeypatch):
    bench = _bench_module()
    (tmp_path / "profiles").mkdir()
    key = f"{bench.KERNEL_NAMES['bwd']}/hist16k"
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {key: {"dram_bytes_per_launch": 1234, "source_sha1": "abc"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "_sha1", lambda paths: "abc")
    assert bench._traffic("bwd", "hist16k") == 1234
    assert bench._traffic("bwd", "stu") is None  # no record for that workload
    assert bench._traffic("fwd", "hist16k") is None  # no record for that kernel
    monkeypatch.setattr(bench, "_sha1", lambda paths: "changed")
    assert bench._traffic("bwd", "hist16k") is None  # sources changed since the capture


def test_source_hash_covers_every_listed_file(tmp_path):
    bench = _bench_module()
    a, b = tmp_path / "a.cu", tmp_path / "b.cuh"
    a.write_text("x")
    b.write_text("y")
    h1 = bench._sha1([str(a), str(b)])
    b.write_text("z")
    assert bench._sha1([str(a), str(b)]) != h1
    assert bench._sha1([str(a), str(tmp_path / "missing.cuh")]) is None


def test_roofline_picks_the_bound_and_the_burst_denominator():
    bench = _bench_module()
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0, "bf16_tflops_sustained": 1400.0,
             "clocks_under_load": {"sm_mhz_median": 1300.0}}
    clk = {"sm_mhz": 1965.0}
    # ridge = 1600e12 / 6400e9 = 250 FLOP/B
    t = bench.roofline(800e9, 1e9, 1.0, peaks, "measured", clk)  # AI 800: tensor roof
    assert t["bound"] == "tensor" and t["unit"] == "TFLOP/s"
    assert abs(t["achieved"] - 800.0) < 1e-9 and abs(t["frac"] - 0.5) < 1e-12
    assert t["peak"] == 1600.0 and abs(t["frac_of_sustained_tensor_peak"] - 800 / 1400) < 1e-12
    assert t["sustained_peak_sm_mhz"] == 1300.0 and t["run_sm_mhz"] == 1965.0
    h = bench.roofline(100e9, 1e9, 0.5, peaks, "measured", clk)  # AI 100: HBM roof
    assert h["bound"] == "hbm" and h["unit"] == "GB/s" and h["peak"] == 6400.0
    assert abs(h["achieved"] - 2000.0) < 1e-9 and abs(h["frac"] - 2000 / 6400) < 1e-12
    assert abs(h["tensor_tflops"] - 200.0) < 1e-9


def test_rank_batches_shard_a_global_batch():
    """N > 1: every sequence of the global batch lands on exactly one rank (by
    length, for the strong split of the workload's one batch), N = 1 is the
    workload's own batch, and the weak split's global batch has N batches'
    sequences."""
    import numpy as np
    from workloads import WORKLOADS, draw_lengths, make_batch
    bench = _bench_module()
    w = WORKLOADS["tiny"]
    b1, info = bench.rank_batch(w, 1, 0)
    assert info is None and np.array_equal(b1.lengths, make_batch(w).lengths)
    for world in (2, 3):
        strong = [bench.rank_batch(w, world, r, strong=True) for r in range(world)]
        got = np.sort(np.concatenate([b.lengths for b, _ in strong]))
        assert np.array_equal(got, np.sort(draw_lengths(w)))
        assert strong[0][1]["global_sequences"] == w.B
        weak = [bench.rank_batch(w, world, r) for r in range(world)]
        assert weak[0][1]["global_sequences"] == world * w.B
        assert sum(len(b.lengths) for b, _ in weak) == world * w.B
