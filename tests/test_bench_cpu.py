"""The benchmark's reference arm (the oracle on the host cores) runs on the
CPU and prints one JSON line with the keys the bench contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert p.returncode == 0 and not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # roofline.traffic comes from profiles/dram_traffic.json only while the
    # kernel sources hash to the value recorded with the capture
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "profiles").mkdir()
    entry = {"bytes_per_launch": 123456, "source_sha": "aaaa"}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({bench.WORKLOAD: {"mrope_apply": entry}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "aaaa")
    assert bench.dram_traffic("mrope_apply") == 123456
    assert bench.dram_traffic("vis_rope2d") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "bbbb")
    assert bench.dram_traffic("mrope_apply") is None


def test_kernel_source_hash_covers_every_kernel_file(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "interpolated_position_encoding_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("one")
    (csrc / "b.cuh").write_text("two")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha()
    (csrc / "b.cuh").write_text("two!")
    assert bench.kernel_source_sha() != h0


def test_cpu_baseline_runs_on_every_core():
    # the oracle baseline: one single-threaded oracle process per host core
    # (bounded by memory), each on its own slice, and the single-thread figure
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    d = bench.cpu_baseline(wl.WORKLOADS[bench.WORKLOAD], rounds=1)
    n, cores = bench.oracle_workers()
    assert d["kind"] == "oracle" and d["cores"] == n and d["host_cores"] == cores
    assert d["single_thread"]["cores"] == 1 and d["single_thread"]["value"] > 0
    if n >= 2:
        assert d["value"] > d["single_thread"]["value"]
