"""Host-side logic of bench.py (no GPU): workload tables, the source hash that
keys the ncu traffic figures, and the reference arm's JSON line on CPU."""
import json
import os
import shutil
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_workload_tables_cover_every_kind():
    kinds = {kind for _, kind, _ in bench.WORKLOADS.values()}
    assert kinds <= set(bench.DEFAULT_STEPS) and kinds <= set(bench.KERNEL_FILE)
    csrc = os.path.join(ROOT, "dequant_gemv_packed_b200", "csrc")
    for files in bench.KERNEL_FILE.values():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), f


def test_workload_config_for_every_workload():
    """The config dict (identical in both arms) names the workload and how the
    timed region keeps L2 from serving repeated inputs, for every workload."""
    from types import SimpleNamespace
    for name, (desc, kind, p) in bench.WORKLOADS.items():
        case = SimpleNamespace(desc_text=desc, M=p.get("M", 1), K=2560, N=9728, bits=4, kind=kind)
        cfg = bench.workload_config(case, 1)
        assert cfg["workload"] == desc and cfg["parallelism"] == "replicas x1"
        assert cfg["l2"].startswith("inputs larger than L2"), name
        json.dumps(cfg)


def test_source_hash_follows_the_kernel_file(tmp_path, monkeypatch):
    """A kind's hash covers its own .cu file and the shared headers, not the
    other kernels' files; the whole-directory hash covers everything."""
    pkg = tmp_path / "dequant_gemv_packed_b200"
    shutil.copytree(os.path.join(ROOT, "dequant_gemv_packed_b200", "csrc"), pkg / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {k: bench.kernel_source_hash(k) for k in (None, "gemv", "gemm", "quantize")}
    assert before["gemv"] == bench.kernel_source_hash("stack")
    assert len(set(before.values())) == 4
    with open(pkg / "csrc" / "qlin_gemm.cu", "a") as f:
        f.write("\n// edit\n")
    after = {k: bench.kernel_source_hash(k) for k in (None, "gemv", "gemm", "quantize")}
    assert after["gemv"] == before["gemv"] and after["quantize"] == before["quantize"]
    assert after["gemm"] != before["gemm"] and after[None] != before[None]
    with open(pkg / "csrc" / "qlin_sm100.cuh", "a") as f:
        f.write("\n// edit\n")
    assert bench.kernel_source_hash("gemv") != before["gemv"]


def test_traffic_lookup_requires_the_same_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(json.dumps(
        {"gateup": {"kernel_hash": "abc", "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("gateup", "abc") == 123
    assert bench.ncu_traffic("gateup", "abd") is None
    assert bench.ncu_traffic("down1", "abc") is None


def test_committed_traffic_table_is_well_formed():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.txt")))
    for name, e in d.items():
        assert name in bench.WORKLOADS
        assert e["dram_bytes_per_launch"] > 0 and len(e["kernel_hash"]) == 16


def test_reference_arm_json_line_on_cpu():
    env = dict(os.environ, QLIN_REFERENCE_BUDGET_S="2")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_config_is_the_workload_config():
    """Both arms print the same `config`: the workload (shapes, widths, inputs),
    not how it was timed (that is `timing` in our arm's line)."""
    from types import SimpleNamespace
    env = dict(os.environ, QLIN_REFERENCE_BUDGET_S="2")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    desc = bench.WORKLOADS["tiny"][0]
    ours = bench.workload_config(SimpleNamespace(desc_text=desc, M=1, K=256, N=512, bits=4, kind="gemv"), 1)
    assert line["config"] == ours
    names = {name for name, _, _ in bench.PER_CONFIG}
    assert names <= set(bench.WORKLOADS) and "gateup" not in names
