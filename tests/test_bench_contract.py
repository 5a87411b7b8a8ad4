"""The bench's reference arm (the float64 oracle on the host cores) prints one JSON line with the
contract's keys for every workload family; runs on the CPU."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
        "e2e"}


@pytest.mark.parametrize("workload", ["mamba130m_layer", "sparc_complex", "pdssm_l5120"])
def test_reference_arm_json_line(workload):
    env = dict(os.environ, OMP_NUM_THREADS="4")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload,
                          "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == workload
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_traffic_records_follow_kernel_code_not_comments(tmp_path):
    """The committed ncu traffic records are keyed to the kernel file's code: an edit of comments
    alone keeps the key, a code edit changes it, and a record whose key matches the current code
    is the value the bench reports (a stale one reads null there, by design)."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    a = tmp_path / "a.cu"
    a.write_text("// header\nint f(int x) {  // doubles\n    return 2 * x;\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("// another header\n\nint f(int x) {\n    return 2 * x;   // twice\n}\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) {\n    return 3 * x;\n}\n")
    assert bench.code_digest(a) == bench.code_digest(b)
    assert bench.code_digest(a) != bench.code_digest(c)
    recs = json.load(open(os.path.join(root, "profiles", "traffic.json")))["records"]
    for rec in recs:
        src = os.path.join(root, "selective_state_space_bwd_b200", "csrc", rec["source"])
        got = bench.measured_traffic(rec["call"], rec["source"], rec["workload"])
        if bench.code_digest(src) == rec["code_sha256"]:
            assert got == float(rec["dram_bytes_per_launch"]), rec["source"]
        else:
            assert got is None


def test_l2_flush_writes_then_reads_buffers_larger_than_l2():
    """The flush between timed steps: a write of 256 MiB (twice the 126 MB L2) and a read of
    another 256 MiB buffer, so that the written lines are evicted (and written back) before the
    step's events start; checked here with CPU tensors."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    f = bench.L2Flush("cpu")
    assert f.wr.numel() * f.wr.element_size() == 256 << 20
    assert f.rd.numel() * f.rd.element_size() == 256 << 20
    assert f.wr.data_ptr() != f.rd.data_ptr()
    f.wr.fill_(7)
    f()
    assert int(f.wr.max()) == 0 and float(f.acc) == 0.0
