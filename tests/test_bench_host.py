"""Host-side logic of bench.py that needs no GPU: the recorded DRAM traffic is reported
only while the kernel sources still hash to the value the profile summary recorded."""
import hashlib
import os

import pytest

import bench


def _setup(tmp_path, monkeypatch, recorded_hash=None):
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    h = recorded_hash or hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "kern_wl.md").write_text(
        "# summary\n\n    traffic_bytes_per_launch: 12345\n    kernel_sources_sha256: %s\n" % h)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "kern", ["k.cu"])
    return src


def test_traffic_reported_while_sources_match(tmp_path, monkeypatch):
    _setup(tmp_path, monkeypatch)
    assert bench.recorded_traffic("kern", "wl") == 12345


def test_traffic_dropped_once_the_kernel_changes(tmp_path, monkeypatch):
    src = _setup(tmp_path, monkeypatch)
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench.recorded_traffic("kern", "wl") is None


def test_traffic_absent_without_summary_or_known_sources(tmp_path, monkeypatch):
    _setup(tmp_path, monkeypatch)
    assert bench.recorded_traffic("kern", "other") is None
    assert bench.recorded_traffic("unknown", "wl") is None


@pytest.mark.parametrize("kernel,workload", [("fused_scan", "lm"), ("chunked_phase_a", "long"),
                                             ("chunked_phase_a", "complex")])
def test_committed_summary_names_known_sources(kernel, workload):
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                        f"{kernel}_{workload}.md")
    with open(path) as f:
        text = f.read()
    assert "traffic_bytes_per_launch:" in text and "kernel_sources_sha256:" in text
    for s in bench.KERNEL_SOURCES[kernel]:
        assert os.path.exists(os.path.join(os.path.dirname(path), "..", s))


def test_reference_arm_prints_one_contract_line():
    """``bench.py --impl reference`` (the oracle on the host cores) prints exactly one
    JSON line with the contract's keys, its e2e and cpu_baseline describing itself."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in res, k
    assert res["impl"] == "reference" and res["steps"] == 2 and res["warmup"] == 3
    assert res["value"] > 0 and res["e2e"]["value"] == res["value"]
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["config"]["workload"].startswith("tiny")


def test_bench_rejects_short_warmup():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "at least 3" in r.stderr


def test_reference_arm_of_the_backward_pass():
    """``--impl reference --pass backward`` times the backward oracle and prints one line."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--pass", "backward",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3", "--tau", "0.5"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["pass"] == "backward" and res["impl"] == "reference" and res["value"] > 0
    assert res["config"]["tau"] == 0.5 and res["cpu_baseline"]["kind"] == "oracle"


def test_backward_bytes_per_token_head():
    """LM workload: s 4 + logits 16 x 2 + d, B, C 3 x 64 x 2 + x, dy 2 x 64 x 2 read, and
    dd, dB, dC, dx, dlogits (3 x 64 + 64 + 16) x 4 written."""
    import workloads
    assert bench.bwd_bytes_per_token_head(workloads.spec("lm")) == 4 + 32 + 384 + 256 + 272 * 4


def test_profiling_overrides_shorten_only_the_named_dimensions():
    """--batch / --seqlen (profiling captures) replace those sizes of the workload and keep
    the rest; without them the workload is the full configuration."""
    import argparse
    import workloads
    full = bench.bench_spec(argparse.Namespace(workload="lm", batch=0, seqlen=0))
    assert full == workloads.spec("lm")
    short = bench.bench_spec(argparse.Namespace(workload="complex", batch=1, seqlen=0))
    assert (short.batch, short.seqlen, short.heads, short.N) == (1, 8192, 64, 128)
    short = bench.bench_spec(argparse.Namespace(workload="lm", batch=0, seqlen=1024))
    assert (short.batch, short.seqlen, short.heads) == (8, 1024, 32)


def test_backward_bytes_cover_complex_gradients():
    """A complex state's dd is complex: 8 bytes an entry instead of 4."""
    import workloads
    sp = workloads.spec("complex")
    # s, bf16 logits, complex d, bf16 B, C, x, complex dy read; complex dd, fp32 dB, dC, dx, dlogits written
    reads = 4 + sp.K * 2 + sp.N * 8 + 2 * sp.N * 2 + sp.P * 2 + sp.P * 8
    assert bench.bwd_bytes_per_token_head(sp) == reads + sp.N * 8 + (2 * sp.N + sp.P + sp.K) * 4
    assert bench.bwd_bytes_per_token_head(workloads.spec("lm")) == 1764
