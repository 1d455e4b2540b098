"""bench.py's contract on CPU (no GPU): the reference arm's JSON line, the
roofline arithmetic, the measured-peaks file and the source-hash gate on the
recorded DRAM traffic.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line with the
    keys the base contract names, the reference-arm extras, and a positive throughput."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-sample-tokens", "8"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == bench.PREFILL
    # the same workload keys as the GPU arm's line, plus the declared sample
    for key in ("num_seqs", "seq_len", "nqk", "nv", "dk", "dv", "chunk", "io", "state", "initial_state"):
        assert key in d["config"], key
    assert d["config"]["sample_tokens_per_seq"] == 8
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_is_at_least_three():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-sample-tokens", "4"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([x for x in r.stdout.splitlines() if x.startswith("{")][0])
    assert d["warmup"] == 3


def test_hbm_line_arithmetic():
    peaks = {"hbm_gbs": 6000.0}
    r = bench.hbm_line(2.0, 6.0e9, peaks, "measured", call="x")
    assert r["ms_per_step"] == 2.0 and r["call"] == "x"
    ro = r["roofline"]
    assert ro["bound"] == "hbm" and ro["unit"] == "GB/s" and ro["peak_source"] == "measured"
    assert abs(ro["achieved"] - 3000.0) < 1e-9          # 6 GB in 2 ms
    assert abs(ro["frac"] - 0.5) < 1e-12
    assert ro["alg_bytes_per_launch"] == 6.0e9 and ro["traffic"] is None


def test_measured_peaks_are_read():
    peaks, src = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        assert src == "measured" and peaks["hbm_gbs"] == float(d["hbm_gbs"])
    else:
        assert src == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_recorded_traffic_is_gated_by_the_source_hash(monkeypatch):
    """The ncu byte counts apply only to the sources they were captured from."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel in rec:
        per_unit = rec[kernel]["bytes_per_unit"]
        monkeypatch.setattr(bench, "source_hash", lambda k, h=rec[kernel]["source_sha256"]: h)
        assert bench.recorded_traffic(kernel, 10) == per_unit * 10
        monkeypatch.setattr(bench, "source_hash", lambda k: "0" * 64)
        assert bench.recorded_traffic(kernel, 10) is None
    assert bench.recorded_traffic("no_such_kernel", 10) is None


def test_source_hash_covers_the_kernel_files():
    for kernel, files in bench.KERNEL_SOURCES.items():
        assert files, kernel
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "gated_deltanet_chunk_b200", "csrc", f)), f
        assert len(bench.source_hash(kernel)) == 64


def test_reference_arm_under_torchrun_two_ranks():
    """The launch the scaling run uses (torchrun, 2 ranks): rank 0 alone prints the line, every rank
    exits 0, and no process group is needed for the CPU oracle."""
    import socket
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-sample-tokens", "4"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
