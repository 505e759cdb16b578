"""Host-side helpers of bench.py, on CPU: the split-scratch byte count, the
recorded-traffic lookup (and its source-hash check), and the CPU baseline's
bounded samples."""
import importlib.util
import os

import numpy as np

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_split_scratch_bytes_counts_multi_partition_sequences():
    bench = _bench()
    w = synth.make_workload("sc", 4, 8, 2, 64, 16, [0, 100, 512, 1000], seed=3, max_blocks_per_seq=64)
    P = 256
    # brute force: per sequence, the partitions that hold a token
    expect = 0
    for L in w.seq_lens.tolist():
        ns = len({t // P for t in range(L)})
        if ns > 1:
            expect += 2 * ns * w.Hq * (w.D + 1) * 4
    assert bench.split_scratch_bytes(w, {"partition_tokens": P}) == expect
    # a window keeps only the partitions that hold its tokens
    W = 300
    expect_w = 0
    for L in w.seq_lens.tolist():
        ns = len({t // P for t in range(max(0, L - W), L)})
        if ns > 1:
            expect_w += 2 * ns * w.Hq * (w.D + 1) * 4
    assert bench.split_scratch_bytes(w, {"partition_tokens": P}, window=W) == expect_w


def test_traffic_is_read_only_for_the_recorded_source(tmp_path, monkeypatch):
    bench = _bench()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "partition_kernel_demo.md").write_text("# demo\n\nsource_sha256: abc123\ndram_bytes_per_launch: 4242\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("demo", "abc123") == 4242
    assert bench.traffic_from_profiles("demo", "other") is None  # the kernel changed since the capture
    assert bench.traffic_from_profiles("missing", "abc123") is None


def test_kernel_source_hash_covers_the_kernel_headers():
    bench = _bench()
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and sha == bench.kernel_source_sha()


def test_cpu_baseline_samples_are_bounded_and_described(monkeypatch):
    bench = _bench()
    w = synth.config("tiny")
    cb = bench.cpu_baseline(w, budget_s=0.2, runs_max=3)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    one = cb["one_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and "whole tiny batch" in one["sample"]
    # a batch too slow for one thread is sampled through its first sequences
    big = synth.make_workload("big", 3, 8, 2, 128, 16, [4096] * 3, seed=4, max_blocks_per_seq=256)
    calls = []

    def prefix(k):
        calls.append(k)
        return synth.make_workload("big", k, 8, 2, 128, 16, [4096] * k, seed=4, max_blocks_per_seq=256)

    clock = iter(np.arange(0, 1e6, 50.0))  # every timed oracle call "takes" 50 s
    monkeypatch.setattr(bench.time, "perf_counter", lambda: float(next(clock)))
    cb2 = bench.cpu_baseline(big, budget_s=1.0, runs_max=1, prefix=prefix)
    assert calls and calls[0] < big.B
    assert cb2["one_thread"]["sample"].startswith(f"first {calls[0]} of {big.B}")


def test_each_kernel_has_its_own_source_hash_and_profile(tmp_path, monkeypatch):
    bench = _bench()
    assert bench.kernel_source_sha("umma_kernel") != bench.kernel_source_sha("partition_kernel")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "umma_kernel_demo.md").write_text("source_sha256: u1\ndram_bytes_per_launch: 77\n")
    (prof / "partition_kernel_demo.md").write_text("source_sha256: p1\ndram_bytes_per_launch: 55\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("demo", "u1", "umma_kernel") == 77
    assert bench.traffic_from_profiles("demo", "p1") == 55
    assert bench.traffic_from_profiles("demo", "p1", "umma_kernel") is None


def test_tcgen05_entry_rejects_what_that_kernel_does_not_take(monkeypatch):
    bench = _bench()
    for extra in (["--kv-dtype", "e4m3"], ["--window", "100"], ["--sinks"]):
        monkeypatch.setattr("sys.argv", ["bench.py", "--entry", "tcgen05", *extra])
        try:
            bench.parse()
        except SystemExit as e:
            assert e.code == 2
        else:
            raise AssertionError(f"--entry tcgen05 {extra} accepted")
    monkeypatch.setattr("sys.argv", ["bench.py", "--entry", "tcgen05", "--workload", "ragged_mqa"])
    args = bench.parse()
    assert args.entry == "tcgen05" and args.kv_dtype == "bf16"


def test_gpus_flag_needs_one_rank_per_gpu(monkeypatch):
    # a single process asked for N > 1 GPUs refuses instead of reporting n_gpus 1
    bench = _bench()
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    for argv in (["--gpus", "8"], ["--gpus", "2", "--impl", "reference"], ["--gpus", "0"]):
        monkeypatch.setattr("sys.argv", ["bench.py", *argv])
        try:
            bench.parse()
        except SystemExit as e:
            assert e.code == 2
        else:
            raise AssertionError(f"{argv} accepted without its ranks")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "2"])
    assert bench.parse().gpus == 2
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "4"])  # ranks and request disagree
    try:
        bench.parse()
    except SystemExit as e:
        assert e.code == 2
    else:
        raise AssertionError("--gpus 4 accepted with WORLD_SIZE 2")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr("sys.argv", ["bench.py"])
    args = bench.parse()
    assert args.gpus == 1 and args.workload == "qwen14b"


def test_reference_arm_prints_one_contract_line():
    # the oracle arm runs on the host cores, so it is checked here end to end
    import json
    import subprocess
    import sys
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--cpu-seconds", "1"], capture_output=True, text=True, cwd=ROOT,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"].startswith("decode attention")
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (1, 1, 1)
    assert d["config"]["workload"] == "qwen14b"
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
