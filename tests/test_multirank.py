"""The N > 1 benchmark path on CPU: two `gloo` ranks run the same aggregation
helpers bench.py uses under torchrun (max over ranks of the device time, sum of
the bytes every rank moved) and the per-rank workload seeding of weak scaling.
No GPU and no data-path collective: the decode itself shards into independent
batches, one per rank."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        # rank r: 10 (r + 1) ms over the timed steps, 100 (r + 1) bytes
        t, nbytes = bench.max_time_sum_bytes(10.0 * (rank + 1), 100 * (rank + 1), cpu, world)
        e2e = bench.max_over_ranks(3.5 * rank, cpu, world)
        base = synth.config("tiny")
        w = synth.config("tiny", seed=bench.rank_seed(base.seed, rank)) if rank else base
        dist.barrier()
        res = {"t": t, "bytes": nbytes, "e2e": e2e, "seed": w.seed,
               "shape": [w.B, w.Hq, w.Hkv, w.D, w.block_size, int(w.block_tables.shape[1])],
               "q0": int(w.q.reshape(-1)[0]), "bytes_alg": w.algorithmic_bytes()}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_benchmark(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    for x in r:
        # whole-job numbers: the slowest rank's time, every rank's bytes
        assert x["t"] == 20.0 and x["bytes"] == 300.0 and x["e2e"] == 3.5
    # weak scaling: same shape and byte count per rank, different data
    assert r[0]["shape"] == r[1]["shape"]
    assert r[0]["seed"] != r[1]["seed"] and r[1]["seed"] == r[0]["seed"] + 1000
    assert r[0]["q0"] != r[1]["q0"]
    assert r[0]["bytes_alg"] == r[1]["bytes_alg"]


def test_single_rank_aggregate_is_the_identity():
    import torch

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_time_sum_bytes(7.5, 123, torch.device("cpu"), 1) == (7.5, 123.0)
    assert bench.max_over_ranks(2.0, torch.device("cpu"), 1) == 2.0
    assert bench.rank_seed(1, 0) == 1 and bench.rank_seed(1, 3) == 3001


def test_reference_arm_other_ranks_exit_quietly(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload = "tiny"
        steps = 1
        warmup = 0
        cpu_seconds = 1.0
        batch = None
        compact_pool = False
    # under torchrun only rank 0 runs and prints the reference line
    assert bench.run_reference(A(), 1, 2) is None
    assert capsys.readouterr().out == ""


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
