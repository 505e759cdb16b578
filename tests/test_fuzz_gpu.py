"""Randomised GPU parity over the whole envelope, against the CPU oracle.

Seeded draws of every parameter the kernel specialises on or branches over:
head_dim 64/128/256; GQA groups 1..40 (8-, 16- and 32-head tiles, one or
several tiles per group, so every warp layout: token groups, head groups,
head_dim pairs); block sizes 1..256; ragged lengths with empty sequences and
sequences shorter than a page; explicit and heuristic partition counts;
sliding window and sinks; bf16 and E4M3 caches with their scales; HND and NHD
cache layouts.  The oracle computes each case in full (cases are small).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu

N_CASES = 160


def draw_case(i):
    r = np.random.default_rng(10_000 + i)
    D = int(r.choice([64, 128, 256]))
    Hkv = int(r.choice([1, 2, 3]))
    g = int(r.choice([1, 2, 4, 5, 8, 9, 12, 16, 17, 20, 24, 32, 33, 40]))
    bs = int(r.choice([1, 2, 4, 8, 16, 32, 64, 128, 256]))
    B = int(r.integers(1, 5))
    lmax = int(r.choice([40, 300, 1500]))
    lens = [int(x) for x in r.integers(0, lmax + 1, size=B)]
    if r.random() < 0.3:
        lens[int(r.integers(B))] = 0
    if r.random() < 0.3:
        lens[int(r.integers(B))] = int(r.integers(1, bs + 1))
    splits = int(r.choice([0, 1, 2, 3, 7]))
    window = int(r.choice([0, 0, 1, 37, 256]))
    sinks = bool(r.random() < 0.35)
    kv = "e4m3" if r.random() < 0.4 else "bf16"
    layout = "nhd" if r.random() < 0.25 else "hnd"
    return dict(D=D, Hkv=Hkv, Hq=g * Hkv, bs=bs, B=B, lens=lens, splits=splits, window=window, sinks=sinks, kv=kv,
                layout=layout, seed=i)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_case_matches_oracle(cuda_device, i):
    c = draw_case(i)
    width = max(1, -(-max(c["lens"]) // c["bs"])) + 1
    w = synth.make_workload(f"fuzz{i}", c["B"], c["Hq"], c["Hkv"], c["D"], c["bs"], c["lens"], seed=c["seed"],
                            max_blocks_per_seq=width, kv_dtype=c["kv"])
    sinks = (np.random.default_rng(i).standard_normal(c["Hq"]) * 2).astype(np.float32) if c["sinks"] else None
    ref_out, ref_lse = oracle.decode_workload(w, window=c["window"], sinks=sinks)
    dev_sinks = torch.from_numpy(sinks).to(cuda_device) if sinks is not None else None
    out, lse = DeviceWorkload(w, cuda_device, layout=c["layout"]).run(
        num_splits=c["splits"], entry=lambda *a, **k: pad.pad_decode(*a, window=c["window"], sinks=dev_sinks, **k))
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, str(c))
    assert pad.pad_check_device_errors() == 0
