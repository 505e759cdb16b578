"""The kernel that ran is the kernel that was planned.

Every decode launch records, from inside the kernel (block 0), which kernel ran
and the plan it was compiled and launched with (pad_last_launch): a
kernel-resident witness of the arm that executed ("perf(BACKEND-ROCM): cooperate
across Q8_K activation blocks", section "What changed").  A silent landing on
another path ("Attention parity: run every attention type on the best available
path on both targets", opening summary) would show here.
"""
import pytest
import torch

import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hkv, D, bs, lens, kv_dtype, splits
    (3, 8, 2, 128, 16, [300, 40, 700], "bf16", 0),
    (3, 8, 2, 128, 16, [300, 40, 700], "e4m3", 3),
    (2, 32, 2, 64, 4, [129, 7], "bf16", 1),
    (2, 32, 4, 256, 16, [333, 48], "e4m3", 0),
    (4, 32, 1, 128, 32, [16, 500, 1000, 77], "bf16", 0),
    (4, 32, 1, 128, 32, [16, 500, 1000, 77], "e4m3", 5),
    (2, 80, 2, 128, 16, [90, 250], "bf16", 2),  # 40 heads per KV head: two tiles
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"D{s[3]}_g{s[1] // s[2]}_{s[6]}_S{s[7]}" for s in SHAPES])
def test_partition_kernel_runs_the_planned_shape(cuda_device, shape):
    B, Hq, Hkv, D, bs, lens, kv, splits = shape
    w = synth.make_workload("wit", B, Hq, Hkv, D, bs, lens, seed=5, max_blocks_per_seq=64, kv_dtype=kv)
    plan = pad.pad_decode_plan(B, Hq, Hkv, D, bs, w.max_blocks_per_seq, num_splits=splits, kv_dtype=kv)
    DeviceWorkload(w, cuda_device).run(num_splits=splits)
    got = pad.pad_last_launch()
    assert got["kernel"] == 1
    assert got["head_dim"] == D
    assert got["kv_dtype"] == (pad.PAD_FP8_E4M3 if kv == "e4m3" else pad.PAD_BF16)
    for key in ("heads_per_tile", "stages", "stage_tokens", "num_splits", "partition_tokens", "ctas"):
        assert got[key] == plan[key], (key, got, plan)
    assert got["warps"] == plan["warps_per_cta"], (got, plan)


def test_tcgen05_entry_runs_the_tcgen05_kernel(cuda_device):
    w = synth.make_workload("wit_tc", 4, 32, 1, 128, 32, [16, 500, 1000, 77], seed=6, max_blocks_per_seq=64)
    DeviceWorkload(w, cuda_device).run(num_splits=4, entry=pad.pad_decode_tcgen05)
    got = pad.pad_last_launch()
    assert (got["kernel"], got["head_dim"], got["heads_per_tile"], got["kv_dtype"]) == (2, 128, 32, pad.PAD_BF16)
    assert got["num_splits"] == 4 and got["ctas"] == 4 * 1 * 1 * 4 and got["warps"] == 6


def test_static_scratch_and_caller_workspace_run_the_partition_kernel(cuda_device):
    w = synth.make_workload("wit_ws", 3, 8, 2, 128, 16, [300, 40, 700], seed=7, max_blocks_per_seq=64)
    dw = DeviceWorkload(w, cuda_device)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=4)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
    pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4, out=out)
    assert pad.pad_last_launch()["kernel"] == 1
    ws = torch.empty(plan["workspace_bytes"] // 4 + 64, dtype=torch.float32, device=cuda_device)
    pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 4, out, None, ws)
    got = pad.pad_last_launch()
    assert got["kernel"] == 1 and got["num_splits"] == plan["num_splits"]
