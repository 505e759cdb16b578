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

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

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
    for key in ("heads_per_tile", "stages", "stage_tokens", "num_splits", "partition_tokens", "ctas", "ctas_per_sm"):
        assert got[key] == plan[key], (key, got, plan)
    assert got["warps"] == plan["warps_per_cta"], (got, plan)


def test_tcgen05_entry_runs_the_tcgen05_kernel(cuda_device):
    w = synth.make_workload("wit_tc", 4, 32, 1, 128, 32, [16, 500, 1000, 77], seed=6, max_blocks_per_seq=64)
    DeviceWorkload(w, cuda_device).run(num_splits=4, entry=pad.pad_decode_tcgen05)
    got = pad.pad_last_launch()
    assert (got["kernel"], got["head_dim"], got["heads_per_tile"], got["kv_dtype"]) == (2, 128, 32, pad.PAD_BF16)
    assert got["num_splits"] == 4 and got["ctas"] == 4 * 1 * 1 * 4 and got["warps"] == 6 and got["ctas_per_sm"] == 2


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


@pytest.mark.parametrize("kv", ["e4m3", "bf16"])
@pytest.mark.parametrize("dense", [False, True], ids=["below", "at"])
def test_8_head_tile_takes_its_dense_build_from_four_waves(cuda_device, dense, kv):
    # Qwen3-14B-shaped heads (40 / 8, one 8-head tile per KV head) at S = 16:
    # 128 units per sequence.  From four full waves at five CTAs per SM on,
    # the plan takes the six-per-SM build; one sequence fewer stays at five.
    # Either way the result is the oracle's.
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    B = -(-4 * 5 * sms // 128) - (0 if dense else 1)
    lens = [int(x) for x in synth.uniform_int(B, 1, 256, 90, synth.S_LENS)]
    w = synth.make_workload("wit_dense", B, 40, 8, 128, 16, lens, seed=91, max_blocks_per_seq=16, kv_dtype=kv)
    plan = pad.pad_decode_plan(B, 40, 8, 128, 16, 16, num_splits=16, kv_dtype=kv)
    assert plan["ctas"] == B * 128 and (plan["ctas"] >= 4 * 5 * sms) == dense
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=16)
    got = pad.pad_last_launch()
    assert got["ctas_per_sm"] == plan["ctas_per_sm"] == (6 if dense else 5), (got, plan)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"{kv} 8-head, {plan['ctas_per_sm']} per SM")
