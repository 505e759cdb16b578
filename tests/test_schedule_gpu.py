"""Launches that order their units longest first.

With heavy units (partition tokens x heads per tile >= 32 K) a one-CTA pass
writes the launch's unit order from the device-resident lengths, and CTA i runs
unit order[i].  The order must be a permutation that changes no result: every
case here is checked against the oracle, with ragged and empty sequences,
windows, sinks, both cache types and both kernels, and the caller's workspace
must hold the order after the partials.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu

LENS = [0, 17, 2048, 3000, 4096, 1500, 2049, 64]


def _round256(x):
    return -(-x // 256) * 256


def _case(kv="bf16", seed=91):
    return synth.make_workload("sched", len(LENS), 32, 1, 128, 16, LENS, seed=seed, max_blocks_per_seq=256,
                               kv_dtype=kv)


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("splits", [2, 4])
def test_scheduled_launch_matches_oracle(cuda_device, kv, splits):
    w = _case(kv)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=splits,
                               kv_dtype=kv)
    assert plan["partition_tokens"] * plan["heads_per_tile"] >= 32768 and plan["num_splits"] > 1
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"scheduled {kv} S={splits}")
    assert pad.pad_last_launch()["kernel"] == 1
    assert pad.pad_check_device_errors() == 0


def test_scheduled_launch_with_window_and_sinks(cuda_device):
    w = _case(seed=92)
    sinks = np.linspace(-1.0, 2.0, w.Hq).astype(np.float32)
    ref_out, ref_lse = oracle.decode_workload(w, window=1100, sinks=sinks)
    dsk = torch.from_numpy(sinks).to(cuda_device)
    out, lse = DeviceWorkload(w, cuda_device).run(
        num_splits=4, entry=lambda *a, **k: pad.pad_decode(*a, window=1100, sinks=dsk, **k))
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "scheduled window+sinks")
    assert pad.pad_check_device_errors() == 0


def test_scheduled_tcgen05_launch(cuda_device):
    w = _case(seed=93)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=2, entry=pad.pad_decode_tcgen05)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "scheduled tcgen05")
    assert pad.pad_last_launch()["kernel"] == 2
    assert pad.pad_check_device_errors() == 0


def test_caller_workspace_holds_the_order_after_the_partials(cuda_device):
    w = _case(seed=94)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=2)
    S, units = plan["num_splits"], plan["ctas"]
    partials = _round256(w.B * w.Hq * S * w.D * 4) + _round256(w.B * w.Hq * S * 4)
    assert plan["workspace_bytes"] == partials + _round256(units * 4)
    dw = DeviceWorkload(w, cuda_device)
    ws = torch.full((plan["workspace_bytes"] // 4,), float("nan"), dtype=torch.float32, device=cuda_device)
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((w.B, w.Hq), float("nan"), device=cuda_device)
    pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 2, out, lse, ws)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "caller workspace, scheduled")
    order = ws[partials // 4: partials // 4 + units].view(torch.int32).cpu().numpy()
    assert sorted(order.tolist()) == list(range(units))  # a permutation of the units
    # longest first, in buckets of P/64 tokens; empty units last
    P = plan["partition_tokens"]
    pairs = w.B * w.Hkv * plan["head_tiles"]
    work = []
    for u in order.tolist():
        s = S - 1 - u // pairs
        b = (u % pairs) // (w.Hkv * plan["head_tiles"])
        L = int(w.seq_lens[b])
        work.append(max(0, min((s + 1) * P, L) - s * P))
    buckets = [63 if x <= 0 else (P - x) * 63 // P for x in work]
    assert buckets == sorted(buckets)


def test_scheduled_launch_replays_in_a_cuda_graph(cuda_device):
    # the schedule pass and the decode launch are both captured (scratch exists
    # after one call outside capture); the replay reads the live lengths
    w = _case(seed=95)
    dw = DeviceWorkload(w, cuda_device)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((w.B, w.Hq), device=cuda_device)
    s = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(s):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=2, out=out, lse=lse)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=2, out=out, lse=lse)
    # new lengths after capture: the replayed pass orders by them
    lens2 = np.asarray([4096, 0, 17, 3000, 64, 2049, 1500, 2048], dtype=np.int32)
    w2 = synth.make_workload("sched", len(lens2), 32, 1, 128, 16, lens2.tolist(), seed=95, max_blocks_per_seq=256)
    dw.lens.copy_(torch.from_numpy(w2.seq_lens))
    dw.tables.copy_(torch.from_numpy(w2.block_tables))
    dw.q.copy_(torch.from_numpy(w2.q).view(torch.bfloat16))
    dw.k.copy_(torch.from_numpy(w2.k_cache).view(torch.bfloat16))
    dw.v.copy_(torch.from_numpy(w2.v_cache).view(torch.bfloat16))
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_workload(w2)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "scheduled graph replay")
    assert pad.pad_check_device_errors() == 0
    del g


def test_stalled_scheduled_launch_then_a_clean_call(cuda_device):
    # the failure-path hook in an ordered launch: partition 0's units give up
    # uncounted, and the next ordinary call is the oracle's
    w = _case(seed=96)
    dw = DeviceWorkload(w, cuda_device)
    pad.pad_inject_stage_timeout(0)
    dw.run(num_splits=2)
    assert pad.pad_check_device_errors() == 0x4
    out, lse = dw.run(num_splits=2)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "after a stalled ordered launch")
    assert pad.pad_check_device_errors() == 0
