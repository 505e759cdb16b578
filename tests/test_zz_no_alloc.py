"""pad_decode_static_scratch: the decode entry point for callers that cannot
allocate device memory (a runtime whose memory is planned up front, a thread
that may not take the allocator's locks or absorb the synchronisation an
allocation can cause).  Its split scratch is a fixed array inside the library.

Checked through the C ABI, on two calls in a row with different inputs (the
shared array keeps the first call's partials; the second must not depend on
them), against pad_decode's output on the same inputs and against the CPU oracle
(a bug the two entry points shared would pass the first check only), within the
parity tolerances the other GPU tests use; and after a launch that left merge
counters set in the array (the call must clear them itself).  This file is named
so that pytest collects it last.
"""
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import LSE_RTOL, OUT_ATOL, DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu


def _static(dw, w, splits):
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=dw.dev)
    lse = torch.full((w.B, w.Hq), float("nan"), device=dw.dev)
    scales = dict(k_scale=w.k_scale, v_scale=w.v_scale) if w.kv_dtype == "e4m3" else {}
    assert not scales or (w.k_scale == 1.0 and w.v_scale == 1.0)  # the entry takes no options
    pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits, out=out, lse=lse)
    torch.cuda.synchronize()
    return out, lse


def test_static_scratch_matches_pad_decode_and_the_oracle_twice(cuda_device):
    # the first call has one partition per sequence (the array's address is
    # looked up all the same); the next two split and use the array
    w0 = synth.make_workload("na0", 3, 8, 2, 128, 16, [100, 1, 256], seed=60, max_blocks_per_seq=16)
    out, lse = _static(DeviceWorkload(w0, cuda_device), w0, 1)
    ref_out, ref_lse = oracle.decode_workload(w0)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "static S=1")
    cases = [
        (synth.make_workload("na1", 8, 32, 8, 128, 16, [700, 33, 1024, 5, 512, 129, 0, 300], seed=61,
                             max_blocks_per_seq=64), 8),
        (synth.make_workload("na2", 4, 20, 4, 128, 32, [2048, 17, 999, 64], seed=62, max_blocks_per_seq=64), 0),
    ]
    for w, splits in cases:
        dw = DeviceWorkload(w, cuda_device)
        plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=splits)
        assert plan["reduce"] == 1  # the split path, which needs scratch
        out, lse = _static(dw, w, splits)
        # the existing entry point on the same inputs
        dec_out, dec_lse = pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits, lse=True)
        torch.cuda.synchronize()
        assert (out.float() - dec_out.float()).abs().max().item() <= OUT_ATOL
        assert torch.equal(torch.isneginf(lse), torch.isneginf(dec_lse))
        fin = ~torch.isneginf(dec_lse)
        assert ((lse[fin] - dec_lse[fin]).abs() / dec_lse[fin].abs().clamp_min(1.0)).max().item() <= LSE_RTOL
        # and the oracle
        ref_out, ref_lse = oracle.decode_workload(w)
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"static {w.name}")
    assert pad.pad_check_device_errors() == 0


def test_static_scratch_e4m3_cache(cuda_device):
    # an E4M3 cache of unit scales (the entry takes no options) through the
    # static array, against the oracle on the same codes
    w = synth.make_workload("na_e4m3", 6, 16, 4, 128, 16, [900, 40, 1024, 0, 333, 129], seed=64,
                            max_blocks_per_seq=64, kv_dtype="e4m3", k_scale=1.0, v_scale=1.0)
    out, lse = _static(DeviceWorkload(w, cuda_device), w, 8)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "static e4m3")


def test_static_scratch_clears_counters_a_failed_launch_left_set(cuda_device):
    # a launch whose partition-0 CTAs give up (the failure-path hook: a bounded
    # wait on a barrier nothing arrives on) leaves the other partitions' counts
    # in the array; pad_check_device_errors re-zeroes only library-owned
    # control blocks, so the next static call is right only if it clears them
    w = synth.make_workload("na_cnt", 4, 16, 4, 128, 16, [256, 200, 129, 64], seed=65, max_blocks_per_seq=16)
    dw = DeviceWorkload(w, cuda_device)
    pad.pad_inject_stage_timeout(0)
    _static(dw, w, 4)
    assert pad.pad_check_device_errors() == 0x4
    ref_out, ref_lse = oracle.decode_workload(w)
    for call in range(2):
        out, lse = _static(dw, w, 4)
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"static after a failed launch, call {call}")
    assert pad.pad_check_device_errors() == 0


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    # 256 partitions of 4 x 64 heads at head_dim 256: 64 MiB of partials, twice the array
    w = synth.make_workload("na_big", 4, 64, 1, 256, 16, [40, 40, 40, 40], seed=63, max_blocks_per_seq=4096)
    dw = DeviceWorkload(w, cuda_device)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=4096)
    assert plan["workspace_bytes"] >= 2 * (32 << 20)
    out = torch.full((w.B, w.Hq, w.D), 2.0, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(pad.PadError) as e:
        pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4096, out=out)
    assert e.value.status == pad.PAD_ERR_WORKSPACE and "static array" in str(e.value)
    # an oversized call that is also malformed reports the malformation, as pad_decode would
    bad = torch.full((w.B, w.Hq, w.D + 8), 2.0, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(pad.PadError) as e:
        pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4096, out=bad)
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(out.float() == 2.0) and torch.all(bad.float() == 2.0)
