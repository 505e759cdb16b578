"""pad_decode_static_scratch: the decode entry point for callers that cannot
allocate device memory (a pre-planned memory arena, a thread that may not touch
the allocator).  Its split scratch is a fixed array inside the library.

Checked through the C ABI against pad_decode on the same inputs, within the
parity tolerances the other GPU tests use, on two calls in a row with different
inputs (the shared array keeps the first call's partials; the second must not
depend on them).  This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, LSE_RTOL, OUT_ATOL

pytestmark = pytest.mark.gpu


def _compare(got_out, got_lse, ref_out, ref_lse):
    d = (got_out.float() - ref_out.float()).abs().max().item()
    assert d <= OUT_ATOL, d
    empty = torch.isneginf(ref_lse)  # L = 0 gives lse = -inf on both sides
    assert torch.equal(torch.isneginf(got_lse), empty)
    fin = ~empty
    rel = ((got_lse[fin] - ref_lse[fin]).abs() / ref_lse[fin].abs().clamp_min(1.0)).max().item()
    assert rel <= LSE_RTOL, rel


def test_static_scratch_matches_pad_decode_twice(cuda_device):
    cases = [
        (synth.make_workload("na1", 8, 32, 8, 128, 16, [700, 33, 1024, 5, 512, 129, 0, 300], seed=61,
                             max_blocks_per_seq=64), 8),
        (synth.make_workload("na2", 4, 20, 4, 128, 32, [2048, 17, 999, 64], seed=62, max_blocks_per_seq=64), 0),
    ]
    for w, splits in cases:
        dw = DeviceWorkload(w, cuda_device)
        plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=splits)
        assert plan["reduce"] == 1  # the split path, which needs scratch
        ref_out, ref_lse = pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits,
                                          lse=True)
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        lse = torch.full((w.B, w.Hq), float("nan"), device=cuda_device)
        pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits,
                                      out=out, lse=lse)
        torch.cuda.synchronize()
        _compare(out, lse, ref_out, ref_lse)


def test_static_scratch_e4m3_cache(cuda_device):
    # an E4M3 cache of unit scales (the entry takes no options) through the
    # static array, against pad_decode on the same inputs
    w = synth.make_workload("na_e4m3", 6, 16, 4, 128, 16, [900, 40, 1024, 0, 333, 129], seed=64,
                            max_blocks_per_seq=64, kv_dtype="e4m3", k_scale=1.0, v_scale=1.0)
    dw = DeviceWorkload(w, cuda_device)
    ref_out, ref_lse = pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=8, lse=True)
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((w.B, w.Hq), float("nan"), device=cuda_device)
    pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=8, out=out, lse=lse)
    torch.cuda.synchronize()
    _compare(out, lse, ref_out, ref_lse)


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    w = synth.make_workload("na_big", 2, 64, 1, 256, 16, [40, 40], seed=63, max_blocks_per_seq=4096)
    dw = DeviceWorkload(w, cuda_device)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=4096)
    assert plan["workspace_bytes"] > 32 << 20
    out = torch.full((w.B, w.Hq, w.D), 2.0, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(pad.PadError) as e:
        pad.pad_decode_static_scratch(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4096, out=out)
    assert e.value.status == pad.PAD_ERR_WORKSPACE and "static array" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(out.float() == 2.0)
