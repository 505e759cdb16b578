"""A bounded wait of the partition kernel that runs out, on the GPU.

Every wait of the partition kernel gives up after a time limit, sets bit 0x4 of
the device error word and returns ("perf(rocke): prepare saved paged decode
bindings once", section "Risk Assessment": focused tests of failure recovery).
pad_inject_stage_timeout makes that happen on purpose and without any fault:
the units of one partition wait, where they would count themselves for the
merge, on a barrier nothing arrives on, with a short limit, and return
uncounted.  The other partitions count themselves, so merge counters are left
set; the tests check that the failure is reported, that the counters are
re-zeroed, and that the next ordinary call on the same stream matches the
oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu


def _case():
    # sequences spanning 1..4 partitions of 64 tokens at S = 4 (capacity 256)
    return synth.make_workload("timeout", 5, 16, 4, 128, 16, [256, 200, 64, 129, 17], seed=81, max_blocks_per_seq=16)


def _poisoned(w, dev):
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.B, w.Hq), float("nan"), device=dev)
    return out, lse


@pytest.mark.parametrize("stalled", [0, 2])
def test_a_stage_wait_that_runs_out_is_reported_and_the_next_call_is_correct(cuda_device, stalled):
    w = _case()
    dw = DeviceWorkload(w, cuda_device)
    ref_out, ref_lse = oracle.decode_workload(w)
    assert pad.pad_check_device_errors() == 0
    stream = torch.cuda.Stream(cuda_device)
    out, lse = _poisoned(w, cuda_device)
    pad.pad_inject_stage_timeout(stalled)
    pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4, out=out, lse=lse, stream=stream)
    # the failure comes back as a status and bit 0x4 (and only that bit)
    lib = pad.load_library()
    import ctypes

    bits = ctypes.c_uint32(0)
    st = lib.pad_check_device_errors(ctypes.c_void_p(stream.cuda_stream), ctypes.byref(bits))
    assert st == pad.PAD_ERR_DEVICE_CHECK and bits.value == 0x4
    assert "bounded wait that gave up" in pad.pad_last_error()
    # the stalled partition never counted: every sequence with several
    # partitions, that one among them, is left unmerged (poisoned); a sequence
    # with one partition wrote its result before the stalled exit
    P = 64
    for b, L in enumerate(w.seq_lens.tolist()):
        unmerged = L > P and L > stalled * P
        assert bool(torch.isnan(out[b].float()).all()) == unmerged, (b, L)
    # the hook was one-shot, and the counters the other partitions left set were
    # re-zeroed by the check: the next call on the same stream is the oracle's
    out, lse = _poisoned(w, cuda_device)
    pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4, out=out, lse=lse, stream=stream)
    stream.synchronize()
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "after the timeout")
    assert pad.pad_check_device_errors(stream) == 0


def test_timeout_with_caller_workspace_then_a_clean_call(cuda_device):
    w = _case()
    dw = DeviceWorkload(w, cuda_device)
    ref_out, ref_lse = oracle.decode_workload(w)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=4)
    ws = torch.empty(plan["workspace_bytes"] // 4, dtype=torch.float32, device=cuda_device)
    out, lse = _poisoned(w, cuda_device)
    pad.pad_inject_stage_timeout(1)
    pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 4, out, lse, ws)
    assert pad.pad_check_device_errors() == 0x4
    for _ in range(2):
        out, lse = _poisoned(w, cuda_device)
        pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 4, out, lse, ws)
        torch.cuda.synchronize()
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "workspace after the timeout")
    assert pad.pad_check_device_errors() == 0


def test_disarmed_hook_changes_nothing(cuda_device):
    w = _case()
    dw = DeviceWorkload(w, cuda_device)
    pad.pad_inject_stage_timeout(0)
    pad.pad_inject_stage_timeout(-1)
    out, lse = dw.run(num_splits=4)
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "disarmed")
    assert pad.pad_check_device_errors() == 0
    assert np.isfinite(lse.cpu().numpy()).all()
