"""Concurrent decodes: several streams, and several host threads each on its own
stream, with split shapes so that every call uses the library-owned partial
scratch and merge counters.  The library keeps those per (device, stream) and
never reuses one stream's scratch for another while work is queued
("perf(rocke): prepare saved paged decode bindings once", section "Technical
Changes": each binding owns its scratch, retained until queued work
completes), so no result may depend on what the other streams do.
"""
import threading

import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, Hq, Hkv, D, bs, lens, kv_dtype, splits
    ("s0", 3, 8, 2, 128, 16, [700, 33, 512], "bf16", 6),
    ("s1", 2, 32, 1, 128, 32, [1500, 90], "bf16", 5),
    ("s2", 2, 16, 4, 256, 16, [900, 257], "e4m3", 4),
    ("s3", 4, 8, 8, 64, 4, [300, 1, 128, 77], "bf16", 7),
]


def _workloads():
    ws = []
    for i, (name, B, Hq, Hkv, D, bs, lens, kv, splits) in enumerate(CASES):
        w = synth.make_workload(name, B, Hq, Hkv, D, bs, lens, seed=40 + i, max_blocks_per_seq=128, kv_dtype=kv)
        ws.append((w, splits))
    return ws


def _call(dw, splits, out, lse, stream):
    w = dw.w
    scales = dict(k_scale=w.k_scale, v_scale=w.v_scale) if w.kv_dtype == "e4m3" else {}
    pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits, out=out, lse=lse,
                   stream=stream, **scales)


def test_streams_interleaved_without_syncs(cuda_device):
    ws = _workloads()
    dws = [DeviceWorkload(w, cuda_device) for w, _ in ws]
    refs = [oracle.decode_workload(w) for w, _ in ws]
    streams = [torch.cuda.Stream(cuda_device) for _ in ws]
    outs = [torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device) for w, _ in ws]
    lses = [torch.empty((w.B, w.Hq), dtype=torch.float32, device=cuda_device) for w, _ in ws]
    torch.cuda.synchronize(cuda_device)
    # six rounds of one call per stream, queued back to back with no host sync:
    # the streams' kernels may overlap, each reusing its own scratch in order
    for _ in range(6):
        for (w, splits), dw, o, l, s in zip(ws, dws, outs, lses, streams):
            with torch.cuda.stream(s):
                o.fill_(float("nan"))
                l.fill_(float("nan"))
            _call(dw, splits, o, l, s)
    torch.cuda.synchronize(cuda_device)
    for (w, _), o, l, (ro, rl) in zip(ws, outs, lses, refs):
        check_parity(to_f64(o), l.cpu().numpy(), ro, rl, f"{w.name} (interleaved streams)")
    assert pad.pad_check_device_errors() == 0


def test_host_threads_each_on_its_own_stream(cuda_device):
    ws = _workloads()
    dws = [DeviceWorkload(w, cuda_device) for w, _ in ws]
    refs = [oracle.decode_workload(w) for w, _ in ws]
    results = [None] * len(ws)
    errors = []
    barrier = threading.Barrier(len(ws))

    def worker(i):
        try:
            torch.cuda.set_device(cuda_device)
            w, splits = ws[i]
            s = torch.cuda.Stream(cuda_device)
            out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
            lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=cuda_device)
            barrier.wait(timeout=60)
            for _ in range(8):
                _call(dws[i], splits, out, lse, s)
            s.synchronize()
            results[i] = (to_f64(out), lse.cpu().numpy())
        except Exception as e:  # reported on the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(ws))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a decode thread did not finish"
    assert not errors, errors
    for (w, _), (o, l), (ro, rl) in zip(ws, results, refs):
        check_parity(o, l, ro, rl, f"{w.name} (thread)")
    assert pad.pad_check_device_errors() == 0


def test_one_stream_many_shapes_reuses_scratch_in_order(cuda_device):
    # one stream, shapes alternating (the scratch grows for the largest and is
    # reused for the others); results equal those of a fresh call per shape
    ws = _workloads()
    dws = [DeviceWorkload(w, cuda_device) for w, _ in ws]
    s = torch.cuda.Stream(cuda_device)
    firsts = []
    for (w, splits), dw in zip(ws, dws):
        o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
        l = torch.empty((w.B, w.Hq), dtype=torch.float32, device=cuda_device)
        _call(dw, splits, o, l, s)
        s.synchronize()
        firsts.append((o.clone(), l.clone()))
    for _ in range(3):
        for (w, splits), dw, (o0, l0) in zip(ws, dws, firsts):
            o = torch.empty_like(o0)
            l = torch.empty_like(l0)
            _call(dw, splits, o, l, s)
            s.synchronize()
            # the same plan on the same inputs: bitwise the same result
            assert torch.equal(o, o0) and torch.equal(torch.nan_to_num(l, neginf=-1e30),
                                                      torch.nan_to_num(l0, neginf=-1e30)), w.name
