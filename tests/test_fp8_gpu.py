"""GPU parity of the E4M3 (8-bit) KV cache against the CPU oracle.

The FP8 decode path beside the non-FP8 one ("perf(rocke): prepare saved paged
decode bindings once", section "Summary") with the reading the oracle states:
OCP E4M3 codes, one fp32 scale per tensor.  The same shape classes as the bf16
parity tests (every head tile, head_dim 64/128/256, block sizes 1..256, ragged
tails, empty sequences), the NHD layout, the window and sink options, and the
four large workloads at full size on sampled outputs.  Poisoned blocks hold the
E4M3 NaN code, so a read outside the live pages fails parity.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, oracle_pairs, sample_pairs, to_f64
from test_parity_gpu import SMALL

pytestmark = pytest.mark.gpu


def _case(name, B, Hq, Hkv, D, bs, lens, **kw):
    return synth.make_workload(name, B, Hq, Hkv, D, bs, lens, seed=zlib.crc32(name.encode()) % 1000,
                               max_blocks_per_seq=max(1, -(-max(lens) // bs)) + 2, kv_dtype="e4m3", **kw)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_e4m3_small_cases_match_oracle(cuda_device, case, splits):
    name, B, Hq, Hkv, D, bs, lens = case
    w = _case("e4m3_" + name, B, Hq, Hkv, D, bs, lens)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"e4m3 {name}/S={splits}")
    assert pad.pad_check_device_errors() == 0


@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.0078125, 3.0), (2.5, 0.001)])
def test_e4m3_scales(cuda_device, scales):
    ks, vs = scales
    w = _case("e4m3_scales", 3, 8, 2, 128, 16, [300, 40, 129], k_scale=ks, v_scale=vs)
    ref_out, ref_lse = oracle.decode_workload(w)
    for splits in (1, 4):
        out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"e4m3 scales {scales}/S={splits}")


@pytest.mark.parametrize("splits", [1, 3])
def test_e4m3_nhd_layout(cuda_device, splits):
    w = _case("e4m3_nhd", 3, 12, 3, 128, 16, [400, 33, 160])
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device, layout="nhd").run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"e4m3 nhd/S={splits}")


@pytest.mark.parametrize("D,bs", [(128, 16), (64, 4), (256, 16), (128, 1)])
def test_e4m3_window_and_sinks(cuda_device, D, bs):
    w = _case(f"e4m3_ws_{D}_{bs}", 3, 8, 2, D, bs, [500, 37, 1000])
    sinks = np.asarray([0.3, -1.0, 2.0, -np.inf, 0.0, 5.0, -3.0, 1.5], dtype=np.float32)
    W = 130
    ref_out, ref_lse = oracle.decode_workload(w, window=W, sinks=sinks)
    dev_sinks = torch.from_numpy(sinks).to(cuda_device)
    for splits in (1, 3, 0):
        out, lse = DeviceWorkload(w, cuda_device).run(
            num_splits=splits, entry=lambda *a, **k: pad.pad_decode(*a, window=W, sinks=dev_sinks, **k))
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"e4m3 window+sinks D{D} bs{bs}/S={splits}")
    assert pad.pad_check_device_errors() == 0


@pytest.mark.parametrize("name", synth.CONFIG_NAMES)
def test_e4m3_named_workload_full_size(cuda_device, name):
    """Each named workload on its E4M3 cache, as benchmarked with --kv-dtype
    e4m3: every (b, head) row against the oracle over the whole batch, after a
    sampled quick check."""
    w = synth.config(name, kv_dtype="e4m3")
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run()
    got_out, got_lse = to_f64(out), lse.cpu().numpy()
    if name != "tiny":
        pairs = sample_pairs(w, 48, seed=11)
        ref_o, ref_l = oracle_pairs(w, pairs)
        idx_b, idx_h = [b for b, _ in pairs], [h for _, h in pairs]
        check_parity(got_out[idx_b, idx_h], got_lse[idx_b, idx_h], ref_o, ref_l, "e4m3 " + name + " (sampled)")
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(got_out, got_lse, ref_out, ref_lse, "e4m3 " + name)
    assert pad.pad_check_device_errors() == 0
    del dw
    torch.cuda.empty_cache()


def test_e4m3_invalid_arguments(cuda_device):
    w = _case("e4m3_bad", 2, 8, 2, 128, 16, [40, 20])
    dw = DeviceWorkload(w, cuda_device)
    mixed = dw.v.view(torch.uint8)  # not a float8 tensor: describe() refuses it
    with pytest.raises(TypeError):
        dw.run(entry=lambda q, k, v, *a, **kw: pad.pad_decode(q, k, mixed, *a, **kw))
    bf16_v = torch.zeros(dw.v.shape, dtype=torch.bfloat16, device=cuda_device)
    for bad in (lambda q, k, v, *a, **kw: pad.pad_decode(q, k, bf16_v, *a, **kw),            # K e4m3, V bf16
                lambda *a, **kw: pad.pad_decode(*a, **{**kw, "k_scale": -1.0}),             # negative scale
                lambda *a, **kw: pad.pad_decode(*a, **{**kw, "v_scale": float("inf")})):   # non-finite scale
        with pytest.raises(pad.PadError) as e:
            dw.run(entry=bad)
        assert e.value.status == pad.PAD_ERR_INVALID_ARG
    # scales on a bf16 cache are an error, 1 (or 0) is not
    wb = synth.make_workload("bf16_scaled", 2, 8, 2, 128, 16, [40, 20], seed=5)
    dwb = DeviceWorkload(wb, cuda_device)
    with pytest.raises(pad.PadError) as e:
        dwb.run(entry=lambda *a, **kw: pad.pad_decode(*a, k_scale=0.5, **kw))
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
    dwb.run(entry=lambda *a, **kw: pad.pad_decode(*a, k_scale=1.0, v_scale=0.0, **kw))
    # the tcgen05 kernel takes bf16 caches only
    w32 = _case("e4m3_g32", 2, 32, 1, 128, 32, [100, 300])
    with pytest.raises(pad.PadError) as e:
        DeviceWorkload(w32, cuda_device).run(
            entry=lambda *a, k_scale=None, v_scale=None, **kw: pad.pad_decode_tcgen05(*a, **kw))
    assert e.value.status == pad.PAD_ERR_UNSUPPORTED


@pytest.mark.parametrize("splits", [1, 5, 0])
def test_caller_workspace_with_options(cuda_device, splits):
    # pad_decode_with_workspace_ex: caller-owned partials with E4M3 scales, a
    # window and sinks together
    w = _case("e4m3_ws_ex", 3, 16, 2, 128, 16, [700, 90, 1200])
    sinks = np.linspace(-2.0, 3.0, w.Hq).astype(np.float32)
    W = 333
    ref_out, ref_lse = oracle.decode_workload(w, window=W, sinks=sinks)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=splits,
                               kv_dtype="e4m3")
    ws = torch.full((plan["workspace_bytes"] // 4 + 64,), float("nan"), dtype=torch.float32, device=cuda_device)
    dev_sinks = torch.from_numpy(sinks).to(cuda_device)

    def entry(q, k, v, t, l, scale, num_splits, out, lse, **kw):
        pad.pad_decode_with_workspace(q, k, v, t, l, scale, num_splits, out, lse, ws if plan["workspace_bytes"] else None,
                                      window=W, sinks=dev_sinks, **kw)

    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits, entry=entry)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"workspace_ex/S={splits}")
    assert pad.pad_check_device_errors() == 0


def test_e4m3_graph_replay_reads_live_inputs(cuda_device):
    # a captured E4M3 decode (scales, window, sinks) replayed after q changed in
    # place: the graph reads the tensors' current contents
    w = _case("e4m3_graph", 3, 8, 2, 128, 16, [300, 45, 700])
    sinks = np.asarray([0.5, -1.0, 2.0, 0.0, -3.0, 1.0, 0.25, -0.5], dtype=np.float32)
    dev_sinks = torch.from_numpy(sinks).to(cuda_device)
    W = 200
    dw = DeviceWorkload(w, cuda_device)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((w.B, w.Hq), device=cuda_device)
    s = torch.cuda.Stream()

    def call():
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=3, out=out, lse=lse, window=W,
                       sinks=dev_sinks, k_scale=w.k_scale, v_scale=w.v_scale)

    with torch.cuda.stream(s):
        call()  # the library's scratch for this shape exists before capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    q2 = synth.bf16_array(w.q.shape, 999, 1)
    dw.q.copy_(torch.from_numpy(q2).view(torch.bfloat16).to(cuda_device))
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    w2 = synth.Workload(**{**w.__dict__, "q": q2})
    ref_out, ref_lse = oracle.decode_workload(w2, window=W, sinks=sinks)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "e4m3 graph replay")
    assert pad.pad_check_device_errors() == 0
