"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element by
element, on the same seeded inputs.

Small cases span several 64-token pipeline stages and ragged tails, every head
tile shape (group 1..32, one or two tiles at D=256), every head_dim, several
block sizes, HND and NHD layouts, explicit and heuristic partition counts, and
the degenerate cases (L = 0, L = 1, L < block_size, one block).  The five named
workloads run at full size in the launch configuration the benchmark times and
are compared on sampled (b, h) outputs the oracle computes one by one.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import (DeviceWorkload, check_parity, oracle_pairs, sample_pairs, to_f64)

pytestmark = pytest.mark.gpu


def _case(name, B, Hq, Hkv, D, bs, lens, seed, **kw):
    return synth.make_workload(name, B, Hq, Hkv, D, bs, lens, seed=seed, **kw)


SMALL = [
    # name, B, Hq, Hkv, D, bs, lens
    ("g4_d128_bs16", 3, 8, 2, 128, 16, [256, 100, 17]),
    ("g5_d128_bs16", 2, 10, 2, 128, 16, [300, 64]),
    ("g1_d128_bs32", 4, 4, 4, 128, 32, [1, 31, 33, 200]),
    ("g8_d64_bs4", 2, 16, 2, 64, 4, [129, 7]),
    ("g12_d64_bs8", 2, 24, 2, 64, 8, [90, 250]),
    ("g32_d128_bs32", 3, 32, 1, 128, 32, [16, 500, 1000]),
    ("g4_d256_bs16", 2, 8, 2, 256, 16, [333, 48]),
    ("g20_d256_bs16", 2, 20, 1, 256, 16, [150, 70]),   # two head tiles at D=256
    ("g2_d128_bs1", 2, 4, 2, 128, 1, [65, 3]),
    ("g3_d128_bs256", 2, 6, 2, 128, 256, [700, 255]),
    ("empty_and_one", 4, 8, 2, 128, 16, [0, 1, 0, 15]),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_small_cases_match_oracle(cuda_device, case, splits):
    name, B, Hq, Hkv, D, bs, lens = case
    w = _case(name, B, Hq, Hkv, D, bs, lens, seed=zlib.crc32(name.encode()) % 1000, max_blocks_per_seq=max(1, -(-max(lens) // bs)) + 2)
    ref_out, ref_lse = oracle.decode_workload(w)
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"{name}/S={splits}")
    assert pad.pad_check_device_errors() == 0


@pytest.mark.parametrize("splits", [1, 2, 5])
def test_nhd_layout_matches_oracle(cuda_device, splits):
    w = _case("nhd", 3, 12, 3, 128, 16, [400, 33, 160], seed=31, max_blocks_per_seq=30)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device, layout="nhd").run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "nhd")


def test_tiny_workload_every_split_count(cuda_device):
    w = synth.config("tiny")
    ref_out, ref_lse = oracle.decode_workload(w)
    dw = DeviceWorkload(w, cuda_device)
    for splits in (1, 2, 3, 4, 5, 8, 16):
        out, lse = dw.run(num_splits=splits)
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"tiny/S={splits}")


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (32, 1, 128), (16, 4, 256)])
@pytest.mark.parametrize("splits", [4, 2, 0])
def test_many_short_units_per_cta(cuda_device, Hq, Hkv, D, splits):
    # Capacity 256 tokens: S=4 gives one-stage (64-token) partitions, S=2
    # two-stage ones with one-stage tails, and ragged lengths (0 .. 256) leave
    # many sequences with a single non-empty partition.  Over a thousand short
    # units run at once, and the split merges of different sequences finish in
    # arbitrary order.
    lens = np.random.default_rng(5).integers(0, 257, size=160).tolist()
    w = _case(f"short_units_g{Hq // Hkv}_d{D}", 160, Hq, Hkv, D, 16, lens, seed=49, max_blocks_per_seq=16)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"short_units/S={splits}")
    assert pad.pad_check_device_errors() == 0


def test_block_table_permutation_is_bitwise_invariant(cuda_device):
    w = _case("perm", 2, 8, 2, 128, 16, [300, 77], seed=41, pool_blocks=60)
    out0, lse0 = DeviceWorkload(w, cuda_device).run(num_splits=3)
    pi = np.random.default_rng(3).permutation(w.num_blocks)
    k2, v2 = np.empty_like(w.k_cache), np.empty_like(w.v_cache)
    k2[pi], v2[pi] = w.k_cache, w.v_cache
    w2 = synth.Workload(**{**w.__dict__, "k_cache": k2, "v_cache": v2,
                           "block_tables": pi[w.block_tables].astype(np.int32)})
    out1, lse1 = DeviceWorkload(w2, cuda_device).run(num_splits=3)
    assert torch.equal(out0.view(torch.int16), out1.view(torch.int16))
    assert torch.equal(lse0, lse1)


def test_constant_values_give_that_constant(cuda_device):
    w = _case("constv", 2, 8, 2, 128, 16, [500, 37], seed=42)
    c = synth.f32_to_bf16_bits(np.linspace(-3, 3, 128, dtype=np.float32))
    w.v_cache[:] = c
    out, _ = DeviceWorkload(w, cuda_device).run(num_splits=0)
    got = to_f64(out)
    want = synth.bf16_to_f64(c)
    # weights sum to 1 in fp32, then one bf16 rounding: within one bf16 ulp of c
    ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7), 2.0 ** -133)
    assert np.all(np.abs(got - want) <= ulp)


def test_lse_none_writes_nothing_else(cuda_device):
    # a call without an LSE output must not write the buffer an earlier call used
    w = _case("nolse", 2, 8, 2, 128, 16, [129, 64], seed=43)
    dw = DeviceWorkload(w, cuda_device)
    for splits in (1, 2):
        lse_buf = torch.empty((w.B, w.Hq), device=cuda_device)
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=splits, out=out, lse=lse_buf)
        lse_buf.fill_(7.25)
        out2, lse2 = dw.run(num_splits=splits, lse=False)
        torch.cuda.synchronize()
        assert lse2 is None and torch.all(lse_buf == 7.25)
        ref_out, _ = oracle.decode_workload(w)
        check_parity(to_f64(out2), None, ref_out, None, "nolse")


def test_strided_outputs(cuda_device):
    # out and lse as views into larger buffers (row strides > D, lse transposed)
    w = _case("strided_out", 3, 8, 2, 128, 16, [90, 200, 5], seed=44)
    dw = DeviceWorkload(w, cuda_device)
    big = torch.full((w.B, w.Hq, 2 * w.D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    out = big[:, :, 64:64 + w.D]
    lse_buf = torch.full((w.Hq, w.B), float("nan"), device=cuda_device)
    lse = lse_buf.t()
    pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=2, out=out, lse=lse)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "strided")
    assert torch.isnan(big[:, :, :64].float()).all() and torch.isnan(big[:, :, 64 + w.D:].float()).all()


def test_invalid_arguments_leave_outputs_untouched(cuda_device):
    w = _case("bad", 2, 8, 2, 128, 16, [40, 20], seed=45)
    dw = DeviceWorkload(w, cuda_device)
    out = torch.full((w.B, w.Hq, w.D), 3.0, dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((w.B, w.Hq), 5.0, device=cuda_device)
    bad_lse = torch.full((w.B, w.Hq + 1), 5.0, device=cuda_device)
    with pytest.raises(pad.PadError) as e:
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, out=out, lse=bad_lse)
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
    with pytest.raises(pad.PadError):
        pad.pad_decode(dw.q, dw.k, dw.v[:, :1], dw.tables, dw.lens, w.scale, out=out, lse=lse)
    with pytest.raises(pad.PadError):
        pad.pad_decode(dw.q[:, :7], dw.k, dw.v, dw.tables, dw.lens, w.scale, out=out[:, :7], lse=lse[:, :7])
    with pytest.raises(pad.PadError):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, float("inf"), out=out, lse=lse)
    with pytest.raises((pad.PadError, ValueError)):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables.cpu(), dw.lens, w.scale, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(out.float() == 3.0) and torch.all(lse == 5.0) and torch.all(bad_lse == 5.0)


def test_bad_device_data_is_flagged_not_dereferenced(cuda_device):
    w = _case("badtable", 2, 8, 2, 128, 16, [64, 64], seed=46)
    dw = DeviceWorkload(w, cuda_device)
    assert pad.pad_check_device_errors() == 0
    dw.tables[1, 2] = w.num_blocks + 1000  # out of range: must be skipped, not read
    dw.run(num_splits=1)
    assert pad.pad_check_device_errors() & 0x1
    dw.tables[1, 2] = int(w.block_tables[1, 2])
    dw.lens[0] = 10_000_000  # beyond the table capacity: clamped
    dw.run(num_splits=2)
    assert pad.pad_check_device_errors() & 0x2
    assert pad.pad_check_device_errors() == 0


def test_plan_matches_launch_and_heuristic_shapes(cuda_device):
    p = pad.pad_decode_plan(64, 40, 8, 128, 16, 512, num_splits=16)
    assert p["num_splits"] == 16 and p["partition_tokens"] == 512 and p["reduce"] == 1
    p = pad.pad_decode_plan(16, 16, 4, 256, 16, 2048, num_splits=32)
    assert p["num_splits"] == 32 and p["partition_tokens"] == 1024
    p = pad.pad_decode_plan(1, 4, 1, 128, 16, 16, num_splits=1)
    assert p["num_splits"] == 1 and p["reduce"] == 0 and p["workspace_bytes"] == 0 and p["ctas"] == 1
    assert p["control_bytes"] == 0
    p = pad.pad_decode_plan(256, 32, 1, 128, 32, 1024, num_splits=0)
    assert p["partition_tokens"] % 32 == 0 and p["heads_per_tile"] == 32


def test_graph_capture_replays(cuda_device):
    w = _case("graph", 4, 8, 2, 128, 16, [300, 40, 129, 512], seed=47)
    dw = DeviceWorkload(w, cuda_device)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((w.B, w.Hq), device=cuda_device)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4, out=out, lse=lse)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=4, out=out, lse=lse)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "graph")
    # growing scratch under capture is refused, with nothing launched
    g2 = torch.cuda.CUDAGraph()
    with pytest.raises(pad.PadError) as e:
        with torch.cuda.graph(g2, stream=s):
            pad.pad_decode(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, num_splits=64, out=out, lse=lse)
    assert e.value.status == pad.PAD_ERR_WORKSPACE


# ---- the five named workloads at full size, every output -------------------

@pytest.mark.parametrize("name", synth.CONFIG_NAMES)
def test_named_workload_full_size(cuda_device, name):
    """The workload exactly as benchmarked (its own partition count, 0 =
    heuristic), every (b, head) row of out and lse against the oracle over the
    whole batch; sampled pairs (longest and shortest sequences, first and last
    heads) run first as a quick check that fails with a small report."""
    w = synth.config(name)
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run()
    got_out, got_lse = to_f64(out), lse.cpu().numpy()
    if name != "tiny":
        pairs = sample_pairs(w, 48, seed=7)
        ref_o, ref_l = oracle_pairs(w, pairs)
        idx_b, idx_h = [b for b, _ in pairs], [h for _, h in pairs]
        check_parity(got_out[idx_b, idx_h], got_lse[idx_b, idx_h], ref_o, ref_l, name + " (sampled)")
    ref_out, ref_lse = oracle.decode_workload(w)
    check_parity(got_out, got_lse, ref_out, ref_lse, name)
    assert pad.pad_check_device_errors() == 0
    del dw
    torch.cuda.empty_cache()


def _round256(x):
    return -(-x // 256) * 256


def test_partition_partials_match_oracle_on_subranges(cuda_device):
    """Caller-owned partials scratch: after the call, partition s of every (b, h)
    whose sequence has several non-empty partitions holds the attention over
    tokens [s*P, min((s+1)*P, L_b)) (normalised by its own sum) and that range's
    LSE, and the merged output is the full result.  The scratch starts as
    garbage (NaN) and is reused by a second call."""
    w = _case("phases", 3, 10, 2, 128, 16, [300, 45, 129], seed=48, max_blocks_per_seq=20)
    dw = DeviceWorkload(w, cuda_device)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=4)
    S, P, HT = plan["num_splits"], plan["partition_tokens"], plan["head_tiles"]
    assert S == 4 and P == 80
    ws = torch.full((plan["workspace_bytes"] // 4,), float("nan"), dtype=torch.float32, device=cuda_device)
    ref_out, ref_lse = oracle.decode_workload(w)
    lse_off = _round256(w.B * w.Hq * S * w.D * 4) // 4
    assert (lse_off + _round256(w.B * w.Hq * S * 4) // 4) * 4 == plan["workspace_bytes"]  # light units: no order
    assert plan["control_bytes"] == _round256(w.B * w.Hkv * HT * 4)
    for call in range(2):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        lse = torch.full((w.B, w.Hq), float("nan"), device=cuda_device)
        pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 4, out, lse, ws)
        torch.cuda.synchronize()
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"workspace call {call}")
        opart = ws[: w.B * w.Hq * S * w.D].view(w.B, w.Hq, S, w.D).cpu().numpy().astype(np.float64)
        lpart = ws[lse_off: lse_off + w.B * w.Hq * S].view(w.B, w.Hq, S).cpu().numpy().astype(np.float64)
        for b in range(w.B):
            L = int(w.seq_lens[b])
            ns = -(-L // P)
            if ns < 2:
                continue
            for s in range(ns):
                a, e = s * P, min((s + 1) * P, L)
                t = np.ascontiguousarray(w.block_tables[b:b + 1, a // 16: -(-e // 16)])
                ro, rl = oracle.decode(np.ascontiguousarray(w.q[b:b + 1]), w.k_cache, w.v_cache, t,
                                       np.asarray([e - a], np.int32), w.scale)
                np.testing.assert_allclose(opart[b, :, s], ro[0], rtol=0, atol=1e-2)
                np.testing.assert_allclose(lpart[b, :, s], rl[0], rtol=1e-4, atol=1e-4)
    # a different shape on the same stream right after (the library's control
    # block is reused and must have been left zero)
    w2 = _case("phases2", 5, 8, 1, 64, 32, [1000, 3, 64, 65, 0], seed=49, max_blocks_per_seq=40)
    out2, lse2 = DeviceWorkload(w2, cuda_device).run(num_splits=0)
    r2o, r2l = oracle.decode_workload(w2)
    check_parity(to_f64(out2), lse2.cpu().numpy(), r2o, r2l, "second shape")
    # too small a workspace is refused before launching
    with pytest.raises(pad.PadError):
        pad.pad_decode_with_workspace(dw.q, dw.k, dw.v, dw.tables, dw.lens, w.scale, 4, out, lse, ws[:16])
