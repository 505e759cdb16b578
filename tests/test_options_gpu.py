"""GPU parity of the decode options against the CPU oracle: sliding window,
attention sinks, both together, and block-sparse attention through a compacted
block table ("Attention parity: run every attention type on the best available
path on both targets", section "Current state", and its "Non-gap: block-sparse
GQA": selected blocks compacted into page tables)."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu

WINDOW_CASES = [
    # name, B, Hq, Hkv, D, bs, lens, window
    ("w64_bs16", 3, 8, 2, 128, 16, [300, 40, 1000], 64),
    ("w1", 2, 8, 2, 128, 16, [129, 2], 1),
    ("w_ragged_bs32", 4, 32, 1, 128, 32, [16, 500, 1000, 77], 100),
    ("w_d64_bs4", 2, 16, 2, 64, 4, [129, 7], 33),
    ("w_d256", 2, 8, 2, 256, 16, [333, 48], 70),
    ("w_bs1", 2, 4, 2, 128, 1, [65, 3], 17),
    ("w_bs256", 2, 6, 2, 128, 256, [700, 255], 300),
    ("w_larger_than_L", 2, 8, 2, 128, 16, [50, 10], 5000),
]


def _case(name, B, Hq, Hkv, D, bs, lens, **kw):
    return synth.make_workload(name, B, Hq, Hkv, D, bs, lens, seed=zlib.crc32(name.encode()) % 1000,
                               max_blocks_per_seq=max(1, -(-max(lens) // bs)) + 2, **kw)


@pytest.mark.parametrize("case", WINDOW_CASES, ids=[c[0] for c in WINDOW_CASES])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_window_matches_oracle(cuda_device, case, splits):
    name, B, Hq, Hkv, D, bs, lens, W = case
    w = _case(name, B, Hq, Hkv, D, bs, lens)
    ref_out, ref_lse = oracle.decode_workload(w, window=W)
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run(num_splits=splits, entry=lambda *a, **k: pad.pad_decode(*a, window=W, **k))
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"{name}/S={splits}")
    assert pad.pad_check_device_errors() == 0


@pytest.mark.parametrize("splits", [1, 4, 0])
def test_window_never_reads_pages_before_it(cuda_device, splits):
    # Table entries wholly before the window hold an out-of-range block id: a
    # kernel that issued a copy for one would flag it in the device error word.
    lens = [1000, 700, 64]
    W, bs = 150, 16
    w = _case("w_skip", 3, 8, 2, 128, bs, lens)
    ref_out, ref_lse = oracle.decode_workload(w, window=W)
    tables = w.block_tables.copy()
    for b, L in enumerate(lens):
        lo = max(0, L - W)
        tables[b, : lo // bs] = 1 << 30
    w2 = synth.Workload(**{**w.__dict__, "block_tables": tables})
    out, lse = DeviceWorkload(w2, cuda_device).run(num_splits=splits,
                                                   entry=lambda *a, **k: pad.pad_decode(*a, window=W, **k))
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"w_skip/S={splits}")
    assert pad.pad_check_device_errors() == 0


def _sinks(Hq, seed):
    r = np.random.default_rng(seed)
    s = (r.standard_normal(Hq) * 2.0).astype(np.float32)
    s[::5] = -np.inf
    if Hq > 3:
        s[3] = 25.0  # a sink far above every score: out -> 0, lse -> sink
    return s


SINK_CASES = [
    ("sink_g4", 3, 8, 2, 128, 16, [300, 40, 1000], 0),
    ("sink_g32", 3, 32, 1, 128, 32, [16, 500, 1000], 0),
    ("sink_empty_seq", 4, 8, 2, 128, 16, [0, 1, 0, 15], 0),
    ("sink_d256_window", 2, 8, 2, 256, 16, [333, 48], 40),
    ("sink_d64_window", 2, 16, 2, 64, 4, [129, 7], 9),
]


@pytest.mark.parametrize("case", SINK_CASES, ids=[c[0] for c in SINK_CASES])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_sinks_match_oracle(cuda_device, case, splits):
    name, B, Hq, Hkv, D, bs, lens, W = case
    w = _case(name, B, Hq, Hkv, D, bs, lens)
    sinks = _sinks(Hq, zlib.crc32(name.encode()))
    ref_out, ref_lse = oracle.decode_workload(w, window=W, sinks=sinks)
    dev_sinks = torch.from_numpy(sinks).to(cuda_device)
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run(num_splits=splits,
                      entry=lambda *a, **k: pad.pad_decode(*a, window=W, sinks=dev_sinks, **k))
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"{name}/S={splits}")
    assert pad.pad_check_device_errors() == 0


def test_block_sparse_through_a_compacted_table(cuda_device):
    # Block-sparse GQA: the selected blocks of a long sequence (a few leading
    # blocks, scattered picks, the local tail) compacted into a block table of
    # their own.  The result must be attention over exactly the selected
    # tokens, computed here from contiguous rows in float64 (no paging at all).
    bs, D, Hq, Hkv = 16, 128, 8, 2
    g = Hq // Hkv
    r = np.random.default_rng(77)
    L_full = 1000
    nblk = -(-L_full // bs)
    k_contig = synth.f32_to_bf16_bits(r.standard_normal((Hkv, nblk * bs, D)).astype(np.float32))
    v_contig = synth.f32_to_bf16_bits(r.standard_normal((Hkv, nblk * bs, D)).astype(np.float32))
    q = synth.f32_to_bf16_bits(r.standard_normal((1, Hq, D)).astype(np.float32))
    selected = sorted({0, 1, 7, 19, 30, 44, 51, nblk - 2, nblk - 1})
    tail = L_full - (nblk - 1) * bs  # the last (local) block is partial
    # physical pool: the selected logical blocks land in a permuted order
    pool = r.permutation(len(selected) + 3)
    kc = np.zeros((len(pool), Hkv, bs, D), dtype=np.uint16)
    vc = np.zeros_like(kc)
    table = np.zeros((1, len(selected)), dtype=np.int32)
    for j, blk in enumerate(selected):
        phys = int(pool[j])
        table[0, j] = phys
        kc[phys] = k_contig[:, blk * bs:(blk + 1) * bs]
        vc[phys] = v_contig[:, blk * bs:(blk + 1) * bs]
    L = (len(selected) - 1) * bs + tail
    w = synth.Workload(name="sparse", B=1, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, q=q, k_cache=kc, v_cache=vc,
                       block_tables=table, seq_lens=np.asarray([L], dtype=np.int32), scale=1 / math.sqrt(D),
                       num_splits=0, want_lse=True, seed=77, recipe="block-sparse selection")
    # reference over the selected tokens, from the contiguous rows
    toks = np.concatenate([np.arange(blk * bs, blk * bs + (tail if blk == nblk - 1 else bs)) for blk in selected])
    f = lambda bits: synth.bf16_to_f64(bits)
    ref_out = np.zeros((1, Hq, D))
    ref_lse = np.zeros((1, Hq))
    for h in range(Hq):
        kh = h // g
        s = (f(k_contig[kh, toks]) @ f(q[0, h])) * w.scale
        m = s.max()
        e = np.exp(s - m)
        ref_out[0, h] = (e / e.sum()) @ f(v_contig[kh, toks])
        ref_lse[0, h] = m + math.log(e.sum())
    for splits in (1, 3, 0):
        out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
        check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"sparse/S={splits}")


def test_invalid_options_are_rejected(cuda_device):
    w = _case("opt_bad", 2, 8, 2, 128, 16, [40, 20])
    dw = DeviceWorkload(w, cuda_device)
    with pytest.raises(pad.PadError) as e:
        dw.run(entry=lambda *a, **k: pad.pad_decode(*a, window=-1, **k))
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
    with pytest.raises(pad.PadError) as e:
        dw.run(entry=lambda *a, **k: pad.pad_decode(*a, sinks=torch.zeros(7, device=cuda_device), **k))
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
    with pytest.raises(pad.PadError) as e:  # fp32 but [2, 4], not [Hq]
        dw.run(entry=lambda *a, **k: pad.pad_decode(*a, sinks=torch.zeros(2, 4, device=cuda_device), **k))
    assert e.value.status == pad.PAD_ERR_INVALID_ARG
