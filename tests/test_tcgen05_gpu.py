"""GPU parity of pad_decode_tcgen05 (the 5th-generation tensor-core kernel)
against the CPU oracle: groups of 17..32 query heads per KV head at head_dim
128, several block sizes, split counts, ragged tails and degenerate lengths, and
the full-size ragged MQA batch on sampled outputs."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
import paged_kv_attention_partition_b200 as pad
from pad_testing import DeviceWorkload, check_parity, oracle_pairs, sample_pairs, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, Hq, Hkv, D, bs, lens
    ("g32_bs32", 3, 32, 1, 128, 32, [16, 500, 1000]),
    ("g32_bs16_two_heads", 2, 64, 2, 128, 16, [129, 300]),
    ("g20_padded_tile", 2, 20, 1, 128, 16, [150, 70]),
    ("g32_bs8_edges", 5, 32, 1, 128, 8, [0, 1, 7, 8, 257]),
    ("g24_bs256", 2, 48, 2, 128, 256, [700, 255]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_tcgen05_matches_oracle(cuda_device, case, splits):
    name, B, Hq, Hkv, D, bs, lens = case
    w = synth.make_workload(name, B, Hq, Hkv, D, bs, lens, seed=zlib.crc32(name.encode()) % 1000,
                            max_blocks_per_seq=max(1, -(-max(lens) // bs)) + 2)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits, entry=pad.pad_decode_tcgen05)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"{name}/S={splits}")
    assert pad.pad_check_device_errors() == 0


@pytest.mark.parametrize("splits", [4, 2, 0])
def test_tcgen05_many_short_units(cuda_device, splits):
    lens = np.random.default_rng(5).integers(0, 257, size=160).tolist()
    w = synth.make_workload("tc_short", 160, 32, 1, 128, 16, lens, seed=49, max_blocks_per_seq=16)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits, entry=pad.pad_decode_tcgen05)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"tc_short/S={splits}")
    assert pad.pad_check_device_errors() == 0


def test_tcgen05_nhd_layout(cuda_device):
    w = synth.make_workload("tc_nhd", 3, 64, 2, 128, 16, [400, 33, 160], seed=31, max_blocks_per_seq=30)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device, layout="nhd").run(num_splits=2, entry=pad.pad_decode_tcgen05)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, "tc_nhd")


def test_tcgen05_ragged_mqa_full_size(cuda_device):
    w = synth.config("ragged_mqa")
    dw = DeviceWorkload(w, cuda_device)
    out, lse = dw.run(entry=pad.pad_decode_tcgen05)
    pairs = sample_pairs(w, 48, seed=11)
    ref_out, ref_lse = oracle_pairs(w, pairs)
    got_out = to_f64(out[[b for b, _ in pairs], [h for _, h in pairs]])
    got_lse = lse[[b for b, _ in pairs], [h for _, h in pairs]].cpu().numpy()
    check_parity(got_out, got_lse, ref_out, ref_lse, "ragged_mqa/tcgen05")
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert pad.pad_check_device_errors() == 0
    del dw
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape", [(2, 8, 2, 128, 16), (2, 32, 1, 64, 16), (2, 32, 1, 128, 4)],
                         ids=["group4", "head_dim64", "block4"])
def test_tcgen05_rejects_other_shapes(cuda_device, shape):
    B, Hq, Hkv, D, bs = shape
    w = synth.make_workload("tc_bad", B, Hq, Hkv, D, bs, [40, 20], seed=3)
    dw = DeviceWorkload(w, cuda_device)
    with pytest.raises(pad.PadError) as e:
        dw.run(entry=pad.pad_decode_tcgen05)
    assert e.value.status == pad.PAD_ERR_UNSUPPORTED
