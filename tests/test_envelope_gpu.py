"""The edges of the supported envelope on the GPU: the largest query-head group
(256 per KV head: 8 tiles of 32 heads at head_dim <= 128, 16 tiles of 16 at
256), the smallest and largest pages (1 and 256 tokens), for both cache types,
against the oracle at the parity bar."""
import pytest

import oracle
import synth
from pad_testing import DeviceWorkload, check_parity, to_f64

pytestmark = pytest.mark.gpu

EDGES = [
    # D, bs, lens, kv, splits
    (64, 1, [70, 1], "bf16", 3),
    (128, 256, [600, 255], "bf16", 0),
    (256, 16, [200, 33], "bf16", 2),
    (128, 8, [300, 9], "e4m3", 0),
    (256, 256, [520, 1], "e4m3", 3),
    (64, 256, [257, 40], "e4m3", 1),
]


@pytest.mark.parametrize("D,bs,lens,kv,splits", EDGES,
                         ids=[f"D{e[0]}_bs{e[1]}_{e[3]}_S{e[4]}" for e in EDGES])
def test_group_of_256_heads(cuda_device, D, bs, lens, kv, splits):
    width = -(-max(lens) // bs) + 1
    w = synth.make_workload(f"edge_{D}_{bs}_{kv}", len(lens), 256, 1, D, bs, lens, seed=70 + D + bs,
                            max_blocks_per_seq=width, kv_dtype=kv)
    ref_out, ref_lse = oracle.decode_workload(w)
    out, lse = DeviceWorkload(w, cuda_device).run(num_splits=splits)
    check_parity(to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, f"g=256 D={D} bs={bs} {kv} S={splits}")
