"""The seeded input generator: deterministic, counter-based, well-formed tables."""
import numpy as np

import synth


def test_fill_is_counter_based_and_thread_independent():
    a = synth.bf16_array((5000,), seed=3, stream=synth.S_K)
    b = synth.bf16_array((5000,), seed=3, stream=synth.S_K)
    assert np.array_equal(a, b)
    # a sub-range regenerated on its own equals the same slice
    lib = synth._l()
    part = np.empty(100, dtype=np.uint16)
    lib.synth_fill_bf16(part.ctypes.data, 100, 1234, 3, synth.S_K, synth.DIST_NORMAL, 1)
    assert np.array_equal(part, a[1234:1334])
    assert not np.array_equal(a, synth.bf16_array((5000,), seed=4, stream=synth.S_K))


def test_distributions_have_the_stated_moments():
    z = synth.bf16_to_f64(synth.bf16_array((400_000,), seed=1, stream=9))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    u = synth.bf16_to_f64(synth.bf16_array((400_000,), seed=1, stream=9, dist=synth.DIST_UNIFORM_PM1))
    assert u.min() >= -1.0 and u.max() <= 1.0 and abs(u.mean()) < 0.01
    assert abs(u.var() - 1.0 / 3.0) < 0.01


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0)
    assert bits[1] == 0x3F80
    # 1 + 3*2^-8 is a tie between 1+2^-7 and 1+2^-6: rounds to even (1+2^-6)
    assert bits[2] == 0x3F82
    assert np.array_equal(synth.bf16_to_f64(bits[[0, 3]]), [1.0, -2.5])


def test_permutation_prefix_is_without_replacement():
    p = synth.permutation_prefix(1000, 1000, seed=7, stream=5)
    assert sorted(p.tolist()) == list(range(1000))
    q = synth.permutation_prefix(300_000, 5000, seed=7, stream=5)
    assert len(set(q.tolist())) == 5000 and q.min() >= 0 and q.max() < 300_000


def test_workload_tables_and_poison():
    w = synth.make_workload("t", 3, 8, 2, 32, 16, [33, 16, 0], seed=5, pool_blocks=20, max_blocks_per_seq=4)
    assert w.block_tables.shape == (3, 4) and w.num_blocks == 21
    poison = w.num_blocks - 1
    live = [w.block_tables[0, :3], w.block_tables[1, :1]]
    assert len(set(np.concatenate(live).tolist())) == 4
    assert (w.block_tables[0, 3:] == poison).all() and (w.block_tables[1, 1:] == poison).all()
    assert (w.block_tables[2] == poison).all()
    assert (w.k_cache[poison] == synth.BF16_NAN).all()
    last = w.block_tables[0, 2]
    assert (w.k_cache[last, :, 1:] == synth.BF16_NAN).all() and (w.v_cache[last, :, 1:] == synth.BF16_NAN).all()
    assert not (w.k_cache[last, :, 0] == synth.BF16_NAN).any()


def test_cyclic_tables_wrap_the_pool():
    w = synth.make_workload("c", 4, 4, 1, 16, 4, [40, 40, 40, 40], seed=6, pool_blocks=25, table_mode="cyclic")
    ids = np.concatenate([w.block_tables[b, :10] for b in range(4)])
    assert ids.max() < 25 and len(set(ids.tolist())) == 25


def test_named_configs_shapes_small():
    w = synth.config("tiny")
    assert (w.B, w.Hq, w.Hkv, w.D, w.block_size) == (1, 4, 1, 128, 16)
    assert sorted(w.block_tables[0].tolist()) == list(range(16)) and int(w.seq_lens[0]) == 256
    assert w.num_splits == 1
