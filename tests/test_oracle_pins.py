"""Pins for the CPU oracle: facts fixed by mathematics or by a library routine,
never by the oracle itself.

The pages print no worked example and no numeric attention value, so every pin
here is a definition-level fact about softmax attention over the tokens a block
table names ("spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm", section
"The gap it specs"; "perf(rocke): prepare saved paged decode bindings once",
section "Summary"):

* brute force: the paged oracle equals torch's float64 scaled-dot-product
  attention on contiguous K/V that a separate routine scatters into pages;
* weights: with V = identity rows the output *is* the weight vector, which must
  equal scipy's softmax of the scaled scores and sum to 1;
* invariants: block-table permutation invariance, layout (HND vs NHD)
  invariance, constant V gives that constant;
* closed forms: q = 0 (uniform weights, lse = ln L, out = mean V), L = 1
  (out = v_0, lse = scale q.k_0), a dominant score (out = v_argmax), L = 0;
* split combine: attention over disjoint token ranges merged by log-sum-exp
  equals attention over the union (the identity the split-KV reduce relies on);
* sliding window: equals torch's SDPA over each sequence's last W contiguous
  tokens; W = 1 gives the last value row exactly;
* attention sinks: equals scipy's softmax over the scores with the sink logit
  appended (zero value row); a -inf sink changes nothing; an empty sequence
  gives out = 0, lse = sink.
* E4M3 cache: every one of the 256 codes, read back through one-token
  sequences, equals torch's float8_e4m3fn widening (and the values the OCP FP8
  definition fixes: 448, 2^-9, 2^-6, +-1, two NaNs) times the tensor's scale;
  the paged oracle equals SDPA on the dequantised contiguous K/V; a
  power-of-two k_scale is the same as scaling the scores, v_scale scales out
  and leaves lse alone; with both scales 1 it equals the bf16 path on the same
  values, bitwise.

``test_planted_mistakes_are_caught`` compiles copies of the oracle with one
plausible mistake each and checks that some pin fails for every one.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth

def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return synth.bf16_to_f64(bits)


def scatter_to_pages(k_contig, v_contig, lens, bs, extra_blocks, seed):
    """Separate routine (not the oracle's gather): place contiguous per-sequence
    K/V [B, Hkv, Lmax, D] (bf16 bits or E4M3 codes) into a paged cache at
    randomly chosen physical blocks."""
    B, Hkv, Lmax, D = k_contig.shape
    nan = synth.E4M3_NAN if k_contig.dtype == np.uint8 else synth.BF16_NAN
    need = [(int(L) + bs - 1) // bs for L in lens]
    nblocks = sum(need) + extra_blocks
    perm = _rng(seed).permutation(nblocks)
    width = max(max(need), 1)
    # entries past the live blocks point at a NaN-filled spare block
    tables = np.full((B, width), int(perm[-1]), dtype=np.int32)
    kc = np.full((nblocks, Hkv, bs, D), nan, dtype=k_contig.dtype)
    vc = np.full((nblocks, Hkv, bs, D), nan, dtype=k_contig.dtype)
    nxt = 0
    for b in range(B):
        for j in range(need[b]):
            phys = int(perm[nxt])
            nxt += 1
            tables[b, j] = phys
            lo, hi = j * bs, min((j + 1) * bs, int(lens[b]))
            kc[phys, :, : hi - lo, :] = k_contig[b, :, lo:hi, :]
            vc[phys, :, : hi - lo, :] = v_contig[b, :, lo:hi, :]
    return kc, vc, tables


def library_attention(q, k_contig, v_contig, lens, scale, kf=None, vf=None):
    """torch float64 SDPA (+ torch.logsumexp) on contiguous K/V, per sequence.
    Query head h reads KV head h // (Hq/Hkv) via repeat_interleave.  kf / vf
    widen the stored K / V elements (default: bf16 bits)."""
    kf = kf or _f
    vf = vf or _f
    B, Hq, D = q.shape
    Hkv = k_contig.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        L = int(lens[b])
        qt = torch.from_numpy(_f(q[b]))[:, None, :]                      # [Hq, 1, D]
        kt = torch.from_numpy(kf(k_contig[b, :, :L])).repeat_interleave(g, 0)  # [Hq, L, D]
        vt = torch.from_numpy(vf(v_contig[b, :, :L])).repeat_interleave(g, 0)
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
        out[b] = o[:, 0, :].numpy()
        lse[b] = torch.logsumexp(scale * (qt @ kt.transpose(1, 2))[:, 0, :], dim=-1).numpy()
    return out, lse


def random_case(seed, B, Hq, Hkv, D, bs, lens, extra=3):
    r = _rng(seed)
    Lmax = max(int(max(lens)), 1)
    q = _bf16(r.standard_normal((B, Hq, D)))
    kc = _bf16(r.standard_normal((B, Hkv, Lmax, D)))
    vc = _bf16(r.standard_normal((B, Hkv, Lmax, D)))
    return q, kc, vc


# ---------------------------------------------------------------------------
# pins (each takes the oracle library path so planted mistakes can be tested)
# ---------------------------------------------------------------------------

BRUTE_CASES = [
    # B, Hq, Hkv, D, bs, lens
    (1, 1, 1, 8, 1, [1]),
    (2, 4, 1, 16, 4, [5, 15]),
    (3, 8, 2, 32, 16, [16, 17, 40]),
    (2, 10, 2, 16, 4, [40, 1]),
    (1, 5, 1, 64, 16, [33]),
    (2, 6, 6, 8, 1, [7, 3]),
]


def pin_bruteforce(lib):
    for i, (B, Hq, Hkv, D, bs, lens) in enumerate(BRUTE_CASES):
        lens = np.asarray(lens, dtype=np.int32)
        q, kc, vc = random_case(100 + i, B, Hq, Hkv, D, bs, lens)
        kp, vp, tables = scatter_to_pages(kc, vc, lens, bs, extra_blocks=2, seed=200 + i)
        scale = 1.0 / math.sqrt(D)
        out, lse = oracle.decode(q, kp, vp, tables, lens, scale, lib_path=lib)
        ref_out, ref_lse = library_attention(q, kc, vc, lens, scale)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def pin_weights_are_softmax(lib):
    # V rows are unit vectors: v_t = e_t, so out[d] = w_d for d < L.
    for (Hq, Hkv, D, bs, L, scale) in [(4, 2, 32, 4, 13, 0.3), (5, 1, 64, 16, 64, 1 / 8), (3, 3, 16, 1, 16, 2.0)]:
        r = _rng(L + D)
        q = _bf16(r.standard_normal((1, Hq, D)))
        kc = _bf16(r.standard_normal((1, Hkv, L, D)))
        eye = np.zeros((1, Hkv, L, D), dtype=np.float32)
        for t in range(L):
            eye[0, :, t, t] = 1.0
        vc = _bf16(eye)
        kp, vp, tables = scatter_to_pages(kc, vc, [L], bs, 1, seed=L)
        out, lse = oracle.decode(q, kp, vp, tables, np.asarray([L], np.int32), scale, lib_path=lib)
        g = Hq // Hkv
        for h in range(Hq):
            s = scale * (_f(kc[0, h // g]) @ _f(q[0, h]))
            w = scipy.special.softmax(s)
            np.testing.assert_allclose(out[0, h, :L], w, rtol=0, atol=1e-13)
            assert abs(out[0, h, :L].sum() - 1.0) <= 1e-12
            assert np.all(out[0, h, L:] == 0.0)
            assert abs(lse[0, h] - scipy.special.logsumexp(s)) <= 1e-12


def pin_permutation_invariance(lib):
    w = synth.make_workload("perm", 3, 8, 2, 32, 4, [9, 30, 17], seed=11, pool_blocks=40)
    out0, lse0 = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    pi = _rng(5).permutation(w.num_blocks)
    k2 = np.empty_like(w.k_cache)
    v2 = np.empty_like(w.v_cache)
    k2[pi] = w.k_cache
    v2[pi] = w.v_cache
    t2 = pi[w.block_tables].astype(np.int32)
    out1, lse1 = oracle.decode(w.q, k2, v2, t2, w.seq_lens, w.scale, lib_path=lib)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


def pin_layout_invariance(lib):
    # the same logical cache stored NHD ([blocks, bs, Hkv, D]) and read through strides
    w = synth.make_workload("nhd", 2, 6, 3, 16, 8, [21, 8], seed=12)
    out0, lse0 = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    k_nhd = np.ascontiguousarray(w.k_cache.transpose(0, 2, 1, 3))
    v_nhd = np.ascontiguousarray(w.v_cache.transpose(0, 2, 1, 3))
    out1, lse1 = oracle.decode(w.q, k_nhd.transpose(0, 2, 1, 3), v_nhd.transpose(0, 2, 1, 3),
                               w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


def pin_constant_v(lib):
    w = synth.make_workload("constv", 2, 4, 2, 32, 4, [23, 64], seed=13)
    c = _bf16(np.linspace(-3, 3, 32, dtype=np.float32))
    v = np.broadcast_to(c, w.v_cache.shape).copy()
    out, _ = oracle.decode(w.q, w.k_cache, v, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    np.testing.assert_allclose(out, np.broadcast_to(_f(c), out.shape), rtol=0, atol=1e-12)


def pin_zero_query(lib):
    w = synth.make_workload("q0", 3, 4, 1, 16, 4, [1, 10, 37], seed=14)
    q = np.zeros_like(w.q)
    out, lse = oracle.decode(q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    for b in range(3):
        L = int(w.seq_lens[b])
        toks = np.stack([_f(w.v_cache[w.block_tables[b, t // 4], 0, t % 4]) for t in range(L)])
        np.testing.assert_allclose(lse[b], math.log(L), rtol=0, atol=1e-12)
        np.testing.assert_allclose(out[b], np.broadcast_to(toks.mean(0), (4, 16)), rtol=0, atol=1e-12)


def pin_single_token(lib):
    w = synth.make_workload("l1", 2, 6, 2, 32, 16, [1, 1], seed=15)
    out, lse = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 0.37, lib_path=lib)
    for b in range(2):
        for h in range(6):
            blk = w.block_tables[b, 0]
            k0 = _f(w.k_cache[blk, h // 3, 0])
            v0 = _f(w.v_cache[blk, h // 3, 0])
            assert np.array_equal(out[b, h], v0)
            assert abs(lse[b, h] - 0.37 * float(_f(w.q[b, h]) @ k0)) <= 1e-12


def pin_dominant_score(lib):
    # with a huge scale the softmax puts all weight on the unique best key
    w = synth.make_workload("argmax", 1, 3, 1, 32, 4, [29], seed=16)
    out, _ = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 1e4, lib_path=lib)
    keys = np.stack([_f(w.k_cache[w.block_tables[0, t // 4], 0, t % 4]) for t in range(29)])
    vals = np.stack([_f(w.v_cache[w.block_tables[0, t // 4], 0, t % 4]) for t in range(29)])
    for h in range(3):
        s = keys @ _f(w.q[0, h])
        top = np.sort(s)[-2:]
        assert top[1] - top[0] > 1e-2  # unique maximum with a margin
        np.testing.assert_allclose(out[0, h], vals[int(np.argmax(s))], rtol=0, atol=1e-12)


def pin_empty_sequence(lib):
    w = synth.make_workload("empty", 3, 4, 2, 16, 4, [0, 5, 0], seed=17)
    out, lse = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    assert np.all(np.isfinite(out[1])) and np.all(np.isfinite(lse[1]))


def pin_split_combine(lib):
    # attention over [0,L) equals the lse-weighted merge of attention over
    # block-aligned sub-ranges, each expressed as a shorter block table
    w = synth.make_workload("split", 2, 5, 1, 32, 4, [45, 64], seed=18)
    full_out, full_lse = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    for P in (4, 8, 12, 64):
        for b in range(2):
            L = int(w.seq_lens[b])
            outs, lses = [], []
            for a in range(0, L, P):
                e = min(a + P, L)
                t = np.ascontiguousarray(w.block_tables[b:b + 1, a // 4: (e + 3) // 4])
                o, l = oracle.decode(np.ascontiguousarray(w.q[b:b + 1]), w.k_cache, w.v_cache, t,
                                     np.asarray([e - a], np.int32), w.scale, lib_path=lib)
                outs.append(o[0])
                lses.append(l[0])
            lses = np.stack(lses)              # [S, Hq]
            merged_lse = scipy.special.logsumexp(lses, axis=0)
            wts = np.exp(lses - merged_lse)    # [S, Hq]
            merged = (wts[:, :, None] * np.stack(outs)).sum(0)
            np.testing.assert_allclose(merged_lse, full_lse[b], rtol=0, atol=1e-12)
            np.testing.assert_allclose(merged, full_out[b], rtol=0, atol=1e-12)


WINDOW_CASES = [
    # B, Hq, Hkv, D, bs, lens, window
    (2, 4, 1, 16, 4, [5, 15], 3),
    (3, 8, 2, 32, 16, [16, 17, 40], 16),
    (2, 10, 2, 16, 4, [40, 1], 7),
    (1, 5, 1, 64, 16, [33], 33),
    (2, 6, 6, 8, 1, [7, 3], 100),
]


def pin_window_bruteforce(lib):
    # Sliding window ("Attention parity: run every attention type on the best
    # available path on both targets", section "Current state"): the last W
    # tokens of each sequence, against SDPA on exactly those contiguous rows.
    for i, (B, Hq, Hkv, D, bs, lens, W) in enumerate(WINDOW_CASES):
        lens = np.asarray(lens, dtype=np.int32)
        q, kc, vc = random_case(300 + i, B, Hq, Hkv, D, bs, lens)
        kp, vp, tables = scatter_to_pages(kc, vc, lens, bs, extra_blocks=2, seed=400 + i)
        scale = 1.0 / math.sqrt(D)
        out, lse = oracle.decode(q, kp, vp, tables, lens, scale, lib_path=lib, window=W)
        lo = np.maximum(lens - W, 0)
        wl = (lens - lo).astype(np.int32)
        kw = np.zeros_like(kc)
        vw = np.zeros_like(vc)
        for b in range(B):
            kw[b, :, : wl[b]] = kc[b, :, lo[b]: lens[b]]
            vw[b, :, : wl[b]] = vc[b, :, lo[b]: lens[b]]
        ref_out, ref_lse = library_attention(q, kw, vw, wl, scale)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def pin_window_one(lib):
    # W = 1: the weight of the last token is 1: out = v_{L-1}, lse = s_{L-1}
    lens = np.asarray([9, 1, 30], dtype=np.int32)
    q, kc, vc = random_case(500, 3, 4, 2, 16, 4, lens)
    kp, vp, tables = scatter_to_pages(kc, vc, lens, 4, extra_blocks=1, seed=501)
    out, lse = oracle.decode(q, kp, vp, tables, lens, 0.25, lib_path=lib, window=1)
    for b in range(3):
        for h in range(4):
            kh = h // 2
            last = int(lens[b]) - 1
            np.testing.assert_array_equal(out[b, h], _f(vc[b, kh, last]))
            assert abs(lse[b, h] - 0.25 * float(_f(q[b, h]) @ _f(kc[b, kh, last]))) <= 1e-12


def pin_sinks_are_softmax_terms(lib):
    # Attention sinks (same page, same section): the sink logit joins the
    # softmax with a zero value row -- scipy's softmax over [scores, sink].
    lens = np.asarray([5, 15, 1], dtype=np.int32)
    B, Hq, Hkv, D, bs = 3, 4, 2, 16, 4
    q, kc, vc = random_case(600, B, Hq, Hkv, D, bs, lens)
    kp, vp, tables = scatter_to_pages(kc, vc, lens, bs, extra_blocks=1, seed=601)
    sinks = np.asarray([0.5, -1.0, 3.0, -30.0], dtype=np.float32)
    scale = 0.25
    out, lse = oracle.decode(q, kp, vp, tables, lens, scale, lib_path=lib, sinks=sinks)
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            sc = scale * (_f(kc[b, kh, :L]) @ _f(q[b, h]))
            logits = np.concatenate([sc, [float(sinks[h])]])
            w = scipy.special.softmax(logits)
            np.testing.assert_allclose(out[b, h], w[:L] @ _f(vc[b, kh, :L]), rtol=0, atol=1e-12)
            assert abs(lse[b, h] - scipy.special.logsumexp(logits)) <= 1e-12


def pin_sink_limits(lib):
    # a -inf sink is no sink; an empty sequence with a sink: out = 0, lse = sink
    w = synth.make_workload("sinklim", 3, 4, 1, 32, 8, [20, 0, 3], seed=21)
    plain = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib)
    ninf = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib,
                         sinks=np.full(4, -np.inf, dtype=np.float32))
    assert np.array_equal(plain[0], ninf[0]) and np.array_equal(plain[1], ninf[1])
    sinks = np.asarray([1.0, -2.0, 0.0, 5.0], dtype=np.float32)
    out, lse = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, lib_path=lib,
                             sinks=sinks)
    assert np.all(out[1] == 0.0) and np.array_equal(lse[1], sinks.astype(np.float64))


# ---- E4M3 cache ("perf(rocke): prepare saved paged decode bindings once" names
# an FP8 decode path; format and per-tensor scales are the reading in the
# oracle's header)

def _e4m3_ref(codes):
    """torch's widening of E4M3 codes (uint8) to float64."""
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _e4m3_codes(x):
    """torch's round-to-nearest of float values onto E4M3 codes."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_code_values(lib):
    codes = np.arange(256, dtype=np.uint8)
    ref = _e4m3_ref(codes)
    # the library agrees with values the format's definition fixes
    for c, val in {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x40: 2.0,
                   0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}.items():
        assert ref[c] == val
    assert np.isnan(ref[0x7F]) and np.isnan(ref[0xFF]) and int(np.isnan(ref).sum()) == 2
    assert math.copysign(1.0, ref[0x80]) < 0 and ref[0x80] == 0.0
    # head h reads KV head h; one token; q = e_0 (bf16 1.0 at d = 0)
    D, H = 8, 256
    q = np.zeros((1, H, D), np.uint16)
    q[0, :, 0] = 0x3F80
    tables, lens = np.asarray([[0]], np.int32), np.asarray([1], np.int32)
    ks, vs, scale = 0.75, 0.3, 0.5
    # K codes vary, V zero: lse_h = scale * k_scale * value(code h)
    k = np.zeros((2, H, 1, D), np.uint8)
    k[0, :, 0, 0] = codes
    _, lse = oracle.decode(q, k, np.zeros_like(k), tables, lens, scale, lib_path=lib, k_scale=ks, v_scale=vs)
    np.testing.assert_array_equal(lse[0], scale * (ks * ref))
    # K zero, V codes vary: weight 1, out_h[0] = v_scale * value(code h)
    v = np.zeros((2, H, 1, D), np.uint8)
    v[0, :, 0, 0] = codes
    out, lse = oracle.decode(q, np.zeros_like(v), v, tables, lens, scale, lib_path=lib, k_scale=ks, v_scale=vs)
    np.testing.assert_array_equal(out[0, :, 0], vs * ref)
    assert np.all(lse == 0.0)


E4M3_CASES = [
    # B, Hq, Hkv, D, bs, lens, k_scale, v_scale
    (2, 4, 1, 16, 4, [5, 15], 0.046875, 0.01953125),
    (3, 8, 2, 32, 16, [16, 17, 40], 0.1, 0.02),
    (2, 6, 6, 8, 1, [7, 3], 1.0, 1.0),
]


def pin_e4m3_bruteforce(lib):
    for i, (B, Hq, Hkv, D, bs, lens, ks, vs) in enumerate(E4M3_CASES):
        lens = np.asarray(lens, dtype=np.int32)
        r = _rng(700 + i)
        Lmax = int(lens.max())
        q = _bf16(r.standard_normal((B, Hq, D)))
        kc = _e4m3_codes(r.standard_normal((B, Hkv, Lmax, D)) / ks)
        vc = _e4m3_codes(r.standard_normal((B, Hkv, Lmax, D)) / vs)
        kp, vp, tables = scatter_to_pages(kc, vc, lens, bs, extra_blocks=2, seed=800 + i)
        scale = 1.0 / math.sqrt(D)
        out, lse = oracle.decode(q, kp, vp, tables, lens, scale, lib_path=lib, k_scale=ks, v_scale=vs)
        ref_out, ref_lse = library_attention(q, kc, vc, lens, scale, kf=lambda c: ks * _e4m3_ref(c),
                                             vf=lambda c: vs * _e4m3_ref(c))
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def pin_e4m3_scales(lib):
    w = synth.make_workload("e4m3s", 3, 8, 2, 32, 8, [20, 1, 37], seed=22, kv_dtype="e4m3", k_scale=1.0,
                            v_scale=1.0)
    base = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 0.125, lib_path=lib)
    # k_scale = 2^j is the score scale times 2^j, exactly
    a = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 0.125, lib_path=lib, k_scale=0.25)
    b = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 0.125 * 0.25, lib_path=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.allclose(a[1], base[1])
    # v_scale multiplies out and leaves lse alone
    c = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, 0.125, lib_path=lib, v_scale=0.37)
    np.testing.assert_allclose(c[0], 0.37 * base[0], rtol=0, atol=1e-14)
    assert np.array_equal(c[1], base[1])


def pin_e4m3_equals_bf16_of_same_values(lib):
    w8 = synth.make_workload("e4m3b", 3, 8, 2, 32, 4, [9, 30, 17], seed=23, kv_dtype="e4m3", k_scale=1.0,
                             v_scale=1.0, poison=False)
    kb = _bf16(_e4m3_ref(w8.k_cache))  # E4M3 values are exact in bf16
    vb = _bf16(_e4m3_ref(w8.v_cache))
    a = oracle.decode(w8.q, w8.k_cache, w8.v_cache, w8.block_tables, w8.seq_lens, w8.scale, lib_path=lib)
    b = oracle.decode(w8.q, kb, vb, w8.block_tables, w8.seq_lens, w8.scale, lib_path=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


PINS = [pin_bruteforce, pin_weights_are_softmax, pin_permutation_invariance, pin_layout_invariance,
        pin_constant_v, pin_zero_query, pin_single_token, pin_dominant_score, pin_empty_sequence,
        pin_split_combine, pin_window_bruteforce, pin_window_one, pin_sinks_are_softmax_terms, pin_sink_limits,
        pin_e4m3_code_values, pin_e4m3_bruteforce, pin_e4m3_scales, pin_e4m3_equals_bf16_of_same_values]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.build())


def test_sampled_pairs_match_full():
    w = synth.make_workload("pairs", 3, 8, 2, 32, 4, [9, 30, 17], seed=19)
    out, lse = oracle.decode_workload(w)
    pairs = [(2, 7), (0, 0), (1, 3), (2, 0)]
    o, l = oracle.decode_pairs(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, pairs)
    for i, (b, h) in enumerate(pairs):
        assert np.array_equal(o[i], out[b, h]) and l[i] == lse[b, h]


def test_thread_count_does_not_change_results():
    w = synth.make_workload("thr", 4, 8, 4, 32, 8, [50, 3, 70, 16], seed=20)
    a = oracle.decode_workload(w, nthreads=1)
    b = oracle.decode_workload(w, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------
# planted mistakes: each must trip at least one pin
# ---------------------------------------------------------------------------

MUTATIONS = {
    "scale_dropped": ("s[t - lo] = p->scale * acc;", "s[t - lo] = acc;"),
    "head_map_modulo": ("const int64_t kh = h / g;", "const int64_t kh = h % p->Hkv;"),
    "slot_from_division": ("int64_t slot = t % p->bs;\n    const int64_t krow",
                           "int64_t slot = (t / p->bs) % p->bs;\n    const int64_t krow"),
    "first_page_only": ("int64_t phys = p->tables[b * p->table_width + t / p->bs];\n    int64_t slot = t % p->bs;\n    const int64_t vrow",
                        "int64_t phys = p->tables[b * p->table_width];\n    int64_t slot = t % p->bs;\n    const int64_t vrow"),
    "unnormalised_weights": ("double w = s[t - lo] / Z;", "double w = s[t - lo];"),
    "lse_without_max": ("*lse = M + log(Z);", "*lse = log(Z);"),
    "lse_log2": ("*lse = M + log(Z);", "*lse = M + log2(Z);"),
    "last_token_dropped": ("for (int64_t t = lo; t < L; ++t) {\n    int64_t phys = p->tables[b * p->table_width + t / p->bs];\n    int64_t slot = t % p->bs;\n    const int64_t vrow",
                           "for (int64_t t = lo; t < L - 1; ++t) {\n    int64_t phys = p->tables[b * p->table_width + t / p->bs];\n    int64_t slot = t % p->bs;\n    const int64_t vrow"),
    "max_over_first_half": ("for (int64_t t = 1; t < n; ++t)\n    if (s[t] > M) M = s[t];",
                            "for (int64_t t = 1; t < n / 2; ++t)\n    if (s[t] > M) M = s[t];"),
    "window_off_by_one": ("L > p->window) ? L - p->window : 0;", "L > p->window) ? L - p->window + 1 : 0;"),
    "window_ignored": ("const int64_t lo = (p->window > 0 && L > p->window) ? L - p->window : 0;",
                       "const int64_t lo = 0;"),
    "sink_ignored": ("if (has_sink) Z += exp(sink - M);", ""),
    "sink_scaled": ("const double sink = has_sink ? (double)p->sinks[h] : 0.0;",
                    "const double sink = has_sink ? (double)p->sinks[h] * p->scale : 0.0;"),
    "empty_sequence_drops_sink": ("*lse = has_sink ? sink : -INFINITY;", "*lse = -INFINITY;"),
    "query_of_kv_head": ("h * p->q_str[1];", "kh * p->q_str[1];"),
    "exp_without_shift": ("s[t] = exp(s[t] - M);", "s[t] = exp(s[t]);"),
    "e4m3_subnormal_as_normal": ("mag = ldexp((double)m / 8.0, -6);", "mag = ldexp(1.0 + (double)m / 8.0, -7);"),
    "e4m3_bias_8": ("mag = ldexp(1.0 + (double)m / 8.0, e - 7);", "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_nan_as_number": ("if (e == 15 && m == 7) return NAN;", ""),
    "e4m3_sign_dropped": ("return sign ? -mag : mag;", "return mag;"),
    "k_scale_dropped": ("krow + d * p->kv_str[3], p->k_scale)", "krow + d * p->kv_str[3], 1.0)"),
    "v_scale_on_keys": ("krow + d * p->kv_str[3], p->k_scale)", "krow + d * p->kv_str[3], p->v_scale)"),
    "v_scale_dropped": ("vrow + d * p->kv_str[3], p->v_scale)", "vrow + d * p->kv_str[3], 1.0)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new, 1))
    lib = oracle.build(force=True, src=str(mutant_src), out=str(tmp_path / "libmutant.so"))
    caught = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(lib)
            except AssertionError:
                caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
