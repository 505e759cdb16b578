"""The C ABI without a GPU: the library loads, exports every function that
include/pad.h declares, plans shapes, and rejects bad arguments before touching
the device (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_attention_partition_b200 as pad
from paged_kv_attention_partition_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return pad.load_library()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(pad_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"pad_decode", "pad_decode_plan", "pad_status_string", "pad_last_error",
            "pad_check_device_errors", "pad_release_workspace", "pad_abi_version"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", pad.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in names:
        getattr(lib, n)


# The source pages, by title; a declaration's comment names one of them with a
# section (or a review finding), or says the pages have no counterpart.
PAGE_TITLES = (
    "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm",
    "feat(rocm): wvSplitK skinny GEMM for decode M<=4",
    "perf(BACKEND-ROCM): cooperate across Q8_K activation blocks",
    "Attention parity: run every attention type on the best available path on both targets",
    "perf(rocke): prepare saved paged decode bindings once",
)


def test_every_declaration_cites_a_passage_or_says_it_has_none():
    src = open(os.path.join(ROOT, "include", "pad.h")).read()
    for name in declared_functions():
        decl = re.search(r"^[A-Za-z_][\w \*]*?\b" + name + r"\s*\(", src, flags=re.M)
        assert decl, name
        # the last block comment starting in column 0 before the declaration
        blocks = [m for m in re.finditer(r"^/\*.*?\*/", src[:decl.start()], flags=re.M | re.S)]
        assert blocks, f"{name}: no comment"
        text = " ".join(re.sub(r"\n\s*\*(?!/)", " ", blocks[-1].group(0)).split())
        cites = any(t in text for t in PAGE_TITLES) and ("section" in text or "review" in text)
        assert cites or "no counterpart" in text, f"{name}: its comment names no page section: {text[:120]}"


def test_resident_ctas_per_sm_in_the_plan(lib):
    # each instantiation's launch bound, and the 8-head tiles' six-per-SM
    # build from four full waves at five per SM (4 * 5 * 148 = 2960 units; the
    # plan counts 148 SMs without a device)
    plan = lambda B, Hq, kv, splits=16: pad.pad_decode_plan(B, Hq, 8, 128, 16, 16, num_splits=splits, kv_dtype=kv)
    for kv in ("e4m3", "bf16"):
        assert plan(23, 40, kv)["ctas"] == 2944 and plan(23, 40, kv)["ctas_per_sm"] == 5
        assert plan(24, 40, kv)["ctas"] == 3072 and plan(24, 40, kv)["ctas_per_sm"] == 6
    assert plan(64, 128, "bf16")["ctas_per_sm"] == 3 and plan(64, 128, "e4m3")["ctas_per_sm"] == 4  # 16-head tiles
    assert plan(4, 256, "bf16")["ctas_per_sm"] == 4 and plan(4, 256, "e4m3")["ctas_per_sm"] == 4  # 32-head tiles
    assert pad.pad_decode_plan(16, 16, 4, 256, 16, 2048, num_splits=32)["ctas_per_sm"] == 3  # D = 256


def test_unit_order_only_for_heavy_units(lib):
    # heavy units (partition tokens x heads per tile >= 32 K) carry the launch's
    # unit order after the partials: 4 bytes per CTA
    r = lambda x: -(-x // 256) * 256
    p = pad.pad_decode_plan(256, 32, 1, 128, 32, 1024, num_splits=0)  # the ragged MQA batch's shape
    S = p["num_splits"]
    assert p["partition_tokens"] * p["heads_per_tile"] >= 32768
    assert p["workspace_bytes"] == r(256 * 32 * S * 128 * 4) + r(256 * 32 * S * 4) + r(p["ctas"] * 4)
    for shape in ((32, 32, 8, 128, 16, 256), (64, 40, 8, 128, 16, 512)):  # llama8b- and qwen14b-shaped
        p = pad.pad_decode_plan(*shape, num_splits=0)
        B, Hq, _, D = shape[:4]
        S = p["num_splits"]
        assert p["partition_tokens"] * p["heads_per_tile"] < 32768
        assert p["workspace_bytes"] == r(B * Hq * S * D * 4) + r(B * Hq * S * 4)


def test_unit_order_needs_the_pairs_to_fit_one_cta(lib):
    # B * S <= 65536 (sequence, partition) pairs: the one-CTA pass handles them;
    # one more pair and the launch keeps its default order
    r = lambda x: -(-x // 256) * 256
    for B, ordered in ((4096, True), (4097, False)):
        p = pad.pad_decode_plan(B, 32, 1, 128, 16, 2048, num_splits=16)  # P = 2048 tokens x 32 heads
        assert p["num_splits"] == 16 and B * 16 <= 65536 or not ordered
        partials = r(B * 32 * 16 * 128 * 4) + r(B * 32 * 16 * 4)
        assert p["workspace_bytes"] == partials + (r(p["ctas"] * 4) if ordered else 0), (B, ordered)


def test_stage_timeout_hook_checks_its_argument(lib):
    assert lib.pad_inject_stage_timeout(-2) == pad.PAD_ERR_INVALID_ARG
    assert lib.pad_inject_stage_timeout(256) == pad.PAD_ERR_INVALID_ARG
    assert lib.pad_inject_stage_timeout(3) == pad.PAD_OK
    assert lib.pad_inject_stage_timeout(-1) == pad.PAD_OK  # disarmed


def test_library_is_built_for_sm100a():
    cmd = _build.compile_command("x.so")
    assert "arch=compute_100a,code=sm_100a" in " ".join(cmd)


def test_status_strings(lib):
    assert pad.pad_status_string(0) == "PAD_OK"
    assert pad.pad_status_string(5) == "PAD_ERR_DEVICE_CHECK"
    assert pad.pad_abi_version() == 3


def test_plan_follows_the_partition_rule(lib):
    # explicit splits: P = round_up(ceil(C / S), bs), S_eff = ceil(C / P)
    p = pad.pad_decode_plan(64, 40, 8, 128, 16, 512, num_splits=16, device=0)
    assert (p["num_splits"], p["partition_tokens"], p["reduce"]) == (16, 512, 1)
    # one CTA per (sequence, KV head, head tile, partition)
    assert p["ctas"] == 64 * 8 * 16 and p["head_tiles"] == 1 and p["heads_per_tile"] == 8
    # bf16 8-head tile at D = 128: head_dim split over warp pairs, 32-token stages, five per SM
    # (8192 units: the six-per-SM build)
    assert p["warps_per_cta"] == 4 and p["stage_tokens"] == 32 and p["stages"] == 2 and p["ctas_per_sm"] == 6
    assert p["workspace_bytes"] >= 64 * 40 * 16 * (128 + 1) * 4 and p["control_bytes"] >= 64 * 8 * 4
    p = pad.pad_decode_plan(16, 16, 4, 256, 16, 2048, num_splits=32, device=0)
    assert (p["num_splits"], p["partition_tokens"]) == (32, 1024)
    p = pad.pad_decode_plan(1, 4, 1, 128, 16, 16, num_splits=1, device=0)
    # one unit: one CTA; no partials, no merge counters
    assert (p["num_splits"], p["reduce"], p["workspace_bytes"], p["ctas"], p["control_bytes"]) == (1, 0, 0, 1, 0)
    # at most 256 partitions per sequence
    p = pad.pad_decode_plan(2, 4, 1, 128, 1, 4096, num_splits=4096, device=0)
    assert (p["num_splits"], p["partition_tokens"]) == (256, 16)
    p = pad.pad_decode_plan(2, 4, 1, 128, 16, 4, num_splits=7, device=0)  # C=64, P=16
    assert (p["num_splits"], p["partition_tokens"]) == (4, 16)
    p = pad.pad_decode_plan(2, 4, 1, 128, 1, 100, num_splits=3, device=0)  # bs=1: P=34, S=3
    assert (p["num_splits"], p["partition_tokens"]) == (3, 34)


def test_heuristic_plans(lib):
    for shape in [(32, 32, 8, 128, 16, 256), (256, 32, 1, 128, 32, 1024), (64, 40, 8, 128, 16, 512),
                  (16, 16, 4, 256, 16, 2048), (1, 4, 1, 128, 16, 16), (3, 64, 1, 128, 16, 4)]:
        p = pad.pad_decode_plan(*shape, num_splits=0, device=0)
        B, Hq, Hkv, D, bs, W = shape
        g = Hq // Hkv
        C = W * bs
        assert p["partition_tokens"] % bs == 0 and p["partition_tokens"] <= max(C, bs)
        assert p["num_splits"] == -(-C // p["partition_tokens"])
        assert p["heads_per_tile"] * p["head_tiles"] >= g and p["heads_per_tile"] <= 32
        # partitions of at least 64 tokens, and the partial each writes (g*D*4
        # bytes) at most 1/16 of the K/V bytes it streams (4*D*P)
        if p["num_splits"] > 1:
            assert p["partition_tokens"] >= 64 and g / p["partition_tokens"] <= 1 / 16 + 1e-9
    # a large batch gets max(512, 64 g) tokens per partition (a power of two); a
    # small batch is cut finer (down to 64 tokens) until the launch has three
    # units per SM (444 on 148 SMs)
    assert pad.pad_decode_plan(32, 32, 8, 128, 16, 256, num_splits=0, device=0)["partition_tokens"] == 512
    assert pad.pad_decode_plan(256, 32, 1, 128, 32, 1024, num_splits=0, device=0)["partition_tokens"] == 2048
    assert pad.pad_decode_plan(1, 32, 8, 128, 16, 256, num_splits=0, device=0)["partition_tokens"] == 64
    assert pad.pad_decode_plan(4, 32, 8, 128, 16, 256, num_splits=0, device=0)["partition_tokens"] == 256
    assert pad.pad_decode_plan(8, 32, 8, 128, 16, 256, num_splits=0, device=0)["partition_tokens"] == 512
    assert pad.pad_decode_plan(2, 40, 8, 128, 16, 512, num_splits=0, device=0)["partition_tokens"] == 256
    # group 20: one 32-head tile at D=128, two 16-head tiles at D=256; group 64: two tiles
    p = pad.pad_decode_plan(2, 20, 1, 128, 16, 10, num_splits=1, device=0)
    assert (p["heads_per_tile"], p["head_tiles"]) == (32, 1)
    p = pad.pad_decode_plan(2, 20, 1, 256, 16, 10, num_splits=1, device=0)
    assert (p["heads_per_tile"], p["head_tiles"]) == (16, 2)
    p = pad.pad_decode_plan(2, 64, 1, 128, 16, 10, num_splits=1, device=0)
    assert (p["heads_per_tile"], p["head_tiles"]) == (32, 2)


def _fake(dtype, shape, strides=None, addr=0x100000):
    t = pad.PadTensor()
    t.data = addr
    t.dtype = dtype
    t.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        t.shape[i] = s
        t.stride[i] = st
    return t


def _call(lib, q, k, v, t, l, out, lse=None, scale=0.1, splits=0):
    r = lambda x: ctypes.byref(x) if x is not None else None
    return lib.pad_decode(r(q), r(k), r(v), r(t), r(l), scale, splits, r(out), r(lse), None)


GOOD = dict(
    q=(pad.PAD_BF16, (2, 8, 128)), k=(pad.PAD_BF16, (10, 2, 16, 128)), v=(pad.PAD_BF16, (10, 2, 16, 128)),
    t=(pad.PAD_I32, (2, 5)), l=(pad.PAD_I32, (2,)), out=(pad.PAD_BF16, (2, 8, 128)), lse=(pad.PAD_F32, (2, 8)))


def _args(**override):
    spec = {**GOOD, **override}
    return {k: (_fake(*v) if v is not None else None) for k, v in spec.items()}


@pytest.mark.parametrize("override,status", [
    (dict(q=(pad.PAD_F32, (2, 8, 128))), pad.PAD_ERR_INVALID_ARG),          # wrong dtype
    (dict(v=(pad.PAD_BF16, (10, 1, 16, 128))), pad.PAD_ERR_INVALID_ARG),    # K/V shapes differ
    (dict(q=(pad.PAD_BF16, (2, 7, 128)), out=(pad.PAD_BF16, (2, 7, 128)), lse=(pad.PAD_F32, (2, 7))),
     pad.PAD_ERR_INVALID_ARG),                                               # Hq % Hkv != 0
    (dict(lse=(pad.PAD_F32, (2, 9))), pad.PAD_ERR_INVALID_ARG),             # lse shape mismatch
    (dict(out=(pad.PAD_BF16, (2, 8, 64))), pad.PAD_ERR_INVALID_ARG),        # out shape mismatch
    (dict(t=(pad.PAD_I32, (3, 5))), pad.PAD_ERR_INVALID_ARG),               # table rows != B
    (dict(l=(pad.PAD_I32, (3,))), pad.PAD_ERR_INVALID_ARG),                 # seq_lens != B
    (dict(q=(pad.PAD_BF16, (2, 8, 96)), k=(pad.PAD_BF16, (10, 2, 16, 96)), v=(pad.PAD_BF16, (10, 2, 16, 96)),
          out=(pad.PAD_BF16, (2, 8, 96))), pad.PAD_ERR_UNSUPPORTED),        # head_dim 96
    (dict(k=(pad.PAD_BF16, (10, 2, 12, 128)), v=(pad.PAD_BF16, (10, 2, 12, 128))), pad.PAD_ERR_UNSUPPORTED),  # bs 12
])
def test_validation_rejects_before_any_launch(lib, override, status):
    a = _args(**override)
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == status
    assert pad.pad_last_error()


def test_validation_scalars_and_alignment(lib):
    a = _args()
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"], scale=float("nan")) == pad.PAD_ERR_INVALID_ARG
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"], splits=-1) == pad.PAD_ERR_INVALID_ARG
    a = _args()
    a["k"].data = 0x100008  # not 16-byte aligned
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == pad.PAD_ERR_INVALID_ARG
    a = _args()
    a["k"].stride[2] = 132  # row stride of 264 bytes: not a multiple of 16
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == pad.PAD_ERR_INVALID_ARG
    a = _args()
    a["q"].stride[2] = 2  # head dim not contiguous
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == pad.PAD_ERR_INVALID_ARG
    assert _call(lib, None, a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == pad.PAD_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(lib):
    a = _args(q=(pad.PAD_BF16, (0, 8, 128)), t=(pad.PAD_I32, (0, 5)), l=(pad.PAD_I32, (0,)),
              out=(pad.PAD_BF16, (0, 8, 128)), lse=(pad.PAD_F32, (0, 8)))
    assert _call(lib, a["q"], a["k"], a["v"], a["t"], a["l"], a["out"], a["lse"]) == pad.PAD_OK


def test_binding_has_no_cpu_path():
    import torch
    import paged_kv_attention_partition_b200 as p
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        p.pad_decode(q, q, q, q, q, 0.1)


def test_e4m3_plan_keeps_partitions_and_scratch(lib):
    # an E4M3 cache streams the same tokens in half the bytes: the same
    # partitions and scratch; at D = 128 (8/16-head tiles) two 64-token stages
    # of half the bytes, at D = 256 two stages of twice the tokens, at D = 64
    # three stages, for 32-head tiles three
    for shape, stage_tokens, stages in (((32, 32, 8, 128, 16, 256), 64, 2), ((256, 32, 1, 128, 32, 1024), 64, 3),
                                        ((16, 16, 4, 256, 16, 2048), 64, 2), ((4, 16, 2, 64, 4, 100), 64, 3),
                                        ((2, 32, 2, 128, 16, 64), 64, 2)):
        b = pad.pad_decode_plan(*shape, num_splits=0, device=0)
        f = pad.pad_decode_plan(*shape, num_splits=0, device=0, kv_dtype="e4m3")
        for k in ("num_splits", "partition_tokens", "heads_per_tile", "head_tiles", "ctas", "workspace_bytes",
                  "control_bytes"):
            assert b[k] == f[k], k
        assert (f["stage_tokens"], f["stages"]) == (stage_tokens, stages), shape
    with pytest.raises(pad.PadError) as e:
        pad.pad_decode_plan(4, 16, 2, 128, 16, 100, kv_dtype="fp4")
    assert e.value.status == pad.PAD_ERR_INVALID_ARG


@pytest.mark.parametrize("value, lines, warned", [("1", 2, False), (None, 0, False), ("", 0, False), ("0", 0, False),
                                                  ("yes", 0, True)])
def test_pad_log_prints_each_plan_once(value, lines, warned):
    # PAD_LOG=1: the plan chosen for each distinct shape, once; other values
    # warn once and stay silent; unset, empty or 0 print nothing
    import sys
    env = {k: v for k, v in os.environ.items() if k != "PAD_LOG"}
    if value is not None:
        env["PAD_LOG"] = value
    code = ("import paged_kv_attention_partition_b200 as pad\n"
            "for _ in range(3): pad.pad_decode_plan(32, 32, 8, 128, 16, 256)\n"
            "pad.pad_decode_plan(64, 40, 8, 128, 16, 512, num_splits=16, kv_dtype='e4m3')\n")
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT, timeout=120)
    assert res.returncode == 0, res.stderr
    plans = [l for l in res.stderr.splitlines() if l.startswith("pad: plan ")]
    assert len(plans) == lines, res.stderr
    if lines:
        assert "B=32 Hq=32 Hkv=8 D=128 bs=16 capacity=4096 kv=bf16 num_splits=0" in plans[0]
        assert "kv=e4m3 num_splits=16" in plans[1] and " S=16 P=512 " in plans[1]
    assert ("ignored" in res.stderr) == warned
