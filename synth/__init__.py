"""Seeded synthetic workloads for paged single-token decode attention.

This module draws inputs only -- no attention arithmetic lives here -- and is the
one thing the GPU path and the CPU oracle share: both consume the bytes it makes.

A workload is one decode step: a query token per sequence (``q``), a paged KV
cache (``k_cache``/``v_cache`` in logical [num_blocks, Hkv, block_size, D]
order), a block table and the sequence lengths, plus the softmax scale and the
requested number of KV splits.

Synthetic stand-ins for the pages' workloads (real-model decode on Qwen3/Llama
geometries: "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm", section "The
gap it specs"; B/KV/Hq/Hkv/D/page-16 one-token split-KV decode: "perf(rocke):
prepare saved paged decode bindings once", section "Runnable saved-binding
HIP-event comparison"). No dataset or checkpoint is involved.

Poisoning: every table entry past ceil(L_b / block_size) points at an extra
physical block filled with NaN (bf16 NaN, or the E4M3 NaN code), and (unless a
block is shared by several sequences) the cache slots past L_b inside a
sequence's last block are NaN too.  A kernel that reads either place produces
NaN and fails parity instead of reading out of bounds.

An 8-bit cache (``kv_dtype="e4m3"``) holds OCP FP8 E4M3 codes with one scale per
tensor: the codes are the seeded samples divided by ``k_scale`` / ``v_scale``
and rounded onto the E4M3 grid, so ``scale * code`` approximates the sample.
"""
from __future__ import annotations

import ctypes
import dataclasses
import functools
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

DIST_NORMAL = 0
DIST_UNIFORM_PM1 = 1
BF16_NAN = 0x7FC0
E4M3_NAN = 0x7F
# default per-tensor scales of an E4M3 cache: not powers of two, exact in fp32
E4M3_K_SCALE = 3.0 / 64.0
E4M3_V_SCALE = 5.0 / 256.0

# stream ids: one independent counter space per drawn quantity
S_Q, S_K, S_V, S_LENS, S_PERM, S_EXTRA = 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    """Compile libsynth.so with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _l():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, u64, i32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int32
        p = ctypes.c_void_p
        lib.synth_fill_bf16.argtypes = [p, i64, i64, u64, u64, ctypes.c_int, ctypes.c_int]
        lib.synth_fill_blocks_bf16.argtypes = [p, p, i64, i64, u64, u64, ctypes.c_int, ctypes.c_int]
        lib.synth_fill_blocks_e4m3.argtypes = [p, p, i64, i64, u64, u64, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_int]
        lib.synth_uniform_f64.argtypes = [p, i64, u64, u64]
        lib.synth_permutation_prefix.argtypes = [p, p, i64, i64, u64, u64]
        lib.synth_uniform_int.argtypes = [p, i64, i32, i32, u64, u64]
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def bf16_array(shape, seed: int, stream: int, dist: int = DIST_NORMAL) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    _l().synth_fill_bf16(out.ctypes.data, out.size, 0, seed, stream, dist, _threads())
    return out


def uniform(n: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _l().synth_uniform_f64(out.ctypes.data, n, seed, stream)
    return out


def uniform_int(n: int, lo: int, hi: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _l().synth_uniform_int(out.ctypes.data, n, lo, hi, seed, stream)
    return out


def permutation_prefix(n: int, k: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(k, dtype=np.int32)
    scratch = np.empty(n, dtype=np.int32)
    _l().synth_permutation_prefix(out.ctypes.data, scratch.ctypes.data, n, k, seed, stream)
    return out


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits (uint16) to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float32 values to raw bf16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + 0x7FFF + ((b >> 16) & 1)
    return (b >> 16).astype(np.uint16)


@dataclasses.dataclass
class Workload:
    """One decode step's inputs (host arrays: raw bf16 bits as uint16; an E4M3
    cache as uint8 codes)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    q: np.ndarray             # uint16 [B, Hq, D]
    k_cache: np.ndarray       # uint16 bf16 / uint8 E4M3 [num_blocks, Hkv, block_size, D] (logical order)
    v_cache: np.ndarray       # same dtype and shape
    block_tables: np.ndarray  # int32 [B, max_blocks_per_seq]
    seq_lens: np.ndarray      # int32 [B]
    scale: float
    num_splits: int           # 0 = let the library choose
    want_lse: bool
    seed: int
    recipe: str = ""
    kv_dtype: str = "bf16"    # "bf16" or "e4m3"
    k_scale: float = 1.0      # dequantisation scales of an E4M3 cache (1 for bf16)
    v_scale: float = 1.0

    @property
    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype == "e4m3" else 2

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    def kv_tokens(self, window: int = 0) -> int:
        L = self.seq_lens.astype(np.int64)
        return int((np.minimum(L, window) if window > 0 else L).sum())

    def algorithmic_bytes(self, window: int = 0, sinks: bool = False) -> int:
        """Minimum bytes one call must move (K+V pages read once, q read, out
        written, live table entries, seq_lens, lse when requested).  With a
        sliding window only the window's tokens and the table entries of the
        pages they touch count; sinks add one fp32 logit per query head."""
        L = self.seq_lens.astype(np.int64)
        lo = np.maximum(L - window, 0) if window > 0 else np.zeros_like(L)
        kv = int((2 * self.kv_elem_bytes * (L - lo) * self.Hkv * self.D).sum())
        qo = 4 * self.B * self.Hq * self.D
        bs = self.block_size
        pages = np.where(L > lo, (L + bs - 1) // bs - lo // bs, 0)
        table = int(4 * pages.sum())
        lse = 4 * self.B * self.Hq if self.want_lse else 0
        return kv + qo + table + 4 * self.B + lse + (4 * self.Hq if sinks else 0)


def make_workload(
    name: str,
    B: int,
    Hq: int,
    Hkv: int,
    D: int,
    block_size: int,
    seq_lens,
    *,
    seed: int,
    pool_blocks: Optional[int] = None,
    max_blocks_per_seq: Optional[int] = None,
    table_mode: str = "unique",
    k_dist: int = DIST_NORMAL,
    v_dist: int = DIST_NORMAL,
    scale: Optional[float] = None,
    num_splits: int = 0,
    want_lse: bool = True,
    poison: bool = True,
    recipe: str = "",
    kv_dtype: str = "bf16",
    k_scale: Optional[float] = None,
    v_scale: Optional[float] = None,
) -> Workload:
    """Build a workload.

    table_mode:
      "unique": block ids drawn without replacement from the pool (a prefix of a
                seeded permutation), each sequence taking the next ceil(L/bs).
      "cyclic": one seeded permutation of the pool; sequences take consecutive
                entries, wrapping around when the pool runs out (blocks may then
                be shared by several sequences, as with prefix sharing).
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int32).reshape(B)
    bs = block_size
    need = (seq_lens.astype(np.int64) + bs - 1) // bs
    demand = int(need.sum())
    width = int(max_blocks_per_seq if max_blocks_per_seq is not None else max(1, int(need.max(initial=1))))
    if int(need.max(initial=0)) > width:
        raise ValueError("max_blocks_per_seq smaller than a sequence's block count")
    pool = int(pool_blocks if pool_blocks is not None else max(demand, 1))
    if table_mode == "unique":
        if demand > pool:
            raise ValueError(f"pool of {pool} blocks cannot hold {demand} distinct blocks")
        ids = permutation_prefix(pool, demand, seed, S_PERM)
    elif table_mode == "cyclic":
        perm = permutation_prefix(pool, pool, seed, S_PERM)
        ids = perm[np.arange(demand) % pool] if demand else perm[:0]
    else:
        raise ValueError(table_mode)

    poison_block = pool  # one extra physical block, never legitimately referenced
    num_blocks = pool + 1
    tables = np.full((B, width), poison_block, dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(need[b])
        tables[b, :n] = ids[off:off + n]
        off += n

    if kv_dtype not in ("bf16", "e4m3"):
        raise ValueError(kv_dtype)
    fp8 = kv_dtype == "e4m3"
    ks = float(np.float32(k_scale if k_scale is not None else (E4M3_K_SCALE if fp8 else 1.0)))
    vs = float(np.float32(v_scale if v_scale is not None else (E4M3_V_SCALE if fp8 else 1.0)))
    shape = (num_blocks, Hkv, bs, D)
    k = np.zeros(shape, dtype=np.uint8 if fp8 else np.uint16)
    v = np.zeros_like(k)
    used = np.unique(ids.astype(np.int64)) if demand else np.zeros(0, np.int64)
    block_elems = Hkv * bs * D
    lib = _l()
    if used.size:
        used = np.ascontiguousarray(used)
        for arr, stream, dist, sc in ((k, S_K, k_dist, ks), (v, S_V, v_dist, vs)):
            if fp8:
                lib.synth_fill_blocks_e4m3(arr.ctypes.data, used.ctypes.data, used.size, block_elems, seed, stream,
                                           dist, 1.0 / sc, _threads())
            else:
                lib.synth_fill_blocks_bf16(arr.ctypes.data, used.ctypes.data, used.size, block_elems, seed, stream,
                                           dist, _threads())
    nan = E4M3_NAN if fp8 else BF16_NAN
    if poison:
        k[poison_block] = nan
        v[poison_block] = nan
        counts = np.bincount(ids.astype(np.int64), minlength=num_blocks) if demand else None
        for b in range(B):
            L = int(seq_lens[b])
            if L % bs and counts is not None:
                last = int(tables[b, L // bs])
                if counts[last] == 1:
                    k[last, :, L % bs:, :] = nan
                    v[last, :, L % bs:, :] = nan
    q = bf16_array((B, Hq, D), seed, S_Q)
    return Workload(
        name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, q=q, k_cache=k, v_cache=v,
        block_tables=tables, seq_lens=seq_lens,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(D)),
        num_splits=num_splits, want_lse=want_lse, seed=seed, recipe=recipe,
        kv_dtype=kv_dtype, k_scale=ks, v_scale=vs,
    )


# ---------------------------------------------------------------------------
# The five named decode workloads.
# ---------------------------------------------------------------------------

CONFIG_NAMES = ("tiny", "llama8b", "qwen14b", "longctx_d256", "ragged_mqa")


def config(name: str, seed: Optional[int] = None, batch: Optional[int] = None,
           compact_pool: bool = False, kv_dtype: str = "bf16") -> Workload:
    """The named decode workloads (seeds 0..4 by default).

    `batch` keeps every other parameter and takes the first `batch` sequences
    (lengths come from a counter-based stream, so they are a prefix of the full
    batch's).  `compact_pool` makes the block pool exactly the blocks the batch
    uses, drawn without replacement: no page is shared between sequences and the
    device holds only what is read.  Both serve reduced profiling cases; the
    llama8b workload with `compact_pool` is also its no-alias variant.
    `kv_dtype="e4m3"` stores the same samples as E4M3 codes with the default
    per-tensor scales (the 8-bit-cache variant of each workload)."""
    w = _config(name, seed, batch, compact_pool, kv_dtype)
    if kv_dtype == "e4m3":
        w.recipe += f"; E4M3 cache, codes = RNE(sample / scale), k_scale {w.k_scale:g}, v_scale {w.v_scale:g}"
    return w


def _config(name, seed, batch, compact_pool, kv_dtype):
    make_workload = functools.partial(_make_workload, kv_dtype=kv_dtype)
    idx = CONFIG_NAMES.index(name)
    seed = idx if seed is None else seed

    def pool(default):
        return None if compact_pool else default

    def nb(default):
        return default if batch is None else int(batch)

    if name == "tiny":
        return make_workload(
            name, nb(1), 4, 1, 128, 16, [256] * nb(1), seed=seed, pool_blocks=pool(16 * nb(1)), max_blocks_per_seq=16,
            num_splits=1, recipe="B1 Hq4/Hkv1 D128 L256 bs16, N(0,1), table = permutation of 16 blocks, S=1")
    if name == "llama8b":
        B = nb(32)
        lens = uniform_int(B, 512, 4096, seed, S_LENS)
        return make_workload(
            name, B, 32, 8, 128, 16, lens, seed=seed, pool_blocks=pool(4096), max_blocks_per_seq=256,
            table_mode="unique" if compact_pool else "cyclic", num_splits=0,
            recipe=("B32 Hq32/Hkv8 D128 bs16, L~U{512..4096}, N(0,1), "
                    + ("blocks without replacement (no aliasing)" if compact_pool
                       else "cyclic over one permutation of a 4096-block pool")))
    if name == "qwen14b":
        B = nb(64)
        return make_workload(
            name, B, 40, 8, 128, 16, [8192] * B, seed=seed, pool_blocks=pool(32768), max_blocks_per_seq=512,
            num_splits=16, want_lse=True,
            recipe="B64 Hq40/Hkv8 D128 L8192 bs16, N(0,1), permutation of a 32768-block pool, 512-token partitions, LSE on")
    if name == "longctx_d256":
        B = nb(16)
        return make_workload(
            name, B, 16, 4, 256, 16, [32768] * B, seed=seed, pool_blocks=pool(32768), max_blocks_per_seq=2048,
            v_dist=DIST_UNIFORM_PM1, num_splits=32,
            recipe="B16 Hq16/Hkv4 D256 L32768 bs16, K~N(0,1), V~U(-1,1), permutation of a 32768-block pool, 1024-token partitions")
    if name == "ragged_mqa":
        B = nb(256)
        u = uniform(B, seed, S_LENS)
        lens = np.clip(np.floor(np.exp(math.log(16) + u * (math.log(32768) - math.log(16)))), 16, 32768).astype(np.int32)
        return make_workload(
            name, B, 32, 1, 128, 32, lens, seed=seed, pool_blocks=pool(300_000), max_blocks_per_seq=1024,
            num_splits=0,
            recipe="B256 Hq32/Hkv1 D128 bs32, L log-uniform [16,32768], N(0,1), without replacement from a 300000-block pool")
    raise KeyError(name)


_make_workload = make_workload
