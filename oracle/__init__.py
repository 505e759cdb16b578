"""CPU double-precision oracle for paged single-token decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``paged_kv_attention_partition_b200``) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, double precision, pthreads); this
module only compiles it with gcc and marshals numpy arrays.  See the header of
``oracle.c`` for the definition it writes out and the passages it follows
("spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm", section "The gap it
specs"; "perf(rocke): prepare saved paged decode bindings once", sections
"Summary" and "Testing Summary").

Every function here is pinned by ``tests/test_oracle_pins.py`` against facts
that do not come from the oracle itself: brute-force unpaged attention through
a library softmax, block-table permutation invariance, softmax invariants and
closed forms.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (idempotent).  ``src``/``out`` let a test
    compile a deliberately broken copy elsewhere."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, out)
    return out


_libs: dict = {}


def _load(path: str = _LIB):
    if path not in _libs:
        if path == _LIB:
            build()
        lib = ctypes.CDLL(path)
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        dbl = ctypes.c_double
        lib.oracle_decode.argtypes = [p, p, p, p, p, p, i64, p, i64, i64, i64, i64, i64,
                                      dbl, i64, p, i64, dbl, dbl, p, p, i32]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode_pairs.argtypes = [p, p, p, p, p, p, i64, p, i64, i64, i64, i64, i64,
                                            dbl, i64, p, i64, dbl, dbl, p, i64, p, p, i32]
        lib.oracle_decode_pairs.restype = ctypes.c_int
        _libs[path] = lib
    return _libs[path]


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _estrides(a: np.ndarray) -> np.ndarray:
    return np.asarray([s // a.itemsize for s in a.strides], dtype=np.int64)


def _check(q, k, v, tables, lens):
    """Returns 1 for an E4M3 cache (uint8 codes), 0 for bf16 (uint16 bits)."""
    assert q.dtype == np.uint16 and k.dtype == v.dtype and k.dtype in (np.uint16, np.uint8)
    assert q.ndim == 3 and k.ndim == 4 and v.shape == k.shape
    assert _estrides(k).tolist() == _estrides(v).tolist(), "K and V must share strides"
    assert tables.dtype == np.int32 and tables.ndim == 2 and tables.flags.c_contiguous
    assert lens.dtype == np.int32 and lens.ndim == 1 and lens.flags.c_contiguous
    return 1 if k.dtype == np.uint8 else 0


def _sinks_arg(sinks, Hq):
    if sinks is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(sinks, dtype=np.float32).reshape(Hq))
    return arr, arr.ctypes.data


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale, nthreads=None, lib_path=_LIB, window=0, sinks=None,
           k_scale=1.0, v_scale=1.0):
    """Full oracle: returns (out [B, Hq, D] float64, lse [B, Hq] float64).

    q: uint16 bf16 bits [B, Hq, D]; k_cache/v_cache: uint16 bf16 bits, or uint8
    E4M3 codes dequantised as k_scale * code / v_scale * code, [num_blocks, Hkv,
    bs, D] (any strides, e.g. a transposed view of an NHD cache); block_tables
    int32 [B, W]; seq_lens int32 [B].  window: 0 = every token, W > 0 = each
    sequence's last W tokens; sinks: None, or fp32 [Hq] sink logits."""
    fp8 = _check(q, k_cache, v_cache, block_tables, seq_lens)
    B, Hq, D = q.shape
    _, Hkv, bs, Dk = k_cache.shape
    assert Dk == D and Hq % Hkv == 0 and seq_lens.shape[0] == B
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    qs, ks = _estrides(q), _estrides(k_cache)
    keep, sp = _sinks_arg(sinks, Hq)
    rc = _load(lib_path).oracle_decode(
        q.ctypes.data, qs.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data, ks.ctypes.data,
        block_tables.ctypes.data, block_tables.shape[1], seq_lens.ctypes.data, B, Hq, Hkv, D, bs,
        float(scale), int(window), sp, fp8, float(k_scale), float(v_scale), out.ctypes.data, lse.ctypes.data,
        nthreads or default_threads())
    if rc:
        raise RuntimeError(f"oracle_decode failed ({rc})")
    return out, lse


def decode_pairs(q, k_cache, v_cache, block_tables, seq_lens, scale, pairs, nthreads=None, lib_path=_LIB, window=0,
                 sinks=None, k_scale=1.0, v_scale=1.0):
    """Oracle for selected (b, h) pairs: returns (out [n, D], lse [n])."""
    fp8 = _check(q, k_cache, v_cache, block_tables, seq_lens)
    B, Hq, D = q.shape
    _, Hkv, bs, _ = k_cache.shape
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    n = pairs.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    qs, ks = _estrides(q), _estrides(k_cache)
    keep, sp = _sinks_arg(sinks, Hq)
    rc = _load(lib_path).oracle_decode_pairs(
        q.ctypes.data, qs.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data, ks.ctypes.data,
        block_tables.ctypes.data, block_tables.shape[1], seq_lens.ctypes.data, B, Hq, Hkv, D, bs,
        float(scale), int(window), sp, fp8, float(k_scale), float(v_scale), pairs.ctypes.data, n,
        out.ctypes.data, lse.ctypes.data, nthreads or default_threads())
    if rc:
        raise RuntimeError(f"oracle_decode_pairs failed ({rc})")
    return out, lse


def decode_workload(w, nthreads=None, window=0, sinks=None):
    """Oracle over a ``synth.Workload`` (bf16 or E4M3 cache, with its scales)."""
    return decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, nthreads, window=window,
                  sinks=sinks, k_scale=w.k_scale, v_scale=w.v_scale)
