"""Paged-KV single-token decode attention for B200 (sm_100a).

A thin Python binding over the C ABI in ``include/pad.h`` (``libpad.so``): it
turns torch tensors into ``pad_tensor`` descriptors and calls the library.  All
arithmetic runs in the library's CUDA kernels; there is no Python or CPU
fallback, and the import fails loudly if ``libpad.so`` has not been built
(``python -m paged_kv_attention_partition_b200._build``).

Functions carry the C names: ``pad_decode``, ``pad_decode_with_workspace``,
``pad_decode_static_scratch``, ``pad_decode_tcgen05``, ``pad_decode_plan``,
``pad_check_device_errors``, ``pad_inject_stage_timeout``, ``pad_last_launch``,
``pad_release_workspace``, ``pad_status_string``, ``pad_last_error``,
``pad_abi_version``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple, Union

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpad.so")

PAD_OK, PAD_ERR_INVALID_ARG, PAD_ERR_UNSUPPORTED, PAD_ERR_WORKSPACE, PAD_ERR_CUDA, PAD_ERR_DEVICE_CHECK = range(6)
PAD_BF16, PAD_F32, PAD_I32, PAD_FP8_E4M3 = 0, 1, 2, 3
_DTYPES = {torch.bfloat16: PAD_BF16, torch.float32: PAD_F32, torch.int32: PAD_I32,
           torch.float8_e4m3fn: PAD_FP8_E4M3}
_KV_DTYPES = {"bf16": PAD_BF16, "e4m3": PAD_FP8_E4M3, torch.bfloat16: PAD_BF16, torch.float8_e4m3fn: PAD_FP8_E4M3}


class PadTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class PadPlan(ctypes.Structure):
    _fields_ = [("num_splits", ctypes.c_int32), ("partition_tokens", ctypes.c_int32),
                ("heads_per_tile", ctypes.c_int32), ("head_tiles", ctypes.c_int32),
                ("warps_per_cta", ctypes.c_int32), ("stage_tokens", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("ctas", ctypes.c_int32), ("ctas_per_sm", ctypes.c_int32),
                ("reduce", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_int64), ("control_bytes", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class PadOptions(ctypes.Structure):
    """pad_decode_options: sliding window, attention sinks, E4M3 cache scales."""
    _fields_ = [("window_left", ctypes.c_int32), ("sinks", ctypes.POINTER(PadTensor)),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


class PadLaunchWitness(ctypes.Structure):
    """pad_launch_witness: what the most recent launch recorded from inside the kernel."""
    _fields_ = [(n, ctypes.c_int32) for n in ("kernel", "head_dim", "heads_per_tile", "kv_dtype", "stages",
                                                  "stage_tokens", "num_splits", "partition_tokens", "ctas",
                                                  "warps", "ctas_per_sm")]


class PadError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


def _status_name(st: int) -> str:
    return ("PAD_OK", "PAD_ERR_INVALID_ARG", "PAD_ERR_UNSUPPORTED", "PAD_ERR_WORKSPACE",
            "PAD_ERR_CUDA", "PAD_ERR_DEVICE_CHECK")[st] if 0 <= st < 6 else f"status {st}"


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpad.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m paged_kv_attention_partition_b200._build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(PadTensor)
    lib.pad_decode.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_int32, P, P, ctypes.c_void_p]
    lib.pad_decode.restype = ctypes.c_int
    lib.pad_decode_static_scratch.argtypes = lib.pad_decode.argtypes
    lib.pad_decode_static_scratch.restype = ctypes.c_int
    lib.pad_decode_tcgen05.argtypes = lib.pad_decode.argtypes
    lib.pad_decode_tcgen05.restype = ctypes.c_int
    lib.pad_decode_ex.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_int32, ctypes.POINTER(PadOptions), P, P,
                                  ctypes.c_void_p]
    lib.pad_decode_ex.restype = ctypes.c_int
    lib.pad_decode_with_workspace.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_int32, P, P, ctypes.c_void_p,
                                              ctypes.c_size_t, ctypes.c_void_p]
    lib.pad_decode_with_workspace.restype = ctypes.c_int
    lib.pad_decode_with_workspace_ex.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_int32,
                                                 ctypes.POINTER(PadOptions), P, P, ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]
    lib.pad_decode_with_workspace_ex.restype = ctypes.c_int
    lib.pad_decode_plan.argtypes = [ctypes.c_int64] * 6 + [ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(PadPlan)]
    lib.pad_decode_plan.restype = ctypes.c_int
    lib.pad_decode_plan_ex.argtypes = [ctypes.c_int64] * 6 + [ctypes.c_int32] * 3 + [ctypes.POINTER(PadPlan)]
    lib.pad_decode_plan_ex.restype = ctypes.c_int
    lib.pad_last_launch.argtypes = [ctypes.POINTER(PadLaunchWitness)]
    lib.pad_last_launch.restype = ctypes.c_int
    lib.pad_status_string.argtypes = [ctypes.c_int]
    lib.pad_status_string.restype = ctypes.c_char_p
    lib.pad_last_error.argtypes = []
    lib.pad_last_error.restype = ctypes.c_char_p
    lib.pad_check_device_errors.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]
    lib.pad_check_device_errors.restype = ctypes.c_int
    lib.pad_inject_stage_timeout.argtypes = [ctypes.c_int32]
    lib.pad_inject_stage_timeout.restype = ctypes.c_int
    lib.pad_release_workspace.argtypes = [ctypes.c_int32]
    lib.pad_release_workspace.restype = ctypes.c_int
    lib.pad_abi_version.argtypes = []
    lib.pad_abi_version.restype = ctypes.c_int32
    _lib = lib
    return lib


def pad_last_error() -> str:
    return load_library().pad_last_error().decode()


def pad_status_string(status: int) -> str:
    return load_library().pad_status_string(status).decode()


def pad_abi_version() -> int:
    return load_library().pad_abi_version()


def _raise(st: int):
    if st != PAD_OK:
        raise PadError(st, pad_last_error())


def describe(t: torch.Tensor) -> PadTensor:
    """pad_tensor descriptor of a torch tensor (pointer, dtype, shape, element strides)."""
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dims")
    d = PadTensor()
    d.data = t.data_ptr()
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream_handle(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def pad_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
               seq_lens: torch.Tensor, scale: float, num_splits: int = 0, out: Optional[torch.Tensor] = None,
               lse: Union[None, bool, torch.Tensor] = None, stream=None, window: int = 0,
               sinks: Optional[torch.Tensor] = None, k_scale: float = 0.0,
               v_scale: float = 0.0) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Paged single-token decode attention (see ``pad_decode`` / ``pad_decode_ex``
    in include/pad.h).

    q [B, Hq, D] bf16; k_cache/v_cache [num_blocks, Hkv, block_size, D] bf16 or
    float8_e4m3fn (any 16-byte-multiple strides on dims 0-2, e.g.
    ``nhd.transpose(1, 2)``); block_tables [B, W] int32; seq_lens [B] int32.
    ``lse=True`` allocates the fp32 [B, Hq] log-sum-exp output, a tensor
    receives it, None skips it.  ``window`` > 0 attends to each sequence's last
    ``window`` tokens; ``sinks`` is an fp32 [Hq] CUDA tensor of per-head sink
    logits; ``k_scale`` / ``v_scale`` dequantise an E4M3 cache (0 = 1).
    Returns (out, lse).  Asynchronous on ``stream`` (default: torch's current)."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor")
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                    ("seq_lens", seq_lens)):
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, q on {dev}")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    if lse is True:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    for name, t in (("out", out), ("lse", lse)):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, q on {dev}")
    if sinks is not None and sinks.device != dev:
        raise ValueError(f"sinks is on {sinks.device}, q on {dev}")
    lib = load_library()
    dq, dk, dv, dt, dl, do = (describe(t) for t in (q, k_cache, v_cache, block_tables, seq_lens, out))
    dlse = describe(lse) if lse is not None else None
    with torch.cuda.device(dev):
        if window or sinks is not None or k_scale or v_scale:
            dsk = describe(sinks) if sinks is not None else None
            opts = PadOptions(int(window), ctypes.pointer(dsk) if dsk is not None else None, float(k_scale),
                              float(v_scale))
            st = lib.pad_decode_ex(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), ctypes.byref(dt),
                                   ctypes.byref(dl), float(scale), int(num_splits), ctypes.byref(opts),
                                   ctypes.byref(do), ctypes.byref(dlse) if dlse is not None else None,
                                   _stream_handle(stream, dev))
        else:
            st = lib.pad_decode(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), ctypes.byref(dt),
                                ctypes.byref(dl), float(scale), int(num_splits), ctypes.byref(do),
                                ctypes.byref(dlse) if dlse is not None else None, _stream_handle(stream, dev))
    _raise(st)
    return out, lse


def pad_decode_static_scratch(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits=0, out=None,
                              lse=None, stream=None):
    """pad_decode for callers that cannot allocate device memory: the split
    scratch is a fixed 32 MiB array inside the library (see include/pad.h).  The
    output tensors are still the caller's; pass them in (``out``, ``lse``) to
    keep the call itself allocation-free.  Calls sharing a device must not
    overlap on the GPU.  Returns (out, lse)."""
    dev = q.device
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    if lse is True:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    descs = [describe(t) for t in (q, k_cache, v_cache, block_tables, seq_lens, out)]
    dlse = describe(lse) if lse is not None else None
    with torch.cuda.device(dev):
        st = load_library().pad_decode_static_scratch(
            *(ctypes.byref(d) for d in descs[:5]), float(scale), int(num_splits), ctypes.byref(descs[5]),
            ctypes.byref(dlse) if dlse is not None else None, _stream_handle(stream, dev))
    _raise(st)
    return out, lse


def pad_decode_tcgen05(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits=0, out=None, lse=None,
                       stream=None):
    """pad_decode on the 5th-generation tensor-core kernel (see
    ``pad_decode_tcgen05`` in include/pad.h): groups of 17..32 query heads per KV
    head at head_dim 128, block_size >= 8.  Returns (out, lse)."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    if lse is True:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    descs = [describe(t) for t in (q, k_cache, v_cache, block_tables, seq_lens, out)]
    dlse = describe(lse) if lse is not None else None
    with torch.cuda.device(dev):
        st = load_library().pad_decode_tcgen05(
            *(ctypes.byref(d) for d in descs[:5]), float(scale), int(num_splits), ctypes.byref(descs[5]),
            ctypes.byref(dlse) if dlse is not None else None, _stream_handle(stream, dev))
    _raise(st)
    return out, lse


def pad_decode_with_workspace(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, workspace,
                              stream=None, window: int = 0, sinks: Optional[torch.Tensor] = None,
                              k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """pad_decode with caller-owned partials scratch (see include/pad.h):
    ``workspace`` is a contiguous device tensor of at least
    ``pad_decode_plan(...)["workspace_bytes"]`` bytes (any contents), or None
    when that is 0.  The options are those of ``pad_decode``
    (``pad_decode_with_workspace_ex`` when any is set)."""
    dev = q.device
    if workspace is not None and (workspace.device != dev or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous tensor on q's device")
    if sinks is not None and sinks.device != dev:
        raise ValueError(f"sinks is on {sinks.device}, q on {dev}")
    descs = [describe(t) for t in (q, k_cache, v_cache, block_tables, seq_lens, out)]
    dlse = describe(lse) if lse is not None else None
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    lib = load_library()
    with torch.cuda.device(dev):
        if window or sinks is not None or k_scale or v_scale:
            dsk = describe(sinks) if sinks is not None else None
            opts = PadOptions(int(window), ctypes.pointer(dsk) if dsk is not None else None, float(k_scale),
                              float(v_scale))
            st = lib.pad_decode_with_workspace_ex(
                *(ctypes.byref(d) for d in descs[:5]), float(scale), int(num_splits), ctypes.byref(opts),
                ctypes.byref(descs[5]), ctypes.byref(dlse) if dlse is not None else None, ws_ptr, ws_bytes,
                _stream_handle(stream, dev))
        else:
            st = lib.pad_decode_with_workspace(
                *(ctypes.byref(d) for d in descs[:5]), float(scale), int(num_splits), ctypes.byref(descs[5]),
                ctypes.byref(dlse) if dlse is not None else None, ws_ptr, ws_bytes, _stream_handle(stream, dev))
    _raise(st)


def pad_decode_plan(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                    max_blocks_per_seq: int, num_splits: int = 0, device: int = -1, kv_dtype="bf16") -> dict:
    """Launch geometry pad_decode would use for this shape (no launch);
    ``kv_dtype`` "bf16" or "e4m3" (or the torch dtype) names the cache."""
    plan = PadPlan()
    lib = load_library()
    if kv_dtype in ("bf16", torch.bfloat16):
        st = lib.pad_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                 num_splits, device, ctypes.byref(plan))
    else:
        st = lib.pad_decode_plan_ex(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                    num_splits, _KV_DTYPES.get(kv_dtype, -1), device, ctypes.byref(plan))
    _raise(st)
    return plan.as_dict()


def pad_check_device_errors(stream=None, device=None) -> int:
    """Synchronise, then read and clear the device's sticky error word.  Returns
    the bits: 0 = clean, 0x1 = an out-of-range block id, 0x2 = an out-of-range
    sequence length, 0x4 = a bounded wait gave up (a stage's copies did not land
    in time, or ``pad_inject_stage_timeout`` stalled the launch; that launch's
    outputs are not valid, and the library's merge counters on the device are
    re-zeroed by this call).  Raises PadError only when the check itself fails."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        st = load_library().pad_check_device_errors(_stream_handle(stream, dev), ctypes.byref(bits))
    if st not in (PAD_OK, PAD_ERR_DEVICE_CHECK):
        _raise(st)
    return bits.value


def pad_inject_stage_timeout(partition: int) -> None:
    """Failure-path test hook (see include/pad.h): in the next partition-kernel
    launch from this thread the units of ``partition`` give up on a bounded wait
    instead of counting themselves for the merge, as on a stage that never
    lands (error bit 0x4).  -1 disarms it."""
    _raise(load_library().pad_inject_stage_timeout(int(partition)))


def pad_last_launch(device=None) -> dict:
    """What the most recent decode launch on the device recorded from inside the
    kernel: ``kernel`` (1 partition kernel, 2 tcgen05 kernel) and the plan it ran
    with.  Synchronises the device."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    w = PadLaunchWitness()
    with torch.cuda.device(dev):
        _raise(load_library().pad_last_launch(ctypes.byref(w)))
    return {name: getattr(w, name) for name, _ in w._fields_}


def pad_release_workspace(device: int = -1) -> None:
    """Free the library's split scratch for one device (all when < 0)."""
    _raise(load_library().pad_release_workspace(device))


__all__ = ["pad_decode", "pad_decode_with_workspace", "pad_decode_static_scratch", "pad_decode_tcgen05", "pad_decode_plan",
           "pad_check_device_errors", "pad_release_workspace",
           "pad_status_string", "pad_last_error", "pad_abi_version", "describe", "load_library",
           "PadError", "PadTensor", "PadPlan", "PadOptions", "PadLaunchWitness", "pad_last_launch",
           "pad_inject_stage_timeout"]
