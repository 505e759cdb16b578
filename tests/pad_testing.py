"""Shared helpers for the GPU tests: move a synth.Workload to the device, call
the library, compare with the oracle under the parity bar.

Parity bar (elementwise, from the target statement of this path):
  out: max |gpu - oracle| <= 2e-2 (gpu bf16 widened exactly, oracle in double)
  lse: |gpu - oracle| <= 1e-3 * max(|oracle|, 1)
"""
import numpy as np
import torch

import oracle
import synth

OUT_ATOL = 2e-2
LSE_RTOL = 1e-3


def bf16_dev(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)


def kv_dev(a: np.ndarray, dev) -> torch.Tensor:
    """A cache array on the device: uint16 bf16 bits, or uint8 E4M3 codes."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.view(torch.float8_e4m3fn if a.dtype == np.uint8 else torch.bfloat16).to(dev)


class DeviceWorkload:
    """A workload's tensors on the device.  layout "hnd" keeps the cache as
    [blocks, Hkv, bs, D]; "nhd" stores it [blocks, bs, Hkv, D] and passes the
    transposed view."""

    def __init__(self, w: synth.Workload, dev, layout: str = "hnd"):
        self.w = w
        self.q = bf16_dev(w.q, dev)
        if layout == "hnd":
            self.k = kv_dev(w.k_cache, dev)
            self.v = kv_dev(w.v_cache, dev)
        elif layout == "nhd":
            self.k = kv_dev(w.k_cache.transpose(0, 2, 1, 3), dev).transpose(1, 2)
            self.v = kv_dev(w.v_cache.transpose(0, 2, 1, 3), dev).transpose(1, 2)
        else:
            raise ValueError(layout)
        self.tables = torch.from_numpy(w.block_tables).to(dev)
        self.lens = torch.from_numpy(w.seq_lens).to(dev)
        self.dev = dev

    def run(self, num_splits=None, lse=True, poison=True, entry=None):
        import paged_kv_attention_partition_b200 as pad

        entry = pad.pad_decode if entry is None else entry
        w = self.w
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=self.dev)
        lse_t = torch.empty((w.B, w.Hq), dtype=torch.float32, device=self.dev) if lse else None
        if poison:  # every element must be written by the call
            out.fill_(float("nan"))
            if lse_t is not None:
                lse_t.fill_(float("nan"))
        splits = w.num_splits if num_splits is None else num_splits
        scales = dict(k_scale=w.k_scale, v_scale=w.v_scale) if w.kv_dtype == "e4m3" else {}
        entry(self.q, self.k, self.v, self.tables, self.lens, w.scale, num_splits=splits, out=out, lse=lse_t,
              **scales)
        torch.cuda.synchronize(self.dev)
        return out, lse_t


def to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


def check_parity(got_out, got_lse, ref_out, ref_lse, what=""):
    """Elementwise parity; returns (max abs out error, max relative lse error)."""
    got_out = np.asarray(got_out, dtype=np.float64)
    assert got_out.shape == ref_out.shape
    assert np.all(np.isfinite(got_out)), f"{what}: non-finite output"
    err = np.abs(got_out - ref_out)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= OUT_ATOL, f"{what}: out max-abs {worst:.4e} > {OUT_ATOL} at {np.unravel_index(err.argmax(), err.shape)}"
    lse_err = 0.0
    if got_lse is not None:
        got_lse = np.asarray(got_lse, dtype=np.float64)
        inf_ref = np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(got_lse), inf_ref), f"{what}: -inf lse mismatch"
        fin = ~inf_ref
        if fin.any():
            rel = np.abs(got_lse[fin] - ref_lse[fin]) / np.maximum(np.abs(ref_lse[fin]), 1.0)
            lse_err = float(rel.max())
            assert lse_err <= LSE_RTOL, f"{what}: lse rel {lse_err:.4e} > {LSE_RTOL}"
    return worst, lse_err


def sample_pairs(w: synth.Workload, n: int, seed: int):
    """(b, h) pairs for sampled full-size parity: always the longest and shortest
    sequences, the first and last heads, then seeded random pairs."""
    rng = np.random.default_rng(seed)
    b_long, b_short = int(np.argmax(w.seq_lens)), int(np.argmin(w.seq_lens))
    pairs = {(b_long, 0), (b_long, w.Hq - 1), (b_short, 0), (b_short, w.Hq - 1), (0, 0), (w.B - 1, w.Hq - 1)}
    while len(pairs) < n:
        pairs.add((int(rng.integers(w.B)), int(rng.integers(w.Hq))))
    return sorted(pairs)


def oracle_pairs(w: synth.Workload, pairs):
    return oracle.decode_pairs(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, pairs,
                               k_scale=w.k_scale, v_scale=w.v_scale)
