"""Writes the fixtures in tests/golden/ from the oracle alone (inputs from synth/).

The pages print no worked example for this operation -- no attention values,
only tolerances and timings ("spec(BACKEND-ROCM): the ROCm head_dim=128 decode
arm", PR #564, and "perf(rocke): prepare saved paged decode bindings once",
PR #13700, section "Testing Summary", state their checks but not their values)
-- so nothing here is a pin.  These files are a tripwire: the oracle's output
on fixed seeded inputs, stored once, so that any later change to its arithmetic
shows up in tests/test_golden.py and has to be justified by a reading of the
pages.  The oracle is pinned by tests/test_oracle_pins.py.

    python tests/golden/make_golden.py      # rewrites tests/golden/oracle_*.txt
"""
import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def cases():
    """name -> (description, workload, window, sinks)."""
    tiny = synth.config("tiny")
    g5 = synth.make_workload("golden_d64_g5", 3, 10, 2, 64, 4, [1, 37, 130], seed=11, max_blocks_per_seq=40)
    sinks = np.linspace(-1.0, 1.0, g5.Hq).astype(np.float32)
    f8 = synth.make_workload("golden_e4m3_g8", 2, 16, 2, 128, 16, [300, 17], seed=12, max_blocks_per_seq=24,
                             kv_dtype="e4m3")
    return {
        "tiny": ("the tiny named workload: B1 Hq4/Hkv1 D128 L256 bs16, one permutation of 16 blocks", tiny, 0, None),
        "d64_g5_window_sinks": ("B3 Hq10/Hkv2 D64 bs4, lengths 1/37/130, last 50 tokens, one sink logit per head "
                                "(linspace -1..1)", g5, 50, sinks),
        "e4m3_g8": ("B2 Hq16/Hkv2 D128 bs16, lengths 300/17, E4M3 cache with the generator's k_scale/v_scale",
                    f8, 0, None),
    }


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a, dtype="<f8").tobytes()).hexdigest()


def compute(w, window, sinks):
    return oracle.decode_workload(w, nthreads=1, window=window, sinks=sinks)


def render(name, desc, out, lse):
    lines = [f"# oracle fixture {name}: {desc}",
             "# written by tests/golden/make_golden.py from oracle/ only (inputs from synth/); not a pin:",
             "# the pages print no worked example.  Values are float64 repr; digests over float64 little-endian.",
             f"shape {out.shape[0]} {out.shape[1]} {out.shape[2]}",
             f"sha256_out {digest(out)}",
             f"sha256_lse {digest(lse)}"]
    B, Hq, _ = out.shape
    for b in range(B):
        for h in range(Hq):
            lines.append(f"lse {b} {h} {float(lse[b, h])!r}")
    for b in range(B):
        for h in range(Hq):
            lines.append(f"rowsum {b} {h} {float(out[b, h].sum())!r}")
    return "\n".join(lines) + "\n"


def main():
    for name, (desc, w, window, sinks) in cases().items():
        out, lse = compute(w, window, sinks)
        path = os.path.join(HERE, f"oracle_{name}.txt")
        with open(path, "w") as f:
            f.write(render(name, desc, out, lse))
        print(path)


if __name__ == "__main__":
    main()
