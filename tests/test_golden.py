"""The oracle against the fixtures in tests/golden/ (CPU).

The pages print no worked example, so these fixtures are the oracle's own
output on fixed seeded inputs, written by tests/golden/make_golden.py (oracle/
and synth/ only): a tripwire, not a pin.  A mismatch means the oracle's
arithmetic changed; such a change must name, in its commit, the passage of the
pages (or the reading of it) that justifies it, and the fixtures are rewritten
with the script.
"""
import importlib.util
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
_spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "golden", "make_golden.py"))
make_golden = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(make_golden)


def _read(path):
    meta, lse, rowsum = {}, {}, {}
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if parts[0] == "lse":
            lse[(int(parts[1]), int(parts[2]))] = float(parts[3])
        elif parts[0] == "rowsum":
            rowsum[(int(parts[1]), int(parts[2]))] = float(parts[3])
        else:
            meta[parts[0]] = parts[1:]
    return meta, lse, rowsum


@pytest.mark.parametrize("name", sorted(make_golden.cases()))
def test_oracle_matches_its_fixture(name):
    desc, w, window, sinks = make_golden.cases()[name]
    out, lse = make_golden.compute(w, window, sinks)
    meta, want_lse, want_rowsum = _read(os.path.join(HERE, "golden", f"oracle_{name}.txt"))
    assert [int(x) for x in meta["shape"]] == list(out.shape)
    # values first, so that a change says where it is
    for (b, h), v in want_lse.items():
        got = float(lse[b, h])
        assert got == v or (np.isneginf(got) and np.isneginf(v)), f"{name}: lse[{b},{h}] {got!r} != {v!r}"
    for (b, h), v in want_rowsum.items():
        assert float(out[b, h].sum()) == v, f"{name}: sum out[{b},{h},:] {float(out[b, h].sum())!r} != {v!r}"
    assert make_golden.digest(out) == meta["sha256_out"][0], f"{name}: out differs from the fixture"
    assert make_golden.digest(lse) == meta["sha256_lse"][0], f"{name}: lse differs from the fixture"


def test_fixtures_cover_every_case():
    files = {f for f in os.listdir(os.path.join(HERE, "golden")) if f.startswith("oracle_") and f.endswith(".txt")}
    assert files == {f"oracle_{n}.txt" for n in make_golden.cases()}
