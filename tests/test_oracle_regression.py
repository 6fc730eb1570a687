"""The oracle against its own stored output (tests/golden/oracle_regression_16x32.txt,
written by tests/golden/make_oracle_regression.py): every stage, bit for
bit, on the stored inputs.  The pins in test_oracle_pins tie the oracle to
the pages and to mathematics; this file makes any later change to its
arithmetic visible as a changed fixture."""
import importlib.util
import os

import numpy as np

from conftest import ROOT

GOLDEN = os.path.join(ROOT, "tests", "golden")


def _generator():
    spec = importlib.util.spec_from_file_location("make_oracle_regression",
                                                  os.path.join(GOLDEN, "make_oracle_regression.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fixture():
    out = {}
    with open(os.path.join(GOLDEN, "oracle_regression_16x32.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, _, v = line.partition(":")
            out[k.strip()] = v.strip()
    return out


def test_every_oracle_stage_matches_the_stored_fixture():
    gen = _generator()
    fx = _fixture()
    O, K, T = (int(v) for v in fx["shape"].split())
    w = np.array([int(v, 16) for v in fx["w"].split()], dtype=np.uint32).view(np.float32).reshape(O, K)
    x = np.array([int(v, 16) for v in fx["x"].split()], dtype=np.uint16).reshape(T, K)
    dy = np.array([int(v, 16) for v in fx["dy"].split()], dtype=np.uint16).reshape(T, O)
    g = np.array([int(v, 16) for v in fx["rmsnorm.g"].split()], dtype=np.uint16)
    got = gen.stages(w, x, dy, g)
    stored = {k: v for k, v in fx.items() if k not in ("shape", "w", "x", "dy", "rmsnorm.g")}
    assert set(got) == set(stored)
    changed = [k for k in sorted(got) if got[k] != stored[k]]
    assert not changed, f"oracle output changed for: {changed}"


def test_fixture_inputs_are_the_seeded_workload_inputs():
    """The stored inputs are the generator's (so the fixture can be rewritten
    from the same seeds), and the stored stages satisfy the method's
    invariants: exactly n kept per group, ternary W_eff, |q| <= 127."""
    gen = _generator()
    fx = _fixture()
    w, x, dy, g = gen.inputs()
    assert fx["w"] == gen.hex32(w) and fx["x"] == gen.hex16(x) and fx["dy"] == gen.hex16(dy)
    O, K, T = (int(v) for v in fx["shape"].split())
    for n, m in gen.PATTERNS:
        mask = np.array(fx[f"{n}of{m}.mask"].split(), dtype=np.int64).reshape(O, K // m, m)
        assert (mask.sum(axis=2) == n).all()
        weff = np.array(fx[f"{n}of{m}.weff"].split(), dtype=np.int64)
        assert set(np.unique(weff)) <= {-1, 0, 1}
        q = np.array(fx[f"{n}of{m}.q"].split(), dtype=np.int64)
        assert np.abs(q).max() == 127
