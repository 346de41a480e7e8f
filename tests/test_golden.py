"""The oracle reproduces its stored batch-1 snapshot (regression guard for oracle edits).

A change to the oracle's arithmetic that moves these values must be justified by the
passage it follows and the snapshot rewritten with tests/golden/make_golden.py.
"""
import os

import numpy as np

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_batch1_snapshot(oracle_mod):
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    got = mg.batch1_lines()
    with open(os.path.join(HERE, "batch1_oracle.txt")) as fh:
        want = [l.rstrip("\n") for l in fh if not l.startswith("#")]
    assert len(got) == len(want)
    for g, w in zip(got, want):
        g, w = g.split(), w.split()
        assert g[:3] == w[:3] and g[-1] == w[-1]
        assert np.allclose(np.array(g[3:-1], float), np.array(w[3:-1], float), rtol=0, atol=1e-15)


def test_next_rows_snapshot(oracle_mod):
    """Phong lighting, point rasterization + compositing and KNN outputs of the oracle stay
    as stored (same rule as the batch-1 snapshot)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    got = mg.next_rows_lines()
    with open(os.path.join(HERE, "next_rows_oracle.txt")) as fh:
        want = [l.rstrip("\n") for l in fh if not l.startswith("#")]
    assert len(got) == len(want)
    ints = {"phong": 3, "points": 7, "knn": 7}          # leading integer fields per tag
    for g, w in zip(got, want):
        g, w = g.split(), w.split()
        n = ints[w[0]]
        assert g[:n] == w[:n], (g[:n], w[:n])
        assert np.allclose(np.array(g[n:], float), np.array(w[n:], float), rtol=1e-14, atol=1e-15)
