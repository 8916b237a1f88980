"""Pins of the oracle's drift-score selection (oracle/ress.py) against facts that do not come
from the oracle itself: the drift identity checked by recomputing the renormalised kept-block
output from scratch, hand-derived golden rows, brute force over all subsets of small rows, and
invariants of the restoration rounds. CPU only."""
import itertools
import os

import numpy as np
import pytest

import oracle
from oracle import ress

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    for line in open(os.path.join(GOLDEN, "ress_cases.txt")):
        if line.strip() and not line.startswith("#"):
            p, v, k, kept, swaps = (x.strip() for x in line.split("|"))
            yield (np.array([float(x) for x in p.split()]),
                   np.array([[float(c) for c in row.split(",")] for row in v.split()]),
                   int(k), [int(x) for x in kept.split()], int(swaps))


def test_golden_rows():
    for p, v, k, kept, swaps in _cases():
        got, n = ress.select_row(p, v, k, rounds=8)
        assert list(np.nonzero(got)[0]) == kept and n == swaps


@pytest.mark.parametrize("seed", range(10))
def test_drift_is_the_shift_of_the_renormalised_output(seed):
    """drift(D) equals |o(kept) - o| with o(kept) = sum_{j kept} p_j v_j / sum_{j kept} p_j."""
    rng = np.random.default_rng(seed)
    B, d = int(rng.integers(2, 12)), int(rng.integers(1, 9))
    p = rng.dirichlet(np.ones(B))
    v = rng.standard_normal((B, d))
    o, delta = ress.drift_vectors(p, v)
    assert np.allclose(delta.sum(axis=0), 0.0, atol=1e-14)          # the deltas cancel
    D = rng.random(B) < 0.5
    D[0], D[1] = True, False
    kept = ~D
    o_kept = (p[kept, None] * v[kept]).sum(axis=0) / p[kept].sum()
    assert np.isclose(ress.drift(delta, p, D), np.linalg.norm(o_kept - (p[:, None] * v).sum(axis=0)), atol=1e-13)


@pytest.mark.parametrize("seed", range(20))
def test_rounds_never_raise_the_drift_and_keep_k(seed):
    rng = np.random.default_rng(100 + seed)
    B, d = int(rng.integers(2, 9)), 3
    p = rng.dirichlet(np.ones(B) * 0.7)
    v = rng.standard_normal((B, d))
    k = int(rng.integers(0, B + 1))
    start, _ = ress.select_row(p, v, k, rounds=0)
    got, swaps = ress.select_row(p, v, k, rounds=8)
    assert got.sum() == k and start.sum() == k and swaps <= 8
    if 0 < k < B:
        _, delta = ress.drift_vectors(p, v)
        d0, d1 = ress.drift(delta, p, ~start), ress.drift(delta, p, ~got)
        assert d1 <= d0 + 1e-15
        best = min(ress.drift(delta, p, ~np.isin(np.arange(B), c)) for c in itertools.combinations(range(B), k))
        assert d1 >= best - 1e-15                                     # brute force lower bound
        if swaps == 0:
            assert np.array_equal(got, start)


def test_start_keeps_the_largest_drift_vectors():
    rng = np.random.default_rng(7)
    p = rng.dirichlet(np.ones(10))
    v = rng.standard_normal((10, 4))
    _, delta = ress.drift_vectors(p, v)
    kept, _ = ress.select_row(p, v, 4, rounds=0)
    norm = np.linalg.norm(delta, axis=1)
    assert set(np.nonzero(kept)[0]) == set(np.argsort(-norm)[:4])


def test_ress_mask_runs_the_rows_from_pooled_tensors():
    rng = np.random.default_rng(9)
    lay = oracle.Layout(2, 30, 5, 2, 8, 10)         # B = 5
    Q, K, V = (rng.standard_normal((lay.N, 2, 8)) for _ in range(3))
    PQ, PK, PV = (oracle.pool(X, lay) for X in (Q, K, V))
    m = ress.ress_mask(PQ, PK, PV, 8, [2, 3], rounds=4)
    probs = oracle.pooled_probs(PQ, PK, 8)
    assert m.shape == (2, 5, 5) and np.all(m[0].sum(axis=1) == 2) and np.all(m[1].sum(axis=1) == 3)
    assert np.array_equal(m[1, 3], ress.select_row(probs[1, 3], PV[1], 3, 4)[0])
