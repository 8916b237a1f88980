"""Pins of the oracle's alternative block selectors (random, fixed-stride uniform, query
probe) against facts that do not come from the oracle itself: the generator's published
known-answer vectors, brute force over small cases, closed forms, the column-mean identity
of the query probe, and the uniformity of the random draw. CPU only."""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import selectors

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kat():
    rows = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        if line.strip() and not line.startswith("#"):
            c, k, out = (part.split() for part in line.split("|"))
            rows.append(([int(x, 16) for x in c], [int(x, 16) for x in k], [int(x, 16) for x in out]))
    return rows


def test_philox_known_answer_vectors():
    for c, k, want in _kat():
        got = selectors.philox4x32_10(*c, *k)
        assert [int(x) for x in got] == want


def test_philox_vectorised_matches_elementwise():
    c0 = np.arange(50)
    got = selectors.philox4x32_10(c0, 3, 7, 0, 11, 0)
    for t in range(0, 50, 7):
        one = selectors.philox4x32_10(t, 3, 7, 0, 11, 0)
        assert [int(w[t]) for w in got] == [int(w) for w in one]


@pytest.mark.parametrize("seed", [0, 1, 2**40 + 5])
def test_random_mask_is_the_k_smallest_keys_by_brute_force(seed):
    lay = oracle.Layout(2, 25, 5, 3, 8, 4)           # B = 10
    kh = [0, 3, 10]
    keys = selectors.random_keys(lay, seed)
    sel = selectors.random_mask(lay, kh, seed)
    for h in range(lay.heads):
        for i in range(lay.B):
            best = sorted((int(keys[h, i, j]), j) for j in range(lay.B))[:kh[h]]
            assert sorted(j for _, j in best) == list(np.nonzero(sel[h, i])[0])
    assert sel[0].sum() == 0 and sel[2].all()


def test_random_mask_keys_follow_the_counter_layout():
    """Key of block j in row (h, i) is word 0 of Philox4x32-10 at counter (j, i, h, 0),
    key (seed low word, seed high word)."""
    lay = oracle.Layout(3, 10, 2, 2, 8, 3)
    seed = (7 << 32) | 12345
    keys = selectors.random_keys(lay, seed)
    for h, i, j in [(0, 0, 0), (1, 2, 5), (1, lay.B - 1, lay.B - 1)]:
        assert keys[h, i, j] == selectors.philox4x32_10(j, i, h, 0, 12345, 7)[0]


def test_random_mask_is_uniform_over_blocks():
    """Across many rows every block is kept with frequency k / B (binomial bound), and the
    draws of different rows and seeds differ."""
    lay = oracle.Layout(8, 64, 0, 4, 8, 4)             # B = 128, 4 x 128 rows
    k = 32
    sel = selectors.random_mask(lay, [k] * 4, seed=9)
    assert np.all(sel.sum(axis=2) == k)
    freq = sel.reshape(-1, lay.B).mean(axis=0)
    n = sel.shape[0] * sel.shape[1]
    sd = math.sqrt(k / lay.B * (1 - k / lay.B) / n)
    assert np.all(np.abs(freq - k / lay.B) < 5 * sd)
    assert not np.array_equal(sel[:, 0], sel[:, 1])
    assert not np.array_equal(sel, selectors.random_mask(lay, [k] * 4, seed=10))


def test_uniform_mask_closed_form():
    lay = oracle.Layout(3, 50, 5, 2, 8, 16)            # Np = 135, B = 9
    for s in (1, 2, 3, 4, 9, 20):
        m = selectors.uniform_mask(lay, s)
        assert np.all(m.sum(axis=2) == -(-lay.B // s))
        assert list(np.nonzero(m[1, 4])[0]) == list(range(0, lay.B, s))
    assert selectors.uniform_mask(lay, 1).all()


def test_probe_scores_are_column_means_of_the_patch_scores():
    """SAF3R's identity: the mean over queries of Q K^T / sqrt(D) equals q_bar K^T / sqrt(D),
    checked against the full patch score matrix; a block's score is the mean of its keys'."""
    rng = np.random.default_rng(4)
    lay = oracle.Layout(3, 23, 4, 2, 16, 5)
    Q = rng.standard_normal((lay.N, 2, 16))
    K = rng.standard_normal((lay.N, 2, 16))
    pr = oracle.patch_rows(lay)
    got = selectors.probe_key_scores(Q, K, lay)
    for h in range(2):
        S = Q[pr, h] @ K[pr, h].T / 4.0                  # [Np, Np] brute force
        assert np.allclose(got[h], S.mean(axis=0), atol=1e-13)
        blocks = selectors.probe_block_scores(Q, K, lay)[h]
        for j in range(lay.B):
            lo, hi = j * lay.block, min((j + 1) * lay.block, lay.Np)
            assert math.isclose(blocks[j], S[:, lo:hi].mean(), abs_tol=1e-13)


def test_probe_mask_keeps_the_top_blocks_for_every_query_block():
    rng = np.random.default_rng(5)
    lay = oracle.Layout(2, 40, 5, 3, 8, 8)             # Np = 70, B = 9 (ragged tail)
    Q = rng.standard_normal((lay.N, 3, 8))
    K = rng.standard_normal((lay.N, 3, 8))
    kh = [1, 4, 9]
    s, m = selectors.probe_mask(Q, K, lay, kh)
    for h in range(3):
        kept = np.nonzero(m[h, 0])[0]
        assert len(kept) == kh[h]
        assert list(kept) == sorted(np.argsort(-s[h], kind="stable")[:kh[h]])
        assert np.all(m[h] == m[h, 0])                   # the same list for every query block
        if kh[h] < lay.B:
            assert s[h, kept].min() >= s[h, ~m[h, 0]].max()


def test_probe_ties_go_to_the_lower_block():
    lay = oracle.Layout(1, 8, 0, 1, 4, 2)              # B = 4
    Q = np.ones((8, 1, 4))
    K = np.zeros((8, 1, 4))
    K[2:4] = 1.0                                       # block 1 high; blocks 0, 2, 3 tie at 0
    _, m = selectors.probe_mask(Q, K, lay, [2])
    assert list(np.nonzero(m[0, 0])[0]) == [0, 1]
