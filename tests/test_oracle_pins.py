"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
closed forms, hand-derived golden cases, brute force over subsets, exact rational
arithmetic, and an independent library routine (torch's scaled-dot-product attention).
All CPU-only."""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle.compare import compare_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.strip() for l in f if l.strip() and not l.startswith("#")]


def _rand_layout(rng, F=None, P=None, S=None, H=2, d=8, b=None):
    F = F or int(rng.integers(1, 5))
    P = P or int(rng.integers(1, 41))
    S = S if S is not None else int(rng.integers(0, 6))
    b = b or int(rng.integers(1, F * P + 1))
    return oracle.Layout(F, P + S, S, H, d, b)


def _sdpa(q, k, v, allowed=None):
    """torch reference: q,k,v [M|N, d] float64, allowed [M, N] bool."""
    mask = None if allowed is None else torch.from_numpy(allowed)
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=mask)
    return o[0].numpy()


# ----------------------------------------------------------------------------- token split

def test_token_split_covers_rows_once():
    lay = oracle.Layout(3, 12, 5, 1, 4, 4)
    sr, pr = oracle.special_rows(lay), oracle.patch_rows(lay)
    assert list(sr) == [0, 1, 2, 3, 4, 12, 13, 14, 15, 16, 24, 25, 26, 27, 28]
    assert sorted(np.concatenate([sr, pr]).tolist()) == list(range(lay.N))
    assert pr[0] == 5 and pr[6] == 11 and pr[7] == 17 and pr[14] == 29   # P = 7 per frame


# ----------------------------------------------------------------------------- pooling

@pytest.mark.parametrize("seed", range(6))
def test_pool_of_arithmetic_sequence_is_block_midpoint(seed):
    """Row value = its patch index p  =>  block mean = (lo + hi - 1) / 2, including
    blocks that straddle frames and a ragged last block."""
    rng = np.random.default_rng(seed)
    lay = _rand_layout(rng, H=3, d=2)
    X = np.full((lay.N, lay.heads, lay.head_dim), -1e9)   # special rows must not leak in
    X[oracle.patch_rows(lay)] = np.arange(lay.Np, dtype=np.float64)[:, None, None]
    PX = oracle.pool(X, lay)
    for j in range(lay.B):
        lo = j * lay.block
        hi = min(lo + lay.block, lay.Np)
        assert np.allclose(PX[:, j, :], (lo + hi - 1) / 2.0, rtol=0, atol=1e-9)


def test_pool_b1_is_identity_and_b_ge_np_is_global_mean():
    rng = np.random.default_rng(1)
    lay = oracle.Layout(2, 9, 2, 2, 4, 1)
    X = rng.standard_normal((lay.N, 2, 4))
    assert np.array_equal(oracle.pool(X, lay), X[oracle.patch_rows(lay)].transpose(1, 0, 2))
    lay2 = oracle.Layout(2, 9, 2, 2, 4, 100)
    assert lay2.B == 1
    ref = X[oracle.patch_rows(lay2)].sum(axis=0) / lay2.Np
    assert np.allclose(oracle.pool(X, lay2)[:, 0], ref, atol=1e-14)


# ----------------------------------------------------------------------------- pooled softmax

def test_pooled_probs_b1_equal_patch_attention_probabilities():
    """b = 1: the pooled distribution is the exact patch-to-patch attention distribution."""
    rng = np.random.default_rng(2)
    lay = oracle.Layout(2, 10, 3, 2, 16, 1)
    Q = rng.standard_normal((lay.N, 2, 16))
    K = rng.standard_normal((lay.N, 2, 16))
    P = oracle.pooled_probs(oracle.pool(Q, lay), oracle.pool(K, lay), 16)
    pr = oracle.patch_rows(lay)
    for h in range(2):
        s = torch.from_numpy(Q[pr, h]) @ torch.from_numpy(K[pr, h]).T / 4.0
        assert np.allclose(P[h], torch.softmax(s, dim=1).numpy(), atol=1e-14)


def test_pooled_probs_uniform_for_identical_keys_and_rows_sum_to_one():
    rng = np.random.default_rng(3)
    PQ = rng.standard_normal((2, 7, 8))
    PK = np.broadcast_to(rng.standard_normal((2, 1, 8)), (2, 7, 8)).copy()
    assert np.allclose(oracle.pooled_probs(PQ, PK, 8), 1.0 / 7, atol=1e-15)
    P = oracle.pooled_probs(PQ, rng.standard_normal((2, 7, 8)), 8)
    assert np.all(P >= 0) and np.allclose(P.sum(axis=2), 1.0, atol=1e-14)


def test_pooled_scores_carry_inverse_sqrt_d():
    """Two blocks with scores s and 0 before scaling: p0 / p1 = exp(s / sqrt(d))."""
    d = 16
    PQ = np.zeros((1, 1, d)); PQ[0, 0, 0] = 2.0
    PK = np.zeros((1, 2, d)); PK[0, 0, 0] = 3.0
    P = oracle.pooled_probs(PQ, PK, d)
    assert math.isclose(P[0, 0, 0] / P[0, 0, 1], math.exp(6.0 / 4.0), rel_tol=1e-14)


# ----------------------------------------------------------------------------- k and budgets

def test_k_from_rho_matches_exact_rational_floor():
    for line in _lines("k_from_rho_cases.txt"):
        B, rho, k = line.split()
        assert oracle.k_from_rho(int(B), float(rho)) == int(k), line
        assert math.floor(int(B) * (1 - Fraction(rho))) == int(k), line
    for B in range(1, 3100, 7):
        for rho in ("0", "0.1", "0.25", "0.5", "0.75", "0.9", "0.95", "1"):
            assert oracle.k_from_rho(B, float(rho)) == math.floor(B * (1 - Fraction(rho)))


def test_k_from_density_golden_cases_with_the_one_block_floor():
    """Hand-derived budgets, including densities whose floor is 0 (clamped to one block)
    and products that land on an integer only in exact arithmetic (10 x 0.7, 100 x 0.29)."""
    lines = _lines("k_from_density_cases.txt")
    assert any(int(l.split()[2]) == 1 and math.floor(int(l.split()[0]) * Fraction(l.split()[1])) == 0
               for l in lines)                                    # the clamp is exercised
    for line in lines:
        B, d, k = line.split()
        assert oracle.k_from_density(int(B), float(d)) == int(k), line
        assert min(int(B), max(1, math.floor(int(B) * Fraction(d)))) == int(k), line


def test_water_fill_golden_cases():
    for line in _lines("water_fill_cases.txt"):
        s, total, cap, want = [x.split() for x in line.split("|")]
        got = oracle.water_fill(np.array([float(x) for x in s]), float(total[0]),
                                float(Fraction(cap[0])))
        assert np.allclose(got, [float(Fraction(x)) for x in want], rtol=0, atol=1e-14), line


@pytest.mark.parametrize("seed", range(20))
def test_water_fill_invariants(seed):
    rng = np.random.default_rng(seed)
    H = int(rng.integers(1, 20))
    s = rng.lognormal(0, 1.5, H)
    cap = float(rng.uniform(0.2, 1.0))
    total = float(rng.uniform(0, H * cap))
    d = oracle.water_fill(s, total, cap)
    assert math.isclose(d.sum(), total, rel_tol=0, abs_tol=1e-12)
    assert np.all(d <= cap + 1e-15) and np.all(d >= 0)
    order = np.argsort(s)
    assert np.all(np.diff(d[order]) >= -1e-15)                 # monotone in the score
    free = d < cap - 1e-12
    if free.sum() >= 2:                                       # proportional where uncapped
        r = d[free] / s[free]
        assert np.allclose(r, r[0], rtol=1e-12)


def test_perhead_budgets_golden():
    from view_transformers_b200 import configs, synth
    vals = dict(l.split(" ", 1) for l in _lines("perhead100_budgets.txt"))
    w = configs.PERHEAD100
    d = oracle.water_fill(synth.head_scores(w), 16 * 0.25, 1.0)
    assert [oracle.k_from_density(608, x) for x in d] == [int(x) for x in vals["k"].split()]


# ----------------------------------------------------------------------------- selection

def test_selection_golden_cases():
    for line in _lines("selection_cases.txt"):
        p, k, tau, want = [x.strip() for x in line.split("|")]
        p = np.array([[float(x) for x in p.split()]])
        _, _, count, sel = oracle.select(p, int(k), float(tau))
        want = [] if want == "-" else [int(x) for x in want.split()]
        assert list(np.nonzero(sel[0])[0]) == want, line
        assert count[0] == len(want)


@pytest.mark.parametrize("seed", range(40))
def test_selection_against_brute_force_over_subsets(seed):
    """n_tau is the smallest size of ANY subset reaching mass tau, and the kept set is
    the size-n subset of maximal mass (distinct probabilities)."""
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 9))
    p = rng.dirichlet(np.ones(B) * float(rng.uniform(0.3, 3)))
    k = int(rng.integers(0, B + 1))
    tau = float(rng.choice([0.0, rng.uniform(0, 1), 1.0]))
    subsets = [c for m in range(B + 1) for c in itertools.combinations(range(B), m)]
    if tau <= 0:
        n_tau = 0
    else:
        sizes = [len(c) for c in subsets if len(c) > 0 and sum(p[list(c)]) >= tau]
        n_tau = min(sizes) if sizes else B
    n = min(B, max(k, n_tau))
    best = max((c for c in subsets if len(c) == n), key=lambda c: sum(p[list(c)]))
    _, _, count, sel = oracle.select(p[None], k, tau)
    if n_tau not in (0, B) and abs(sum(sorted(p)[::-1][:n_tau]) - tau) < 1e-12:
        pytest.skip("tau sits on a partial sum; the brute force's sums are not order-exact")
    assert count[0] == n
    assert set(np.nonzero(sel[0])[0]) == set(best)


@pytest.mark.parametrize("seed", range(10))
def test_selection_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 300))
    P = rng.dirichlet(np.ones(B) * 0.5, size=16)
    k = int(rng.integers(0, B + 1))
    tau = float(rng.uniform(0, 1))
    order, cum, count, sel = oracle.select(P, k, tau)
    for i in range(16):
        n = count[i]
        assert n >= min(k, B) and sel[i].sum() == n
        if n < B:
            assert P[i][sel[i]].sum() >= tau - 1e-12
        if n > k:
            assert cum[i, n - 2] < tau if n >= 2 else True        # minimality
        if 0 < n < B:
            assert P[i][sel[i]].min() >= P[i][~sel[i]].max()


def test_selection_extremes():
    P = np.random.default_rng(5).dirichlet(np.ones(12), size=3)
    assert oracle.select(P, oracle.k_from_rho(12, 0.0), 0.0)[3].all()       # rho = 0 -> dense
    assert oracle.select(P, 0, 1.0)[3].all()                                # tau = 1 -> dense
    assert not oracle.select(P, oracle.k_from_rho(12, 1.0), 0.0)[3].any()   # rho = 1, tau = 0


# ----------------------------------------------------------------------------- attention

@pytest.mark.parametrize("seed", range(5))
def test_attend_matches_torch_sdpa(seed):
    rng = np.random.default_rng(seed)
    M, N, d = int(rng.integers(1, 30)), int(rng.integers(1, 60)), 16
    q, k, v = rng.standard_normal((M, d)) * 2, rng.standard_normal((N, d)) * 2, rng.standard_normal((N, d))
    o, lse = oracle.attend(q, k, v)
    assert np.allclose(o, _sdpa(q, k, v), atol=1e-12)
    ref = torch.logsumexp(torch.from_numpy(q @ k.T / 4.0), dim=1).numpy()
    assert np.allclose(lse, ref, atol=1e-12)


def test_attend_closed_forms():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((5, 8))
    k = rng.standard_normal((9, 8))
    c = rng.standard_normal(8)
    o, _ = oracle.attend(q, k, np.tile(c, (9, 1)))
    assert np.allclose(o, c, atol=1e-14)                       # constant values
    v = rng.standard_normal((9, 8))
    o, lse = oracle.attend(q, np.tile(k[0], (9, 1)), v)
    assert np.allclose(o, v.mean(axis=0), atol=1e-14)          # identical keys -> mean
    assert np.allclose(lse, q @ k[0] / math.sqrt(8) + math.log(9), atol=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_lse_merge_of_a_key_partition_is_the_joint_softmax(seed):
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((7, 8)), rng.standard_normal((40, 8)) * 3, rng.standard_normal((40, 8))
    part = rng.random(40) < 0.3
    part[0], part[1] = True, False
    oa, la = oracle.attend(q, k[part], v[part])
    ob, lb = oracle.attend(q, k[~part], v[~part])
    o, L = oracle.merge(oa[:, None], la[None], ob[:, None], lb[None])
    oj, lj = oracle.attend(q, k, v)
    assert np.allclose(o[:, 0], oj, atol=1e-13) and np.allclose(L[0], lj, atol=1e-12)


def _token_mask(lay, selected, h):
    """Eq. (2) with excluded masked entries, built at token level from the block mask."""
    allowed = np.zeros((lay.N, lay.N), dtype=bool)
    sr, pr = oracle.special_rows(lay), oracle.patch_rows(lay)
    allowed[sr, :] = True
    allowed[:, sr] = True
    blk = np.arange(lay.Np) // lay.block
    allowed[np.ix_(pr, pr)] = selected[h][blk[:, None], blk[None, :]]
    return allowed


@pytest.mark.parametrize("seed", range(8))
def test_layer_forward_matches_torch_masked_sdpa(seed):
    rng = np.random.default_rng(seed)
    lay = _rand_layout(rng, H=2, d=8)
    Q, K, V = (rng.standard_normal((lay.N, 2, 8)) for _ in range(3))
    sel = rng.random((2, lay.B, lay.B)) < 0.5
    sel[:, np.arange(lay.B), np.arange(lay.B)] = True
    out = oracle.layer_forward(Q, K, V, lay, sel)
    for h in range(2):
        ref = _sdpa(Q[:, h], K[:, h], V[:, h], _token_mask(lay, sel, h))
        assert np.allclose(out[:, h], ref, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_rho0_layer_is_dense_attention(seed):
    rng = np.random.default_rng(seed)
    lay = _rand_layout(rng, H=2, d=16)
    st = [rng.standard_normal((lay.N, 2, 16)).astype(np.float32) for _ in range(3)]
    res = oracle.run_layer(*st, "f32", lay, rho=0.0, tau=float(rng.uniform(0, 1)))
    Q, K, V = (x.astype(np.float64) for x in st)
    assert res.mask.selected.all()
    for h in range(2):
        assert np.allclose(res.out[:, h], _sdpa(Q[:, h], K[:, h], V[:, h]), atol=1e-12)
    res1 = oracle.run_layer(*st, "f32", lay, rho=0.5, tau=1.0)                 # tau = 1 -> dense
    assert np.allclose(res1.out, res.out, atol=1e-12)


def test_single_block_is_always_kept():
    rng = np.random.default_rng(9)
    lay = oracle.Layout(2, 12, 5, 2, 8, 64)
    st = [rng.standard_normal((lay.N, 2, 8)).astype(np.float32) for _ in range(3)]
    res = oracle.run_layer(*st, "f32", lay, rho=0.9, tau=0.5)
    assert lay.B == 1 and res.mask.selected.all()


def test_partials_merge_to_the_layer_output():
    rng = np.random.default_rng(11)
    lay = oracle.Layout(3, 20, 5, 2, 8, 6)
    Q, K, V = (rng.standard_normal((lay.N, 2, 8)) for _ in range(3))
    sel = rng.random((2, lay.B, lay.B)) < 0.4
    o_pp, l_pp, o_ps, l_ps = oracle.partials(Q, K, V, lay, sel)
    has = sel.any(axis=2)                       # rows whose block kept no patch key
    l_pp = np.where(np.repeat(has, lay.block, axis=1)[:, :lay.Np], l_pp, -np.inf)
    o_pp = np.nan_to_num(o_pp)
    merged, _ = oracle.merge(o_pp, l_pp, o_ps, l_ps)
    out = oracle.layer_forward(Q, K, V, lay, sel)
    assert np.allclose(merged, out[oracle.patch_rows(lay)], atol=1e-12)


def test_bf16_decoding_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F, 0x0080], dtype=np.uint16)
    want = [1.0, -1.0, 3.140625, 0.0, -0.0, 3.3895313892515355e38, 1.1754943508222875e-38]
    assert oracle.to_f64(bits, "bf16").tolist() == want


# ----------------------------------------------------------------------------- acceptance rule

def test_mask_comparison_rule_accepts_near_ties_only():
    p = np.array([[[0.3, 0.3 + 5e-7, 0.2, 0.2 - 5e-7]]])
    p = p / p.sum(axis=2, keepdims=True)
    order, cum, count, sel = oracle.select(p[0], 1, 0.0)
    m = oracle.MaskResult(p, order[None], cum[None], count[None], sel[None])
    swapped = np.zeros((1, 1, 4), dtype=bool); swapped[0, 0, 0] = True      # near-tie swap
    assert compare_mask(m, swapped, 0.0).exempt == 1
    wrong = np.zeros((1, 1, 4), dtype=bool); wrong[0, 0, 2] = True          # far from the cut
    assert compare_mask(m, wrong, 0.0).failed == 1
    assert compare_mask(m, sel[None], 0.0).exact == 1


@pytest.mark.parametrize("seed", range(3))
def test_layer_rows_match_layer_forward(seed):
    rng = np.random.default_rng(seed)
    lay = _rand_layout(rng, H=3, d=8, S=int(rng.integers(1, 6)))
    Q, K, V = (rng.standard_normal((lay.N, 3, 8)) for _ in range(3))
    sel = rng.random((3, lay.B, lay.B)) < 0.5
    full = oracle.layer_forward(Q, K, V, lay, sel)
    rows = rng.integers(0, lay.N, 40)
    heads = rng.integers(0, 3, 40)
    got = oracle.layer_rows(Q.astype(np.float32), K.astype(np.float32), V.astype(np.float32), lay, sel,
                            rows, heads)
    Q, K, V = (x.astype(np.float32).astype(np.float64) for x in (Q, K, V))
    full = oracle.layer_forward(Q, K, V, lay, sel)
    assert np.allclose(got, full[rows, heads], atol=1e-12)
