"""GPU parity of the ablation and alternative selector rows, through the C ABI on cuda:0:

  * random block selection (bit-exact lists against the oracle's Philox4x32-10 draw), with and
    without the dense special path ("Block-Sparse Global Attention for Efficient Multi-View
    Geometry Transformers", 消融实验, 图 10);
  * the CDF threshold alone (rho = 1, so k = 0) and the layer without the dense special path
    (the special tokens read as patch tokens), through the same mask prediction (same table);
  * fixed-stride uniform sampling (bit-exact) and the query-probe Top-K ("SAF3R: Dynamic Sparse
    Attention for Feed-Forward 3D Reconstruction Transformers", 四、1. and 四、3.): the probe lists
    match the oracle's fp64 ranking except near-ties within the fp32 rounding of the pooled
    means (compare_probe).

Outputs are compared with the oracle fed the device's lists, at the layer's tolerances
(relative L2 2e-3, max-abs 2e-2 for bf16 inputs)."""
import numpy as np
import pytest

import oracle
from oracle import selectors
from oracle.compare import compare_mask, compare_probe, max_abs, rel_l2
from view_transformers_b200 import configs

from gpu_common import exact, head_density, inputs, sample_pairs

pytestmark = pytest.mark.gpu

BF16_TOL = (2e-3, 2e-2)


def _lay(w):
    return oracle.Layout(w.frames, w.tokens_per_frame, w.layer_special, w.heads, w.head_dim, w.block)


def _run(w, x, dens):
    import torch
    from view_transformers_b200 import layer
    L = layer.BlockSparseLayer.for_workload(w, head_density=dens)
    q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, x.v))
    out = L.forward(q, k, v).float().cpu().numpy()
    torch.cuda.synchronize()
    status = L.check_status()
    kv_cnt = L.buf.kv_cnt.cpu().numpy()
    kv_idx = L.buf.kv_idx.cpu().numpy().view(np.uint16)
    return L, status, out, L.selected(), kv_cnt, kv_idx


def _check_lists(sel, cnt, idx):
    assert np.array_equal(sel.sum(axis=2), cnt)
    H, B, _ = sel.shape
    for h in range(H):
        for i in range(0, B, max(1, B // 16)):
            assert np.array_equal(np.nonzero(sel[h, i])[0], idx[h, i, :cnt[h, i]])


def _check_output(w, x, lay, sel, out):
    Q, K, V = (exact(a, w.dtype) for a in (x.q, x.k, x.v))
    if lay.N * lay.heads <= 40000:
        ref = oracle.layer_forward(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), lay, sel)
        got = out
    else:
        rows, heads = sample_pairs(w, 2048)
        ref = oracle.layer_rows(Q, K, V, lay, sel, rows, heads)
        got = out[rows, heads]
    e2, ea = rel_l2(got, ref), max_abs(got, ref)
    print(f"{w.name}: rel_l2 {e2:.3e} max_abs {ea:.3e}")
    assert e2 <= BF16_TOL[0] and ea <= BF16_TOL[1]


SMALL = dict(frames=3, heads=4)
RANDOM = [
    configs.RANDOM100.with_(name="random_f3_b128", **SMALL),
    configs.RANDOM100.with_(name="random_f3_b64", block=64, **SMALL),
    configs.RANDOM_NOSPECIAL100.with_(name="random_nospecial_f3", **SMALL),
    configs.RANDOM100.with_(name="random_f3_seed", seed=(5 << 32) | 77, head_budgets=False, rho=0.3, **SMALL),
    configs.RANDOM100.with_(name="random_f3_k0", head_budgets=False, rho=1.0, **SMALL),
    configs.RANDOM100.with_(name="random_f3_dense", head_budgets=False, rho=0.0, **SMALL),
    configs.RANDOM100,
    configs.RANDOM_NOSPECIAL100,
]


@pytest.mark.parametrize("w", RANDOM, ids=lambda w: w.name)
def test_random_selection(w):
    x = inputs(w)
    dens = head_density(w, x)
    L, status, out, sel, cnt, idx = _run(w, x, dens)
    assert status == 0
    lay = _lay(w)
    kh = oracle.head_k(lay, w.rho, dens)
    ref = selectors.random_mask(lay, kh, w.seed)
    assert np.array_equal(sel, ref)                       # integer work: bit-exact
    assert np.array_equal(cnt, np.broadcast_to(np.minimum(kh, lay.B)[:, None], cnt.shape))
    _check_lists(sel, cnt, idx)
    if np.any(kh > 0):
        _check_output(w, x, lay, sel, out)


UNIFORM = [
    configs.UNIFORM100.with_(name="uniform_f3_s4", **SMALL),
    configs.UNIFORM100.with_(name="uniform_f3_s3_b64", block=64, stride=3, **SMALL),
    configs.UNIFORM100.with_(name="uniform_f3_s1", stride=1, **SMALL),
    configs.UNIFORM100.with_(name="uniform_f3_s50", stride=50, **SMALL),
    configs.UNIFORM100,
]


@pytest.mark.parametrize("w", UNIFORM, ids=lambda w: w.name)
def test_uniform_sampling(w):
    x = inputs(w)
    L, status, out, sel, cnt, idx = _run(w, x, None)
    assert status == 0
    lay = _lay(w)
    assert np.array_equal(sel, selectors.uniform_mask(lay, w.stride))
    _check_lists(sel, cnt, idx)
    _check_output(w, x, lay, sel, out)


PROBE = [
    configs.PROBE100.with_(name="probe_f3", **SMALL),
    configs.PROBE100.with_(name="probe_f3_b64", block=64, **SMALL),
    configs.PROBE100.with_(name="probe_f4_rho", frames=4, heads=3, head_budgets=False, rho=0.5),
    configs.PROBE100,
]


@pytest.mark.parametrize("w", PROBE, ids=lambda w: w.name)
def test_query_probe_topk(w):
    x = inputs(w)
    dens = head_density(w, x)
    L, status, out, sel, cnt, idx = _run(w, x, dens)
    assert status == 0
    lay = _lay(w)
    Q, K = (exact(a, w.dtype) for a in (x.q, x.k))
    kh = oracle.head_k(lay, w.rho, dens)
    scores, ref = selectors.probe_mask(Q, K, lay, kh)
    assert np.all(sel == sel[:, :1])                       # one list per head
    rep = compare_probe(scores, selectors.probe_score_scale(Q, K, lay), kh, sel[:, 0])
    print(f"{w.name}: heads {rep.rows} exact {rep.exact} exempt {rep.exempt} failed {rep.failed}")
    assert rep.ok, rep.failures
    _check_lists(sel, cnt, idx)
    _check_output(w, x, lay, sel, out)


ABLATION = [
    configs.CDF_ONLY100.with_(name="cdf_only_f3", **SMALL),
    configs.CDF_ONLY100.with_(name="cdf_only_f3_tau90", tau=0.9, **SMALL),
    configs.CDF_ONLY100.with_(name="cdf_only_f3_b64", block=64, **SMALL),
    configs.NOSPECIAL100.with_(name="nospecial_f3", **SMALL),
    configs.NOSPECIAL100.with_(name="nospecial_f3_b64", block=64, head_budgets=False, rho=0.7, **SMALL),
    configs.CDF_ONLY100,
    configs.NOSPECIAL100,
]


@pytest.mark.parametrize("w", ABLATION, ids=lambda w: w.name)
def test_ablation_masks_and_layer(w):
    """The same mask prediction and attention under the CDF-only setting (k = 0) and under
    the no-dense-special reading (every token of a frame pooled and sparsified)."""
    x = inputs(w)
    dens = head_density(w, x)
    L, status, out, sel, cnt, idx = _run(w, x, dens)
    assert status == 0
    lay = _lay(w)
    Q, K = (exact(a, w.dtype) for a in (x.q, x.k))
    kh = oracle.head_k(lay, w.rho, dens)
    if w.rho == 1.0:
        assert np.all(kh == 0)
    om = oracle.predict_mask(oracle.pool(Q, lay), oracle.pool(K, lay), lay.head_dim, kh, w.tau)
    rep = compare_mask(om, sel, w.tau)
    print(f"{w.name}: mask rows {rep.rows} exact {rep.exact} exempt {rep.exempt} failed {rep.failed}; "
          f"density {sel.mean():.3f}")
    assert rep.ok, rep.failures
    _check_lists(sel, cnt, idx)
    _check_output(w, x, lay, sel, out)


RESS = [
    configs.RESS100.with_(name="ress_f3", **SMALL),
    configs.RESS100.with_(name="ress_f3_b64", block=64, **SMALL),
    configs.RESS100.with_(name="ress_f3_r0", rounds=0, **SMALL),
    configs.RESS100.with_(name="ress_f4_rho_r32", frames=4, heads=3, head_budgets=False, rho=0.5, rounds=32),
    configs.RESS100.with_(name="ress_f3_k0", head_budgets=False, rho=1.0, **SMALL),
    configs.RESS100,
]


@pytest.mark.parametrize("w", RESS, ids=lambda w: w.name)
def test_drift_score_selection(w):
    """Drift-score rows ("ReSS...", 技术框架 / 关键设计) against the oracle run on the device's own
    pooled means (fp32 values, exact in fp64), so that both sides take every decision in fp64
    on the same numbers: rows must match exactly unless one of the oracle's decisions had a
    relative gap below 1e-9 (a rounding-level tie). The pooled V is checked against the
    oracle's pooling, and the layer output against the oracle fed the device's lists."""
    from oracle import ress
    x = inputs(w)
    dens = head_density(w, x)
    L, status, out, sel, cnt, idx = _run(w, x, dens)
    assert status == 0
    lay = _lay(w)
    PQd = L.buf.pq.cpu().numpy().astype(np.float64)
    PKd = L.buf.pk.cpu().numpy().astype(np.float64).transpose(0, 2, 1)
    PVd = L.pv.cpu().numpy().astype(np.float64).transpose(0, 2, 1)
    V = exact(x.v, w.dtype)
    assert max_abs(PVd, oracle.pool(V, lay)) < 1e-5
    kh = oracle.head_k(lay, w.rho, dens)
    probs = oracle.pooled_probs(PQd, PKd, lay.head_dim)
    H, B = lay.heads, lay.B
    pairs = [(h, i) for h in range(H) for i in range(B)]
    if len(pairs) > 400:
        g = np.random.default_rng(11)
        pairs = [pairs[t] for t in g.choice(len(pairs), 96, replace=False)]
    exact_rows = exempt = 0
    for h, i in pairs:
        margins = []
        ref, _ = ress.select_row(probs[h, i], PVd[h], int(kh[h]), w.rounds, margins)
        if np.array_equal(ref, sel[h, i]):
            exact_rows += 1
        else:
            assert margins and min(margins) < 1e-9, (h, i, np.nonzero(ref ^ sel[h, i])[0])
            exempt += 1
    print(f"{w.name}: rows {len(pairs)} exact {exact_rows} exempt {exempt}; density {sel.mean():.3f}")
    assert np.array_equal(cnt, np.broadcast_to(np.minimum(kh, B)[:, None], cnt.shape))
    _check_lists(sel, cnt, idx)
    if np.any(kh > 0):
        _check_output(w, x, lay, sel, out)
