"""GPU parity: every step of the layer, through the C ABI on cuda:0, against the fp64 oracle.

Tolerances (from the acceptance rule of the layer): block masks bit-exact except blocks
whose pooled-probability gap to the cut (or whose CDF crossing) is below 1e-6; outputs
within relative L2 2e-3 and max-abs 2e-2 for bf16 inputs, 1e-5 for f32 inputs. Pooled
means are fp32 sums of at most b values: within 1e-5 absolute.
Full-size workloads are checked on 2,048 seeded (row, head) samples of the output, the
mask on every row."""
import numpy as np
import pytest

import oracle
from oracle.compare import compare_mask, max_abs, nmse_per_head, rel_l2
from view_transformers_b200 import configs

from gpu_common import exact, head_density, inputs, oracle_layout, run_gpu, sample_pairs

pytestmark = pytest.mark.gpu

BF16_TOL = (2e-3, 2e-2)
F32_TOL = (1e-5, 1e-5)

SMALL_BF16 = [
    configs.VGGT518.with_(name="vggt518_f3", frames=3, heads=4),
    configs.SWEEP_TAU0.with_(name="sweep_tau0_f4", frames=4, heads=3),
    configs.PERHEAD100.with_(name="perhead_f3", frames=3, heads=4, head_budgets=False, rho=0.6),
]
FULL = [configs.TINY, configs.TINY_TAU0, configs.VGGT518, configs.SWEEP_R50, configs.SWEEP_R75,
        configs.SWEEP_R90, configs.SWEEP_TAU0, configs.PERHEAD100, configs.PERHEAD100_TAU95]


def _oracle_mask(w, x, res):
    lay = oracle_layout(w)
    Q, K = exact(x.q, w.dtype), exact(x.k, w.dtype)
    PQ, PK = oracle.pool(Q, lay), oracle.pool(K, lay)
    dens = None if x.scores is None else oracle.water_fill(x.scores, w.heads * (1.0 - w.rho), 1.0)
    kh = oracle.head_k(lay, w.rho, dens)
    return lay, PQ, PK, kh, oracle.predict_mask(PQ, PK, lay.head_dim, kh, w.tau)


def _rows_with_same_mask(lay, om_selected, dev_selected):
    """[N, H] bool: output rows whose keys are the same under the oracle's own mask and the
    device's (every special row; a patch row when its query block's kept set matches)."""
    same_blk = np.all(om_selected == dev_selected, axis=2)                  # [H, B]
    ok = np.ones((lay.N, lay.heads), dtype=bool)
    pr = oracle.patch_rows(lay)
    ok[pr] = same_blk[:, np.arange(lay.Np) // lay.block].T
    return ok


def _check_lists(res, B):
    """kv_idx rows are ascending, distinct, and agree with the mask bits and counts."""
    sel, idx, cnt = res["selected"], res["kv_idx"], res["kv_cnt"]
    assert np.array_equal(sel.sum(axis=2), cnt)
    H = sel.shape[0]
    for h in range(H):
        for i in range(0, B, max(1, B // 64)):
            lst = idx[h, i, :cnt[h, i]]
            assert np.all(np.diff(lst.astype(np.int64)) > 0)
            assert np.array_equal(np.nonzero(sel[h, i])[0], lst)


@pytest.mark.parametrize("w", FULL + SMALL_BF16, ids=lambda w: w.name)
def test_mask_and_layer(w):
    x = inputs(w)
    dens = head_density(w, x)
    res = run_gpu(w, x, dens)
    assert res["status"] == 0
    lay, PQ, PK, kh, om = _oracle_mask(w, x, res)
    # pooling
    assert max_abs(res["pq"], PQ) < 1e-5 and max_abs(res["pk"], PK.transpose(0, 2, 1)) < 1e-5
    # mask
    rep = compare_mask(om, res["selected"], w.tau)
    print(f"{w.name}: mask rows {rep.rows} exact {rep.exact} exempt {rep.exempt} failed {rep.failed}")
    assert rep.ok, rep.failures
    assert np.all(res["kv_cnt"] >= np.minimum(kh, lay.B)[:, None])
    _check_lists(res, lay.B)
    # output, against the oracle fed the device mask
    Q, K, V = (exact(a, w.dtype) for a in (x.q, x.k, x.v))
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    small = lay.N * lay.heads <= 4096
    rows, heads = (None, None) if small else sample_pairs(w, 2048)

    def reference(selected):
        if small:
            return oracle.layer_forward(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64),
                                        lay, selected)
        return oracle.layer_rows(Q, K, V, lay, selected, rows, heads)

    pick = (lambda a: a) if small else (lambda a: a[rows, heads])
    ref = reference(res["selected"])
    if small:
        print(f"{w.name}: nmse/head {nmse_per_head(res['out'], ref)}")
    for key in ("out", "out_fused"):
        if res[key] is None:
            continue
        got = pick(res[key])
        e2, ea = rel_l2(got, ref), max_abs(got, ref)
        print(f"{w.name} {key}: rel_l2 {e2:.3e} max_abs {ea:.3e}")
        assert e2 <= tol[0] and ea <= tol[1]
    # output, against the oracle fed its own mask, on the rows whose kept sets agree (the
    # others differ only by near-tie exemptions of the mask rule)
    keep = pick(_rows_with_same_mask(lay, om.selected, res["selected"]))
    ref_own = ref if np.array_equal(om.selected, res["selected"]) else reference(om.selected)
    assert keep.mean() > 0.5
    got = pick(res["out_fused"] if res["out_fused"] is not None else res["out"])
    e2, ea = rel_l2(got[keep], ref_own[keep]), max_abs(got[keep], ref_own[keep])
    print(f"{w.name} own-mask rows {keep.sum()}/{keep.size}: rel_l2 {e2:.3e} max_abs {ea:.3e}")
    assert e2 <= tol[0] and ea <= tol[1]
    # forward(): pooling folded into the packing pass, then mask and fused attention
    fwd = res["forward"]
    if fwd is not None:
        assert max_abs(fwd["pq"], PQ) < 1e-5 and max_abs(fwd["pk"], PK.transpose(0, 2, 1)) < 1e-5
        rep = compare_mask(om, fwd["selected"], w.tau)
        assert rep.ok, rep.failures
        ref_f = ref if np.array_equal(fwd["selected"], res["selected"]) else reference(fwd["selected"])
        got = pick(fwd["out"])
        e2, ea = rel_l2(got, ref_f), max_abs(got, ref_f)
        print(f"{w.name} forward: rel_l2 {e2:.3e} max_abs {ea:.3e}")
        assert e2 <= tol[0] and ea <= tol[1]


@pytest.mark.parametrize("w", SMALL_BF16 + [configs.TINY], ids=lambda w: w.name)
def test_partials(w):
    """o_pp / lse_pp (kept patch keys) and o_ps / lse_ps (special keys) element by element."""
    x = inputs(w)
    res = run_gpu(w, x, head_density(w, x))
    lay = oracle_layout(w)
    Q, K, V = (exact(a, w.dtype).astype(np.float64) for a in (x.q, x.k, x.v))
    o_pp, l_pp, o_ps, l_ps = oracle.partials(Q, K, V, lay, res["selected"])
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    for got, ref in ((res["o_pp"], o_pp), (res["o_ps"], o_ps)):
        assert rel_l2(got, ref) <= tol[0] and max_abs(got, ref) <= tol[1]
    assert max_abs(res["lse_pp"], l_pp) < 1e-4 and max_abs(res["lse_ps"], l_ps) < 1e-4


@pytest.mark.slow
def test_long500_mask_full_and_sampled_rows():
    w = configs.LONG500
    x = inputs(w)
    res = run_gpu(w, x)
    assert res["status"] == 0
    lay, PQ, PK, kh, om = _oracle_mask(w, x, res)
    assert max_abs(res["pq"], PQ) < 1e-5
    rep = compare_mask(om, res["selected"], w.tau)
    print(f"long500: mask rows {rep.rows} exact {rep.exact} exempt {rep.exempt} failed {rep.failed}")
    assert rep.ok, rep.failures
    rows, heads = sample_pairs(w, 2048)
    Q, K, V = (exact(a, w.dtype) for a in (x.q, x.k, x.v))
    ref = oracle.layer_rows(Q, K, V, lay, res["selected"], rows, heads)
    for key in ("out", "out_fused"):
        got = res[key][rows, heads]
        print(f"long500 {key}: rel_l2 {rel_l2(got, ref):.3e} max_abs {max_abs(got, ref):.3e}")
        assert rel_l2(got, ref) <= BF16_TOL[0] and max_abs(got, ref) <= BF16_TOL[1]


@pytest.mark.slow
def test_long_rows_twelve_row_mask_variant():
    """B = 3,643 blocks (600 frames, 2 heads): past the 14-row long-row CTA's shared memory, so
    the mask kernel runs 12 rows per CTA; every row against the oracle."""
    import torch
    from view_transformers_b200 import layer
    w = configs.LONG500.with_(name="long600_h2", frames=600, heads=2, tau=0.0)
    x = inputs(w)
    L = layer.BlockSparseLayer.for_workload(w)
    assert L.B == 3643
    q, k = (layer.to_device(a, w.dtype) for a in (x.q, x.k))
    L.predict(q, k)
    torch.cuda.synchronize()
    assert L.check_status() == 0
    lay, PQ, PK, kh, om = _oracle_mask(w, x, {})
    rep = compare_mask(om, L.selected(), w.tau)
    print(f"long600_h2: mask rows {rep.rows} exact {rep.exact} exempt {rep.exempt} failed {rep.failed}")
    assert rep.ok, rep.failures


# ------------------------------------------------------------------ edge cases

EDGE = [
    configs.Workload("no_special", 3, 777, 0, 2, 64, 128, 0.5, 0.5, "bf16", "five_percent"),
    configs.Workload("empty_lists", 3, 777, 5, 2, 64, 128, 1.0, 0.0, "bf16", "five_percent"),
    configs.Workload("one_block", 1, 100, 5, 2, 64, 128, 0.5, 0.5, "bf16", "five_percent"),
    configs.Workload("b64_odd_tail", 3, 777, 5, 2, 64, 64, 0.7, 0.0, "bf16", "five_percent"),
    configs.Workload("dense_rho0", 2, 300, 5, 2, 64, 64, 0.0, 0.0, "bf16", "five_percent"),
    configs.Workload("f32_ragged", 3, 37, 4, 2, 64, 10, 0.6, 0.3, "f32", "tiny"),
    configs.Workload("f32_no_special", 2, 40, 0, 2, 64, 16, 0.5, 0.5, "f32", "tiny"),
    # a last block of one token, and a block count just above a multiple of 32
    configs.Workload("tail1_b64", 3, 43, 5, 2, 64, 64, 0.5, 0.0, "bf16", "five_percent"),
    configs.Workload("tail1_b128", 1, 129, 5, 2, 64, 128, 0.5, 0.0, "bf16", "five_percent"),
    configs.Workload("b33_blocks", 3, 703, 5, 2, 64, 64, 0.6, 0.0, "bf16", "five_percent"),
    configs.Workload("f32_tail1", 3, 11, 4, 2, 64, 16, 0.5, 0.3, "f32", "tiny"),
    # an odd number of (query tile, head) items at b = 128 (the fused kernel pairs them), with
    # uneven kept counts between the rows of a pair
    configs.Workload("odd_items_b128", 3, 777, 5, 3, 64, 128, 0.5, 0.5, "bf16", "five_percent"),
    # more than 32 heads: the attention kernels keep the plain head order (no work ranking)
    configs.Workload("many_heads_b128", 1, 300, 5, 40, 64, 128, 0.5, 0.0, "bf16", "five_percent"),
    configs.Workload("many_heads_b64", 1, 300, 5, 40, 64, 64, 0.5, 0.5, "bf16", "five_percent"),
]


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_edge_cases(w):
    x = inputs(w)
    res = run_gpu(w, x)
    assert res["status"] == 0
    lay, PQ, PK, kh, om = _oracle_mask(w, x, res)
    assert compare_mask(om, res["selected"], w.tau).ok
    Q, K, V = (exact(a, w.dtype).astype(np.float64) for a in (x.q, x.k, x.v))
    if w.name == "empty_lists":
        assert res["kv_cnt"].max() == 0
        assert np.all(res["lse_pp"] == -np.inf) and np.all(res["o_pp"] == 0)
    if w.name == "dense_rho0":
        assert res["selected"].all()
    ref = oracle.layer_forward(Q, K, V, lay, res["selected"])
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    for key in ("out", "out_fused"):
        if res[key] is not None:
            assert rel_l2(res[key], ref) <= tol[0] and max_abs(res[key], ref) <= tol[1], key


def test_out_of_range_block_index_is_reported_not_faulted():
    w = configs.VGGT518.with_(name="tamper", frames=2, heads=2)
    x = inputs(w)

    def tamper(L):
        import torch
        L.buf.kv_idx[0, 0, 0] = 30000          # >= B: must be skipped and reported
        torch.cuda.synchronize()

    res = run_gpu(w, x, tamper=tamper)
    assert res["status"] == 5                   # BSA_ERR_DEVICE_BOUNDS
    assert np.isfinite(res["out"]).all()


def test_deterministic():
    w = SMALL_BF16[0]
    x = inputs(w)
    a, b = run_gpu(w, x), run_gpu(w, x)
    assert np.array_equal(a["selected"], b["selected"])
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["out_fused"], b["out_fused"])


def test_v_beyond_fp16_range_is_reported():
    """V is the fp16 operand of the P.V product: a bf16 V element of magnitude >= 65536 is
    reported as BSA_ERR_RANGE by every packing path; the largest bf16 magnitude below it
    (65280) packs exactly and the layer still matches the oracle."""
    import torch
    from view_transformers_b200 import _lib, layer, synth

    w = configs.VGGT518.with_(name="v_range", frames=2, heads=2, tau=0.0)
    x = inputs(w)
    lay = oracle_layout(w)
    for big, want in ((1.0e5, _lib.BSA_ERR_RANGE), (65280.0, 0)):
        v_st = x.v.copy()
        v_st[7, 1, 3] = synth.f64_to_bf16_bits(np.array([big]))[0]
        v_st[800, 0, 60] = synth.f64_to_bf16_bits(np.array([-big]))[0]
        L = layer.BlockSparseLayer.for_workload(w)
        q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, v_st))
        out = L.forward(q, k, v).float().cpu().numpy()          # one-pass pack + pool
        assert L.check_status() == want
        L.attend(q, k, v)                                       # separate packing pass
        assert L.check_status() == want
        o2 = torch.empty_like(L.buf.out)
        _lib.bsa_attention_noalloc(L.layout, q.data_ptr(), k.data_ptr(), v.data_ptr(), L.buf.kv_idx.data_ptr(),
                                   L.buf.kv_cnt.data_ptr(), o2.data_ptr(), L.buf.status.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
        assert L.check_status() == want
        if want == 0:
            Q, K, V = (exact(a, w.dtype).astype(np.float64) for a in (x.q, x.k, v_st))
            ref = oracle.layer_forward(Q, K, V, lay, L.selected())
            assert np.isfinite(out).all() and rel_l2(out, ref) <= BF16_TOL[0]
