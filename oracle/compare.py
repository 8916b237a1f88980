"""Acceptance rules for comparing a device result with the oracle (test infrastructure only).

Mask rule (block mask of the dual threshold, "Block-Sparse Global Attention for
Efficient Multi-View Geometry Transformers", 关键设计 2): a device row matches the
oracle row when the selected sets are equal, or when every difference is explained
by floating-point near-ties of the oracle's own fp64 values:
  * the counts differ by at most one, and when they differ the oracle's cumulative
    mass at the smaller count lies within `eps` of tau (the CDF crossing moved);
  * every block in the symmetric difference between the device set and the oracle's
    top-n_device prefix has an oracle probability within `eps` of the oracle's
    probability at rank n_device (a near-tie at the cut).
Output rule: relative L2 over the tensor, max-abs, and per-head NMSE
E = ||O_ref - O||^2 / ||O_ref||^2 (the error measure of "SAF3R: Dynamic Sparse
Attention for Feed-Forward 3D Reconstruction Transformers", 离线头分析).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass
class MaskReport:
    rows: int = 0
    exact: int = 0
    exempt: int = 0
    failed: int = 0
    failures: list = field(default_factory=list)

    @property
    def ok(self) -> bool:
        return self.failed == 0


def compare_mask(oracle_mask, device_selected: np.ndarray, tau: float, eps: float = 1e-6,
                 rows=None, max_failures: int = 10) -> MaskReport:
    """oracle_mask: MaskResult; device_selected: bool [H, B, B] (or [H, R, B] for `rows`)."""
    probs, order, cum, count = oracle_mask.probs, oracle_mask.order, oracle_mask.cum, oracle_mask.count
    sel_o = oracle_mask.selected
    if rows is not None:
        probs, order, cum, count, sel_o = (probs[:, rows], order[:, rows], cum[:, rows],
                                           count[:, rows], sel_o[:, rows])
    rep = MaskReport()
    H, R, B = sel_o.shape
    rep.rows = H * R
    same = np.all(sel_o == device_selected, axis=2)
    rep.exact = int(same.sum())
    for h, i in zip(*np.nonzero(~same)):
        dev = device_selected[h, i]
        n_g = int(dev.sum())
        n_o = int(count[h, i])
        ok = True
        if n_g != n_o:
            m = min(n_g, n_o)
            c_m = 0.0 if m == 0 else float(cum[h, i, m - 1])
            ok = abs(n_g - n_o) == 1 and abs(c_m - tau) < eps
        if ok and n_g > 0:
            ref = np.zeros(B, dtype=bool)
            ref[order[h, i, :n_g]] = True
            diff = np.nonzero(ref ^ dev)[0]
            thr = probs[h, i, order[h, i, n_g - 1]]
            ok = bool(np.all(np.abs(probs[h, i, diff] - thr) < eps))
        if ok:
            rep.exempt += 1
        else:
            rep.failed += 1
            if len(rep.failures) < max_failures:
                rep.failures.append((int(h), int(i), n_o, n_g))
    return rep


def rel_l2(x: np.ndarray, ref: np.ndarray) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_abs(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(np.asarray(x, dtype=np.float64) - ref))) if np.size(ref) else 0.0


def nmse_per_head(x: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """x, ref: [rows, H, d]."""
    x = np.asarray(x, dtype=np.float64)
    num = ((x - ref) ** 2).sum(axis=(0, 2))
    den = (ref ** 2).sum(axis=(0, 2))
    return num / np.maximum(den, 1e-300)


def compare_probe(scores: np.ndarray, scale: np.ndarray, k_per_head, device_selected: np.ndarray,
                  rel: float = 2e-5) -> MaskReport:
    """Query-probe Top-K rule ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D
    Reconstruction Transformers", 四、1. and 四、3.): per head, the device keeps k_h blocks, and
    every block where it differs from the oracle's fp64 top-k has an oracle score within
    rel * (scale_j + scale_cut) of the oracle's k-th score, where scale_j bounds the size of
    the terms of block j's score (sum_d |q_bar_d| |P_b(K)_jd| / sqrt(d)).
    scores, scale: [H, B]; device_selected: [H, B] bool (one row per head)."""
    rep = MaskReport()
    H, B = scores.shape
    rep.rows = H
    for h in range(H):
        k = min(int(k_per_head[h]), B)
        order = np.argsort(-scores[h], kind="stable")
        ref = np.zeros(B, dtype=bool)
        ref[order[:k]] = True
        dev = device_selected[h]
        if np.array_equal(ref, dev):
            rep.exact += 1
            continue
        ok = int(dev.sum()) == k and k > 0
        if ok:
            cut = order[k - 1]
            diff = np.nonzero(ref ^ dev)[0]
            ok = bool(np.all(np.abs(scores[h, diff] - scores[h, cut]) <= rel * (scale[h, diff] + scale[h, cut])))
        if ok:
            rep.exempt += 1
        else:
            rep.failed += 1
            rep.failures.append((h, k, int(dev.sum())))
    return rep
