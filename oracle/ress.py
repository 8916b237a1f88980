"""Plain fp64 CPU oracle of drift-score block selection (test infrastructure only; only the
tests, the package smoke check and the benchmark's CPU leg import it, and it imports nothing
from the CUDA package).

"ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers" (摘要, 技术框架,
关键设计) selects blocks by the drift that dropping them leaves in the attention output (the
residual stream), not by their attention mass: a drift score per block, and an iterative
residual restoration that refines the whole drop set, because the drift of a set depends on
the directions of the blocks' contribution vectors. The page prints no formula. Reading taken
here, at the pooled resolution of the block-mask predictor of "Block-Sparse Global Attention
for Efficient Multi-View Geometry Transformers" (关键设计 1), per head h and query block i:

  * p_j   = the pooled block probabilities softmax_j(P_b(Q)_i . P_b(K)_j / sqrt(d));
  * o     = sum_j p_j P_b(V)_j, the pooled attention output (P_b(V) = block means of V);
  * delta_j = p_j (o - P_b(V)_j), block j's drift vector: dropping a set D and renormalising
    the softmax over the kept blocks moves the output by exactly
        o(kept) - o = (sum_{j in D} delta_j) / (1 - sum_{j in D} p_j),
    so drift(D) = |sum_{j in D} delta_j| / (1 - sum_{j in D} p_j) (Euclidean norm);
  * start: keep the k blocks of largest |delta_j| (ties to the lower index), drop the rest;
  * restoration rounds (at most `rounds`): restore the dropped block l whose removal from D
    gives the smallest drift, then drop the kept block m whose addition gives the smallest
    drift; keep the swap if the drift of the new set is below the old one (ties to the lower
    index), else stop.

k is the layer's k_h (k = floor(B (1 - rho)), or the per-head budget), as for the other
selectors. The decisions are taken in float64 on both sides.
"""
from __future__ import annotations

import numpy as np

from .bsa_oracle import pooled_probs


def drift_vectors(p_row: np.ndarray, pv: np.ndarray):
    """(o [d], delta [B, d]) of one row: p_row [B] pooled probabilities, pv [B, d] pooled V."""
    o = p_row @ pv
    return o, p_row[:, None] * (o[None, :] - pv)


def drift(delta: np.ndarray, p_row: np.ndarray, dropped: np.ndarray) -> float:
    """|sum_{j in D} delta_j| / (1 - sum_{j in D} p_j) for the bool drop mask D."""
    mass = float(p_row[dropped].sum())
    if mass >= 1.0:
        return float("inf")
    return float(np.linalg.norm(delta[dropped].sum(axis=0))) / (1.0 - mass)


def _gap(vals) -> float:
    """Relative gap between the smallest and the second-smallest value (inf if fewer than 2)."""
    v = np.sort(np.asarray(vals, dtype=np.float64))
    if len(v) < 2 or not np.isfinite(v[1]):
        return float("inf")
    return float((v[1] - v[0]) / max(abs(v[0]), abs(v[1]), 1e-300))


def select_row(p_row: np.ndarray, pv: np.ndarray, k: int, rounds: int, margins: list | None = None):
    """Kept-block mask [B] of one row and the number of swaps taken. When `margins` is a list,
    the relative gap of every decision is appended to it (the start cut, each argmin, each
    keep-or-undo comparison), so that a comparison with another evaluation can tell a
    rounding-level tie from a real difference."""
    B = len(p_row)
    k = min(max(k, 0), B)
    _, delta = drift_vectors(p_row, pv)
    norm = np.sqrt((delta * delta).sum(axis=1))
    order = np.lexsort((np.arange(B), -norm))           # |delta| descending, index ascending
    kept = np.zeros(B, dtype=bool)
    kept[order[:k]] = True
    if margins is not None and 0 < k < B:
        margins.append(_gap([-norm[order[k - 1]], -norm[order[k]]]))
    if k == 0 or k == B:
        return kept, 0
    swaps = 0
    for _ in range(rounds):
        cur = drift(delta, p_row, ~kept)
        # restore the dropped block whose return lowers the drift most
        cand = np.nonzero(~kept)[0]
        vals = [drift(delta, p_row, (~kept) & (np.arange(B) != l)) for l in cand]
        if margins is not None:
            margins.append(_gap(vals))
        l = int(cand[int(np.argmin(vals))])
        kept[l] = True
        # drop the kept block whose removal raises it least
        cand = np.nonzero(kept & (np.arange(B) != l))[0]
        vals = [drift(delta, p_row, (~kept) | (np.arange(B) == m)) for m in cand]
        if margins is not None:
            margins.append(_gap(vals))
        m = int(cand[int(np.argmin(vals))])
        new = min(vals)
        if margins is not None:
            margins.append(_gap([new, cur]))
        if new < cur:
            kept[m] = False
            swaps += 1
        else:
            kept[l] = False
            break
    return kept, swaps


def ress_mask(PQ: np.ndarray, PK: np.ndarray, PV: np.ndarray, head_dim: int, k_per_head, rounds: int):
    """Kept-block mask [H, B, B] from pooled Q, K, V [H, B, d] (float64 values)."""
    probs = pooled_probs(PQ, PK, head_dim)
    H, B, _ = probs.shape
    out = np.zeros((H, B, B), dtype=bool)
    for h in range(H):
        for i in range(B):
            out[h, i], _ = select_row(probs[h, i], PV[h], int(k_per_head[h]), rounds)
    return out
