"""Plain fp64 / integer CPU oracle of the alternative block selectors (test infrastructure only).

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the package smoke
check and the benchmark's CPU-baseline leg import it, and it imports nothing from the CUDA
package.

Each selector emits, per head h and patch query block i, the set of kept patch key blocks
(bool [H, B, B]) that the same block-sparse attention then computes:

  * random        -- "Block-Sparse Global Attention for Efficient Multi-View Geometry
                     Transformers", 消融实验 (图 10), rows "Random" / "Random w/ dense
                     special": k_h blocks per row drawn uniformly without replacement.
  * CDF only      -- same page and table, row "CDF only": the dual threshold with no Top-K
                     floor (rho = 1, so k = 0); it needs no code of its own (bsa_oracle.select).
  * uniform       -- "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
                     Transformers", 四、1. 均匀采样核 (scanning heads): keys kept at a fixed
                     stride, the same for every query.
  * query probe   -- same page, 四、1. Query-Probe Top-K 核 and 四、3. (its acceleration): keys
                     ranked by the scores of the mean query q_bar, q_bar K^T / sqrt(D), which
                     equal the column means of Q K^T / sqrt(D); the top K are kept for every
                     query.

Readings taken where the pages are silent (each is tested):
  * the SAF3R selectors act on the patch key blocks of the layer (the special keys stay
    dense), so that their lists feed the same block-sparse kernel; a block's probe score is
    the mean of its keys' probe scores, q_bar . P_b(K)_j / sqrt(d);
  * q_bar is the mean of the patch queries (the queries whose keys are being selected);
  * the number of probe blocks per head is the layer's k_h (k = floor(B (1 - rho)), or the
    per-head budget), ties to the lower block index;
  * uniform sampling keeps blocks j = 0, s, 2s, ... for a stride s >= 1;
  * the random draw is keyed by a counter-based generator, Philox4x32-10 (Salmon, Moraes,
    Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): for block j of
    row (h, i) the 32-bit key is word 0 of Philox4x32-10 with counter (j, i, h, 0) and key
    (seed mod 2^32, seed >> 32); a row keeps the k_h blocks with the smallest (key, j),
    which is a uniformly random k_h-subset.
"""
from __future__ import annotations

import math

import numpy as np

from .bsa_oracle import Layout, patch_rows

# Philox4x32 constants as published with the generator: round multipliers and the Weyl
# increments of the key schedule.
PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds on numpy arrays of counters (any broadcastable shapes,
    values < 2^32). One round maps (c0, c1, c2, c3) under key (k0, k1) to
    (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the key gains the
    Weyl increments between rounds. Returns the four output words as uint64 arrays."""
    c = [np.asarray(x, dtype=np.uint64) & _U32 for x in (c0, c1, c2, c3)]
    k = [np.asarray(k0, dtype=np.uint64) & _U32, np.asarray(k1, dtype=np.uint64) & _U32]
    for r in range(10):
        if r:
            k = [(k[0] + np.uint64(PHILOX_W0)) & _U32, (k[1] + np.uint64(PHILOX_W1)) & _U32]
        p0 = np.uint64(PHILOX_M0) * c[0]          # < 2^64: exact in uint64
        p1 = np.uint64(PHILOX_M1) * c[2]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ k[0], p1 & _U32, (p0 >> np.uint64(32)) ^ c[3] ^ k[1], p0 & _U32]
    return c


def random_keys(lay: Layout, seed: int) -> np.ndarray:
    """uint32 key [H, B, B] of every (head, query block, key block)."""
    H, B = lay.heads, lay.B
    h, i, j = np.meshgrid(np.arange(H), np.arange(B), np.arange(B), indexing="ij")
    seed = int(seed)
    return philox4x32_10(j, i, h, 0, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)[0]


def smallest_k(keys: np.ndarray, k_per_head) -> np.ndarray:
    """bool [H, R, B]: per row, the k_h entries with the smallest (key, index)."""
    H, R, B = keys.shape
    order = np.argsort(keys, axis=-1, kind="stable")       # stable: equal keys by index
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.broadcast_to(np.arange(B), keys.shape).copy(), axis=-1)
    k = np.minimum(np.asarray(k_per_head, dtype=np.int64), B)
    return rank < k[:, None, None]


def random_mask(lay: Layout, k_per_head, seed: int) -> np.ndarray:
    """Random block selection [BSGA 消融实验]: k_h uniformly random blocks per row."""
    return smallest_k(random_keys(lay, seed), k_per_head)


def uniform_mask(lay: Layout, stride: int) -> np.ndarray:
    """Fixed-stride uniform sampling [SAF3R 四、1.]: key blocks 0, s, 2s, ... for every row."""
    if stride < 1:
        raise ValueError("stride >= 1")
    keep = (np.arange(lay.B) % stride) == 0
    return np.broadcast_to(keep, (lay.heads, lay.B, lay.B)).copy()


def mean_query(Q: np.ndarray, lay: Layout) -> np.ndarray:
    """q_bar [H, d]: the mean of the patch query rows, in float64."""
    return Q[patch_rows(lay)].astype(np.float64).mean(axis=0)


def probe_key_scores(Q: np.ndarray, K: np.ndarray, lay: Layout) -> np.ndarray:
    """[H, Np]: q_bar . k_t / sqrt(d) for every patch key t [SAF3R 四、3.]."""
    qbar = mean_query(Q, lay)
    Kp = K[patch_rows(lay)].astype(np.float64)            # [Np, H, d]
    return np.einsum("hd,thd->ht", qbar, Kp) / math.sqrt(lay.head_dim)


def probe_block_scores(Q: np.ndarray, K: np.ndarray, lay: Layout) -> np.ndarray:
    """[H, B]: mean probe score of the keys of each patch block."""
    s = probe_key_scores(Q, K, lay)
    out = np.empty((lay.heads, lay.B))
    for j in range(lay.B):
        lo, hi = j * lay.block, min((j + 1) * lay.block, lay.Np)
        out[:, j] = s[:, lo:hi].mean(axis=1)
    return out


def probe_score_scale(Q: np.ndarray, K: np.ndarray, lay: Layout) -> np.ndarray:
    """[H, B]: sum_d |q_bar_d| |P_b(K)_jd| / sqrt(d), the size of the terms of each block's
    probe score (the conditioning of its floating-point evaluation)."""
    from .bsa_oracle import pool
    qbar = mean_query(Q, lay)
    return np.einsum("hd,hjd->hj", np.abs(qbar), np.abs(pool(K.astype(np.float64), lay))) / math.sqrt(lay.head_dim)


def probe_mask(Q: np.ndarray, K: np.ndarray, lay: Layout, k_per_head):
    """Query-probe Top-K [SAF3R 四、1., 四、3.]: per head, the k_h blocks of highest probe score
    (ties to the lower index), kept by every query block. Returns (scores [H, B], mask)."""
    s = probe_block_scores(Q, K, lay)
    sel = smallest_k(-s[:, None, :], k_per_head)[:, 0]    # [H, B]
    return s, np.broadcast_to(sel[:, None, :], (lay.heads, lay.B, lay.B)).copy()
