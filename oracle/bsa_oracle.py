"""Plain fp64 CPU oracle of the block-sparse global attention layer.

TEST INFRASTRUCTURE ONLY. Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module. It imports nothing from the
CUDA package, and the CUDA package never imports it.

Every step is written the plain way, in float64, with numpy's matmul, sort and
sum as the only library primitives, and follows these pages:

  [BSGA] "Block-Sparse Global Attention for Efficient Multi-View Geometry
         Transformers" (CVPR 2026 paper notes):
           - 方法详解 / 整体框架, flowchart: split special tokens from patch tokens,
             predict the block mask on the patch tokens, block-sparse attention on
             the selected blocks, dense attention for the special tokens, merge.
           - 关键设计 1: average pooling P_b of Q and K by block size b,
             S = P_b(Q) P_b(K)^T followed by softmax; Eq. (1) dense attention;
             Eq. (2) attention under a binary block mask M.
           - 关键设计 2: Top-K + CDF dual threshold, k = floor(B (1 - rho)).
           - 关键设计 3: 1 camera + 4 register tokens per frame stay dense
             (self attention and both cross directions with the patch tokens).
  [HeSS] "HeSS: Head Sensitivity Score for Sparsity Redistribution in VGGT",
         提案手法: the layer's attention budget is redistributed across heads in
         proportion to the head scores with an iterative capping procedure.

Readings taken where the pages are silent (each is tested):
  * special tokens are the first S tokens of each frame;
  * blocks are runs of b consecutive tokens of the concatenated patch sequence
    (they may straddle frames); the last block is the mean over its real count;
  * the pooled scores carry the 1/sqrt(d) of Eq. (1) (the page prints none);
  * masked entries of Eq. (2) are excluded from the softmax (-inf), since only the
    selected blocks are computed;
  * ties in the block ranking go to the lower block index;
  * k = floor(B (1 - rho) + 1e-9) in fp64 (1e-9 absorbs the rounding of 1 - rho);
    with per-head densities k_h = clamp(floor(B d_h + 1e-9), 1, B);
  * the merge is one softmax over {special keys} U {selected patch keys}; the
    partial results combine exactly through their log-sum-exp values.
"""
from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np

TIE_EPS = 1e-9


@dataclass(frozen=True)
class Layout:
    frames: int            # F
    tokens_per_frame: int  # T = P + S
    special_per_frame: int  # S
    heads: int             # H
    head_dim: int          # d
    block: int             # b

    @property
    def P(self) -> int:
        return self.tokens_per_frame - self.special_per_frame

    @property
    def N(self) -> int:
        return self.frames * self.tokens_per_frame

    @property
    def Np(self) -> int:
        return self.frames * self.P

    @property
    def Ns(self) -> int:
        return self.frames * self.special_per_frame

    @property
    def B(self) -> int:
        return -(-self.Np // self.block)


# ----------------------------------------------------------------------------- inputs

def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage bits -> float64 exactly. bf16 is the top half of an IEEE fp32."""
    if dtype == "bf16":
        bits = np.asarray(a, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------- token split

def special_rows(lay: Layout) -> np.ndarray:
    """Rows of the special tokens X_s: the first S tokens of every frame [BSGA 关键设计 3]."""
    f = np.repeat(np.arange(lay.frames), lay.special_per_frame)
    s = np.tile(np.arange(lay.special_per_frame), lay.frames)
    return f * lay.tokens_per_frame + s


def patch_rows(lay: Layout) -> np.ndarray:
    """Row of patch token p (0 <= p < Np) of the concatenated patch sequence X_p."""
    p = np.arange(lay.Np)
    return (p // lay.P) * lay.tokens_per_frame + lay.special_per_frame + (p % lay.P)


def block_bounds(lay: Layout, j: int) -> tuple[int, int]:
    """Patch index range [lo, hi) of block j."""
    lo = j * lay.block
    return lo, min(lo + lay.block, lay.Np)


# ----------------------------------------------------------------------------- mask prediction

def pool(X: np.ndarray, lay: Layout) -> np.ndarray:
    """P_b(X): mean of each block of b consecutive patch tokens, per head [BSGA 关键设计 1].

    X is [N, H, d] holding exact values (float32 or float64); sums are taken in float64.
    Returns [H, B, d] float64.
    """
    Xp = X[patch_rows(lay)]
    out = np.zeros((lay.heads, lay.B, lay.head_dim))
    for j in range(lay.B):
        lo, hi = block_bounds(lay, j)
        out[:, j, :] = Xp[lo:hi].sum(axis=0, dtype=np.float64) / (hi - lo)
    return out


def pooled_probs(PQ: np.ndarray, PK: np.ndarray, head_dim: int) -> np.ndarray:
    """softmax_j( P_b(Q)_i . P_b(K)_j / sqrt(d) ) per head and row i [BSGA 关键设计 1]."""
    s = np.einsum("hid,hjd->hij", PQ, PK) / math.sqrt(head_dim)
    s = s - s.max(axis=2, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=2, keepdims=True)


def k_from_rho(B: int, rho: float) -> int:
    """Top-K floor k = floor(B (1 - rho)) [BSGA 关键设计 2]."""
    return int(math.floor(B * (1.0 - rho) + TIE_EPS))


def k_from_density(B: int, density: float) -> int:
    """Per-head block budget from a per-head density [HeSS 提案手法]."""
    return int(min(B, max(1, math.floor(B * density + TIE_EPS))))


def water_fill(scores: np.ndarray, total: float, cap: float = 1.0) -> np.ndarray:
    """Iterative capped redistribution of a layer budget across heads [HeSS 提案手法].

    density_h = (total - cap * #capped) * s_h / sum_{uncapped} s, repeated after
    capping every head whose density exceeds `cap`, until no new head is capped.
    """
    s = np.asarray(scores, dtype=np.float64)
    H = s.shape[0]
    if not (0.0 <= total <= H * cap + 1e-12) or np.any(s <= 0):
        raise ValueError("need 0 <= total <= H*cap and positive scores")
    density = np.zeros(H)
    capped = np.zeros(H, dtype=bool)
    for _ in range(H + 1):
        free = ~capped
        density[capped] = cap
        if not free.any():
            break
        remaining = total - cap * capped.sum()
        density[free] = remaining * s[free] / s[free].sum()
        newly = free & (density > cap)
        if not newly.any():
            break
        capped |= newly
    return density


@dataclass
class MaskResult:
    probs: np.ndarray     # [H, B, B] pooled block probabilities
    order: np.ndarray     # [H, B, B] blocks sorted by (p desc, index asc)
    cum: np.ndarray       # [H, B, B] prefix sums of the sorted probabilities
    count: np.ndarray     # [H, B]    number of selected blocks n
    selected: np.ndarray  # [H, B, B] bool block mask M


def select(probs_row_major: np.ndarray, k: int, tau: float):
    """Dual threshold on one head's rows [BSGA 关键设计 2].

    Rank blocks by probability (descending; ties to the lower index), take the
    cumulative sum C(n) and keep the first n = min(B, max(k, n_tau)) blocks, where
    n_tau is the smallest n >= 1 with C(n) >= tau (0 when tau <= 0, B when the sum
    never reaches tau). The top-k set and the CDF set are both prefixes of the same
    ranking, so their union is the longer prefix.
    """
    p = probs_row_major
    B = p.shape[-1]
    order = np.argsort(-p, axis=-1, kind="stable")
    cum = np.cumsum(np.take_along_axis(p, order, axis=-1), axis=-1)
    if tau <= 0.0:
        n_tau = np.zeros(p.shape[:-1], dtype=np.int64)
    else:
        reach = cum >= tau
        n_tau = np.where(reach.any(axis=-1), reach.argmax(axis=-1) + 1, B)
    count = np.minimum(B, np.maximum(k, n_tau))
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.arange(B)[None, :].repeat(p.shape[0], 0), axis=-1)
    selected = rank < count[:, None]
    return order, cum, count, selected


def predict_mask(PQ: np.ndarray, PK: np.ndarray, head_dim: int, k_per_head, tau: float) -> MaskResult:
    probs = pooled_probs(PQ, PK, head_dim)
    H, B, _ = probs.shape
    order = np.empty((H, B, B), dtype=np.int64)
    cum = np.empty((H, B, B))
    count = np.empty((H, B), dtype=np.int64)
    selected = np.empty((H, B, B), dtype=bool)
    for h in range(H):
        order[h], cum[h], count[h], selected[h] = select(probs[h], int(k_per_head[h]), tau)
    return MaskResult(probs, order, cum, count, selected)


def head_k(lay: Layout, rho: float, density=None) -> np.ndarray:
    if density is None:
        return np.full(lay.heads, k_from_rho(lay.B, rho), dtype=np.int64)
    return np.array([k_from_density(lay.B, float(x)) for x in density], dtype=np.int64)


# ----------------------------------------------------------------------------- attention

def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """softmax(q k^T / sqrt(d)) v for a set of query rows over a set of keys [BSGA Eq. (1)].

    Returns (output [M, d], natural-log log-sum-exp of the scaled scores [M]).
    """
    d = q.shape[-1]
    s = q @ k.T / math.sqrt(d)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1)
    return (e @ v) / l[:, None], m[:, 0] + np.log(l)


def patch_keys_of(lay: Layout, selected_row: np.ndarray) -> np.ndarray:
    """Rows of the patch tokens in the selected key blocks of one query block."""
    pr = patch_rows(lay)
    return np.concatenate([pr[slice(*block_bounds(lay, j))] for j in np.nonzero(selected_row)[0]]
                          or [np.zeros(0, dtype=np.int64)])


def layer_forward(Q, K, V, lay: Layout, selected: np.ndarray, heads=None, qblocks=None,
                  special_chunk: int = 512):
    """Full layer output [N, H, d] under the block mask [BSGA Eq. (2), 关键设计 3, flowchart].

    Special query rows attend densely over all N keys. Patch query rows of block i
    attend over every special key and the patch keys of the blocks selected for
    (head, i); all other keys are excluded. `heads` / `qblocks` restrict the work
    (rows not computed stay NaN).
    """
    out = np.full((lay.N, lay.heads, lay.head_dim), np.nan)
    sr = special_rows(lay)
    pr = patch_rows(lay)
    heads = range(lay.heads) if heads is None else heads
    for h in heads:
        for c in range(0, len(sr), special_chunk):
            rows = sr[c:c + special_chunk]
            out[rows, h], _ = attend(Q[rows, h], K[:, h], V[:, h])
        for i in (range(lay.B) if qblocks is None else qblocks):
            rows = pr[slice(*block_bounds(lay, i))]
            keys = np.concatenate([sr, patch_keys_of(lay, selected[h, i])])
            out[rows, h], _ = attend(Q[rows, h], K[keys, h], V[keys, h])
    return out


def allowed_keys(lay: Layout, selected: np.ndarray, h: int, row: int) -> np.ndarray:
    """Token-level key mask [N] of query row `row` in head h: every key for a special
    query; the special keys plus the patch keys of the kept blocks for a patch query."""
    T, S = lay.tokens_per_frame, lay.special_per_frame
    token = np.arange(lay.N)
    is_special = (token % T) < S
    if (row % T) < S:
        return np.ones(lay.N, dtype=bool)
    patch_index = (token // T) * lay.P + (token % T) - S          # valid where not special
    i = ((row // T) * lay.P + (row % T) - S) // lay.block
    kept = np.zeros(lay.N, dtype=bool)
    kept[~is_special] = selected[h, i][patch_index[~is_special] // lay.block]
    return is_special | kept


def layer_rows(Q, K, V, lay: Layout, selected: np.ndarray, rows, heads, chunk: int = 32):
    """Layer output for the (row, head) pairs only: the same keys as layer_forward, with
    excluded keys removed from the softmax. Q, K, V hold exact values (float32/float64);
    returns [len(rows), d] float64."""
    rows = np.asarray(rows)
    heads = np.asarray(heads)
    out = np.empty((len(rows), lay.head_dim))
    for h in np.unique(heads):
        sel_pairs = np.nonzero(heads == h)[0]
        Kh = K[:, h, :].astype(np.float64)
        Vh = V[:, h, :].astype(np.float64)
        for c in range(0, len(sel_pairs), chunk):
            idx = sel_pairs[c:c + chunk]
            q = Q[rows[idx], h, :].astype(np.float64)
            s = q @ Kh.T / math.sqrt(lay.head_dim)
            for a, r in enumerate(rows[idx]):
                s[a, ~allowed_keys(lay, selected, int(h), int(r))] = -np.inf
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            out[idx] = (e @ Vh) / e.sum(axis=1)[:, None]
    return out


def partials(Q, K, V, lay: Layout, selected: np.ndarray, heads=None):
    """Per patch row: (O_pp, lse_pp) over the selected patch keys and (O_ps, lse_ps)
    over the special keys, laid out [Np, H, d] and [H, Np]."""
    Np, H, d = lay.Np, lay.heads, lay.head_dim
    o_pp = np.full((Np, H, d), np.nan)
    o_ps = np.full((Np, H, d), np.nan)
    lse_pp = np.full((H, Np), np.nan)
    lse_ps = np.full((H, Np), np.nan)
    sr = special_rows(lay)
    pr = patch_rows(lay)
    for h in (range(H) if heads is None else heads):
        for i in range(lay.B):
            lo, hi = block_bounds(lay, i)
            rows = pr[lo:hi]
            keys = patch_keys_of(lay, selected[h, i])
            o_pp[lo:hi, h], lse_pp[h, lo:hi] = attend(Q[rows, h], K[keys, h], V[keys, h])
            o_ps[lo:hi, h], lse_ps[h, lo:hi] = attend(Q[rows, h], K[sr, h], V[sr, h])
    return o_pp, lse_pp, o_ps, lse_ps


def merge(o_a, lse_a, o_b, lse_b):
    """Exact combination of two softmax-normalised partial outputs over disjoint key sets:
    L = log(e^lse_a + e^lse_b); o = e^(lse_a - L) o_a + e^(lse_b - L) o_b.
    o_* are [rows, H, d], lse_* are [H, rows]."""
    L = np.logaddexp(lse_a, lse_b)
    wa = np.exp(lse_a - L).T[:, :, None]
    wb = np.exp(lse_b - L).T[:, :, None]
    return wa * o_a + wb * o_b, L


# ----------------------------------------------------------------------------- whole layer

@dataclass
class LayerResult:
    k: np.ndarray
    density: np.ndarray | None
    PQ: np.ndarray
    PK: np.ndarray
    mask: MaskResult
    out: np.ndarray | None


def run_layer(q_store, k_store, v_store, dtype: str, lay: Layout, rho: float, tau: float,
              scores=None, cap: float = 1.0, compute_output: bool = True) -> LayerResult:
    """Pool -> pooled softmax -> dual threshold -> masked attention with the dense
    special path, from storage arrays (bf16 bits or float32)."""
    Q, K, V = to_f64(q_store, dtype), to_f64(k_store, dtype), to_f64(v_store, dtype)
    density = None
    if scores is not None:
        density = water_fill(scores, lay.heads * (1.0 - rho), cap)
    kh = head_k(lay, rho, density)
    PQ, PK = pool(Q, lay), pool(K, lay)
    mask = predict_mask(PQ, PK, lay.head_dim, kh, tau)
    out = layer_forward(Q, K, V, lay, mask.selected) if compute_output else None
    return LayerResult(kh, density, PQ, PK, mask, out)
