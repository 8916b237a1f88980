"""Plain fp64 CPU oracle of the steps on either side of the global-attention layer (test
infrastructure only; only the tests, the package smoke check and the benchmark's CPU leg
import it, and it imports nothing from the CUDA package).

The pages place the global attention inside an aggregator that alternates frame-wise and
global attention blocks, each a multi-head self-attention with its projections
("Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers", 研究背景与动机:
the VGGT aggregator; "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
Transformers", 图2: local and global attention modules, each multi-head attention plus a
feed-forward network). These are the steps written here:

  * linear        y = x W^T + b (the QKV and output projections);
  * qkv_project   the QKV projection of C = H d channels into 3C, split as [Q | K | V], each
                  C wide with channel c = h d + e (head h, dimension e);
  * out_project   the heads concatenated back to C channels, then the output projection;
  * frame_attention
                  dense softmax attention (Eq. (1) of the first page) of every token over the
                  T tokens of its own frame, special tokens included.

Readings (the pages print no projection code): the split [Q | K | V] with head-major channels
is the usual multi-head layout; weights are stored [out features, in features].
"""
from __future__ import annotations

import numpy as np

from .bsa_oracle import attend


def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """x [N, Cin] @ w[Cout, Cin]^T + b[Cout], in float64."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    return y if b is None else y + np.asarray(b, dtype=np.float64)[None, :]


def qkv_project(x, w_qkv, b_qkv, heads: int, head_dim: int):
    """Q, K, V [N, H, d] from x [N, C] with w_qkv [3C, C] and b_qkv [3C]."""
    C = heads * head_dim
    y = linear(x, w_qkv, b_qkv)
    N = y.shape[0]
    return tuple(y[:, t * C:(t + 1) * C].reshape(N, heads, head_dim) for t in range(3))


def out_project(o, w_o, b_o):
    """o [N, H, d] -> heads concatenated to [N, C] -> o W_o^T + b_o."""
    N = o.shape[0]
    return linear(np.asarray(o).reshape(N, -1), w_o, b_o)


def frame_attention(Q, K, V, frames: int, tokens_per_frame: int):
    """Every token attends over the T tokens of its frame, per head. Q, K, V [F T, H, d]."""
    N, H, d = Q.shape
    T = tokens_per_frame
    out = np.empty((N, H, d))
    for f in range(frames):
        rows = slice(f * T, (f + 1) * T)
        for h in range(H):
            out[rows, h], _ = attend(np.asarray(Q[rows, h], dtype=np.float64),
                                     np.asarray(K[rows, h], dtype=np.float64),
                                     np.asarray(V[rows, h], dtype=np.float64))
    return out


def frame_attention_rows(Q, K, V, tokens_per_frame: int, rows, heads):
    """frame_attention at the (row, head) pairs only; returns [len(rows), d]."""
    T = tokens_per_frame
    out = np.empty((len(rows), Q.shape[2]))
    for a, (r, h) in enumerate(zip(np.asarray(rows), np.asarray(heads))):
        f = int(r) // T
        keys = slice(f * T, (f + 1) * T)
        o, _ = attend(np.asarray(Q[r:r + 1, h], dtype=np.float64), np.asarray(K[keys, h], dtype=np.float64),
                      np.asarray(V[keys, h], dtype=np.float64))
        out[a] = o[0]
    return out
