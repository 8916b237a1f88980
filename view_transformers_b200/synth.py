"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle's tests.

This module draws random numbers and rounds them to the storage dtype; it holds
none of the attention method's arithmetic. Both sides consume the exact bits it
returns.

Recipe (all draws in fp64, then rounded to the storage type with round-to-nearest-even):
  * Q, K, V ~ N(0, 1) i.i.d. over [F*T, H, d]. Tensor t in {Q:0, K:1, V:2}, frame f,
    is drawn from Generator(PCG64(SeedSequence([seed, t, f]))).standard_normal(T*H*d)
    in row-major [token, head, dim] order. Special tokens are ordinary N(0, 1).
  * "tiny" planting (planted cross-frame correspondences): for every frame f, with
    g = (f + 1) mod F and a permutation pi_f of the P patches,
    K[g, S + pi_f(i)] = Q[f, S + i] + 0.1 * eps for every head (eps fresh per
    row/head/dim).
  * "five_percent" planting: for every frame, n = round(0.05 P) distinct source
    patches; each gets a target (another frame uniformly, a patch uniformly, redrawn
    when that target was already used); K[target] = 3 * (Q[source] + 0.1 * eps), the
    same pairs for every head.
  * per-head sensitivity scores ~ LogNormal(0, 1), drawn from Generator(PCG64(seed)).
Planting draws come from Generator(PCG64(SeedSequence([seed, 99]))).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

from .configs import Workload

_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    sign = ((u >> np.uint64(63)).astype(np.uint16)) << np.uint16(15)
    mag = u & np.uint64(0x7FFFFFFFFFFFFFFF)
    lsb = (mag >> np.uint64(45)) & np.uint64(1)
    r = (mag + np.uint64((1 << 44) - 1) + lsb) >> np.uint64(45)   # exp11 << 7 | mant7
    e8 = (r >> np.uint64(7)).astype(np.int64) - 1023 + 127
    zero = mag == 0
    if np.any(((e8 < 1) | (e8 > 254)) & ~zero):
        raise ValueError("value outside the bfloat16 normal range")
    bits = (e8 << 7) | (r & np.uint64(0x7F)).astype(np.int64)
    bits = np.where(zero, 0, bits).astype(np.uint16)
    return bits | sign


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class LayerInputs:
    """Q, K, V as storage arrays of shape [F*T, H, d] (uint16 bf16 bits or float32)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    dtype: str
    scores: np.ndarray | None = None   # per-head sensitivity scores (fp64) or None


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _draw_tensor(w: Workload, name: str) -> np.ndarray:
    F, T, H, d = w.frames, w.tokens_per_frame, w.heads, w.head_dim
    tid = _TENSOR_ID[name]
    out = np.empty((F, T * H * d), dtype=np.uint16 if w.dtype == "bf16" else np.float32)

    def frame(f: int) -> None:
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, tid, f])))
        x = g.standard_normal(T * H * d)
        out[f] = f64_to_bf16_bits(x) if w.dtype == "bf16" else x.astype(np.float32)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(frame, range(F)))
    return out.reshape(F * T, H, d)


def _decode(a: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_to_f32(a).astype(np.float64) if dtype == "bf16" else a.astype(np.float64)


def _encode(x: np.ndarray, dtype: str) -> np.ndarray:
    return f64_to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float32)


def _plant(w: Workload, q: np.ndarray, k: np.ndarray) -> None:
    F, P, S, T, H, d = (w.frames, w.patch_per_frame, w.special_per_frame,
                        w.tokens_per_frame, w.heads, w.head_dim)
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, 99])))
    if w.planting == "tiny":
        for f in range(F):
            other = (f + 1) % F
            perm = g.permutation(P)
            src = f * T + S + np.arange(P)
            dst = other * T + S + perm
            eps = g.standard_normal((P, H, d))
            k[dst] = _encode(_decode(q[src], w.dtype) + 0.1 * eps, w.dtype)
    elif w.planting == "five_percent":
        if F < 2:
            return
        n = int(round(0.05 * P))
        used = set()
        for f in range(F):
            sources = g.choice(P, size=n, replace=False)
            for s in sources:
                while True:
                    tf = int(g.integers(0, F - 1))
                    tf = tf + 1 if tf >= f else tf          # uniform over the other frames
                    tp = int(g.integers(0, P))
                    if (tf, tp) not in used:
                        break
                used.add((tf, tp))
                eps = g.standard_normal((H, d))
                src_row = f * T + S + int(s)
                dst_row = tf * T + S + tp
                k[dst_row] = _encode(3.0 * (_decode(q[src_row], w.dtype) + 0.1 * eps), w.dtype)
    else:
        raise ValueError(f"unknown planting {w.planting!r}")


def head_scores(w: Workload) -> np.ndarray:
    """Per-head sensitivity scores ~ LogNormal(0, 1) (stand-in for calibrated HeSS)."""
    return np.random.Generator(np.random.PCG64(w.seed)).lognormal(0.0, 1.0, w.heads)


def make_inputs(w: Workload) -> LayerInputs:
    q = _draw_tensor(w, "q")
    k = _draw_tensor(w, "k")
    v = _draw_tensor(w, "v")
    _plant(w, q, k)
    return LayerInputs(q, k, v, w.dtype, head_scores(w) if w.head_budgets else None)


def decode(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array (bf16 bits or float32) -> float64, exactly."""
    return _decode(a, dtype)


@dataclass
class BlockInputs:
    """Synthetic inputs of one attention block: tokens x [N, C] and random-init projection
    weights (bf16 bits), biases fp32. W ~ N(0, 1/C) keeps the projected values near unit
    scale; biases ~ N(0, 0.02^2)."""
    x: np.ndarray        # uint16 [N, C]
    w_qkv: np.ndarray    # uint16 [3C, C]
    b_qkv: np.ndarray    # float32 [3C]
    w_o: np.ndarray      # uint16 [C, C]
    b_o: np.ndarray      # float32 [C]


def make_block_inputs(w: Workload) -> BlockInputs:
    """Drawn from Generator(PCG64(SeedSequence([seed, 10 + t]))) for t = x, w_qkv, b_qkv, w_o,
    b_o in that order, in fp64, then rounded (bf16 RNE, or fp32 for the biases)."""
    C = w.heads * w.head_dim
    N = w.n_tokens

    def draw(t, shape, std):
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, 10 + t])))
        return g.standard_normal(shape) * std

    return BlockInputs(
        x=f64_to_bf16_bits(draw(0, (N, C), 1.0)),
        w_qkv=f64_to_bf16_bits(draw(1, (3 * C, C), C ** -0.5)),
        b_qkv=draw(2, 3 * C, 0.02).astype(np.float32),
        w_o=f64_to_bf16_bits(draw(3, (C, C), C ** -0.5)),
        b_o=draw(4, C, 0.02).astype(np.float32),
    )
