"""Shared helpers of the GPU tests: seeded inputs (cached), one layer run through the C ABI,
and the oracle pieces they are compared with."""
from __future__ import annotations

import functools

import numpy as np

import oracle
from view_transformers_b200 import configs, synth


@functools.lru_cache(maxsize=2)
def inputs(w: configs.Workload) -> synth.LayerInputs:
    return synth.make_inputs(w)


def exact(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage -> float32 holding the exact input values (bf16 and f32 are exact in fp32)."""
    return synth.bf16_bits_to_f32(a) if dtype == "bf16" else np.asarray(a, dtype=np.float32)


def oracle_layout(w: configs.Workload) -> oracle.Layout:
    return oracle.Layout(w.frames, w.tokens_per_frame, w.special_per_frame, w.heads, w.head_dim, w.block)


def head_density(w: configs.Workload, x: synth.LayerInputs):
    """Per-head densities from the library's own capped water-filling (the step the
    product runs), checked against the oracle's on the way."""
    if x.scores is None:
        return None
    from view_transformers_b200 import _lib
    dens = _lib.bsa_head_budgets(x.scores, w.rho, 1.0)
    assert np.allclose(dens, oracle.water_fill(x.scores, w.heads * (1.0 - w.rho), 1.0), rtol=0, atol=1e-12)
    return dens


def run_gpu(w: configs.Workload, x: synth.LayerInputs, density=None, tamper=None):
    """Runs the layer on cuda:0; returns host copies of every intermediate."""
    import torch
    from view_transformers_b200 import layer
    L = layer.BlockSparseLayer.for_workload(w, head_density=density)
    q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, x.v))
    L.predict(q, k)
    if tamper is not None:
        tamper(L)
    L.attend(q, k, v)
    torch.cuda.synchronize()
    status = L.check_status()
    out = L.buf.out.float().cpu().numpy()
    out_fused = None
    if w.dtype == "bf16":
        L.buf.out.zero_()
        L.attend_fused(q, k, v)
        torch.cuda.synchronize()
        status = status or L.check_status()
        out_fused = L.buf.out.float().cpu().numpy()
    res = dict(
        layer=L, status=status, out=out, out_fused=out_fused, selected=L.selected(),
        kv_idx=L.buf.kv_idx.cpu().numpy().view(np.uint16), kv_cnt=L.buf.kv_cnt.cpu().numpy(),
        pq=L.buf.pq.cpu().numpy(), pk=L.buf.pk.cpu().numpy(),
        o_pp=L.buf.o_pp.cpu().numpy(), lse_pp=L.buf.lse_pp.cpu().numpy(),
        o_ps=L.buf.o_ps.cpu().numpy(), lse_ps=L.buf.lse_ps.cpu().numpy(), forward=None)
    if w.dtype == "bf16":
        # the whole layer through forward(): one-pass packing + pooling, mask, fused attention
        L.buf.pq.zero_()
        L.buf.pk.zero_()
        L.buf.out.zero_()
        L.forward(q, k, v)
        torch.cuda.synchronize()
        res["status"] = res["status"] or L.check_status()
        res["forward"] = dict(pq=L.buf.pq.cpu().numpy(), pk=L.buf.pk.cpu().numpy(), selected=L.selected(),
                              out=L.buf.out.float().cpu().numpy())
    return res


def sample_pairs(w: configs.Workload, n: int, seed: int = 1234):
    """Seeded (row, head) pairs, rows uniform without replacement over all N tokens."""
    g = np.random.default_rng(seed)
    rows = g.choice(w.n_tokens, size=min(n, w.n_tokens), replace=False)
    heads = g.integers(0, w.heads, size=len(rows))
    return rows, heads
