"""Seeded generator: determinism, exact bf16 rounding, planting structure (CPU-only)."""
import numpy as np
import torch

from view_transformers_b200 import configs, synth


def test_bf16_rounding_ties_to_even_and_matches_torch_for_fp32_inputs():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> ties to even (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -30,
                  0.0, -0.0, 3.0e38])
    bits = synth.f64_to_bf16_bits(x)
    assert bits.tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81, 0x0000, 0x8000, 0x7F62]
    r = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    ref = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f64_to_bf16_bits(r.astype(np.float64)), ref)


def test_inputs_are_deterministic_and_shaped():
    w = configs.TINY
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    assert a.q.shape == (w.n_tokens, w.heads, w.head_dim) and a.q.dtype == np.float32
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    w2 = configs.VGGT518.with_(frames=3, heads=2)
    c = synth.make_inputs(w2)
    assert c.q.dtype == np.uint16 and c.q.shape == (3 * 1374, 2, 64)
    v = synth.decode(c.v, "bf16")
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01


def test_tiny_planting_copies_queries_into_the_other_frame():
    w = configs.TINY
    x = synth.make_inputs(w)
    q, k = x.q.astype(np.float64), x.k.astype(np.float64)
    T, S, P = w.tokens_per_frame, w.special_per_frame, w.patch_per_frame
    qa = q[S:T]                      # frame 0 patches
    kb = k[T + S:2 * T]              # frame 1 patches (a permutation of frame-0 queries + noise)
    dist = np.linalg.norm(qa[:, None] - kb[None], axis=-1).sum(-1)      # [P, P]
    best = dist.argmin(axis=1)
    assert len(set(best.tolist())) == P                                # a permutation
    assert np.all(dist[np.arange(P), best] < 0.15 * np.sqrt(64) * 2 * 2)


def test_five_percent_planting_scales_keys():
    w = configs.SWEEP_R50.with_(frames=4, heads=2)
    x = synth.make_inputs(w)
    k = synth.decode(x.k, "bf16")
    norms = np.linalg.norm(k.reshape(k.shape[0], -1), axis=1)
    planted = norms > 2.0 * np.sqrt(2 * 64)
    assert planted.sum() == 4 * round(0.05 * w.patch_per_frame)
    rows = np.nonzero(planted)[0] % w.tokens_per_frame
    assert rows.min() >= w.special_per_frame


def test_head_scores_are_seeded_lognormal():
    s = synth.head_scores(configs.PERHEAD100)
    assert s.shape == (16,) and np.all(s > 0)
    assert np.array_equal(s, np.random.Generator(np.random.PCG64(0)).lognormal(0, 1, 16))
