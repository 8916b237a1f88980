"""Pins of the oracle's projection and frame-attention steps against facts that do not come
from the oracle itself: torch's fp64 linear layer and masked scaled-dot-product attention
(independent library routines), closed forms and the channel layout of the QKV split. CPU only."""
import numpy as np
import pytest
import torch

import oracle
from oracle import layer_io


@pytest.mark.parametrize("seed", range(3))
def test_linear_matches_torch(seed):
    rng = np.random.default_rng(seed)
    x, w, b = rng.standard_normal((37, 24)), rng.standard_normal((40, 24)), rng.standard_normal(40)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b)).numpy()
    assert np.allclose(layer_io.linear(x, w, b), ref, atol=1e-12)
    assert np.allclose(layer_io.linear(x, w, None), ref - b, atol=1e-12)


def test_linear_closed_forms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 8))
    assert np.allclose(layer_io.linear(x, np.eye(8), np.arange(8.0)), x + np.arange(8.0), atol=1e-15)
    w = rng.standard_normal((6, 8))
    assert np.allclose(layer_io.linear(np.eye(8), w, None), w.T, atol=1e-15)   # one-hot rows pick columns


def test_qkv_split_is_q_k_v_with_head_major_channels():
    """With x = 0 the projection returns the bias, so bias[c] = c exposes where channel c lands:
    Q[n, h, e] = h d + e, K = C + h d + e, V = 2C + h d + e."""
    H, d = 3, 4
    C = H * d
    q, k, v = layer_io.qkv_project(np.zeros((2, C)), np.zeros((3 * C, C)), np.arange(3.0 * C), H, d)
    idx = np.arange(H)[:, None] * d + np.arange(d)[None, :]
    for t, a in enumerate((q, k, v)):
        assert a.shape == (2, H, d) and np.array_equal(a[1], t * C + idx)


def test_out_project_concatenates_heads_in_order():
    rng = np.random.default_rng(2)
    o = rng.standard_normal((4, 3, 4))
    w, b = rng.standard_normal((5, 12)), rng.standard_normal(5)
    ref = torch.nn.functional.linear(torch.from_numpy(np.concatenate([o[:, h] for h in range(3)], axis=1)),
                                     torch.from_numpy(w), torch.from_numpy(b)).numpy()
    assert np.allclose(layer_io.out_project(o, w, b), ref, atol=1e-12)


@pytest.mark.parametrize("seed", range(3))
def test_frame_attention_matches_block_diagonal_sdpa(seed):
    rng = np.random.default_rng(seed)
    F, T, H, d = 3, int(rng.integers(1, 20)), 2, 8
    Q, K, V = (rng.standard_normal((F * T, H, d)) for _ in range(3))
    out = layer_io.frame_attention(Q, K, V, F, T)
    frame = np.arange(F * T) // T
    allowed = torch.from_numpy(frame[:, None] == frame[None, :])
    for h in range(H):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[:, h])[None], torch.from_numpy(K[:, h])[None], torch.from_numpy(V[:, h])[None],
            attn_mask=allowed)[0].numpy()
        assert np.allclose(out[:, h], ref, atol=1e-12)
    rows = rng.integers(0, F * T, 10)
    heads = rng.integers(0, H, 10)
    assert np.allclose(layer_io.frame_attention_rows(Q, K, V, T, rows, heads), out[rows, heads], atol=1e-13)


def test_frame_attention_of_one_frame_is_dense_and_constant_values_pass_through():
    rng = np.random.default_rng(3)
    Q, K = rng.standard_normal((9, 1, 8)), rng.standard_normal((9, 1, 8))
    V = np.tile(rng.standard_normal(8), (9, 1, 1))
    assert np.allclose(layer_io.frame_attention(Q, K, V, 3, 3), V, atol=1e-14)
    V = rng.standard_normal((9, 1, 8))
    o, _ = oracle.attend(Q[:, 0], K[:, 0], V[:, 0])
    assert np.allclose(layer_io.frame_attention(Q, K, V, 1, 9)[:, 0], o, atol=1e-14)
