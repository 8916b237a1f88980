"""GPU parity of the steps on either side of the layer, through the C ABI on cuda:0, against
the fp64 oracle (oracle/layer_io.py):

  * the QKV and output projections (tcgen05 GEMM): every element within one bf16 unit in the
    last place of the oracle's value (fp32 accumulation of exact bf16 products, then one
    rounding to bf16), and relative L2 <= 2e-3 (bf16 rounding alone gives about 1.7e-3 on
    Gaussian data);
  * the frame-wise attention: relative L2 <= 2e-3 and max-abs <= 2e-2 (the layer's bf16
    tolerance), on every row of small layers and on 2,048 sampled (row, head) pairs of the
    100-frame layer;
  * one whole block (projections around the block-sparse global layer and around the frame
    attention) against the oracle chained on the device's own intermediate tensors."""
import numpy as np
import pytest

import oracle
from oracle import layer_io
from oracle.compare import max_abs, rel_l2
from view_transformers_b200 import configs, synth

from gpu_common import sample_pairs

pytestmark = pytest.mark.gpu

def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _dev(a, dtype="bf16"):
    import torch
    from view_transformers_b200 import layer
    if a.dtype == np.float32:
        return torch.from_numpy(a).cuda()
    return layer.to_device(a, dtype)


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_close_ulp(got, ref, absdot, K):
    """|got - ref| <= half a bf16 ulp (the final rounding) + K 2^-24 sum_i |x_i w_i| (the
    standard bound of a K-term fp32 accumulation of exact products)."""
    bound = 0.5 * np.maximum(_bf16_ulp(ref), _bf16_ulp(got)) + K * 2.0 ** -24 * absdot + 1e-30
    worst = float(np.max(np.abs(got - ref) / bound))
    print(f"  max error / bound {worst:.3f}, rel_l2 {rel_l2(got, ref):.3e}")
    assert worst <= 1.0
    assert rel_l2(got, ref) <= 2e-3


PROJ = [
    configs.VGGT518.with_(name="proj_h16", frames=3),               # C = 1024, N = 4122 (ragged M)
    configs.VGGT518.with_(name="proj_h2", frames=2, heads=2),       # C = 128: 3C = 384, partial N tile
    configs.VGGT518.with_(name="proj_h3", frames=1, heads=3),       # C = 192: 3C = 576, tiles straddle q/k
    # fewer rows than one 256-row tile of a CTA pair: the second CTA's rows all lie past the end
    configs.VGGT518.with_(name="proj_m105", frames=1, heads=2, patch_per_frame=100),
    configs.PERHEAD100,                                             # full size, sampled rows
]


@pytest.mark.parametrize("w", PROJ, ids=lambda w: w.name)
def test_qkv_and_out_projection(w):
    import torch
    from view_transformers_b200 import _lib
    bi = synth.make_block_inputs(w)
    lay = _lib.layout_of(w)
    N, H, d = w.n_tokens, w.heads, w.head_dim
    x, wq, bq, wo, bo = (_dev(a) for a in (bi.x, bi.w_qkv, bi.b_qkv, bi.w_o, bi.b_o))
    q, k, v, y = (torch.empty((N, H * d), dtype=torch.bfloat16, device="cuda") for _ in range(4))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    _lib.bsa_qkv_project(lay, x.data_ptr(), wq.data_ptr(), bq.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                         status.data_ptr(), st)
    _lib.bsa_out_project(lay, q.data_ptr(), wo.data_ptr(), bo.data_ptr(), y.data_ptr(), status.data_ptr(), st)
    torch.cuda.synchronize()
    assert _lib.bsa_check_status(status.data_ptr(), st) == 0
    X = synth.bf16_bits_to_f32(bi.x).astype(np.float64)
    rows = np.arange(N) if N <= 5000 else np.sort(np.random.default_rng(3).choice(N, 2048, replace=False))
    Wq = synth.bf16_bits_to_f32(bi.w_qkv).astype(np.float64)
    Wo = synth.bf16_bits_to_f32(bi.w_o).astype(np.float64)
    C = H * d
    ref = layer_io.qkv_project(X[rows], Wq, bi.b_qkv, H, d)
    absdot = np.abs(X[rows]) @ np.abs(Wq).T
    for t, (name, got, want) in enumerate(zip("qkv", (q, k, v), ref)):
        print(name, end="")
        _check_close_ulp(_host(got)[rows], want.reshape(len(rows), -1), absdot[:, t * C:(t + 1) * C], C)
    # the output projection of the device's own q (as [N, H, d])
    Qd = _host(q)[rows]
    want = layer_io.out_project(Qd.reshape(len(rows), H, d), Wo, bi.b_o)
    print("y", end="")
    _check_close_ulp(_host(y)[rows], want, np.abs(Qd) @ np.abs(Wo).T, C)


FRAME = [
    configs.VGGT518.with_(name="frame_t782", frames=2, heads=2, patch_per_frame=777),   # 7 tiles, 14-row tail
    configs.VGGT518.with_(name="frame_t129", frames=3, heads=2, patch_per_frame=124),   # one-row tail
    configs.VGGT518.with_(name="frame_t128", frames=2, heads=3, patch_per_frame=123),   # whole tiles
    configs.VGGT518.with_(name="frame_t50_s0", frames=4, heads=2, patch_per_frame=50, special_per_frame=0),
    configs.PERHEAD100,                                                                # 100 frames, sampled
]


@pytest.mark.parametrize("w", FRAME, ids=lambda w: w.name)
def test_frame_attention(w):
    import torch
    from view_transformers_b200 import _lib, layer
    x = synth.make_inputs(w)
    lay = _lib.layout_of(w)
    q, k, v = (layer.to_device(a, "bf16") for a in (x.q, x.k, x.v))
    out = torch.full_like(q, float("nan"))
    nbytes = _lib.bsa_frame_workspace_size(lay)
    ws = torch.empty(nbytes + 1024, dtype=torch.uint8, device="cuda")
    ptr = (ws.data_ptr() + 1023) // 1024 * 1024
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    _lib.bsa_pack_frames(lay, q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr, nbytes, status.data_ptr(), st)
    _lib.bsa_frame_attention(lay, ptr, nbytes, out.data_ptr(), status.data_ptr(), st)
    torch.cuda.synchronize()
    assert _lib.bsa_check_status(status.data_ptr(), st) == 0
    got = _host(out)
    assert np.isfinite(got).all()                   # every row written
    Q, K, V = (synth.bf16_bits_to_f32(a) for a in (x.q, x.k, x.v))
    T = w.tokens_per_frame
    if w.n_tokens * w.heads <= 20000:
        ref = layer_io.frame_attention(Q, K, V, w.frames, T)
        g = got
    else:
        rows, heads = sample_pairs(w, 2048)
        ref = layer_io.frame_attention_rows(Q, K, V, T, rows, heads)
        g = got[rows, heads]
    e2, ea = rel_l2(g, ref), max_abs(g, ref)
    print(f"{w.name}: rel_l2 {e2:.3e} max_abs {ea:.3e}")
    assert e2 <= 2e-3 and ea <= 2e-2


@pytest.mark.parametrize("global_layer", [True, False], ids=["global", "frame"])
def test_whole_block(global_layer):
    """x -> QKV projection -> attention -> output projection, checked step by step against the
    oracle on the device's own intermediate tensors (each step's error is its own)."""
    import torch
    from view_transformers_b200 import layer
    w = configs.VGGT518.with_(name="block_f3", frames=3, heads=4, tau=0.0)
    bi = synth.make_block_inputs(w)
    x, wq, bq, wo, bo = (_dev(a) for a in (bi.x, bi.w_qkv, bi.b_qkv, bi.w_o, bi.b_o))
    L = layer.BlockSparseLayer.for_workload(w) if global_layer else None
    blk = layer.AttentionBlock(w.frames, w.tokens_per_frame, w.special_per_frame, w.heads, w.head_dim,
                               wq, bq, wo, bo, L)
    y = _host(blk.forward(x))
    torch.cuda.synchronize()
    assert blk.check_status() == 0
    H, d = w.heads, w.head_dim
    X = synth.bf16_bits_to_f32(bi.x).astype(np.float64)
    Wq = synth.bf16_bits_to_f32(bi.w_qkv).astype(np.float64)
    Wo = synth.bf16_bits_to_f32(bi.w_o).astype(np.float64)
    C = H * d
    absdot = np.abs(X) @ np.abs(Wq).T
    for t, (got, want) in enumerate(zip((blk.q, blk.k, blk.v), layer_io.qkv_project(X, Wq, bi.b_qkv, H, d))):
        _check_close_ulp(_host(got).reshape(len(X), -1), want.reshape(len(X), -1), absdot[:, t * C:(t + 1) * C], C)
    Qd, Kd, Vd = (_host(t) for t in (blk.q, blk.k, blk.v))
    if global_layer:
        lay = oracle.Layout(w.frames, w.tokens_per_frame, w.special_per_frame, H, d, w.block)
        ref_o = oracle.layer_forward(Qd, Kd, Vd, lay, L.selected())
    else:
        ref_o = layer_io.frame_attention(Qd, Kd, Vd, w.frames, w.tokens_per_frame)
    o = _host(blk.o)
    assert rel_l2(o, ref_o) <= 2e-3 and max_abs(o, ref_o) <= 2e-2
    o2 = o.reshape(len(X), -1)
    _check_close_ulp(y, layer_io.out_project(o.reshape(len(X), H, d), Wo, bi.b_o), np.abs(o2) @ np.abs(Wo).T, C)
