"""Out-of-bounds writes: every output buffer of every entry point sits between canary
regions, and the canaries must be intact after each call (compute-sanitizer is not
available, so the kernels' own index arithmetic is checked this way)."""
import numpy as np
import pytest

from view_transformers_b200 import _lib, configs, layer, synth

pytestmark = pytest.mark.gpu

PAD = 4096   # bytes of canary on each side of every buffer

CASES = [
    configs.VGGT518.with_(name="canary_b64", frames=3, heads=3, rho=0.6, tau=0.0),
    configs.PERHEAD100.with_(name="canary_b128", frames=2, heads=3, head_budgets=False, rho=0.5),
    configs.Workload("canary_tail1_b64", 3, 43, 5, 2, 64, 64, 0.5, 0.0, "bf16", "five_percent"),
    configs.Workload("canary_f32_tail1", 3, 11, 4, 2, 64, 16, 0.5, 0.3, "f32", "tiny"),
]


class Guarded:
    """A device buffer of `nbytes` at `align`-byte alignment inside a canary-filled block."""

    def __init__(self, torch, nbytes: int, align: int = 16, fill: int = 0xA5):
        self.fill = fill
        self.nbytes = max(int(nbytes), 0)
        self.raw = torch.full((self.nbytes + 2 * PAD + align,), fill, dtype=torch.uint8, device="cuda")
        base = self.raw.data_ptr()
        self.start = (base + PAD + align - 1) // align * align
        self.off = self.start - base
        self.ptr = self.start

    def intact(self) -> bool:
        h = self.raw.cpu().numpy()
        return bool(np.all(h[: self.off] == self.fill) and np.all(h[self.off + self.nbytes:] == self.fill))


def _check_all(bufs, where):
    bad = [name for name, b in bufs.items() if not b.intact()]
    assert not bad, f"canary overwritten after {where}: {bad}"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_no_writes_outside_the_buffers(w):
    import torch
    x = synth.make_inputs(w)
    lay = _lib.layout_of(w)
    B = _lib.bsa_num_blocks(lay)
    ws_bytes = _lib.bsa_workspace_size(lay)
    H, d, N = w.heads, w.head_dim, w.n_tokens
    Np = w.n_patch
    e = 2 if w.dtype == "bf16" else 4
    words = (B + 31) // 32
    q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, x.v))
    g = {
        "pq": Guarded(torch, H * B * d * 4), "pk": Guarded(torch, H * d * B * 4),
        "mask_bits": Guarded(torch, H * B * words * 4), "kv_idx": Guarded(torch, H * B * B * 2),
        "kv_cnt": Guarded(torch, H * B * 4), "ws": Guarded(torch, ws_bytes, align=1024),
        "o_pp": Guarded(torch, Np * H * d * 4), "lse_pp": Guarded(torch, H * Np * 4),
        "o_ps": Guarded(torch, Np * H * d * 4), "lse_ps": Guarded(torch, H * Np * 4),
        "out": Guarded(torch, N * H * d * e), "out2": Guarded(torch, N * H * d * e),
    }
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    sp = status.data_ptr()
    P = {n: b.ptr for n, b in g.items()}
    qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
    ws = P["ws"] if ws_bytes else None

    def run(name, fn):
        fn()
        torch.cuda.synchronize()
        _check_all(g, name)

    run("pool", lambda: _lib.bsa_pool_qk(lay, qp, kp, P["pq"], P["pk"], sp, st))
    run("mask", lambda: _lib.bsa_predict_mask(lay, P["pq"], P["pk"], w.rho, w.tau, None, P["mask_bits"],
                                              P["kv_idx"], P["kv_cnt"], sp, st))
    run("pack", lambda: _lib.bsa_pack_qkv(lay, qp, kp, vp, ws, ws_bytes, sp, st))
    run("special", lambda: _lib.bsa_special_dense(lay, qp, kp, vp, ws, ws_bytes, P["out"], P["o_ps"],
                                                  P["lse_ps"], sp, st))
    run("sparse", lambda: _lib.bsa_block_sparse_attn(lay, qp, kp, vp, ws, ws_bytes, P["kv_idx"], P["kv_cnt"],
                                                     P["o_pp"], P["lse_pp"], sp, st))
    run("merge", lambda: _lib.bsa_merge(lay, P["o_pp"], P["lse_pp"], P["o_ps"], P["lse_ps"], P["out"], sp, st))
    run("pack_pool", lambda: _lib.bsa_pack_pool_qkv(lay, qp, kp, vp, ws, ws_bytes, P["pq"], P["pk"], sp, st))
    if w.dtype == "bf16":
        run("special rows", lambda: _lib.bsa_special_dense(lay, qp, kp, vp, ws, ws_bytes, P["out2"], None, None,
                                                           sp, st))
        run("fused", lambda: _lib.bsa_block_sparse_attn_fused(lay, qp, kp, vp, ws, ws_bytes, P["kv_idx"],
                                                              P["kv_cnt"], P["out2"], sp, st))
        # the fused path and the five-call path agree (same mask, same arithmetic up to rounding)
        n = N * H * d
        a = g["out"].raw[g["out"].off: g["out"].off + n * 2].view(torch.bfloat16).float()
        b = g["out2"].raw[g["out2"].off: g["out2"].off + n * 2].view(torch.bfloat16).float()
        assert torch.linalg.vector_norm(a - b) <= 3e-3 * torch.linalg.vector_norm(a)
    # the other block selectors write the same list buffers
    run("random", lambda: _lib.bsa_random_mask(lay, w.rho, None, 7, P["mask_bits"], P["kv_idx"], P["kv_cnt"], sp, st))
    run("uniform", lambda: _lib.bsa_uniform_mask(lay, 3, P["mask_bits"], P["kv_idx"], P["kv_cnt"], sp, st))
    run("probe", lambda: _lib.bsa_probe_mask(lay, P["pq"], P["pk"], w.rho, None, P["mask_bits"], P["kv_idx"],
                                             P["kv_cnt"], sp, st))
    g["pv"] = Guarded(torch, H * d * B * 4)
    P["pv"] = g["pv"].ptr
    run("pool_v", lambda: _lib.bsa_pool_v(lay, vp, P["pv"], sp, st))
    rws = _lib.bsa_ress_workspace_size(lay)
    g["rws"] = Guarded(torch, rws)
    P["rws"] = g["rws"].ptr
    run("ress", lambda: _lib.bsa_ress_mask(lay, P["pq"], P["pk"], P["pv"], w.rho, None, 4, P["rws"], rws,
                                           P["mask_bits"], P["kv_idx"], P["kv_cnt"], sp, st))
    if w.dtype == "bf16":
        # the steps on either side of the layer
        C = H * d
        bi = synth.make_block_inputs(w)
        xd, wq, wo = (layer.to_device(a, "bf16") for a in (bi.x, bi.w_qkv, bi.w_o))
        bq, bo = torch.from_numpy(bi.b_qkv).cuda(), torch.from_numpy(bi.b_o).cuda()
        for name in ("q2", "k2", "v2", "y"):
            g[name] = Guarded(torch, N * C * 2)
        fws = _lib.bsa_frame_workspace_size(lay)
        g["fws"] = Guarded(torch, fws, align=1024)
        P.update({n: g[n].ptr for n in ("q2", "k2", "v2", "y", "fws")})
        run("qkv_project", lambda: _lib.bsa_qkv_project(lay, xd.data_ptr(), wq.data_ptr(), bq.data_ptr(), P["q2"],
                                                        P["k2"], P["v2"], sp, st))
        run("out_project", lambda: _lib.bsa_out_project(lay, P["q2"], wo.data_ptr(), bo.data_ptr(), P["y"], sp, st))
        run("pack_frames", lambda: _lib.bsa_pack_frames(lay, qp, kp, vp, P["fws"], fws, sp, st))
        run("frame_attention", lambda: _lib.bsa_frame_attention(lay, P["fws"], fws, P["out2"], sp, st))
    assert _lib.bsa_check_status(sp, st) == _lib.BSA_OK
