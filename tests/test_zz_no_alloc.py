"""The allocation-free entry point, for callers that cannot allocate device memory (a host
framework's memory pool owns every allocation, or a latency-critical loop may not call
cudaMalloc/cudaFree because they can synchronize the device). It must give the same layer
output as the workspace-based entry points and as the fp64 oracle, call after call, although
every call reuses the library's one static scratch array. Collected last on purpose."""
import ctypes

import numpy as np
import pytest

from view_transformers_b200 import _lib, configs


def test_layers_beyond_the_scratch_limit_are_rejected_before_launch():
    lay = _lib.layout_of(configs.PERHEAD100)          # needs about 500 MB of packed data
    assert _lib.bsa_workspace_size(lay) > 64 << 20
    A = 0x10000
    assert _lib.load().bsa_attention_noalloc(ctypes.byref(lay), A, A, A, A, A, A, None,
                                             None) == _lib.BSA_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_matches_workspace_path_and_oracle_on_two_calls_in_a_row():
    """Per case, two calls back to back with different kept-block lists (two budgets on the
    same Q, K, V); the second case is a smaller layer than the first. Each output is checked
    against the workspace path and against the oracle fed the same lists."""
    import torch

    import oracle
    from oracle.compare import max_abs, rel_l2
    from view_transformers_b200 import layer, synth

    cases = [configs.VGGT518.with_(name="noalloc_b64", frames=4, tau=0.0),            # b = 64, 16 heads
             configs.PERHEAD100.with_(name="noalloc_b128", frames=4, head_budgets=False, rho=0.6)]
    st = torch.cuda.current_stream().cuda_stream
    for w in cases:
        x = synth.make_inputs(w)
        q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, x.v))
        lay = oracle.Layout(w.frames, w.tokens_per_frame, w.special_per_frame, w.heads, w.head_dim, w.block)
        Q, K, V = (oracle.to_f64(a, w.dtype) for a in (x.q, x.k, x.v))
        masks = []
        for rho in (w.rho, 0.85):
            L = layer.BlockSparseLayer.for_workload(w.with_(rho=rho))
            assert L.ws_bytes <= 64 << 20
            ref = L.forward(q, k, v, fused=True).float().cpu().numpy()
            assert L.check_status() == 0
            masks.append((L, ref))
        assert not np.array_equal(masks[0][0].selected(), masks[1][0].selected())
        for L, ref in masks:                      # two calls in a row, each with its own lists
            out = torch.full_like(L.buf.out, float("nan"))
            _lib.bsa_attention_noalloc(L.layout, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       L.buf.kv_idx.data_ptr(), L.buf.kv_cnt.data_ptr(), out.data_ptr(),
                                       L.buf.status.data_ptr(), st)
            torch.cuda.synchronize()
            assert L.check_status() == 0
            got = out.float().cpu().numpy()
            assert np.isfinite(got).all()                   # every row written
            assert rel_l2(got, ref) <= 2e-3 and max_abs(got, ref) <= 2e-2, w.name
            want = oracle.layer_forward(Q, K, V, lay, L.selected())
            assert rel_l2(got, want) <= 2e-3 and max_abs(got, want) <= 2e-2, w.name
