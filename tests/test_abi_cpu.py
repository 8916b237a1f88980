"""C ABI checks that need no GPU: the library loads, exports every entry point declared in
include/bsa.h, its host helpers agree with the oracle, and invalid arguments are rejected
before anything is launched."""
import ctypes
import subprocess

import numpy as np
import pytest

import oracle
from view_transformers_b200 import _lib, build, configs, synth

E = _lib


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _lib.declared_symbols()
    assert len(declared) >= 13
    for name in ("bsa_pool_qk", "bsa_predict_mask", "bsa_block_sparse_attn", "bsa_special_dense", "bsa_merge"):
        assert name in declared
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    for name in declared:
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in range(7):
        assert _lib.status_string(code)
    assert _lib.status_string(99) == "unknown status"


@pytest.mark.parametrize("w", [configs.TINY, configs.VGGT518, configs.SWEEP_R50, configs.PERHEAD100, configs.LONG500])
def test_num_blocks_and_k(lib, w):
    lay = _lib.layout_of(w)
    B = _lib.bsa_num_blocks(lay)
    assert B == w.n_blocks
    assert _lib.bsa_k_from_rho(B, w.rho) == oracle.k_from_rho(B, w.rho)


def test_k_helpers_match_oracle(lib):
    for B in range(1, 4000, 37):
        for rho in (0.0, 0.1, 0.25, 0.5, 0.75, 0.9, 0.95, 1.0):
            assert _lib.bsa_k_from_rho(B, rho) == oracle.k_from_rho(B, rho)
        for d in (0.0, 0.013, 0.25, 0.5, 0.85, 1.0):
            assert _lib.bsa_k_from_density(B, d) == oracle.k_from_density(B, d)


def test_k_from_density_golden_cases(lib):
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "k_from_density_cases.txt")
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            B, d, k = line.split()
            assert _lib.bsa_k_from_density(int(B), float(d)) == int(k), line


@pytest.mark.parametrize("seed", range(10))
def test_head_budgets_match_oracle(lib, seed):
    rng = np.random.default_rng(seed)
    H = int(rng.integers(1, 64))
    s = rng.lognormal(0, 1.5, H)
    rho = float(rng.uniform(0, 1))
    got = _lib.bsa_head_budgets(s, rho, 1.0)
    assert np.allclose(got, oracle.water_fill(s, H * (1 - rho), 1.0), rtol=0, atol=1e-12)


def test_perhead_budgets(lib):
    w = configs.PERHEAD100
    d = _lib.bsa_head_budgets(synth.head_scores(w), w.rho, 1.0)
    ks = [_lib.bsa_k_from_density(608, x) for x in d]
    assert ks == [159, 122, 266, 155, 82, 201, 517, 361, 69, 39, 75, 146, 13, 112, 40, 67]


def test_workspace_size(lib):
    w = configs.PERHEAD100
    n = _lib.bsa_workspace_size(_lib.layout_of(w))
    # key-range splits of the 512 special queries (4 tiles x 16 heads = 64 CTAs per split)
    # over 4 + 608 key tiles: 9 splits fill 576 of the 592 slots of two waves (97%)
    np_pad, ns_pad, nsplit = 77824, 512, 9
    assert n == 3 * 16 * (np_pad + ns_pad) * 128 + nsplit * 16 * ns_pad * (64 + 1) * 4
    assert _lib.bsa_workspace_size(_lib.layout_of(configs.TINY)) == 0


# ------------------------------------------------------------------ validation (no launch)

A = 0x10000   # aligned fake device address (never dereferenced: validation fails first)


def _call(fn, *args):
    return getattr(_lib.load(), fn)(*args)


def _lay(**kw):
    base = dict(frames=2, tokens_per_frame=69, special_per_frame=5, heads=2, head_dim=64, block=16, dtype="f32")
    base.update(kw)
    return _lib.make_layout(**base)


def test_invalid_layouts(lib):
    out = ctypes.c_int32()
    nb = lambda l: lib.bsa_num_blocks(ctypes.byref(l), ctypes.byref(out))
    assert nb(_lay()) == E.BSA_OK and out.value == 8
    assert nb(_lay(head_dim=32)) == E.BSA_ERR_UNSUPPORTED
    assert nb(_lay(frames=0)) == E.BSA_ERR_INVALID_ARG
    assert nb(_lay(special_per_frame=69)) == E.BSA_ERR_INVALID_ARG
    assert nb(_lay(block=0)) == E.BSA_ERR_INVALID_ARG
    assert nb(_lay(heads=129)) == E.BSA_ERR_UNSUPPORTED
    assert nb(_lay(frames=100000, block=1, dtype="bf16")) == E.BSA_ERR_UNSUPPORTED   # B > 8192
    bad = _lay()
    bad.dtype = 7
    assert nb(bad) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_num_blocks(None, ctypes.byref(out)) == E.BSA_ERR_INVALID_ARG


def test_step_argument_validation(lib):
    lay = ctypes.byref(_lay())
    assert lib.bsa_pool_qk(lay, None, A, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pool_qk(lay, A + 4, A, A, A, None, None) == E.BSA_ERR_INVALID_ARG          # misaligned
    assert lib.bsa_predict_mask(lay, A, A, 1.5, 0.5, None, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_predict_mask(lay, A, A, 0.5, -0.1, None, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    dens = (ctypes.c_double * 2)(0.5, 0.6)                                                  # sum != H (1 - rho)
    assert lib.bsa_predict_mask(lay, A, A, 0.5, 0.5, dens, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_predict_mask(lay, A, A, 0.5, 0.5, None, None, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_block_sparse_attn(lay, A, A, A, None, 0, A, A, A, None, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_special_dense(lay, A, A, A, None, 0, None, None, None, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_merge(lay, A, A, A, A, None, None, None) == E.BSA_ERR_INVALID_ARG
    # one-pass packing + pooling: pooled outputs required; bf16 also needs V and the workspace
    assert lib.bsa_pack_pool_qkv(lay, A, A, A, None, 0, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pack_pool_qkv(lay, A, A + 8, A, None, 0, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    bf = _lay(dtype="bf16", block=64)
    ws = ctypes.c_size_t()
    assert lib.bsa_workspace_size(ctypes.byref(bf), ctypes.byref(ws)) == E.BSA_OK and ws.value > 0
    bfr = ctypes.byref(bf)
    assert lib.bsa_pack_pool_qkv(bfr, A, A, None, A, ws.value, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pack_pool_qkv(bfr, A, A, A, None, ws.value, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pack_pool_qkv(bfr, A, A, A, A, ws.value - 1, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    bf = _lay(dtype="bf16", block=64, tokens_per_frame=782, frames=4)
    ws = ctypes.c_size_t()
    assert lib.bsa_workspace_size(ctypes.byref(bf), ctypes.byref(ws)) == E.BSA_OK
    # bf16 attention needs the packed workspace, 1024-byte aligned and large enough
    assert lib.bsa_block_sparse_attn(ctypes.byref(bf), A, A, A, None, ws.value, A, A, A, A, None,
                                     None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_block_sparse_attn(ctypes.byref(bf), A, A, A, A + 16, ws.value, A, A, A, A, None,
                                     None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_block_sparse_attn(ctypes.byref(bf), A, A, A, A, ws.value - 1, A, A, A, A, None,
                                     None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pack_qkv(ctypes.byref(bf), A, A, A, A, ws.value - 1, None, None) == E.BSA_ERR_INVALID_ARG
    odd = _lay(dtype="bf16", block=32, tokens_per_frame=782, frames=4)
    assert lib.bsa_block_sparse_attn(ctypes.byref(odd), A, A, A, A, 1 << 40, A, A, A, A, None,
                                     None) == E.BSA_ERR_UNSUPPORTED
    assert lib.bsa_check_status(None, None) == E.BSA_ERR_INVALID_ARG


def test_head_budgets_validation(lib):
    s = (ctypes.c_double * 3)(1.0, -1.0, 2.0)
    d = (ctypes.c_double * 3)()
    assert lib.bsa_head_budgets(s, 3, 0.5, 1.0, d) == E.BSA_ERR_INVALID_ARG
    s2 = (ctypes.c_double * 3)(1.0, 1.0, 2.0)
    assert lib.bsa_head_budgets(s2, 3, 0.5, 0.1, d) == E.BSA_ERR_INVALID_ARG   # budget above H * cap


def test_selector_and_projection_argument_validation(lib):
    """The selectors, the projections and the frame-wise attention reject bad arguments on the
    host, before anything is launched (A is never dereferenced)."""
    lay = ctypes.byref(_lay())
    # random selection: rho in [0, 1], lists required and aligned; densities validated as in the mask
    assert lib.bsa_random_mask(lay, 1.5, None, 0, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_random_mask(lay, 0.5, None, 0, None, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_random_mask(lay, 0.5, None, 0, A + 4, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    dens = (ctypes.c_double * 2)(0.5, 0.6)
    assert lib.bsa_random_mask(lay, 0.5, dens, 0, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    # uniform sampling: stride >= 1
    assert lib.bsa_uniform_mask(lay, 0, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_uniform_mask(lay, 2, None, A, None, None, None) == E.BSA_ERR_INVALID_ARG
    # query probe: pooled tensors required
    assert lib.bsa_probe_mask(lay, None, A, 0.5, None, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_probe_mask(lay, A, A, -0.1, None, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    # drift scores: rounds in range, workspace large enough, pooled V required
    rws = ctypes.c_size_t()
    assert lib.bsa_ress_workspace_size(lay, ctypes.byref(rws)) == E.BSA_OK
    assert rws.value == 2 * 8 * 8 * 8                                    # H B B doubles, B = 8
    assert lib.bsa_ress_mask(lay, A, A, A, 0.5, None, -1, A, rws.value, None, A, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_ress_mask(lay, A, A, A, 0.5, None, 2000, A, rws.value, None, A, A, None,
                             None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_ress_mask(lay, A, A, A, 0.5, None, 4, A, rws.value - 1, None, A, A, None,
                             None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_ress_mask(lay, A, A, None, 0.5, None, 4, A, rws.value, None, A, A, None,
                             None) == E.BSA_ERR_INVALID_ARG
    big = _lay(frames=100, tokens_per_frame=782, block=64, dtype="bf16")   # B = 1215: P_b(V) exceeds shared memory
    assert lib.bsa_ress_mask(ctypes.byref(big), A, A, A, 0.5, None, 4, A, 1 << 40, None, A, A, None,
                             None) == E.BSA_ERR_UNSUPPORTED
    assert lib.bsa_pool_v(lay, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    # projections and frame-wise attention: bf16 layouts only, pointers required
    assert lib.bsa_qkv_project(lay, A, A, None, A, A, A, None, None) == E.BSA_ERR_UNSUPPORTED          # f32 layout
    bf = ctypes.byref(_lay(dtype="bf16", block=64))
    assert lib.bsa_qkv_project(bf, A, A, None, A, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_qkv_project(bf, A, A, A + 4, A, A, A, None, None) == E.BSA_ERR_INVALID_ARG        # bias misaligned
    assert lib.bsa_out_project(bf, A, None, None, A, None, None) == E.BSA_ERR_INVALID_ARG
    fws = ctypes.c_size_t()
    assert lib.bsa_frame_workspace_size(bf, ctypes.byref(fws)) == E.BSA_OK
    assert fws.value == 3 * 2 * 2 * 128 * 128                            # H F t_pad rows of 128 bytes, x3
    assert lib.bsa_pack_frames(bf, A, A, A, A, fws.value - 1, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_pack_frames(bf, A, A, A, A + 16, fws.value, None, None) == E.BSA_ERR_INVALID_ARG  # 1024-byte alignment
    assert lib.bsa_frame_attention(bf, A, fws.value, None, None, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_frame_attention(lay, A, fws.value, A, None, None) == E.BSA_ERR_UNSUPPORTED          # f32 layout
