"""ctypes binding of libbsa.so (argument marshalling only; every step runs in the library).

The functions keep the C names of include/bsa.h. Device pointers are plain integers
(e.g. torch's `tensor.data_ptr()`), streams are `cudaStream_t` handles as integers.
Loading fails loudly when the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbsa.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "bsa.h")

(BSA_OK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA, BSA_ERR_TIMEOUT, BSA_ERR_DEVICE_BOUNDS,
 BSA_ERR_RANGE) = range(7)
BSA_F32, BSA_BF16 = 0, 1
DTYPES = {"f32": BSA_F32, "bf16": BSA_BF16}


class bsa_layout(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("special_per_frame", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class BsaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {code})")
        self.code = code


_vp, _sz, _i32p, _st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
_LP = ctypes.POINTER(bsa_layout)
_SIGS = {
    "bsa_pool_qk": [_LP, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_predict_mask": [_LP, _vp, _vp, ctypes.c_double, ctypes.c_double, ctypes.c_void_p, _vp, _vp, _vp, _i32p, _st],
    "bsa_pack_qkv": [_LP, _vp, _vp, _vp, _vp, _sz, _i32p, _st],
    "bsa_pack_pool_qkv": [_LP, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _i32p, _st],
    "bsa_block_sparse_attn": [_LP, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_special_dense": [_LP, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _i32p, _st],
    "bsa_merge": [_LP, _vp, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_block_sparse_attn_fused": [_LP, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _i32p, _st],
    "bsa_attention_noalloc": [_LP, _vp, _vp, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_qkv_project": [_LP, _vp, _vp, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_out_project": [_LP, _vp, _vp, _vp, _vp, _i32p, _st],
    "bsa_pack_frames": [_LP, _vp, _vp, _vp, _vp, _sz, _i32p, _st],
    "bsa_frame_attention": [_LP, _vp, _sz, _vp, _i32p, _st],
    "bsa_frame_workspace_size": [_LP, ctypes.POINTER(ctypes.c_size_t)],
    "bsa_pool_v": [_LP, _vp, _vp, _i32p, _st],
    "bsa_ress_mask": [_LP, _vp, _vp, _vp, ctypes.c_double, ctypes.c_void_p, ctypes.c_int32, _vp, _sz, _vp, _vp,
                      _vp, _i32p, _st],
    "bsa_ress_workspace_size": [_LP, ctypes.POINTER(ctypes.c_size_t)],
    "bsa_random_mask": [_LP, ctypes.c_double, ctypes.c_void_p, ctypes.c_uint64, _vp, _vp, _vp, _i32p, _st],
    "bsa_uniform_mask": [_LP, ctypes.c_int32, _vp, _vp, _vp, _i32p, _st],
    "bsa_probe_mask": [_LP, _vp, _vp, ctypes.c_double, ctypes.c_void_p, _vp, _vp, _vp, _i32p, _st],
    "bsa_num_blocks": [_LP, ctypes.POINTER(ctypes.c_int32)],
    "bsa_workspace_size": [_LP, ctypes.POINTER(ctypes.c_size_t)],
    "bsa_k_from_rho": [ctypes.c_int32, ctypes.c_double, ctypes.POINTER(ctypes.c_int32)],
    "bsa_k_from_density": [ctypes.c_int32, ctypes.c_double, ctypes.POINTER(ctypes.c_int32)],
    "bsa_head_budgets": [ctypes.POINTER(ctypes.c_double), ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                         ctypes.POINTER(ctypes.c_double)],
    "bsa_check_status": [_i32p, _st],
    "bsa_selftest_wait_timeout": [_i32p, ctypes.c_uint32, _st],
    "bsa_status_string": [ctypes.c_int],
}

_lib = None


def load() -> ctypes.CDLL:
    """Loads the in-tree libbsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m view_transformers_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "bsa_status_string" else ctypes.c_int
        _lib = lib
    return _lib


def declared_symbols() -> list[str]:
    """Entry points declared in include/bsa.h."""
    with open(HEADER) as f:
        return re.findall(r"^BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", f.read(), flags=re.M)


def status_string(code: int) -> str:
    return load().bsa_status_string(code).decode()


def _check(fn: str, code: int) -> None:
    if code != BSA_OK:
        raise BsaError(fn, code, status_string(code))


def make_layout(frames: int, tokens_per_frame: int, special_per_frame: int, heads: int, head_dim: int,
                block: int, dtype: str) -> bsa_layout:
    return bsa_layout(frames, tokens_per_frame, special_per_frame, heads, head_dim, block, DTYPES[dtype])


def layout_of(w) -> bsa_layout:
    """Layout of a configs.Workload."""
    return make_layout(w.frames, w.tokens_per_frame, w.special_per_frame, w.heads, w.head_dim, w.block, w.dtype)


# ------------------------------------------------------------------ host helpers

def bsa_num_blocks(layout: bsa_layout) -> int:
    out = ctypes.c_int32()
    _check("bsa_num_blocks", load().bsa_num_blocks(ctypes.byref(layout), ctypes.byref(out)))
    return out.value


def bsa_workspace_size(layout: bsa_layout) -> int:
    out = ctypes.c_size_t()
    _check("bsa_workspace_size", load().bsa_workspace_size(ctypes.byref(layout), ctypes.byref(out)))
    return out.value


def bsa_k_from_rho(num_blocks: int, rho: float) -> int:
    out = ctypes.c_int32()
    _check("bsa_k_from_rho", load().bsa_k_from_rho(num_blocks, rho, ctypes.byref(out)))
    return out.value


def bsa_k_from_density(num_blocks: int, density: float) -> int:
    out = ctypes.c_int32()
    _check("bsa_k_from_density", load().bsa_k_from_density(num_blocks, density, ctypes.byref(out)))
    return out.value


def bsa_head_budgets(scores, rho: float, cap: float = 1.0) -> list[float]:
    n = len(scores)
    s = (ctypes.c_double * n)(*[float(x) for x in scores])
    d = (ctypes.c_double * n)()
    _check("bsa_head_budgets", load().bsa_head_budgets(s, n, rho, cap, d))
    return list(d)


def bsa_selftest_wait_timeout(status_ptr: int, limit_us: int, stream: int = 0) -> None:
    _check("bsa_selftest_wait_timeout", load().bsa_selftest_wait_timeout(status_ptr, limit_us, stream))


def bsa_check_status(status_ptr: int, stream: int = 0) -> int:
    """Returns the device status code (0 = ok) and resets it."""
    return load().bsa_check_status(status_ptr, stream)


# ------------------------------------------------------------------ device steps

def bsa_pool_qk(layout, q, k, pq, pk, status=0, stream=0) -> None:
    _check("bsa_pool_qk", load().bsa_pool_qk(ctypes.byref(layout), q, k, pq, pk, status, stream))


def bsa_predict_mask(layout, pq, pk, rho, tau, head_density, mask_bits, kv_idx, kv_cnt, status=0,
                     stream=0) -> None:
    dens = None
    if head_density is not None:
        dens = (ctypes.c_double * len(head_density))(*[float(x) for x in head_density])
    _check("bsa_predict_mask", load().bsa_predict_mask(ctypes.byref(layout), pq, pk, rho, tau,
                                                       ctypes.cast(dens, ctypes.c_void_p) if dens else None,
                                                       mask_bits, kv_idx, kv_cnt, status, stream))


def _densities(head_density):
    if head_density is None:
        return None, None
    dens = (ctypes.c_double * len(head_density))(*[float(x) for x in head_density])
    return dens, ctypes.cast(dens, ctypes.c_void_p)


def bsa_random_mask(layout, rho, head_density, seed, mask_bits, kv_idx, kv_cnt, status=0, stream=0) -> None:
    keep, dens = _densities(head_density)
    _check("bsa_random_mask", load().bsa_random_mask(ctypes.byref(layout), rho, dens, int(seed), mask_bits,
                                                     kv_idx, kv_cnt, status, stream))


def bsa_pool_v(layout, v, pv, status=0, stream=0) -> None:
    _check("bsa_pool_v", load().bsa_pool_v(ctypes.byref(layout), v, pv, status, stream))


def bsa_ress_workspace_size(layout) -> int:
    out = ctypes.c_size_t()
    _check("bsa_ress_workspace_size", load().bsa_ress_workspace_size(ctypes.byref(layout), ctypes.byref(out)))
    return out.value


def bsa_ress_mask(layout, pq, pk, pv, rho, head_density, rounds, workspace, workspace_bytes, mask_bits, kv_idx,
                  kv_cnt, status=0, stream=0) -> None:
    keep, dens = _densities(head_density)
    _check("bsa_ress_mask", load().bsa_ress_mask(ctypes.byref(layout), pq, pk, pv, rho, dens, int(rounds), workspace,
                                                 workspace_bytes, mask_bits, kv_idx, kv_cnt, status, stream))


def bsa_uniform_mask(layout, stride, mask_bits, kv_idx, kv_cnt, status=0, stream=0) -> None:
    _check("bsa_uniform_mask", load().bsa_uniform_mask(ctypes.byref(layout), int(stride), mask_bits, kv_idx,
                                                       kv_cnt, status, stream))


def bsa_probe_mask(layout, pq, pk, rho, head_density, mask_bits, kv_idx, kv_cnt, status=0, stream=0) -> None:
    keep, dens = _densities(head_density)
    _check("bsa_probe_mask", load().bsa_probe_mask(ctypes.byref(layout), pq, pk, rho, dens, mask_bits, kv_idx,
                                                   kv_cnt, status, stream))


def bsa_pack_qkv(layout, q, k, v, workspace, workspace_bytes, status=0, stream=0) -> None:
    _check("bsa_pack_qkv", load().bsa_pack_qkv(ctypes.byref(layout), q, k, v, workspace, workspace_bytes,
                                               status, stream))


def bsa_pack_pool_qkv(layout, q, k, v, workspace, workspace_bytes, pq, pk, status=0, stream=0) -> None:
    _check("bsa_pack_pool_qkv", load().bsa_pack_pool_qkv(ctypes.byref(layout), q, k, v, workspace,
                                                         workspace_bytes, pq, pk, status, stream))


def bsa_block_sparse_attn(layout, q, k, v, workspace, workspace_bytes, kv_idx, kv_cnt, o_pp, lse_pp,
                          status=0, stream=0) -> None:
    _check("bsa_block_sparse_attn", load().bsa_block_sparse_attn(
        ctypes.byref(layout), q, k, v, workspace, workspace_bytes, kv_idx, kv_cnt, o_pp, lse_pp, status, stream))


def bsa_special_dense(layout, q, k, v, workspace, workspace_bytes, out, o_ps, lse_ps, status=0,
                      stream=0) -> None:
    _check("bsa_special_dense", load().bsa_special_dense(
        ctypes.byref(layout), q, k, v, workspace, workspace_bytes, out, o_ps, lse_ps, status, stream))


def bsa_merge(layout, o_pp, lse_pp, o_ps, lse_ps, out, status=0, stream=0) -> None:
    _check("bsa_merge", load().bsa_merge(ctypes.byref(layout), o_pp, lse_pp, o_ps, lse_ps, out, status, stream))


def bsa_block_sparse_attn_fused(layout, q, k, v, workspace, workspace_bytes, kv_idx, kv_cnt, out, status=0,
                                stream=0) -> None:
    _check("bsa_block_sparse_attn_fused", load().bsa_block_sparse_attn_fused(
        ctypes.byref(layout), q, k, v, workspace, workspace_bytes, kv_idx, kv_cnt, out, status, stream))


def bsa_qkv_project(layout, x, w_qkv, b_qkv, q, k, v, status=0, stream=0) -> None:
    _check("bsa_qkv_project", load().bsa_qkv_project(ctypes.byref(layout), x, w_qkv, b_qkv, q, k, v, status, stream))


def bsa_out_project(layout, o, w_o, b_o, y, status=0, stream=0) -> None:
    _check("bsa_out_project", load().bsa_out_project(ctypes.byref(layout), o, w_o, b_o, y, status, stream))


def bsa_frame_workspace_size(layout) -> int:
    out = ctypes.c_size_t()
    _check("bsa_frame_workspace_size", load().bsa_frame_workspace_size(ctypes.byref(layout), ctypes.byref(out)))
    return out.value


def bsa_pack_frames(layout, q, k, v, workspace, workspace_bytes, status=0, stream=0) -> None:
    _check("bsa_pack_frames", load().bsa_pack_frames(ctypes.byref(layout), q, k, v, workspace, workspace_bytes,
                                                     status, stream))


def bsa_frame_attention(layout, workspace, workspace_bytes, out, status=0, stream=0) -> None:
    _check("bsa_frame_attention", load().bsa_frame_attention(ctypes.byref(layout), workspace, workspace_bytes, out,
                                                             status, stream))


def bsa_attention_noalloc(layout, q, k, v, kv_idx, kv_cnt, out, status=0, stream=0) -> None:
    """Steps 4-6 for bf16 layers with the library's static scratch (no workspace argument)."""
    _check("bsa_attention_noalloc", load().bsa_attention_noalloc(
        ctypes.byref(layout), q, k, v, kv_idx, kv_cnt, out, status, stream))
