"""Runs one block-sparse global-attention layer through the C ABI.

Torch provides the device buffers and the stream; each step is one library call.
forward() on a bf16 layer: pack + pool -> predict mask -> special queries -> fused patch
rows. The step-by-step path (predict(), attend(); f32 layers, or fused=False):
  pool -> predict mask -> pack -> special dense -> block-sparse attention -> merge.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class Buffers:
    pq: torch.Tensor
    pk: torch.Tensor
    mask_bits: torch.Tensor
    kv_idx: torch.Tensor
    kv_cnt: torch.Tensor
    workspace: torch.Tensor
    out: torch.Tensor
    status: torch.Tensor
    # fp32 partial results of the step-by-step path, allocated on its first use
    o_pp: torch.Tensor | None = None
    lse_pp: torch.Tensor | None = None
    o_ps: torch.Tensor | None = None
    lse_ps: torch.Tensor | None = None


class BlockSparseLayer:
    """One global-attention layer of fixed geometry and selection hyper-parameters."""

    SELECTORS = ("predict", "random", "uniform", "probe", "ress")

    def __init__(self, frames: int, tokens_per_frame: int, special_per_frame: int, heads: int,
                 head_dim: int, block: int, dtype: str, rho: float, tau: float, head_density=None,
                 device: str | torch.device = "cuda", selector: str = "predict", seed: int = 0,
                 stride: int = 4, rounds: int = 8):
        """selector: how the kept blocks are chosen -- "predict" (pooled softmax and the dual
        threshold), "random" (k_h blocks uniformly at random, keyed by `seed`), "uniform"
        (every `stride`-th block), "probe" (the k_h blocks of highest mean-query score) or
        "ress" (the k_h blocks by drift score, refined by up to `rounds` restoration swaps)."""
        if selector not in self.SELECTORS:
            raise ValueError(f"selector must be one of {self.SELECTORS}")
        self.layout = _lib.make_layout(frames, tokens_per_frame, special_per_frame, heads, head_dim, block, dtype)
        self.dtype = dtype
        self.selector, self.seed, self.stride, self.rounds = selector, int(seed), int(stride), int(rounds)
        self.rho, self.tau = float(rho), float(tau)
        self.head_density = None if head_density is None else [float(x) for x in head_density]
        self.device = torch.device(device)
        self.B = _lib.bsa_num_blocks(self.layout)
        self.ws_bytes = _lib.bsa_workspace_size(self.layout)
        F, T, S, H, d = frames, tokens_per_frame, special_per_frame, heads, head_dim
        self.N, self.Np, self.H, self.d = F * T, F * (T - S), H, d
        B, dev = self.B, self.device
        words = (B + 31) // 32
        self.buf = Buffers(
            pq=torch.empty((H, B, d), dtype=torch.float32, device=dev),
            pk=torch.empty((H, d, B), dtype=torch.float32, device=dev),   # dimension-major
            mask_bits=torch.empty((H, B, words), dtype=torch.int32, device=dev),
            kv_idx=torch.empty((H, B, B), dtype=torch.int16, device=dev),
            kv_cnt=torch.empty((H, B), dtype=torch.int32, device=dev),
            # 1024-byte alignment for the TMA tiles: over-allocate and offset
            workspace=torch.empty(max(self.ws_bytes, 1) + 1024, dtype=torch.uint8, device=dev),
            out=torch.empty((self.N, H, d), dtype=_TORCH_DTYPE[dtype], device=dev),
            status=torch.zeros(1, dtype=torch.int32, device=dev),
        )
        # pooled V, dimension-major [H, d, B], and the Gram-matrix workspace of the drift-score selector
        self.pv = torch.empty((H, d, B), dtype=torch.float32, device=dev) if selector == "ress" else None
        self.ress_ws_bytes = _lib.bsa_ress_workspace_size(self.layout) if selector == "ress" else 0
        self.ress_ws = torch.empty(max(self.ress_ws_bytes, 1), dtype=torch.uint8, device=dev) if selector == "ress" else None
        base = self.buf.workspace.data_ptr()
        self.ws_ptr = (base + 1023) // 1024 * 1024 if self.ws_bytes else 0

    @classmethod
    def for_workload(cls, w, head_density=None, device="cuda") -> "BlockSparseLayer":
        return cls(w.frames, w.tokens_per_frame, w.layer_special, w.heads, w.head_dim, w.block,
                   w.dtype, w.rho, w.tau, head_density, device, w.selector, w.seed, w.stride, w.rounds)

    # individual steps -------------------------------------------------------------
    def predict(self, q: torch.Tensor, k: torch.Tensor, stream: int | None = None, v: torch.Tensor | None = None) -> None:
        """Block selection from Q and K (and V for the drift-score selector)."""
        st = self._stream(stream)
        b = self.buf
        if self.selector in ("predict", "probe", "ress"):
            _lib.bsa_pool_qk(self.layout, q.data_ptr(), k.data_ptr(), b.pq.data_ptr(), b.pk.data_ptr(),
                             b.status.data_ptr(), st)
        self._select(st, v)

    def _select(self, st, v: torch.Tensor | None = None) -> None:
        """The block selection step, from the pooled means already in pq / pk (the drift-score
        selector also pools v)."""
        b = self.buf
        args = (b.mask_bits.data_ptr(), b.kv_idx.data_ptr(), b.kv_cnt.data_ptr(), b.status.data_ptr(), st)
        if self.selector == "ress":
            if v is None:
                raise ValueError("the drift-score selector needs v")
            _lib.bsa_pool_v(self.layout, v.data_ptr(), self.pv.data_ptr(), b.status.data_ptr(), st)
            _lib.bsa_ress_mask(self.layout, b.pq.data_ptr(), b.pk.data_ptr(), self.pv.data_ptr(), self.rho,
                               self.head_density, self.rounds, self.ress_ws.data_ptr(), self.ress_ws_bytes, *args)
        elif self.selector == "predict":
            _lib.bsa_predict_mask(self.layout, b.pq.data_ptr(), b.pk.data_ptr(), self.rho, self.tau,
                                  self.head_density, *args)
        elif self.selector == "random":
            _lib.bsa_random_mask(self.layout, self.rho, self.head_density, self.seed, *args)
        elif self.selector == "uniform":
            _lib.bsa_uniform_mask(self.layout, self.stride, *args)
        else:
            _lib.bsa_probe_mask(self.layout, b.pq.data_ptr(), b.pk.data_ptr(), self.rho, self.head_density, *args)

    def partials(self) -> Buffers:
        """The layer's buffers, with the fp32 partials of the step-by-step path allocated."""
        b = self.buf
        if b.o_pp is None:
            H, d, dev = self.H, self.d, self.device
            b.o_pp = torch.empty((self.Np, H, d), dtype=torch.float32, device=dev)
            b.lse_pp = torch.empty((H, self.Np), dtype=torch.float32, device=dev)
            b.o_ps = torch.empty((self.Np, H, d), dtype=torch.float32, device=dev)
            b.lse_ps = torch.empty((H, self.Np), dtype=torch.float32, device=dev)
        return b

    def attend(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream: int | None = None,
               out: torch.Tensor | None = None) -> torch.Tensor:
        st = self._stream(stream)
        b = self.partials()
        o = self._out(out)
        qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
        _lib.bsa_pack_qkv(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.status.data_ptr(), st)
        _lib.bsa_special_dense(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, o.data_ptr(),
                               b.o_ps.data_ptr(), b.lse_ps.data_ptr(), b.status.data_ptr(), st)
        _lib.bsa_block_sparse_attn(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.kv_idx.data_ptr(),
                                   b.kv_cnt.data_ptr(), b.o_pp.data_ptr(), b.lse_pp.data_ptr(),
                                   b.status.data_ptr(), st)
        _lib.bsa_merge(self.layout, b.o_pp.data_ptr(), b.lse_pp.data_ptr(), b.o_ps.data_ptr(),
                       b.lse_ps.data_ptr(), o.data_ptr(), b.status.data_ptr(), st)
        return o

    def attend_fused(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     stream: int | None = None) -> torch.Tensor:
        """Steps 4-6 with the patch rows in one pass (bf16): pack, special rows, fused patch rows."""
        st = self._stream(stream)
        b = self.buf
        qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
        _lib.bsa_pack_qkv(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.status.data_ptr(), st)
        _lib.bsa_special_dense(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.out.data_ptr(),
                               None, None, b.status.data_ptr(), st)
        _lib.bsa_block_sparse_attn_fused(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes,
                                         b.kv_idx.data_ptr(), b.kv_cnt.data_ptr(), b.out.data_ptr(),
                                         b.status.data_ptr(), st)
        return b.out

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream: int | None = None,
                fused: bool | None = None, out: torch.Tensor | None = None,
                kernel_events=None) -> torch.Tensor:
        """The whole layer: [N, H, d] tensors in the layer dtype, on this device. bf16 layers
        use the fused patch-row pass unless fused=False. The result goes to `out` when given
        (an [N, H, d] contiguous tensor of the layer dtype), else to the layer's own buffer.
        kernel_events: optional pair of CUDA events recorded on the calling stream right
        before and after the patch-row attention launch (to time that kernel in place)."""
        if fused is None:
            fused = self.dtype == "bf16"
        if not fused:
            self.predict(q, k, stream, v)
            return self.attend(q, k, v, stream, out)
        st = self._stream(stream)
        b = self.buf
        o = self._out(out)
        qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
        # packing and pooling in one pass over Q, K, V; then mask, special rows, patch rows.
        # (Running the special rows on a second stream next to the mask and the patch rows
        # was measured slower: both attention passes are compute-bound and share the SMs.)
        if self.selector in ("predict", "probe", "ress"):
            _lib.bsa_pack_pool_qkv(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.pq.data_ptr(),
                                   b.pk.data_ptr(), b.status.data_ptr(), st)
        else:   # the selection reads no pooled means
            _lib.bsa_pack_qkv(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, b.status.data_ptr(), st)
        self._select(st, v)
        _lib.bsa_special_dense(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes, o.data_ptr(),
                               None, None, b.status.data_ptr(), st)
        main = None
        if kernel_events is not None:
            main = torch.cuda.current_stream(self.device) if stream is None else torch.cuda.ExternalStream(stream)
            kernel_events[0].record(main)
        _lib.bsa_block_sparse_attn_fused(self.layout, qp, kp, vp, self.ws_ptr, self.ws_bytes,
                                         b.kv_idx.data_ptr(), b.kv_cnt.data_ptr(), o.data_ptr(),
                                         b.status.data_ptr(), st)
        if kernel_events is not None:
            kernel_events[1].record(main)
        return o

    def check_status(self, stream: int | None = None) -> int:
        return _lib.bsa_check_status(self.buf.status.data_ptr(), self._stream(stream))

    # helpers ----------------------------------------------------------------------
    def _out(self, out):
        b = self.buf
        if out is None:
            return b.out
        if (out.shape != b.out.shape or out.dtype != b.out.dtype or out.device != b.out.device
                or not out.is_contiguous()):
            raise ValueError(f"out must be a contiguous {tuple(b.out.shape)} {b.out.dtype} tensor on {b.out.device}")
        return out

    def _stream(self, stream):
        return torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream

    def selected(self):
        """Kept-block mask [H, B, B] (numpy bool, host) from the mask bits."""
        import numpy as np
        words = self.buf.mask_bits.cpu().numpy().view(np.uint32)
        bits = np.unpackbits(words.view(np.uint8), axis=-1, bitorder="little")
        return bits[..., :self.B].astype(bool)


class AttentionBlock:
    """The projections around one attention layer of the aggregator: x [N, C] -> QKV projection
    -> attention (global block-sparse `layer`, or frame-wise when layer is None) -> output
    projection -> y [N, C] (bf16). Weights are device tensors: w_qkv [3C, C], b_qkv [3C] fp32 or
    None, w_o [C, C], b_o [C] fp32 or None."""

    def __init__(self, frames: int, tokens_per_frame: int, special_per_frame: int, heads: int, head_dim: int,
                 w_qkv, b_qkv, w_o, b_o, layer: "BlockSparseLayer | None" = None, device="cuda"):
        self.layout = _lib.make_layout(frames, tokens_per_frame, special_per_frame, heads, head_dim,
                                       layer.layout.block if layer is not None else 128, "bf16")
        self.w_qkv, self.b_qkv, self.w_o, self.b_o = w_qkv, b_qkv, w_o, b_o
        self.layer = layer
        self.device = torch.device(device)
        N = frames * tokens_per_frame
        shape = (N, heads, head_dim)
        self.q, self.k, self.v, self.o = (torch.empty(shape, dtype=torch.bfloat16, device=self.device)
                                          for _ in range(4))
        self.y = torch.empty((N, heads * head_dim), dtype=torch.bfloat16, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.frame_ws_bytes = _lib.bsa_frame_workspace_size(self.layout) if layer is None else 0
        self.frame_ws = torch.empty(self.frame_ws_bytes + 1024, dtype=torch.uint8, device=self.device)
        self.frame_ws_ptr = (self.frame_ws.data_ptr() + 1023) // 1024 * 1024

    def forward(self, x: torch.Tensor, stream: int | None = None) -> torch.Tensor:
        st = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        s = self.status.data_ptr()
        ptr = (lambda t: 0 if t is None else t.data_ptr())
        _lib.bsa_qkv_project(self.layout, x.data_ptr(), self.w_qkv.data_ptr(), ptr(self.b_qkv), self.q.data_ptr(),
                             self.k.data_ptr(), self.v.data_ptr(), s, st)
        if self.layer is None:
            _lib.bsa_pack_frames(self.layout, self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                 self.frame_ws_ptr, self.frame_ws_bytes, s, st)
            _lib.bsa_frame_attention(self.layout, self.frame_ws_ptr, self.frame_ws_bytes, self.o.data_ptr(), s, st)
        else:
            self.layer.forward(self.q, self.k, self.v, stream=st, out=self.o)
        _lib.bsa_out_project(self.layout, self.o.data_ptr(), self.w_o.data_ptr(), ptr(self.b_o), self.y.data_ptr(),
                             s, st)
        return self.y

    def check_status(self, stream: int | None = None) -> int:
        st = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        code = _lib.bsa_check_status(self.status.data_ptr(), st)
        if self.layer is not None:
            code = code or self.layer.check_status(stream)
        return code


def to_device(x, dtype: str, device="cuda") -> torch.Tensor:
    """Storage array from synth (uint16 bf16 bits or float32) -> device tensor of the layer dtype."""
    import numpy as np
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device)
