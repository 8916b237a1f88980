"""The benchmark's parity samples (bench.py): on CPU, with stand-ins for the device tensors
built from the oracle itself, a correct result reports agreement at rounding level and a
planted error shows up (no GPU needed)."""
import numpy as np
import pytest

import bench
import oracle
from oracle import layer_io
from view_transformers_b200 import configs, synth

torch = pytest.importorskip("torch")


class _Buf:
    pass


class _StandIn:
    """The two members of a layer that sample_parity reads: buf.out and selected()."""

    def __init__(self, out: np.ndarray, selected: np.ndarray):
        self.buf = _Buf()
        self.buf.out = torch.from_numpy(out.astype(np.float32))
        self._sel = selected

    def selected(self):
        return self._sel


@pytest.mark.parametrize("name", ["tiny", "tiny_tau0"])
def test_layer_parity_sample_agrees_and_catches_a_planted_error(name):
    w = configs.ALL[name]
    x = synth.make_inputs(w)
    keep = {}
    bench.oracle_layer_sample(w, x, budget_s=0.5, keep=keep)
    assert keep["rows"] and keep["mask"] is not None
    lay = oracle.Layout(w.frames, w.tokens_per_frame, w.layer_special, w.heads, w.head_dim, w.block)
    Q, K, V = (oracle.to_f64(a, w.dtype) for a in (x.q, x.k, x.v))
    full = oracle.layer_forward(Q, K, V, lay, keep["mask"].selected)
    rep = bench.sample_parity(torch, _StandIn(full, keep["mask"].selected), w, keep)
    assert rep["rel_l2"] < 1e-6 and rep["max_abs"] < 1e-5
    assert rep["mask"]["failed"] == 0 and rep["mask"]["rows"] == w.heads * lay.B
    # a wrong output value in a sampled row, and a wrong mask row
    rows, h, _ = keep["rows"][0]
    bad = full.copy()
    bad[rows[0], h, 0] += 1.0
    sel = keep["mask"].selected.copy()
    sel[0, 0] = ~sel[0, 0]
    rep = bench.sample_parity(torch, _StandIn(bad, sel), w, keep)
    assert rep["max_abs"] > 0.5
    assert rep["mask"]["failed"] >= 1


@pytest.mark.parametrize("kind", ["frame", "frame_block"])
def test_block_parity_sample_stages(kind):
    w = configs.ALL["frame_block100"].with_(name="fb3", frames=3, kind=kind)
    x = synth.make_inputs(w)
    bf = (lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16))
    t = {k_: bf(synth.decode(a, "bf16")) for k_, a in (("q", x.q), ("k", x.k), ("v", x.v))}
    H, d = w.heads, w.head_dim
    if kind == "frame_block":
        bi = synth.make_block_inputs(w)
        t["x"], t["w_qkv"], t["w_o"] = (bf(synth.decode(a, "bf16")) for a in (bi.x, bi.w_qkv, bi.w_o))
        t["b_qkv"], t["b_o"] = torch.from_numpy(bi.b_qkv), torch.from_numpy(bi.b_o)
        q, k, v = layer_io.qkv_project(t["x"].double().numpy(), t["w_qkv"].double().numpy(), bi.b_qkv, H, d)
        t["q"], t["k"], t["v"] = bf(q), bf(k), bf(v)
    o = layer_io.frame_attention(t["q"].double().numpy(), t["k"].double().numpy(), t["v"].double().numpy(),
                                 w.frames, w.tokens_per_frame)
    t["o"] = bf(o)
    if kind == "frame_block":
        t["y"] = bf(layer_io.out_project(t["o"].double().numpy(), t["w_o"].double().numpy(), bi.b_o))
    rep = bench.block_parity_sample(torch, w, t)
    stages = ("qkv_projection", "frame_attention", "out_projection") if kind == "frame_block" else ("frame_attention",)
    assert set(rep) == set(stages)
    for s in stages:   # the stand-ins are the oracle's values rounded to bf16
        assert rep[s]["rel_l2"] < 4e-3, (s, rep[s])
    t["o"] = t["o"] + 1.0   # every attention output off by one
    assert bench.block_parity_sample(torch, w, t)["frame_attention"]["max_abs"] > 0.5
