"""Workload table for the block-sparse global attention layer.

Each workload is one global-attention layer of a VGGT-style multi-view geometry
transformer: F frames, each with P patch tokens and S special tokens (1 camera +
4 register), H heads of width d, and the block-selection hyper-parameters b
(block size), rho (sparsity floor) and tau (CDF coverage) named in
"Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers",
section 损失函数 / 训练策略 (the only tunables are tau, rho and b).

Shapes follow that page's workloads: 518x518 input -> 37x37 = 1369 patches per
frame; 294x518 input -> 21x37 = 777 patches per frame.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    frames: int            # F
    patch_per_frame: int   # P
    special_per_frame: int  # S (prefix of each frame)
    heads: int             # H
    head_dim: int          # d
    block: int             # b
    rho: float             # sparsity floor: k = floor(B (1 - rho))
    tau: float             # CDF coverage threshold
    dtype: str             # "f32" or "bf16"
    planting: str          # "tiny" (permuted cross-frame copies) or "five_percent"
    head_budgets: bool = False  # per-head densities from capped water-filling
    seed: int = 0
    # block selector: "predict" (pooled softmax + dual threshold), "random" (k_h uniformly
    # random blocks), "uniform" (every `stride`-th block), "probe" (mean-query Top-K), "ress"
    # (drift scores with restoration rounds)
    selector: str = "predict"
    stride: int = 4
    rounds: int = 8   # restoration rounds of the drift-score selector
    # the ablation without the dense special path: the layer reads the S special tokens of
    # every frame as patch tokens (pooled and sparsified with them)
    sparse_specials: bool = False
    # what one step runs: "global" (the block-sparse global attention layer), "frame" (the
    # frame-wise dense attention), "block" / "frame_block" (that attention between the QKV and
    # output projections, from tokens x [N, C] to y [N, C])
    kind: str = "global"

    @property
    def layer_special(self) -> int:
        """Special tokens per frame as the layer reads them."""
        return 0 if self.sparse_specials else self.special_per_frame

    def layer_view(self) -> "Workload":
        """The workload as the layer reads it (the inputs are drawn from `self`): with
        sparse_specials every token of a frame is a patch token."""
        if not self.sparse_specials:
            return self
        return replace(self, patch_per_frame=self.tokens_per_frame, special_per_frame=0, sparse_specials=False)

    @property
    def tokens_per_frame(self) -> int:
        return self.patch_per_frame + self.special_per_frame

    @property
    def n_tokens(self) -> int:
        return self.frames * self.tokens_per_frame

    @property
    def n_patch(self) -> int:
        return self.frames * self.patch_per_frame

    @property
    def n_special(self) -> int:
        return self.frames * self.special_per_frame

    @property
    def n_blocks(self) -> int:
        return -(-self.n_patch // self.block)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny", 2, 64, 5, 2, 64, 16, 0.5, 0.9, "f32", "tiny")
VGGT518 = Workload("vggt518", 10, 1369, 5, 16, 64, 64, 0.5, 0.9, "bf16", "five_percent")
SWEEP_R50 = Workload("sweep_r50", 32, 777, 5, 16, 64, 64, 0.5, 0.95, "bf16", "five_percent")
SWEEP_R75 = SWEEP_R50.with_(name="sweep_r75", rho=0.75)
SWEEP_R90 = SWEEP_R50.with_(name="sweep_r90", rho=0.9)
# tau is not given for the per-head-budget workload; tau = 0 makes each head keep
# exactly its budgeted k_h blocks so that the layer density is the budget (1 - rho).
PERHEAD100 = Workload("perhead100", 100, 777, 5, 16, 64, 128, 0.75, 0.0, "bf16",
                      "five_percent", head_budgets=True)
PERHEAD100_TAU95 = PERHEAD100.with_(name="perhead100_tau95", tau=0.95)
LONG500 = Workload("long500", 500, 777, 5, 16, 64, 128, 0.9, 0.95, "bf16", "five_percent")

# Non-degenerate variants: with the near-uniform pooled distributions of this
# generator, tau >= 0.9 keeps almost every block; tau = 0 exercises the top-k floor.
TINY_TAU0 = TINY.with_(name="tiny_tau0", tau=0.0)
SWEEP_TAU0 = SWEEP_R75.with_(name="sweep_tau0", tau=0.0)

# Ablation rows of "Block-Sparse Global Attention for Efficient Multi-View Geometry
# Transformers", 消融实验 (图 10), at the 100-frame shape: CDF threshold alone (no Top-K
# floor: rho = 1, k = 0; tau = 0.25 keeps about a quarter of the blocks on these inputs),
# without the dense special path, and random selection with and without it (same k_h).
CDF_ONLY100 = PERHEAD100.with_(name="cdf_only100", head_budgets=False, rho=1.0, tau=0.25)
NOSPECIAL100 = PERHEAD100.with_(name="nospecial100", sparse_specials=True)
RANDOM100 = PERHEAD100.with_(name="random100", selector="random")
RANDOM_NOSPECIAL100 = PERHEAD100.with_(name="random_nospecial100", selector="random", sparse_specials=True)
# Key selectors of "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
# Transformers", 四、1.: fixed-stride uniform sampling (every 4th block: 25% kept) and the
# query-probe Top-K (the per-head budgets of the 100-frame workload).
UNIFORM100 = PERHEAD100.with_(name="uniform100", selector="uniform", stride=4, head_budgets=False)
PROBE100 = PERHEAD100.with_(name="probe100", selector="probe")
# Drift-score selection of "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers"
# (技术框架 / 关键设计), with the per-head budgets of the 100-frame workload.
RESS100 = PERHEAD100.with_(name="ress100", selector="ress")

# The steps on either side of the layer ("Block-Sparse Global Attention...", 研究背景与动机: the
# aggregator alternates frame-wise and global attention; "SAF3R...", 图2): frame-wise dense
# attention over the 782 tokens of each frame as a second workload, and whole blocks with the
# QKV and output projections (random-init weights).
FRAME100 = PERHEAD100.with_(name="frame100", kind="frame", head_budgets=False)
BLOCK100 = PERHEAD100.with_(name="block100", kind="block")
FRAME_BLOCK100 = PERHEAD100.with_(name="frame_block100", kind="frame_block", head_budgets=False)

ALL = {w.name: w for w in (FRAME100, BLOCK100, FRAME_BLOCK100, TINY, VGGT518, SWEEP_R50, SWEEP_R75, SWEEP_R90, PERHEAD100,
                           PERHEAD100_TAU95, LONG500, TINY_TAU0, SWEEP_TAU0, CDF_ONLY100, NOSPECIAL100,
                           RANDOM100, RANDOM_NOSPECIAL100, UNIFORM100, PROBE100, RESS100)}
