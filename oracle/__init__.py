"""fp64 CPU oracle of the block-sparse global attention layer (test infrastructure only).

Only tests, the package smoke check and the benchmark's CPU-baseline leg import
this package; the CUDA library never does.
"""
from .bsa_oracle import *  # noqa: F401,F403
from .bsa_oracle import Layout, MaskResult, LayerResult  # noqa: F401
