"""Block-sparse global attention for multi-view geometry transformers on NVIDIA B200.

The compute lives in libbsa.so (C ABI in include/bsa.h, CUDA kernels for sm_100a).
`_lib` binds it with ctypes, `layer.BlockSparseLayer` runs one layer through it, and
`configs` / `synth` describe the workloads and draw their seeded inputs. Importing the
package does not load the library; the first library call does, and fails loudly when the
library has not been built.
"""
__all__ = ["configs", "synth"]
