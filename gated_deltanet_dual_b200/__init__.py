"""B200-native dual-stream Gated DeltaNet forward (clean causal stream + block-bidirectional
noisy stream), as a C-ABI CUDA library (libgdn_dual.so) with a thin Python binding.

Importing the package loads nothing; the library is loaded by the first binding call.
"""
from . import synth  # noqa: F401  (seeded input generator; no method arithmetic)

__all__ = ["synth", "binding", "build"]
