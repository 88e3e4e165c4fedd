"""B200-native chunked H2O sparse-attention step.

The step (per chunk of T tokens): SDPA of the chunk against a C-slot KV cache
plus itself, per-slot attention-weight sums added to the H2O scores, and
eviction back to C slots -- "Learning how to Forget: Fine-tuning for
Long-Context Sparse Attention", paper page, sections "Improvements to
Heavy-Hitter Oracle (H2O)" and "Kernel Support Needs". The work runs in the
CUDA kernels of ``libh2o.so``; this package holds its ctypes binding
(``H2OCache``) and the seeded synthetic inputs (``synth``).
"""
from ._lib import (H2O_BF16, H2O_FP32, H2OError, lib)  # noqa: F401
from .cache import H2OCache  # noqa: F401
