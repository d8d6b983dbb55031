"""B200-native locality-constrained block-sparse causal attention (LCSA).

The package holds the CUDA sources of the hot path (``csrc/``), the build step
that compiles them into ``liblcsa.so`` and a thin ctypes binding
(``diffusion_vsr_b200.lcsa``).  Importing the package loads nothing; the
library is loaded on first use of the binding and fails loudly if missing.
"""

__all__ = ["workloads"]
