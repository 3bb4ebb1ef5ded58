"""B200-native routed-expert MoE prefill layer.

The layer (top-k routing over the experts, grouping of the token/expert pairs
by expert, gate/up projection over on-the-fly decoded 1-2-bit block weights,
SwiGLU, the decoded down projection and the routing-weighted combine in
selection order) runs in the CUDA kernels of ``librl_moe.so``; this package
only marshals arguments to that library (``api``) and generates seeded
synthetic inputs (``synth``).  Importing the package loads nothing; the first
call into ``api`` loads the shared library and raises if it is missing.
"""

__all__ = ["api", "synth"]
