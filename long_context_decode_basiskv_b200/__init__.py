"""BasisKV decode hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libbasiskv.so`` (hand-written CUDA behind a C ABI,
declared in ``include/basiskv.h``); ``binding`` marshals torch tensors into
that ABI.  ``workloads`` draws seeded synthetic decode steps.  Importing the
package does not load the CUDA library; ``binding.lib()`` does, and raises
if it is missing.
"""
__all__ = ["binding", "workloads"]
