"""Absorbed Multi-head Latent Attention (MLA) decode for B200 (sm_100a).

The compute path lives in the CUDA library ``libmla.so`` (sources in
``csrc/``, C-ABI declared in ``include/mla.h``); ``binding`` marshals torch
tensors into it.  ``workload`` holds the seeded synthetic inputs.
Importing this package does not load the CUDA library; ``binding.load()``
does, and raises if it is missing.
"""

__all__ = ["binding", "workload"]
