"""SALS latent-space sparse attention decode for B200 (sm_100a).

The compute path is the CUDA library ``csrc/libsalsc.so`` behind the C ABI in
``include/salsc.h``; :mod:`latent_space_sparse_b200.salsc` is its thin ctypes
binding.  ``workloads`` and ``synth`` hold the decode shapes and the seeded
synthetic input generators.
"""
__all__ = ["workloads", "synth", "salsc"]
