"""B200-native contextual token sparsity: block scoring, selection and
permutation-free token movement on sm_100a.

The compute lives in ``liblemo.so`` (CUDA C++ for sm_100a, C ABI declared in
``include/lemo.h``).  ``contextual_token_sparsity_b200.lemo`` is the thin
ctypes binding with the same entry-point names; ``synth`` draws the seeded
synthetic inputs.  The binding loads the library on first use and raises if
it is missing; there is no CPU fallback.
"""

__all__ = ["lemo", "synth"]
