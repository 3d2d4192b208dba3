"""B200-native (sm_100a) CUDA library for OAL causal grouped positive-quadratic attention.

``positive_quadratic_b200.oal`` is the Python binding of the C ABI in include/oal.h;
``positive_quadratic_b200.inputs`` generates the seeded synthetic workloads;
``positive_quadratic_b200.build`` compiles liboal.so; ``positive_quadratic_b200.seqpar``
splits one long prefill over ranks.  Submodules are imported on demand so
that importing the package needs neither torch nor a GPU.
"""
__all__ = ["oal", "inputs", "build", "seqpar"]
