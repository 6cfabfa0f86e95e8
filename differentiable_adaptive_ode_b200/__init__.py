"""B200-native record-and-replay discrete adjoint for ensembles of adaptive ODE solves.

The compute path is the CUDA library libgradsolve_b200.so (C ABI in include/gradsolve_b200.h);
`gradsolve` is its thin Python binding and `workloads` the seeded synthetic ensembles.
"""
__all__ = ["gradsolve", "workloads"]
