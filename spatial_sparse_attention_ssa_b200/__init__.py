"""Spatial sparse attention (SSA) over sparse 3D voxel tokens, for NVIDIA B200 (sm_100a).

The compute runs in libssa.so (hand-written CUDA, C ABI in include/ssa.h);
`ssa` is its thin ctypes binding and `workloads` the seeded synthetic inputs.
"""
__all__ = ["ssa", "workloads"]
