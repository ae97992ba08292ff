"""Packed 3D Gaussian Splatting forward+backward step for B200 (sm_100a).

The compute path is libss.so (hand-written CUDA, C ABI in include/ss.h);
`ss` is its ctypes binding, `scenes` the seeded synthetic workloads.
"""
