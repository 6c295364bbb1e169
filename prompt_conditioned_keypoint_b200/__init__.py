"""B200-native GKDT parameter-free detection head.

The head's steps run as CUDA kernels for sm_100a inside the C-ABI library
`libgkd.so` (declared in include/gkd.h). This package holds that library's
sources (csrc/), a thin ctypes binding with the same entry-point names
(`binding`), and the seeded synthetic-input generator (`synthetic`).
"""
