"""SpliceGEMM hot path of FourSight for NVIDIA B200 (sm_100a).

Python binding of the C ABI in ``include/foursight.h``: every function here only marshals
torch tensors into pointers, sizes and the current CUDA stream and calls the library of the
same name; all arithmetic runs in the hand-written CUDA kernels of ``csrc/``.
"""
from ._lib import (FS_COMPACT_K, FS_DTYPE_BF16, FS_DTYPE_F32, FS_FAULT_NO_COPIES, FS_GAIN_EXACT, FS_KEY_M2,  # noqa: F401
                   FS_OUT_BF16, FS_PATH_DECODE, FS_PATH_TENSOR, FS_RESIDUAL, FoursightError, load)
from .foursight import *  # noqa: F401,F403
