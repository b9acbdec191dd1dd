"""ctypes loader for libfoursight.so and the declarations of its C ABI (include/foursight.h).

The library is built in place by ``nvfp4_w4a4_gemm_fs_b200.build``.  Loading fails loudly when
it is missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfoursight.so")

FS_OK, FS_ERR_INVALID_ARGUMENT, FS_ERR_UNSUPPORTED, FS_ERR_CUDA, FS_ERR_RANGE, FS_ERR_TIMEOUT = range(6)
FS_DTYPE_BF16, FS_DTYPE_F32 = 0, 1
FS_RESIDUAL, FS_KEY_M2, FS_GAIN_EXACT, FS_OUT_BF16, FS_PATH_TENSOR, FS_PATH_DECODE = 1, 2, 4, 8, 16, 32
FS_FAULT_NO_COPIES, FS_COMPACT_K = 64, 128

P = C.c_void_p
i32, i64, u32, f32 = C.c_int32, C.c_int64, C.c_uint32, C.c_float

# name -> (restype, argtypes); mirrors include/foursight.h
SIGNATURES = {
    "fs_status_string": (C.c_char_p, [C.c_int]),
    "fs_last_error": (C.c_char_p, []),
    "fs_version": (C.c_char_p, []),
    "fs_side_cols": (i32, [i32]),
    "fs_compact_cols": (i32, [i32, i32]),
    "fs_sf_bytes": (i64, [i64, i32]),
    "fs_grouped_rows": (i64, [i64, i32]),
    "fs_channel_stats": (C.c_int, [P, i32, i64, i32, i64, i32, P, P, P, P, P, P]),
    "fs_stats_check": (C.c_int, [P, i32, P]),
    "fs_select_topk": (C.c_int, [i32, i32, P, P, P, P, P, i32, u32, P, P, P, i32, P]),
    "fs_prepare_weights": (C.c_int, [P, i32, i32, i32, i64, P, i32, u32, P, P, P, P, P, P, P]),
    "fs_quantize_splice": (C.c_int, [P, i32, i64, i32, i64, P, i32, P, u32, P, P, P, P]),
    "fs_quantize_splice_grouped": (C.c_int, [P, i32, i32, P, i64, i32, i64, P, i32, P, u32, P, P, P, P]),
    "fs_quantize_splice_stats": (C.c_int, [P, i32, i64, i32, i64, P, i32, P, u32, P, P, P, i32, P, P, P, P, P, P]),
    "fs_plan_create": (C.c_int, [C.POINTER(P), i32, i32, i32, u32]),
    "fs_plan_destroy": (C.c_int, [P]),
    "fs_plan_check": (C.c_int, [P, P]),
    "fs_splice_gemm": (C.c_int, [P, i64, i32, P, P, P, P, P, P, P, P, i64, P]),
    "fs_splice_gemm_segmented": (C.c_int, [P, i64, i32, P, P, P, P, P, P, i32, P, P, P, i64, P]),
    "fs_splice_gemm_grouped": (C.c_int, [P, i32, P, i64, i32, P, P, P, P, P, P, P, P, i64, P]),
    "fs_decode_splice_gemm": (C.c_int, [P, i64, i32, P, i64, P, P, u32, P, P, P, i32, P, P, P, i64, P]),
    "fs_seq_filter": (C.c_int, [P, i64, P, i32, i32, f32, i32, i32, i32, P, P, P, P, P, P]),
    "fs_splice_gemm_noalloc": (C.c_int, [i32, i32, u32, i64, i32, P, P, P, P, P, P, P, P, i64, i32, P]),
    "fs_gemm_bf16": (C.c_int, [P, i64, i32, i32, P, i64, P, i64, P, P, i64, P]),
    "fs_transpose_bf16": (C.c_int, [i64, i64, P, i64, P, i64, P]),
    "fs_ste_backward_work_bytes": (i64, [i64, i32, i32]),
    "fs_ste_backward": (C.c_int, [P, i64, i32, i32, P, i64, P, i64, P, i64, P, i64, P, i64, P, i64, P]),
    "fs_grpo_objective": (C.c_int, [P, P, i64, P, i32, i32, P, f32, P, P, P, i64, P]),
    "fs_k3_work_bytes": (i64, [i32]),
    "fs_k3_kl": (C.c_int, [P, P, i64, P, i32, i32, P, P, P, P]),
}

_lib = None


def load() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m nvfp4_w4a4_gemm_fs_b200.build` "
                              "(the SpliceGEMM path has no CPU fallback)")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class FoursightError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        self.status = status
        name = lib.fs_status_string(status).decode()
        detail = lib.fs_last_error().decode()
        super().__init__(f"{where}: {name}: {detail}")


def check(status: int, where: str) -> None:
    if status != FS_OK:
        raise FoursightError(status, where)
