"""The C-ABI library loads, exports every symbol include/foursight.h declares, and rejects bad
arguments on the host before touching the GPU (no compute calls here)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "foursight.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fs_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from nvfp4_w4a4_gemm_fs_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from nvfp4_w4a4_gemm_fs_b200 import build
        build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    from nvfp4_w4a4_gemm_fs_b200 import _lib
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def _declared_arity():
    """Parameter count of every function the header declares (FS_API prototypes)."""
    src = open(os.path.join(ROOT, "include", "foursight.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for name, params in re.findall(r"\b(fs_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    from nvfp4_w4a4_gemm_fs_b200 import _lib
    arity = _declared_arity()
    assert len(arity) >= 15
    for name, n in arity.items():
        assert len(_lib.SIGNATURES[name][1]) == n, f"{name}: header {n} parameters, binding {len(_lib.SIGNATURES[name][1])}"


def test_status_strings_and_sizes(lib):
    assert lib.fs_status_string(0) == b"FS_OK"
    assert lib.fs_status_string(5) == b"FS_ERR_TIMEOUT"
    assert lib.fs_side_cols(64) == 64 and lib.fs_side_cols(65) == 80 and lib.fs_side_cols(0) == 0
    assert lib.fs_sf_bytes(8192, 4096) == 8192 * 256
    assert lib.fs_sf_bytes(1, 64) == 128 * 4
    assert lib.fs_sf_bytes(129, 80) == 256 * 8
    assert lib.fs_grouped_rows(100, 4) >= 100 + 4 * 127


def test_host_validation_rejects_bad_arguments(lib):
    dummy = C.c_void_p(256)
    # K not a multiple of 8
    assert lib.fs_channel_stats(dummy, 0, 4, 12, 16, 1, dummy, dummy, dummy, dummy, dummy, None) == 1
    assert b"K" in lib.fs_last_error()
    # row_stride 0, bad dtype, null state
    assert lib.fs_channel_stats(dummy, 0, 4, 16, 16, 0, dummy, dummy, dummy, dummy, dummy, None) == 1
    assert lib.fs_channel_stats(dummy, 7, 4, 16, 16, 1, dummy, dummy, dummy, dummy, dummy, None) == 1
    assert lib.fs_channel_stats(dummy, 0, 4, 16, 16, 1, None, dummy, dummy, dummy, dummy, None) == 1
    # M == 0 is a no-op that succeeds without a GPU
    assert lib.fs_channel_stats(dummy, 0, 0, 16, 16, 1, dummy, dummy, dummy, dummy, dummy, None) == 0
    # select: p > K, p > 256
    assert lib.fs_select_topk(1, 64, dummy, dummy, dummy, dummy, dummy, 65, 0, dummy, dummy, dummy, 0, None) == 1
    assert lib.fs_select_topk(1, 4096, dummy, dummy, dummy, dummy, dummy, 300, 0, dummy, dummy, dummy, 0, None) == 1
    # quantise: K % 64, p without mask, misaligned X
    assert lib.fs_quantize_splice(dummy, 0, 4, 48, 48, None, 0, dummy, 0, dummy, dummy, None, None) == 1
    assert lib.fs_quantize_splice(dummy, 0, 4, 64, 64, None, 4, dummy, 0, dummy, dummy, dummy, None) == 1
    assert lib.fs_quantize_splice(C.c_void_p(258), 0, 4, 64, 64, None, 0, dummy, 0, dummy, dummy, None, None) == 1
    assert lib.fs_quantize_splice(dummy, 0, 0, 64, 64, None, 0, dummy, 0, dummy, dummy, None, None) == 0
    # weights: N == 0, missing alpha
    assert lib.fs_prepare_weights(dummy, 0, 0, 64, 64, None, 0, 0, dummy, dummy, dummy, None, dummy, dummy, None) == 1
    assert lib.fs_prepare_weights(dummy, 0, 4, 64, 64, None, 0, 0, dummy, dummy, dummy, None, dummy, None, None) == 1
    # an empty batch is a no-op that reads no operand (allocation-free entry: no plan needed)
    assert lib.fs_splice_gemm_noalloc(256, 512, 0, 0, 64, None, None, None, None, None, None, None, None, 256, 0,
                                      None) == 0
    assert lib.fs_splice_gemm(None, 0, 0, None, None, None, None, None, None, None, None, 256, None) == 1   # null plan
    # segmented GEMM: a plan is required before the segments are looked at
    seg = (C.c_int32 * 3)(0, 128, 256)
    assert lib.fs_splice_gemm_segmented(None, 8, 0, dummy, dummy, None, dummy, dummy, None, 2, seg, dummy, dummy, 256,
                                        None) == 1
    assert b"plan" in lib.fs_last_error()
    # filter: K1 < 1, rewards without G
    assert lib.fs_seq_filter(dummy, 64, None, 4, 64, -9.0, 0, 5, 0, None, None, dummy, dummy, dummy, None) == 1
    assert lib.fs_seq_filter(dummy, 64, None, 4, 64, -9.0, 3, 5, 3, dummy, dummy, dummy, dummy, dummy, None) == 1
    assert lib.fs_seq_filter(dummy, 64, None, 0, 64, -9.0, 3, 5, 0, None, None, dummy, dummy, dummy, None) == 0


def test_host_validation_of_the_later_entries(lib):
    """The grouped quantiser, the fused statistics + quantise pass, the fused decode GEMM and the
    selection refuse bad arguments on the host, before any device call."""
    dummy = C.c_void_p(256)
    # grouped quantise: E out of range, null offsets; no routed rows is a no-op
    assert lib.fs_quantize_splice_grouped(dummy, 0, 0, dummy, 8, 64, 64, None, 0, dummy, 0, dummy, dummy, None,
                                          None) == 1
    assert lib.fs_quantize_splice_grouped(dummy, 0, 257, dummy, 8, 64, 64, None, 0, dummy, 0, dummy, dummy, None,
                                          None) == 1
    assert lib.fs_quantize_splice_grouped(dummy, 0, 4, None, 8, 64, 64, None, 0, dummy, 0, dummy, dummy, None,
                                          None) == 1
    assert lib.fs_quantize_splice_grouped(dummy, 0, 4, dummy, 0, 64, 64, None, 0, dummy, 0, dummy, dummy, None,
                                          None) == 0
    # fused statistics + quantise: fp32 activations unsupported (2), row_stride 0, K % 64
    stats = [dummy] * 5
    assert lib.fs_quantize_splice_stats(dummy, 1, 4, 64, 64, None, 0, dummy, 0, dummy, dummy, None, 1, *stats,
                                        None) == 2
    assert lib.fs_quantize_splice_stats(dummy, 0, 4, 64, 64, None, 0, dummy, 0, dummy, dummy, None, 0, *stats,
                                        None) == 1
    assert lib.fs_quantize_splice_stats(dummy, 0, 4, 96, 96, None, 0, dummy, 0, dummy, dummy, None, 1, *stats,
                                        None) == 1
    # fused decode GEMM: a plan is required
    assert lib.fs_decode_splice_gemm(None, 4, 0, dummy, 64, None, dummy, 0, dummy, dummy, None, 1, None, dummy,
                                     dummy, 256, None) == 1
    # selection: K above 16384
    assert lib.fs_select_topk(1, 16416, dummy, dummy, dummy, dummy, dummy, 8, 0, dummy, dummy, dummy, 0, None) == 1
    # grouped GEMM: a plan is required; E must be positive
    assert lib.fs_splice_gemm_grouped(None, 4, dummy, 8, 0, dummy, dummy, None, dummy, dummy, None, dummy, dummy,
                                      256, None) == 1
