"""The hand-placed swizzles in shared memory against the TMA swizzle modes' definition.

A tensor map with SWIZZLE_128B (or 64B) stores the 16-byte granule at byte address a of a box
row at a ^ (((a >> 7) & 7) << 4) (or & 3): granule bits [4, 7) (or [4, 6)) XOR address bits
[7, 10) (or [7, 9)), of the absolute shared-memory address, so a buffer must start on a multiple
of the pattern's repeat (1024 or 512 bytes).  The kernels write such boxes by hand:
* the tensor-core GEMM's epilogue stages 32 x 32 output chunks for a TMA store: fp32 rows of 128
  bytes with chunk j of row r at j ^ (r & 7), bf16 rows of 64 bytes at j ^ ((r >> 1) & 3);
* the fused decode preparation writes the 16-row X box the MMA's 128-byte-swizzle descriptor
  reads: chunk c of row r at c ^ (r & 7).
Each placement must equal the definition, and each staging buffer must start on the repeat.
"""
import pytest


def tma_swizzle(addr: int, mode_bytes: int) -> int:
    bits = {128: 7, 64: 3, 32: 1}[mode_bytes]
    return addr ^ (((addr >> 7) & bits) << 4)


@pytest.mark.parametrize("row_bytes,mode,placement", [
    (128, 128, lambda r, j: 128 * r + ((j ^ (r & 7)) << 4)),            # fp32 output chunk
    (64, 64, lambda r, j: 64 * r + ((j ^ ((r >> 1) & 3)) << 4)),        # bf16 output chunk
])
def test_epilogue_staging_matches_the_store_maps_swizzle(row_bytes, mode, placement):
    for buf in range(0, 4 * 3 * 4096, 4096):                           # every staging buffer start
        assert buf % (8 * mode) == 0                                   # the pattern's repeat
        for r in range(32):
            for j in range(row_bytes // 16):
                assert buf + placement(r, j) == tma_swizzle(buf + row_bytes * r + 16 * j, mode)


def test_decode_x_box_matches_the_128_byte_swizzle():
    for r in range(16):
        for c in range(8):
            assert 128 * r + 16 * (c ^ (r & 7)) == tma_swizzle(128 * r + 16 * c, 128)


@pytest.mark.parametrize("BN,CG", [(256, 2), (256, 1), (128, 1)])
def test_staging_area_starts_on_the_repeat(BN, CG):
    """Stages are A (128 rows x 128 B), this CTA's B rows, SFA (128 x 16 B), SFB (BN x 16 B); the
    staging area follows STAGES of them from a 1024-byte-aligned base and holds 4 warps x buffers
    x 4096 bytes."""
    b_rows = BN // CG
    stage = 128 * 128 + b_rows * 128 + 128 * 16 + BN * 16
    stages = 5 if CG == 2 else (3 if BN == 256 else 4)
    assert stage % 1024 == 0 and (stages * stage) % 1024 == 0
