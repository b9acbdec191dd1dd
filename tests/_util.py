"""Shared helpers of the GPU tests: numpy <-> torch marshalling and oracle adapters."""
import numpy as np
import torch

from oracle import nvfp4


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def f32_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)


def mask_tensor(mask_u32: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(mask_u32, dtype=np.uint32).view(np.int32)).to(device)


def check_packed(packed, ref, rows, K, p):
    """Bit-exact comparison of a packed operand with the oracle's codes, scales and side values."""
    q = u8(packed.q)[:rows]
    assert np.array_equal(q, nvfp4.pack_codes(ref["codes"])), "E2M1 payload differs"
    sf = nvfp4.sf_from_tiled(u8(packed.sf), rows, K)
    assert np.array_equal(sf, ref["sf"].astype(np.uint8)), "block scales differ"
    tiled = u8(packed.sf)
    assert np.array_equal(tiled, nvfp4.sf_to_tiled(ref["sf"], K)), "tiled scale array (incl. padding) differs"
    if p:
        side = bf16_bits_of(packed.side)[:rows]
        key = "xs" if "xs" in ref else "ws"
        assert np.array_equal(side, nvfp4.bf16_bits(ref[key])), "side buffer differs"
