"""Transfers between numpy arrays (oracle side) and CUDA tensors (library side) for the
parity tests. Bit patterns move unchanged; no arithmetic happens here."""
import numpy as np
import torch

DEV = "cuda"


def bf16_from_bits(bits):
    """numpy uint16 bf16 bit patterns -> torch.bfloat16 CUDA tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(DEV)


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def f16_from_values(a):
    """float64 values that are exactly binary16 -> torch.float16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64).astype(np.float16)).to(DEV)


def bits16(t):
    """torch 16-bit tensor -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f16_bits_of(values):
    """float64 binary16 values (oracle) -> uint16 bit patterns."""
    return np.asarray(values, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_to_f64(t):
    u = bits16(t).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def to_np(t):
    return t.detach().cpu().numpy()
