"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds none of LiteLA's arithmetic: it only draws and packs the bf16 qkv
buffers that both the CUDA path and the fp64 oracle then read.  Sana's real activations
need trained weights, so i.i.d. N(0, 1) values of Sana's shapes stand in for them.

Packed layout of one token row (the qkv projection's output): [q | k | v], each
head-major, i.e. element (b, n, h, c) of q/k/v sits at ((b*N + n)*3*H + {0,1,2}*H + h)*d + c.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = ["make_qkv", "to_bits", "pack_qkv", "config_seed", "WORKLOADS"]


# Sana's shapes for the LiteLA forward (heads of dim 32; hidden = heads * 32).
WORKLOADS = {
    "sana600m_512px": dict(B=1, N=16 * 16, H=36, d=32),
    "sana1600m_1024px": dict(B=2, N=32 * 32, H=70, d=32),
    "sana1600m_2048px": dict(B=2, N=64 * 64, H=70, d=32),
    "sana4800m_4096px": dict(B=2, N=128 * 128, H=70, d=32),
    "block_causal_16x1024": dict(B=1, N=16 * 1024, H=70, d=32, tokens_per_block=1024),
}


def config_seed(index: int, buffer: int = 0) -> int:
    """Seed of buffer `buffer` of workload `index` (0-based order of WORKLOADS):
    workload k uses 1000 + k; the 60 buffers of the 4096px workload use 4000 + i."""
    if buffer:
        return 4000 + buffer
    return 1000 + index


def make_qkv(B: int, N: int, H: int, d: int, seed: int, device="cpu",
             qk_shift: float = 0.0) -> torch.Tensor:
    """Packed bf16 qkv [B, N, 3*H*d] with i.i.d. N(0,1) entries drawn in float32 from a
    seeded torch generator on `device`, optionally shifting q and k (not v) by qk_shift
    before the bf16 cast (qk_shift = -1.5 gives the mostly-negative, sparse-ReLU input)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn((B, N, 3 * H * d), generator=g, dtype=torch.float32, device=device)
    if qk_shift:
        x[..., : 2 * H * d] += qk_shift
    return x.to(torch.bfloat16)


def to_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host uint16 numpy array."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def pack_qkv(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> torch.Tensor:
    """Pack float arrays q, k, v of shape [B, N, H, d] into a bf16 qkv tensor
    [B, N, 3*H*d] (values are rounded to bf16; exact for small dyadic values)."""
    q, k, v = (np.asarray(a, dtype=np.float32) for a in (q, k, v))
    B, N, H, d = q.shape
    x = np.stack([q, k, v], axis=2).reshape(B, N, 3 * H * d)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)
