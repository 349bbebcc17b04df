"""fp64 CPU oracle for the ELU+1 variant of kernelised linear attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module: only the test-suite may.  It shares no code with the CUDA library.

What it computes
----------------
The Sana tutorial page (aifetchly), in its linear-attention block, uses the feature map
phi(x) = ELU(x) + 1 (exp(x) for x <= 0, x + 1 for x > 0; strictly positive), scales phi(q)
by 1/sqrt(d), accumulates the context phi(K)^T V and the key sum sum_j phi(k_j), and divides
the numerator by the denominator clamped from below at 1e-6 instead of adding an eps.  Per
(batch, head), as a quadratic form (equal by associativity to the context route):

    w_ij  = (phi(q_i) / sqrt(d)) . phi(k_j)       (j over the keys query i sees)
    out_i = (sum_j w_ij v_j) / max(sum_j w_ij, clamp_min)

Block-causal masking is the same as for LiteLA (oracle/litela_oracle.py).  Readings where the
page is silent: ELU's alpha is 1 (PyTorch's default); inputs are the exactly decoded bf16 values.

Parity status: phi_elu1 and elu1_fwd are pinned by tests/test_oracle_elu_pins.py (closed
forms of phi, the context route evaluated independently, invariants, the clamp branch).
"""
from __future__ import annotations

import math

import numpy as np

from .litela_oracle import decode_bf16, unpack_qkv, visible_key_count

__all__ = ["phi_elu1", "elu1_rows", "elu1_fwd"]


def phi_elu1(x: np.ndarray) -> np.ndarray:
    """ELU(x) + 1 with alpha = 1: x + 1 for x > 0, exp(x) for x <= 0 (float64)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def elu1_rows(q_rows, k, v, clamp_min, n_visible=None):
    """Quadratic form for a set of queries of ONE (batch, head); q_rows [R, d], k, v [N, d]."""
    d = q_rows.shape[1]
    pq = phi_elu1(q_rows) / math.sqrt(d)
    pk = phi_elu1(k)
    w = pq @ pk.T
    if n_visible is not None:
        cols = np.arange(k.shape[0])[None, :]
        w = np.where(cols < np.asarray(n_visible)[:, None], w, 0.0)
    num = w @ v
    den = np.maximum(w.sum(axis=1, keepdims=True), clamp_min)
    return num / den


def elu1_fwd(qkv_bits, B: int, N: int, H: int, d: int, clamp_min: float = 1e-6,
             tokens_per_block: int | None = None, rows=None, chunk: int = 2048) -> np.ndarray:
    """ELU+1 linear attention on packed bf16 qkv bits [B, N, 3*H*d]; block-causal when
    tokens_per_block is given.  Returns float64 [B, len(rows), H, d]."""
    x = decode_bf16(np.asarray(qkv_bits).reshape(B, N, 3 * H * d))
    q, k, v = unpack_qkv(x, H, d)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    if tokens_per_block is not None and int(tokens_per_block) <= 0:
        raise ValueError("tokens_per_block must be positive")
    out = np.empty((B, rows.size, H, d))
    for b in range(B):
        for h in range(H):
            kk, vv = np.ascontiguousarray(k[b, :, h]), np.ascontiguousarray(v[b, :, h])
            for s in range(0, rows.size, chunk):
                r = rows[s:s + chunk]
                nv = None if tokens_per_block is None else visible_key_count(r, N, int(tokens_per_block))
                out[b, s:s + chunk, h] = elu1_rows(q[b, r, h], kk, vv, clamp_min, nv)
    return out
