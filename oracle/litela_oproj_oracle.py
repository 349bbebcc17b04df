"""fp64 CPU oracle for LiteLA followed by the attention block's output projection.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module: only the test-suite, the smoke check and the benchmark's CPU leg may.  It shares no
code with the CUDA library.

What it computes
----------------
In Sana's linear DiT block, LiteLA sits between the qkv projection and the output
projection (Sana explainer, section "What LiteLA actually computes"); the FLOP ledger of
section "Two levers" counts "qkv + out proj" as 4 N d^2 multiply-adds per layer, i.e. the out
projection is one dense d x d linear map of every token's hidden vector (d = H * d_h, the
heads' outputs side by side, head-major).  Reading where the pages are silent: the map is a
linear layer in PyTorch's convention, y = x W^T + b, with W [C_out, C_in] (C_in = H * d_h)
and an optional bias b [C_out]; x is LiteLA's output.  The oracle evaluates it exactly as
written, in fp64, on the exactly decoded bf16 inputs and weights:

    y[b, n, o] = sum_{h, c} x[b, n, h, c] * W[o, h * d_h + c]  (+ bias[o])
    x          = LiteLA (the quadratic form of oracle/litela_oracle.py)

`linear` is the projection alone on a given bf16 input (the second step of the unfused
chain).  No blocking, fusion or reordering: one library matmul per (batch).

Parity status: linear and lite_la_oproj (non-causal and block-causal) are pinned by
tests/test_oracle_oproj_pins.py: an exact rational route (the pages' padded-state form, then
the projection as explicit sums of products) on tiny shapes, W = identity giving LiteLA's
output itself, a head permutation applied to q, k, v and to W's column blocks leaving y
unchanged, linearity in W and the bias.
"""
from __future__ import annotations

import numpy as np

from .litela_oracle import decode_bf16, lite_la_block_causal_fwd, lite_la_fwd

__all__ = ["linear", "lite_la_oproj"]


def linear(x: np.ndarray, w_bits: np.ndarray, C_out: int, C_in: int, bias=None) -> np.ndarray:
    """y = x W^T + b in fp64.  x: float64 [..., C_in] (or bf16 bit patterns, uint16);
    w_bits: bf16 bits [C_out, C_in]; bias: float [C_out] or None.  Returns float64 [..., C_out]."""
    x = decode_bf16(x) if np.asarray(x).dtype == np.uint16 else np.asarray(x, dtype=np.float64)
    w = decode_bf16(np.asarray(w_bits).reshape(C_out, C_in))
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y


def lite_la_oproj(qkv_bits: np.ndarray, w_bits: np.ndarray, B: int, N: int, H: int, d: int, C_out: int,
                  eps: float, bias=None, tokens_per_block: int | None = None, rows=None) -> np.ndarray:
    """LiteLA on packed bf16 qkv bits [B, N, 3*H*d] (non-causal, or block-causal with
    tokens_per_block), then the output projection W (bf16 bits [C_out, H*d]) and bias.
    Returns float64 [B, len(rows), C_out] (all N tokens when rows is None)."""
    if tokens_per_block:
        x = lite_la_block_causal_fwd(qkv_bits, B, N, H, d, eps, tokens_per_block, rows=rows)
    else:
        x = lite_la_fwd(qkv_bits, B, N, H, d, eps, rows=rows)
    R = x.shape[1]
    return linear(x.reshape(B, R, H * d), w_bits, C_out, H * d, bias)
