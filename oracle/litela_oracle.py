"""fp64 CPU oracle for the LiteLA forward pass (Sana's ReLU linear self-attention).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module: only the test-suite, the package smoke check and the benchmark's CPU-baseline leg
do.  It shares no code with the CUDA library and imports nothing from it.

What it computes
----------------
LiteLA (Sana explainer, "Sana: the autoencoder does more of the work than the linear
attention", section "What LiteLA actually computes") applies phi = ReLU to q and k, pads v
with a row of ones, forms the (d+1) x d state  vk = [V;1] . phi(K)^T, applies it to phi(Q)
and divides the first d rows by the last row plus eps.  By associativity that is exactly
(up to rounding order) the quadratic form of kernelised linear attention ("How Linear
Attention Improves Efficiency in DiT for High-Resolution Images", section "Mathematical
Foundation"):

    out_i = sum_j w_ij v_j / (sum_j w_ij + eps),   w_ij = phi(q_i) . phi(k_j).

This oracle is that plain definition written out in float64: one weight per (query, key)
pair, a weighted sum and a division.  It never forms the state; the state route is what
the CUDA path takes, and the tests pin this oracle against the state route done in exact
rational arithmetic, against invariants and against special cases with closed forms.

Block-causal variant ("Block-Linear Attention", same instagit page, section "Video
Generation and Constant-Memory KV Cache"; "block causal linear attention", evermx overview,
section "Model Family"): tokens are cut into consecutive blocks of T tokens; a query in
block b sees exactly the keys/values of blocks 0..b (inclusive; a ragged last block is
allowed).  The oracle is the same quadratic form with the key set restricted to that
prefix.

Readings taken where the pages are silent:
  * phi is ReLU on q and k only; v is not passed through phi.
  * eps is ADDED to the denominator, never used as a clamp; no 1/sqrt(d) scale.
  * bf16 inputs are decoded exactly (bits << 16 -> float32 -> float64).
  * den = 0 gives 0 / eps = 0.
  * Packed layout of one batch row: [q | k | v], each head-major (H heads x d channels).

Parity status: every public function here is pinned by tests/test_oracle_pins.py and
tests/test_golden.py (no function is "parity unpinned").
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "decode_bf16",
    "unpack_qkv",
    "relu",
    "lite_la_rows",
    "lite_la_fwd",
    "lite_la_block_causal_fwd",
    "visible_key_count",
]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """Exact decode of raw bf16 bit patterns (uint16/int16) to float64.

    A bf16 value is the top half of an IEEE binary32 word, so shifting the 16 bits into
    the high half of a 32-bit word gives the float32 with the same value; float32 ->
    float64 is exact.
    """
    b = np.asarray(bits)
    if b.dtype not in (np.uint16, np.int16):
        raise TypeError("decode_bf16 expects 16-bit raw patterns, got %s" % b.dtype)
    words = b.view(np.uint16).astype(np.uint32) << np.uint32(16)
    return words.view(np.float32).astype(np.float64)


def unpack_qkv(qkv: np.ndarray, H: int, d: int):
    """Split a packed [B, N, 3*H*d] array into q, k, v of shape [B, N, H, d].

    Layout (the packed qkv projection output): within one token row the first H*d entries
    are q, the next H*d are k, the last H*d are v, each head-major (head h owns channels
    h*d .. h*d+d-1).
    """
    B, N, W = qkv.shape
    if W != 3 * H * d:
        raise ValueError("last axis is %d, expected 3*H*d = %d" % (W, 3 * H * d))
    x = qkv.reshape(B, N, 3, H, d)
    return x[:, :, 0], x[:, :, 1], x[:, :, 2]


def relu(x: np.ndarray) -> np.ndarray:
    """phi = ReLU, the LiteLA kernel function (Sana explainer, "What LiteLA actually
    computes": `kernel_func` is nn.ReLU)."""
    return np.maximum(x, 0.0)


def visible_key_count(n: np.ndarray, N: int, tokens_per_block: int | None) -> np.ndarray:
    """Number of leading keys a query at token index n may attend to.

    Non-causal (tokens_per_block None): all N.  Block-causal with block size T: query n is
    in block floor(n/T) and sees blocks 0..floor(n/T), i.e. the first
    min((floor(n/T)+1)*T, N) tokens.
    """
    n = np.asarray(n, dtype=np.int64)
    if tokens_per_block is None:
        return np.full(n.shape, N, dtype=np.int64)
    T = int(tokens_per_block)
    if T <= 0:
        raise ValueError("tokens_per_block must be positive")
    return np.minimum((n // T + 1) * T, N)


def lite_la_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, eps: float,
                 n_visible: np.ndarray | None = None) -> np.ndarray:
    """Quadratic-form LiteLA for a set of queries of ONE (batch, head).

    q_rows: [R, d] float64 raw queries; k, v: [N, d] float64 raw keys/values;
    n_visible: [R] number of leading keys each query sees (None = all N).
    Returns [R, d] float64:  out_i = sum_j w_ij v_j / (sum_j w_ij + eps),
    w_ij = relu(q_i) . relu(k_j), j over the visible keys.
    """
    pq = relu(q_rows)
    pk = relu(k)
    w = pq @ pk.T                                    # [R, N]: w_ij = phi(q_i).phi(k_j)
    if n_visible is not None:
        cols = np.arange(k.shape[0])[None, :]
        w = np.where(cols < np.asarray(n_visible)[:, None], w, 0.0)
    num = w @ v                                      # [R, d]: sum_j w_ij v_j
    den = w.sum(axis=1, keepdims=True)               # [R, 1]: sum_j w_ij
    return num / (den + eps)


def _forward(qkv_bits: np.ndarray, B: int, N: int, H: int, d: int, eps: float,
             tokens_per_block: int | None, rows, chunk: int) -> np.ndarray:
    x = decode_bf16(np.asarray(qkv_bits).reshape(B, N, 3 * H * d))
    q, k, v = unpack_qkv(x, H, d)
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((B, rows.size, H, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kk = np.ascontiguousarray(k[b, :, h, :])
            vv = np.ascontiguousarray(v[b, :, h, :])
            for s in range(0, rows.size, chunk):
                r = rows[s:s + chunk]
                nv = None if tokens_per_block is None else visible_key_count(r, N, tokens_per_block)
                out[b, s:s + chunk, h, :] = lite_la_rows(q[b, r, h, :], kk, vv, eps, nv)
    return out


def lite_la_fwd(qkv_bits: np.ndarray, B: int, N: int, H: int, d: int, eps: float,
                rows=None, chunk: int = 2048) -> np.ndarray:
    """Non-causal LiteLA forward on packed bf16 qkv bits [B, N, 3*H*d].

    Returns float64 [B, len(rows), H, d] (all N query tokens when rows is None); rows
    selects query token indices so that full-size inputs can be checked on a sample.
    """
    return _forward(qkv_bits, B, N, H, d, eps, None, rows, chunk)


def lite_la_block_causal_fwd(qkv_bits: np.ndarray, B: int, N: int, H: int, d: int,
                             eps: float, tokens_per_block: int, rows=None,
                             chunk: int = 2048) -> np.ndarray:
    """Block-causal LiteLA forward: a query in block b sees the keys of blocks 0..b."""
    if int(tokens_per_block) <= 0:
        raise ValueError("tokens_per_block must be positive")
    return _forward(qkv_bits, B, N, H, d, eps, int(tokens_per_block), rows, chunk)
