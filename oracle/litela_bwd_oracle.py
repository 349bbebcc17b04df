"""fp64 CPU oracle for the LiteLA backward pass (gradients of Sana's ReLU linear attention).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module: only the test-suite may.  It shares no code with the CUDA library.

What it computes
----------------
The pages give the forward pass only (Sana explainer, "What LiteLA actually computes";
"How Linear Attention Improves Efficiency in DiT for High-Resolution Images", sections
"Mathematical Foundation" and "Video Generation and Constant-Memory KV Cache"); Sana trains
with it, and the gradient it trains with is the derivative of that forward.  So this oracle
is the chain rule applied to the plain quadratic form the forward oracle evaluates,

    out_i = num_i / den_i,  num_i = sum_j w_ij v_j,  den_i = sum_j w_ij + eps,
    w_ij  = relu(q_i) . relu(k_j)   (j over the keys query i sees),

for the scalar L = sum_i dout_i . out_i (dout is the incoming gradient):

    dL/dnum_i = dout_i / den_i                        (d-vector)
    dL/dden_i = -(dout_i . out_i) / den_i             (scalar)
    dL/dw_ij  = dL/dnum_i . v_j + dL/dden_i           (visible pairs only)
    dL/dv_j   = sum_i w_ij dL/dnum_i
    dL/dq_i   = relu'(q_i) * sum_j dL/dw_ij relu(k_j)
    dL/dk_j   = relu'(k_j) * sum_i dL/dw_ij relu(q_i)

It forms one weight per (query, key) pair and never the (d+1) x d state; the state route is
what the CUDA path takes.  Readings where the pages are silent: relu'(x) = 1 for x > 0 and 0
otherwise (0 at x = 0, as PyTorch's ReLU backward); eps is a constant; the ones row that pads
v is a constant and gets no gradient.

Error magnitudes (magnitudes=True).  A gradient element is a sum of terms of both signs and
may cancel to far below the size of its terms (for N = 1, dq is exactly eps-small), so a
floating-point evaluation of it errs in proportion to its terms, not to itself.  With
magnitudes=True each function also returns, per element, the same sums taken over absolute
values, with |dL/dden_i| replaced by the bound sum_r |dout_ir| (sum_j w_ij |v_jr|) / den_i^2 of
its own terms:
    M(dq_i) = sum_j (|dL/dnum_i| . |v_j| + B_i) relu(k_j)
    M(dk_j) = sum_i (|dL/dnum_i| . |v_j| + B_i) relu(q_i)
    M(dv_j) = sum_i w_ij |dL/dnum_i|
These bound what any route that reassociates the sums (such as the state route) adds up, so
a computed gradient is compared with tolerance rtol * |g| + atol * M.

Parity status: lite_la_bwd_head, lite_la_bwd and lite_la_block_causal_bwd are pinned by
tests/test_oracle_bwd_pins.py (central finite differences of the pinned forward oracle,
PyTorch autograd of the quadratic form, closed-form identities from homogeneity and
linearity, ReLU masks and block-causal special cases); the error magnitudes are pinned from
both sides by the sums of the absolute values of every chain-rule term, written out per
(query, key) pair in exact rational arithmetic on tiny inputs.
"""
from __future__ import annotations

import numpy as np

from .litela_oracle import decode_bf16, relu, unpack_qkv, visible_key_count

__all__ = ["lite_la_bwd_head", "lite_la_bwd", "lite_la_block_causal_bwd"]


def _weights(pq_rows, pk, n_visible):
    w = pq_rows @ pk.T                                           # w_ij = relu(q_i).relu(k_j)
    if n_visible is None:
        return w, None
    mask = np.arange(pk.shape[0])[None, :] < np.asarray(n_visible)[:, None]
    return np.where(mask, w, 0.0), mask


def lite_la_bwd_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray, eps: float,
                     tokens_per_block: int | None = None, rows=None, chunk: int = 1024,
                     magnitudes: bool = False):
    """Gradients of L = sum(dout * out) for ONE (batch, head).

    q, k, v, dout: [N, d] float64 (raw q and k; relu is applied here).  rows: token indices
    whose gradients are returned (None = all N); every query contributes to dk and dv.
    Returns (dq, dk, dv), each [len(rows), d] float64, followed by their error magnitudes
    (mq, mk, mv) when `magnitudes` is set.
    """
    N, d = q.shape
    T = None if tokens_per_block is None else int(tokens_per_block)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    pq, pk = relu(q), relu(k)
    v_rows = v[rows]

    av = np.abs(v)
    # dq for the selected queries: sum over the keys each one sees
    dq = np.zeros((rows.size, d))
    mq = np.zeros((rows.size, d))
    for s in range(0, rows.size, chunk):
        r = rows[s:s + chunk]
        nv = None if T is None else visible_key_count(r, N, T)
        w, mask = _weights(pq[r], pk, nv)
        den = w.sum(axis=1) + eps
        out = (w @ v) / den[:, None]
        dnum = dout[r] / den[:, None]
        dden = -(dout[r] * out).sum(axis=1) / den
        dw = dnum @ v.T + dden[:, None]
        if mask is not None:
            dw = np.where(mask, dw, 0.0)
        dq[s:s + chunk] = (dw @ pk) * (q[r] > 0)
        if magnitudes:
            bnd = (np.abs(dout[r]) * (w @ av)).sum(axis=1) / den ** 2
            aw = np.abs(dnum) @ av.T + bnd[:, None]
            if mask is not None:
                aw = np.where(mask, aw, 0.0)
            mq[s:s + chunk] = aw @ pk

    # dk and dv for the selected keys: sum over every query that sees them
    dkt = np.zeros((rows.size, d))
    dv = np.zeros((rows.size, d))
    mk = np.zeros((rows.size, d))
    mv = np.zeros((rows.size, d))
    av_rows = av[rows]
    for s in range(0, N, chunk):
        i = np.arange(s, min(s + chunk, N), dtype=np.int64)
        nv = None if T is None else visible_key_count(i, N, T)
        w, mask = _weights(pq[i], pk, nv)
        den = w.sum(axis=1) + eps
        out = (w @ v) / den[:, None]
        dnum = dout[i] / den[:, None]
        dden = -(dout[i] * out).sum(axis=1) / den
        w_sel = w[:, rows]                                       # [C, R]
        dw_sel = dnum @ v_rows.T + dden[:, None]
        if mask is not None:
            dw_sel = np.where(mask[:, rows], dw_sel, 0.0)
        dv += w_sel.T @ dnum
        dkt += dw_sel.T @ pq[i]
        if magnitudes:
            bnd = (np.abs(dout[i]) * (w @ av)).sum(axis=1) / den ** 2
            aw_sel = np.abs(dnum) @ av_rows.T + bnd[:, None]
            if mask is not None:
                aw_sel = np.where(mask[:, rows], aw_sel, 0.0)
            mv += w_sel.T @ np.abs(dnum)
            mk += aw_sel.T @ pq[i]
    dk = dkt * (k[rows] > 0)
    if magnitudes:
        return dq, dk, dv, mq, mk, mv
    return dq, dk, dv


def _backward(qkv_bits, dout_bits, B, N, H, d, eps, tokens_per_block, rows, heads, chunk, magnitudes=False):
    x = decode_bf16(np.asarray(qkv_bits).reshape(B, N, 3 * H * d))
    g = decode_bf16(np.asarray(dout_bits).reshape(B, N, H, d))
    q, k, v = unpack_qkv(x, H, d)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    res = [np.full((B, rows.size, H, d), np.nan) for _ in range(6 if magnitudes else 3)]
    for (b, h) in heads:
        got = lite_la_bwd_head(np.ascontiguousarray(q[b, :, h]), np.ascontiguousarray(k[b, :, h]),
                               np.ascontiguousarray(v[b, :, h]), np.ascontiguousarray(g[b, :, h]),
                               eps, tokens_per_block, rows, chunk, magnitudes)
        for dst, src in zip(res, got):
            dst[b, :, h] = src
    return tuple(res)


def lite_la_bwd(qkv_bits, dout_bits, B: int, N: int, H: int, d: int, eps: float,
                rows=None, heads=None, chunk: int = 1024, magnitudes: bool = False):
    """Non-causal LiteLA backward on packed bf16 qkv bits [B, N, 3*H*d] and bf16 dout bits
    [B, N, H*d].  Returns float64 (dq, dk, dv), each [B, len(rows), H, d] (then their error
    magnitudes when `magnitudes` is set); rows selects token indices (None = all), heads a list
    of (b, h) to evaluate (None = all; the others are NaN)."""
    return _backward(qkv_bits, dout_bits, B, N, H, d, eps, None, rows, heads, chunk, magnitudes)


def lite_la_block_causal_bwd(qkv_bits, dout_bits, B: int, N: int, H: int, d: int, eps: float,
                             tokens_per_block: int, rows=None, heads=None, chunk: int = 1024,
                             magnitudes: bool = False):
    """Block-causal LiteLA backward: query i sees the keys of blocks 0..floor(i/T)."""
    if int(tokens_per_block) <= 0:
        raise ValueError("tokens_per_block must be positive")
    return _backward(qkv_bits, dout_bits, B, N, H, d, eps, int(tokens_per_block), rows, heads, chunk,
                     magnitudes)
