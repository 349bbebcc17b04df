"""Exact rational LiteLA by the padded-state route, used to pin the fp64 oracle.

The oracle evaluates the quadratic form (one weight per query/key pair).  This helper takes
the other route the pages give, in exact rational arithmetic (fractions.Fraction), so the
two agree only if both are right: phi = ReLU on q and k, V padded with a row of ones, the
(d+1) x d state vk = [V;1] . phi(K)^T, y = vk . phi(q), out = y[:d] / (y[d] + eps) (Sana
explainer, section "What LiteLA actually computes").  The block-causal form sums the
per-block states of blocks 0..b for a query in block b (instagit page "How Linear Attention
Improves Efficiency in DiT for High-Resolution Images", section "Video Generation and
Constant-Memory KV Cache").  Pure Python loops: tiny inputs only.
"""
from fractions import Fraction


def _relu(x):
    return x if x > 0 else Fraction(0)


def state_of(k_rows, v_rows):
    """(d+1) x d state of a list of tokens: rows r < d are sum_n v[n][r] * relu(k[n][c]);
    row d (the ones pad) is sum_n relu(k[n][c])."""
    d = len(k_rows[0]) if k_rows else 0
    S = [[Fraction(0)] * d for _ in range(d + 1)]
    for kn, vn in zip(k_rows, v_rows):
        vpad = [Fraction(x) for x in vn] + [Fraction(1)]
        pk = [_relu(Fraction(x)) for x in kn]
        for r in range(d + 1):
            for c in range(d):
                S[r][c] += vpad[r] * pk[c]
    return S


def apply_state(S, q_row, eps):
    d = len(q_row)
    pq = [_relu(Fraction(x)) for x in q_row]
    y = [sum((S[r][c] * pq[c] for c in range(d)), Fraction(0)) for r in range(d + 1)]
    den = y[d] + Fraction(eps)
    if den == 0:
        return [Fraction(0)] * d
    return [y[r] / den for r in range(d)]


def lite_la_exact(q, k, v, eps, tokens_per_block=None):
    """q, k, v: lists of N rows of d numbers (one batch, one head).  Returns N rows of d
    Fractions."""
    N = len(q)
    if N == 0:
        return []
    d = len(q[0])
    if tokens_per_block is None:
        S = state_of(k, v)
        return [apply_state(S, q[n], eps) for n in range(N)]
    T = int(tokens_per_block)
    nblk = (N + T - 1) // T
    block_states = [state_of(k[b * T:(b + 1) * T], v[b * T:(b + 1) * T]) for b in range(nblk)]
    out = []
    prefix = [[Fraction(0)] * d for _ in range(d + 1)]
    for b in range(nblk):
        prefix = [[prefix[r][c] + block_states[b][r][c] for c in range(d)] for r in range(d + 1)]
        for n in range(b * T, min((b + 1) * T, N)):
            out.append(apply_state(prefix, q[n], eps))
    return out
