"""Pins for the fp64 backward oracle (oracle/litela_bwd_oracle.py), independent of its own
formulas: central finite differences of the pinned forward oracle, PyTorch autograd of the
quadratic form, closed-form identities that follow from the forward's homogeneity and
linearity, the ReLU masks, and the block-causal special cases.  CPU only."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_diffusion_litela_b200.inputs import to_bits

def bits_of(a):
    """bf16 bit patterns of a float32 array (round to nearest even)."""
    return to_bits(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16))


D = 32


def away_from_kinks(rng, shape, lo=0.05):
    """Gaussian values with |x| >= lo, so relu is differentiable within a small step."""
    x = rng.standard_normal(shape)
    return np.where(np.abs(x) < lo, np.sign(x + 1e-300) * lo, x)


def loss(q, k, v, g, eps, T):
    N = q.shape[0]
    nv = None if T is None else oracle.visible_key_count(np.arange(N), N, T)
    return float((oracle.lite_la_rows(q, k, v, eps, nv) * g).sum())


def finite_difference(q, k, v, g, eps, T, h=1e-6):
    grads = []
    for which in range(3):
        x = [q.copy(), k.copy(), v.copy()]
        out = np.zeros_like(x[which])
        for idx in np.ndindex(*out.shape):
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += h
            xm[which][idx] -= h
            out[idx] = (loss(*xp, g, eps, T) - loss(*xm, g, eps, T)) / (2 * h)
        grads.append(out)
    return grads


@pytest.mark.parametrize("N,T,eps", [(1, None, 1e-15), (5, None, 1e-15), (6, None, 0.3), (7, 2, 1e-15),
                                     (6, 1, 0.2), (5, 3, 1e-15)])
def test_matches_central_finite_differences_of_the_forward_oracle(N, T, eps):
    rng = np.random.default_rng(100 + N + (T or 0))
    q, k, v, g = (away_from_kinks(rng, (N, D)) for _ in range(4))
    dq, dk, dv = oracle.lite_la_bwd_head(q, k, v, g, eps, T)
    fq, fk, fv = finite_difference(q, k, v, g, eps, T)
    # relative to the gradient's overall size: a tensor whose true gradient is eps-small (the
    # queries and keys when N = 1) is checked to be that small
    scale = max(np.abs(f).max() for f in (fq, fk, fv))
    for got, want in ((dq, fq), (dk, fk), (dv, fv)):
        assert np.abs(got - want).max() <= 1e-6 * scale


@pytest.mark.parametrize("T", [None, 3])
def test_matches_torch_autograd_of_the_quadratic_form(T):
    rng = np.random.default_rng(7)
    N, eps = 11, 1e-3
    q, k, v, g = (rng.standard_normal((N, D)) for _ in range(4))
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    w = torch.relu(tq) @ torch.relu(tk).T
    if T is not None:
        i = torch.arange(N)[:, None]
        j = torch.arange(N)[None, :]
        w = torch.where(j // T <= i // T, w, torch.zeros_like(w))
    out = (w @ tv) / (w.sum(1, keepdim=True) + eps)
    (out * torch.tensor(g)).sum().backward()
    dq, dk, dv = oracle.lite_la_bwd_head(q, k, v, g, eps, T)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)


def forward_parts(q, k, v, eps, T=None):
    """num_i and den_i (eps included) of the quadratic form, for the identities below."""
    N = q.shape[0]
    w = np.maximum(q, 0) @ np.maximum(k, 0).T
    if T is not None:
        w = np.where(np.arange(N)[None, :] // T <= np.arange(N)[:, None] // T, w, 0.0)
    return w @ v, w.sum(1) + eps


@pytest.mark.parametrize("T", [None, 4])
def test_homogeneity_and_linearity_identities(T):
    """out is unchanged (up to eps) by scaling one query or all keys, affine in V:
      q_i . dq_i          = eps * (dout_i . num_i) / den_i^2
      sum_j k_j . dk_j    = eps * sum_i (dout_i . num_i) / den_i^2
      sum_j dv_j          = sum_i dout_i * (den_i - eps) / den_i
      sum_j v_j . dv_j    = sum_i dout_i . out_i
    With a large eps every one of them is far from 0 and tests its eps term."""
    rng = np.random.default_rng(11)
    N, eps = 20, 0.7
    q, k, v, g = (rng.standard_normal((N, D)) for _ in range(4))
    dq, dk, dv = oracle.lite_la_bwd_head(q, k, v, g, eps, T)
    num, den = forward_parts(q, k, v, eps, T)
    e = eps * (g * num).sum(1) / den ** 2
    np.testing.assert_allclose((q * dq).sum(1), e, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose((k * dk).sum(), e.sum(), rtol=1e-10)
    np.testing.assert_allclose(dv.sum(0), (g * ((den - eps) / den)[:, None]).sum(0), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose((v * dv).sum(), (g * num / den[:, None]).sum(), rtol=1e-10)


def test_relu_masks_and_a_query_that_sees_nothing():
    rng = np.random.default_rng(12)
    N = 9
    q, k, v, g = (rng.standard_normal((N, D)) for _ in range(4))
    q[4] = -np.abs(q[4])                       # relu(q_4) = 0: out_4 = 0 whatever the keys
    dq, dk, dv = oracle.lite_la_bwd_head(q, k, v, g, 1e-15)
    assert np.all(dq[q <= 0] == 0.0) and np.all(dk[k <= 0] == 0.0)
    assert np.all(dq[4] == 0.0)
    g2 = g.copy()
    g2[4] = 100.0 * rng.standard_normal(D)      # that row's incoming gradient reaches nothing
    dq2, dk2, dv2 = oracle.lite_la_bwd_head(q, k, v, g2, 1e-15)
    np.testing.assert_allclose(dk2, dk, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dv2, dv, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(np.delete(dq2, 4, 0), np.delete(dq, 4, 0))


def test_block_causal_special_cases():
    rng = np.random.default_rng(13)
    N, eps = 10, 1e-15
    q, k, v, g = (rng.standard_normal((N, D)) for _ in range(4))
    full = oracle.lite_la_bwd_head(q, k, v, g, eps)
    for T in (N, N + 5):                       # one block: the non-causal gradient
        for a, b in zip(oracle.lite_la_bwd_head(q, k, v, g, eps, T), full):
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)
    # token-causal (T = 1): the last key is seen by the last query only, so
    # dv_{N-1} = w_{N-1,N-1} dout_{N-1} / den_{N-1}
    dq, dk, dv = oracle.lite_la_bwd_head(q, k, v, g, eps, 1)
    num, den = forward_parts(q, k, v, eps, 1)
    w_last = np.maximum(q[-1], 0) @ np.maximum(k[-1], 0)
    np.testing.assert_allclose(dv[-1], w_last * g[-1] / den[-1], rtol=1e-12, atol=1e-15)
    # keys of the last block get gradient only from queries of the last block
    T = 4
    g_early = g.copy()
    g_early[8:] = 0.0
    _, dk_e, dv_e = oracle.lite_la_bwd_head(q, k, v, g_early, eps, T)
    assert np.all(dk_e[8:] == 0.0) and np.all(dv_e[8:] == 0.0)


def test_rows_select_the_full_result_and_packed_entry_points_agree():
    rng = np.random.default_rng(14)
    B, N, H = 2, 13, 3
    qkv = rng.standard_normal((B, N, 3 * H * D)).astype(np.float32)
    dout = rng.standard_normal((B, N, H * D)).astype(np.float32)
    qb, gb = bits_of(qkv), bits_of(dout)
    x = oracle.decode_bf16(qb)
    q, k, v = oracle.unpack_qkv(x, H, D)
    g = oracle.decode_bf16(gb).reshape(B, N, H, D)
    rows = np.array([0, 5, 12])
    for T in (None, 4):
        if T is None:
            dq, dk, dv = oracle.lite_la_bwd(qb, gb, B, N, H, D, 1e-15)
            sq, sk, sv = oracle.lite_la_bwd(qb, gb, B, N, H, D, 1e-15, rows=rows, heads=[(1, 2)])
        else:
            dq, dk, dv = oracle.lite_la_block_causal_bwd(qb, gb, B, N, H, D, 1e-15, T)
            sq, sk, sv = oracle.lite_la_block_causal_bwd(qb, gb, B, N, H, D, 1e-15, T, rows=rows, heads=[(1, 2)])
        for b in range(B):
            for h in range(H):
                ref = oracle.lite_la_bwd_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h], 1e-15, T)
                for got, want in zip((dq, dk, dv), ref):
                    np.testing.assert_array_equal(got[b, :, h], want)
        for full, samp in ((dq, sq), (dk, sk), (dv, sv)):
            np.testing.assert_allclose(samp[1, :, 2], full[1, rows, 2], rtol=1e-13, atol=1e-16)
            assert np.isnan(samp[0]).all()
    with pytest.raises(ValueError):
        oracle.lite_la_block_causal_bwd(qb, gb, B, N, H, D, 1e-15, 0)


@pytest.mark.parametrize("T", [None, 3])
def test_error_magnitudes_bound_the_gradients(T):
    """M >= |gradient| elementwise, with equality for dv when dout and v are non-negative (then
    no term of dv = sum_i w_ij dout_i / den_i is negative); flipping signs of v or dout entries
    leaves M unchanged."""
    rng = np.random.default_rng(15)
    N, eps = 12, 1e-15
    q, k, v, g = (rng.standard_normal((N, D)) for _ in range(4))
    dq, dk, dv, mq, mk, mv = oracle.lite_la_bwd_head(q, k, v, g, eps, T, magnitudes=True)
    for grad, mag in ((dq, mq), (dk, mk), (dv, mv)):
        assert np.all(mag >= np.abs(grad) * (1 - 1e-12))
    flip = np.where(rng.random((N, D)) < 0.5, -1.0, 1.0)
    _, _, _, mq2, mk2, mv2 = oracle.lite_la_bwd_head(q, k, v * flip, g * flip[::-1], eps, T, magnitudes=True)
    for a, b in ((mq, mq2), (mk, mk2), (mv, mv2)):
        np.testing.assert_allclose(a, b, rtol=1e-12)
    _, _, dvp, _, _, mvp = oracle.lite_la_bwd_head(q, k, np.abs(v), np.abs(g), eps, T, magnitudes=True)
    np.testing.assert_allclose(mvp, dvp, rtol=1e-12)
    # for N = 1 dq is eps-small while its magnitude is not
    dq1, _, _, mq1, _, _ = oracle.lite_la_bwd_head(q[:1], k[:1], v[:1], g[:1], eps, None, magnitudes=True)
    assert np.abs(dq1).max() < 1e-12 * mq1.max()


# ---------------------------------------------------------------------------------------------
# The error magnitudes, pinned from above: every chain-rule term written out per (query, key)
# pair in exact rational arithmetic.

def _explicit_terms(q, k, v, g, eps, T):
    """The gradients of L = sum_i dout_i . out_i expanded into elementary products, with
    exact Fractions on tiny inputs.  With out_i = num_i / den_i, num_i = sum_j w_ij v_j,
    den_i = sum_j w_ij + eps and w_ij = relu(q_i) . relu(k_j) (j visible to i):

        dq_ic = sum_j relu(k_jc) [ sum_r g_ir v_jr / den_i  -  sum_r sum_j' g_ir w_ij' v_j'r / den_i^2 ]
        dk_jc = sum_i relu(q_ic) [ the same bracket ]          (i that see j)
        dv_jr = sum_i w_ij g_ir / den_i

    (the masks relu'(q), relu'(k) left off, as in the magnitudes).  Each product above is one
    term; w_ij and den_i are sums of non-negative terms and enter as they are.  Returns the
    signed sums (the gradients before the ReLU masks) and the sums of the terms' absolute
    values (what any reassociation of these sums adds up)."""
    from fractions import Fraction as F
    N, d = len(q), len(q[0])
    fr = lambda a: [[F(x) for x in row] for row in a]
    q, k, v, g = fr(q), fr(k), fr(v), fr(g)
    eps = F(eps)
    rq = [[max(x, F(0)) for x in row] for row in q]
    rk = [[max(x, F(0)) for x in row] for row in k]
    vis = lambda i, j: T is None or j // T <= i // T
    w = [[sum(rq[i][c] * rk[j][c] for c in range(d)) if vis(i, j) else F(0) for j in range(N)] for i in range(N)]
    den = [sum(w[i]) + eps for i in range(N)]
    zero = lambda: [[F(0)] * d for _ in range(N)]
    dq, dk, dv, aq, ak, av = zero(), zero(), zero(), zero(), zero(), zero()
    for i in range(N):
        for j in range(N):
            if not vis(i, j):
                continue
            # the bracket of pair (i, j): its terms, each with its sign
            terms = [g[i][r] * v[j][r] / den[i] for r in range(d)]
            terms += [-(g[i][r] * w[i][jj] * v[jj][r]) / den[i] ** 2 for r in range(d) for jj in range(N) if vis(i, jj)]
            s, a = sum(terms), sum(abs(t) for t in terms)
            for c in range(d):
                dq[i][c] += rk[j][c] * s
                aq[i][c] += rk[j][c] * a
                dk[j][c] += rq[i][c] * s
                ak[j][c] += rq[i][c] * a
            for r in range(d):
                t = w[i][j] * g[i][r] / den[i]
                dv[j][r] += t
                av[j][r] += abs(t)
    as_np = lambda a: np.array([[float(x) for x in row] for row in a])
    return tuple(as_np(a) for a in (dq, dk, dv, aq, ak, av))


def _dyadic(rng, shape, scale=8):
    """Small values exactly representable in binary (multiples of 1/scale), some negative."""
    return rng.integers(-2 * scale, 2 * scale + 1, size=shape) / scale


def _check_magnitudes(got, explicit, masks):
    """The oracle's (dq, dk, dv, mq, mk, mv) against the explicit term sums, to 1e-12."""
    dq, dk, dv, mq, mk, mv = got
    eq, ek, ev, aq, ak, av = explicit
    mask_q, mask_k = masks
    ok = True
    # the signed sums cancel (dq is eps-small for N = 1): they are compared relative to their
    # own terms' magnitudes; the magnitudes relative to themselves
    for x, want, size in ((dq, eq * mask_q, aq), (dk, ek * mask_k, ak), (dv, ev, av),
                          (mq, aq, aq), (mk, ak, ak), (mv, av, av)):
        ok &= bool(np.all(np.abs(x - want) <= 1e-12 * size + 1e-300))
    return ok


MAG_CASES = [(1, 2, None, 1e-15), (3, 3, None, 1e-15), (4, 4, None, 0.25), (5, 2, 2, 1e-15),
             (6, 3, 2, 0.5), (6, 4, None, 1e-15), (5, 4, 3, 1e-15)]


@pytest.mark.parametrize("N,d,T,eps", MAG_CASES)
def test_error_magnitudes_equal_the_explicit_term_sums(N, d, T, eps):
    """M(dq), M(dk) and M(dv) equal, to 1e-12, the sums of the absolute values of every term of
    the chain rule written out pair by pair in exact rational arithmetic (and the signed sums
    of the same terms reproduce the gradients, so the term list is the gradient's own).  This
    bounds the magnitudes from above as well as from below: a magnitude counted twice, or a
    term missing its 1/den, fails here."""
    rng = np.random.default_rng(900 + 10 * N + d + (T or 0))
    q, k, v, g = (_dyadic(rng, (N, d)) for _ in range(4))
    got = oracle.lite_la_bwd_head(q, k, v, g, eps, T, magnitudes=True)
    explicit = _explicit_terms(q, k, v, g, eps, T)
    assert _check_magnitudes(got, explicit, ((q > 0).astype(float), (k > 0).astype(float)))


def _planted(src_old, src_new):
    """A copy of the backward oracle module with one slip planted in its source text."""
    import importlib.util
    import types
    spec = importlib.util.find_spec("oracle.litela_bwd_oracle")
    src = open(spec.origin).read()
    assert src.count(src_old) >= 1, src_old
    mod = types.ModuleType("planted_bwd_oracle")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src.replace(src_old, src_new), spec.origin, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("old,new", [
    ("mq[s:s + chunk] = aw @ pk", "mq[s:s + chunk] = 2 * (aw @ pk)"),            # M(dq) doubled
    ("mk += aw_sel.T @ pq[i]", "mk += 2 * (aw_sel.T @ pq[i])"),                  # M(dk) doubled
    ("/ den ** 2\n            aw = ", "/ den\n            aw = "),                # bnd without one 1/den (dq side)
    ("/ den ** 2\n            aw_sel", "/ den\n            aw_sel"),              # the same on the dk side
    ("aw = np.abs(dnum) @ av.T + bnd[:, None]", "aw = np.abs(dnum) @ av.T"),    # the denominator's terms dropped
    ("mv += w_sel.T @ np.abs(dnum)", "mv += w_sel.T @ np.abs(dout[i])"),       # M(dv) without 1/den
])
def test_a_planted_magnitude_slip_fails_the_explicit_pin(old, new):
    """Each slip, planted in a copy of the oracle's source, fails the explicit-term pin on at
    least one of the cases above (the pin is sensitive to it)."""
    mod = _planted(old, new)
    caught = False
    for N, d, T, eps in MAG_CASES:
        rng = np.random.default_rng(900 + 10 * N + d + (T or 0))
        q, k, v, g = (_dyadic(rng, (N, d)) for _ in range(4))
        got = mod.lite_la_bwd_head(q, k, v, g, eps, T, magnitudes=True)
        explicit = _explicit_terms(q, k, v, g, eps, T)
        if not _check_magnitudes(got, explicit, ((q > 0).astype(float), (k > 0).astype(float))):
            caught = True
            break
    assert caught
