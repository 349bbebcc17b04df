"""Pins for the fp64 oracle of LiteLA + output projection (oracle/litela_oproj_oracle.py),
independent of its own formulas: an exact rational route (the pages' padded-state form for
LiteLA, then the projection as explicit sums of products), the identity and permutation
special cases, and linearity.  CPU only."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from linear_attention_diffusion_litela_b200.inputs import pack_qkv, to_bits
from tests.exact_state_form import lite_la_exact

D = 32


def bf16_bits(a):
    return to_bits(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16))


def dyadic(rng, shape, scale=8, span=2):
    """Values exactly representable in bf16 and as small binary fractions."""
    return rng.integers(-span * scale, span * scale + 1, size=shape) / scale


def exact_oproj(q, k, v, w, bias, eps, T=None):
    """LiteLA by the padded-state route in Fractions, per (batch, head), then
    y[o] = sum_{h,c} x[h][c] * W[o][h*d + c] + bias[o] as explicit sums."""
    B, N, H, d = q.shape
    C_out = w.shape[0]
    y = np.zeros((B, N, C_out))
    for b in range(B):
        x = [lite_la_exact(q[b, :, h].tolist(), k[b, :, h].tolist(), v[b, :, h].tolist(), Fraction(eps), T)
             for h in range(H)]
        for n in range(N):
            for o in range(C_out):
                acc = Fraction(0) if bias is None else Fraction(float(bias[o]))
                for h in range(H):
                    for c in range(d):
                        acc += x[h][n][c] * Fraction(float(w[o, h * d + c]))
                y[b, n, o] = float(acc)
    return y


@pytest.mark.parametrize("B,N,H,C_out,T,eps,with_bias", [
    (1, 3, 1, 5, None, 1e-15, True), (2, 4, 2, 8, None, 0.25, False), (1, 5, 2, 3, 2, 1e-15, True),
    (2, 6, 3, 4, 4, 0.5, True), (1, 1, 1, 2, None, 1e-15, False)])
def test_matches_the_exact_padded_state_route_then_explicit_sums(B, N, H, C_out, T, eps, with_bias):
    rng = np.random.default_rng(31 * N + 7 * H + C_out + (T or 0))
    # d = 32 as everywhere; a few channels nonzero keeps the exact route quick but every index used
    q, k, v = (dyadic(rng, (B, N, H, D)) for _ in range(3))
    w = dyadic(rng, (C_out, H * D), scale=4)
    bias = dyadic(rng, (C_out,), scale=16) if with_bias else None
    qkv_bits = to_bits(pack_qkv(q, k, v))
    got = oracle.lite_la_oproj(qkv_bits, bf16_bits(w), B, N, H, D, C_out, eps, bias, T)
    want = exact_oproj(q, k, v, w, bias, eps, T)
    scale = np.abs(w).sum() * (np.abs(v).max() + 1) + 1
    assert np.all(np.abs(got - want) <= 1e-12 * scale)


def test_linear_matches_explicit_sums_of_products():
    rng = np.random.default_rng(5)
    M, C_in, C_out = 4, 12, 7
    x = dyadic(rng, (M, C_in))
    w = dyadic(rng, (C_out, C_in), scale=4)
    bias = dyadic(rng, (C_out,), scale=16)
    got = oracle.linear(bf16_bits(x), bf16_bits(w), C_out, C_in, bias)
    for m in range(M):
        for o in range(C_out):
            acc = Fraction(float(bias[o]))
            for i in range(C_in):
                acc += Fraction(float(x[m, i])) * Fraction(float(w[o, i]))
            assert got[m, o] == float(acc)        # small dyadic values: exact in fp64
    # float input is taken as it is; no bias means none
    np.testing.assert_array_equal(oracle.linear(x, bf16_bits(w), C_out, C_in), x @ w.T)


@pytest.mark.parametrize("T", [None, 3])
def test_identity_projection_gives_lite_la_itself(T):
    rng = np.random.default_rng(8)
    B, N, H = 2, 7, 3
    qkv = pack_qkv(*(rng.standard_normal((B, N, H, D)) for _ in range(3)))
    bits = to_bits(qkv)
    eye = bf16_bits(np.eye(H * D))
    y = oracle.lite_la_oproj(bits, eye, B, N, H, D, H * D, 1e-15, None, T)
    x = (oracle.lite_la_block_causal_fwd(bits, B, N, H, D, 1e-15, T) if T else
         oracle.lite_la_fwd(bits, B, N, H, D, 1e-15))
    np.testing.assert_array_equal(y, x.reshape(B, N, H * D))
    # a projection that keeps head 1's channels reversed, scaled by 2, gives exactly that
    sel = np.zeros((D, H * D))
    for c in range(D):
        sel[c, D + (D - 1 - c)] = 2.0
    y = oracle.lite_la_oproj(bits, bf16_bits(sel), B, N, H, D, D, 1e-15, None, T)
    np.testing.assert_array_equal(y, 2.0 * x[:, :, 1, ::-1])


def test_permuting_heads_with_the_weight_blocks_leaves_the_output_unchanged():
    """y = sum_h x_h W_h^T over head blocks: permuting the heads of q, k, v together with the
    column blocks of W changes nothing (up to the order of the sum)."""
    rng = np.random.default_rng(9)
    B, N, H, C_out = 2, 9, 4, 6
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    w = rng.standard_normal((C_out, H * D))
    bias = rng.standard_normal(C_out)
    perm = np.array([2, 0, 3, 1])
    y = oracle.lite_la_oproj(to_bits(pack_qkv(q, k, v)), bf16_bits(w), B, N, H, D, C_out, 1e-15, bias)
    wp = w.reshape(C_out, H, D)[:, perm].reshape(C_out, H * D)
    yp = oracle.lite_la_oproj(to_bits(pack_qkv(q[:, :, perm], k[:, :, perm], v[:, :, perm])), bf16_bits(wp),
                              B, N, H, D, C_out, 1e-15, bias)
    np.testing.assert_allclose(yp, y, rtol=1e-12, atol=1e-12)
    # rows select tokens of the full result
    rows = np.array([0, 4, 8])
    ys = oracle.lite_la_oproj(to_bits(pack_qkv(q, k, v)), bf16_bits(w), B, N, H, D, C_out, 1e-15, bias, rows=rows)
    np.testing.assert_allclose(ys, y[:, rows], rtol=1e-13, atol=1e-13)


def test_linear_in_the_weights_and_affine_in_the_bias():
    rng = np.random.default_rng(10)
    B, N, H, C_out = 1, 6, 2, 5
    bits = to_bits(pack_qkv(*(rng.standard_normal((B, N, H, D)) for _ in range(3))))
    w1, w2 = dyadic(rng, (C_out, H * D), scale=4), dyadic(rng, (C_out, H * D), scale=4)
    bias = dyadic(rng, (C_out,), scale=16)
    f = lambda w, b: oracle.lite_la_oproj(bits, bf16_bits(w), B, N, H, D, C_out, 1e-15, b)
    np.testing.assert_allclose(f(w1 + w2, bias), f(w1, bias) + f(w2, None), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(3 * w1, None), 3 * f(w1, None), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(f(0 * w1, bias), np.broadcast_to(bias, (B, N, C_out)))


def test_a_transposed_weight_fails_the_exact_route():
    """Planted slip: W applied untransposed (square case) is caught by the exact route."""
    rng = np.random.default_rng(11)
    B, N, H = 1, 3, 1
    q, k, v = (dyadic(rng, (B, N, H, D)) for _ in range(3))
    w = dyadic(rng, (H * D, H * D), scale=4)
    bits = to_bits(pack_qkv(q, k, v))
    want = exact_oproj(q, k, v, w, None, 1e-15)
    good = oracle.lite_la_oproj(bits, bf16_bits(w), B, N, H, D, H * D, 1e-15)
    slip = oracle.lite_la_oproj(bits, bf16_bits(w.T), B, N, H, D, H * D, 1e-15)
    assert np.allclose(good, want, rtol=1e-12, atol=1e-12)
    assert not np.allclose(slip, want, rtol=1e-6, atol=1e-6)
