"""Pins of the fp64 oracle to what the pages and the mathematics fix (CPU only).

Each test would fail under a plausible slip in the oracle: a dropped eps or ones row, ReLU
applied to v or missing on q/k, q/k/v swapped in the packed layout, a transposed operand,
a wrong block boundary.
"""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_litela_b200.inputs import make_qkv, pack_qkv, to_bits
from oracle import (decode_bf16, lite_la_block_causal_fwd, lite_la_fwd, unpack_qkv,
                    visible_key_count)
from tests.exact_state_form import lite_la_exact

EPS = 1e-15


def dyadic(rng, shape, lo=-8, hi=8, denom=4):
    """Small dyadic values (multiples of 1/denom), exact in bf16."""
    return rng.integers(lo * denom, hi * denom + 1, size=shape).astype(np.float64) / denom


def qkv_arrays(bits, B, N, H, d):
    x = decode_bf16(bits).reshape(B, N, 3 * H * d)
    return unpack_qkv(x, H, d)


# --- bf16 decoding -------------------------------------------------------------------

def test_decode_bf16_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x3F81, 0x7F7F, 0x0080, 0x4049],
                    dtype=np.uint16)
    want = [1.0, -2.0, 0.0, -0.0, 1.0 + 2.0 ** -7, (2.0 - 2.0 ** -7) * 2.0 ** 127,
            2.0 ** -126, 3.140625]
    got = decode_bf16(bits)
    assert list(got) == want
    assert np.signbit(got[3])


def test_decode_bf16_matches_torch_conversion():
    t = make_qkv(1, 64, 2, 32, seed=7)
    np.testing.assert_array_equal(decode_bf16(to_bits(t)), t.to(torch.float64).numpy())


# --- exact rational state route (brute force on tiny inputs) -------------------------

@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 1), (1, 2, 1, 2), (1, 3, 2, 3), (2, 7, 3, 4),
                                     (1, 16, 1, 5), (2, 33, 1, 3)])
def test_oracle_equals_exact_state_route(B, N, H, d):
    rng = np.random.default_rng(100 + N * 7 + d)
    q, k, v = (dyadic(rng, (B, N, H, d)) for _ in range(3))
    bits = to_bits(pack_qkv(q, k, v))
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    for b in range(B):
        for h in range(H):
            ex = lite_la_exact(q[b, :, h].tolist(), k[b, :, h].tolist(), v[b, :, h].tolist(), EPS)
            np.testing.assert_allclose(got[b, :, h], np.array(ex, dtype=np.float64),
                                       rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("N,T", [(7, 1), (7, 2), (7, 3), (8, 4), (9, 4), (5, 5), (5, 9), (16, 5)])
def test_block_causal_oracle_equals_exact_state_route(N, T):
    B, H, d = 2, 2, 3
    rng = np.random.default_rng(200 + N * 11 + T)
    q, k, v = (dyadic(rng, (B, N, H, d)) for _ in range(3))
    bits = to_bits(pack_qkv(q, k, v))
    got = lite_la_block_causal_fwd(bits, B, N, H, d, EPS, T)
    for b in range(B):
        for h in range(H):
            ex = lite_la_exact(q[b, :, h].tolist(), k[b, :, h].tolist(), v[b, :, h].tolist(), EPS, T)
            np.testing.assert_allclose(got[b, :, h], np.array(ex, dtype=np.float64),
                                       rtol=1e-12, atol=1e-300)


def test_layout_q_k_v_not_interchangeable():
    """Swapping the roles of q, k or v changes the result (guards the unpacking order)."""
    rng = np.random.default_rng(5)
    B, N, H, d = 1, 9, 2, 4
    q, k, v = (dyadic(rng, (B, N, H, d)) for _ in range(3))
    base = lite_la_fwd(to_bits(pack_qkv(q, k, v)), B, N, H, d, EPS)
    for perm in [(k, q, v), (q, v, k), (v, k, q)]:
        other = lite_la_fwd(to_bits(pack_qkv(*perm)), B, N, H, d, EPS)
        assert not np.allclose(base, other)


# --- invariants and closed forms ------------------------------------------------------

def seeded(B, N, H, d, seed, shift=0.0):
    t = make_qkv(B, N, H, d, seed=seed, qk_shift=shift)
    return t, to_bits(t)


def test_key_value_permutation_invariance():
    B, N, H, d = 2, 40, 3, 32
    t, bits = seeded(B, N, H, d, 11)
    perm = np.random.default_rng(1).permutation(N)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 1:] = x[:, perm][:, :, 1:]        # permute (k_j, v_j) pairs jointly
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    np.testing.assert_allclose(lite_la_fwd(bits2, B, N, H, d, EPS), lite_la_fwd(bits, B, N, H, d, EPS),
                               rtol=1e-12, atol=1e-15)


def test_block_causal_permutation_within_a_block_invariance():
    B, N, H, d, T = 1, 30, 2, 8, 10
    t, bits = seeded(B, N, H, d, 12)
    perm = np.concatenate([np.random.default_rng(2).permutation(T) + b * T for b in range(3)])
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 1:] = x[:, perm][:, :, 1:]
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    np.testing.assert_allclose(lite_la_block_causal_fwd(bits2, B, N, H, d, EPS, T),
                               lite_la_block_causal_fwd(bits, B, N, H, d, EPS, T),
                               rtol=1e-12, atol=1e-15)
    # a permutation across blocks is NOT an invariance of the block-causal form
    perm_x = np.random.default_rng(3).permutation(N)
    y = t.view(B, N, 3, H, d).clone()
    y[:, :, 1:] = y[:, perm_x][:, :, 1:]
    bits3 = to_bits(y.view(B, N, 3 * H * d))
    assert not np.allclose(lite_la_block_causal_fwd(bits3, B, N, H, d, EPS, T),
                           lite_la_block_causal_fwd(bits, B, N, H, d, EPS, T))


def test_query_permutation_equivariance():
    B, N, H, d = 1, 33, 2, 32
    t, bits = seeded(B, N, H, d, 13)
    perm = np.random.default_rng(4).permutation(N)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 0] = x[:, perm][:, :, 0]
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    np.testing.assert_allclose(lite_la_fwd(bits2, B, N, H, d, EPS),
                               lite_la_fwd(bits, B, N, H, d, EPS)[:, perm], rtol=1e-12, atol=1e-15)


def test_constant_v_gives_c_times_den_over_den_plus_eps():
    B, N, H, d = 1, 50, 2, 32
    t, bits = seeded(B, N, H, d, 14)
    x = t.view(B, N, 3, H, d).clone()
    c = 0.375
    x[:, :, 2] = c
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    q, k, _ = qkv_arrays(bits2, B, N, H, d)
    den = np.einsum("bnhc,bhc->bnh", np.maximum(q, 0), np.maximum(k, 0).sum(axis=1))
    got = lite_la_fwd(bits2, B, N, H, d, EPS)
    np.testing.assert_allclose(got, np.broadcast_to((c * den / (den + EPS))[..., None], got.shape),
                               rtol=1e-13, atol=0)
    np.testing.assert_allclose(got[den > 1e-6], c, rtol=1e-12)


def test_all_negative_q_row_gives_zero():
    B, N, H, d = 1, 20, 2, 32
    t, _ = seeded(B, N, H, d, 15)
    x = t.view(B, N, 3, H, d).clone()
    x[0, 5, 0, 1] = -x[0, 5, 0, 1].abs() - 0.5       # token 5, head 1: every q channel < 0
    bits = to_bits(x.view(B, N, 3 * H * d))
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    assert np.all(got[0, 5, 1] == 0.0)
    assert np.any(got[0, 5, 0] != 0.0)


def test_all_negative_k_gives_zero():
    B, N, H, d = 1, 20, 2, 32
    t, _ = seeded(B, N, H, d, 16)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 1, 0] = -x[:, :, 1, 0].abs() - 0.25     # head 0: every key channel < 0
    bits = to_bits(x.view(B, N, 3 * H * d))
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    assert np.all(got[:, :, 0] == 0.0)
    assert np.all(np.abs(got[:, :, 1]) > 0.0)


@pytest.mark.parametrize("gamma", [0.25, 2.0, 8.0])
def test_degree_zero_homogeneity_in_q(gamma):
    B, N, H, d = 1, 30, 2, 32
    t, bits = seeded(B, N, H, d, 17)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 0] *= gamma                             # powers of two: exact in bf16
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    np.testing.assert_allclose(lite_la_fwd(bits2, B, N, H, d, EPS), lite_la_fwd(bits, B, N, H, d, EPS),
                               rtol=1e-12, atol=1e-15)


def test_output_in_convex_hull_of_values():
    B, N, H, d = 2, 64, 3, 32
    _, bits = seeded(B, N, H, d, 18)
    _, _, v = qkv_arrays(bits, B, N, H, d)
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    lo, hi = v.min(axis=1, keepdims=True), v.max(axis=1, keepdims=True)
    nz = got != 0
    assert np.all((got >= lo - 1e-12) | ~nz) and np.all((got <= hi + 1e-12) | ~nz)


def test_affine_in_v():
    B, N, H, d = 1, 40, 2, 32
    t, _ = seeded(B, N, H, d, 19)
    alpha, beta = -2.0, 0.5
    x = t.view(B, N, 3, H, d).to(torch.float64).clone()
    x[:, :, 2] = torch.from_numpy(dyadic(np.random.default_rng(9), (B, N, H, d)))  # few-bit V
    x2 = x.clone()
    x2[:, :, 2] = alpha * x[:, :, 2] + beta                 # exact in bf16 for few-bit V
    t1, t2 = x.to(torch.bfloat16), x2.to(torch.bfloat16)
    assert torch.equal(t1.to(torch.float64), x) and torch.equal(t2.to(torch.float64), x2)
    bits = to_bits(t1.view(B, N, 3 * H * d))
    bits2 = to_bits(t2.view(B, N, 3 * H * d))
    q, k, _ = qkv_arrays(bits, B, N, H, d)
    den = np.einsum("bnhc,bhc->bnh", np.maximum(q, 0), np.maximum(k, 0).sum(axis=1))[..., None]
    want = alpha * lite_la_fwd(bits, B, N, H, d, EPS) + beta * den / (den + EPS)
    np.testing.assert_allclose(lite_la_fwd(bits2, B, N, H, d, EPS), want, rtol=1e-11, atol=1e-13)


def test_heads_and_batches_are_independent():
    B, N, H, d = 2, 24, 3, 32
    t, bits = seeded(B, N, H, d, 20)
    x = t.view(B, N, 3, H, d).clone()
    x[1, :, :, 2] = torch.randn(N, 3, d).to(torch.bfloat16)   # change batch 1, head 2 only
    bits2 = to_bits(x.view(B, N, 3 * H * d))
    a, b = lite_la_fwd(bits, B, N, H, d, EPS), lite_la_fwd(bits2, B, N, H, d, EPS)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1, :, :2], b[1, :, :2])
    assert not np.allclose(a[1, :, 2], b[1, :, 2])


def test_identical_keys_reduce_to_mean_of_values():
    """All keys equal: every weight is the same, the output is numpy's plain mean of V."""
    B, N, H, d = 1, 17, 1, 32
    t, _ = seeded(B, N, H, d, 21)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 1] = x[:, :1, 1].abs() + 0.125
    bits = to_bits(x.view(B, N, 3 * H * d))
    _, _, v = qkv_arrays(bits, B, N, H, d)
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    np.testing.assert_allclose(got[0, :, 0], np.broadcast_to(v[0, :, 0].mean(axis=0), (N, d)),
                               rtol=1e-12, atol=1e-14)


def test_single_active_channel_is_weighted_average():
    """Only channel c of q and k positive: the output is numpy's weighted average of V with
    weights relu(k_jc), whatever the query's magnitude."""
    B, N, H, d, c = 1, 25, 1, 32, 7
    t, _ = seeded(B, N, H, d, 22)
    x = t.view(B, N, 3, H, d).clone()
    x[:, :, 0:2] = -x[:, :, 0:2].abs() - 0.125
    x[:, :, 0, 0, c] = x[:, :, 0, 0, c].abs() + 0.5
    x[:, ::2, 1, 0, c] = x[:, ::2, 1, 0, c].abs()
    bits = to_bits(x.view(B, N, 3 * H * d))
    _, k, v = qkv_arrays(bits, B, N, H, d)
    w = np.maximum(k[0, :, 0, c], 0)
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    np.testing.assert_allclose(got[0, :, 0], np.broadcast_to(np.average(v[0, :, 0], axis=0, weights=w), (N, d)),
                               rtol=1e-12, atol=1e-14)


# --- block-causal special cases ------------------------------------------------------

def test_block_covering_everything_is_non_causal():
    B, N, H, d = 1, 37, 2, 32
    _, bits = seeded(B, N, H, d, 23)
    ref = lite_la_fwd(bits, B, N, H, d, EPS)
    for T in (N, N + 1, 10 * N):
        np.testing.assert_array_equal(lite_la_block_causal_fwd(bits, B, N, H, d, EPS, T), ref)


@pytest.mark.parametrize("T", [1, 4, 16, 13])
def test_block_output_equals_non_causal_on_the_visible_prefix(T):
    B, N, H, d = 1, 40, 2, 32
    t, bits = seeded(B, N, H, d, 24)
    got = lite_la_block_causal_fwd(bits, B, N, H, d, EPS, T)
    for blk in range((N + T - 1) // T):
        end = min((blk + 1) * T, N)
        sub = to_bits(t[:, :end].contiguous())
        ref = lite_la_fwd(sub, B, end, H, d, EPS)
        np.testing.assert_allclose(got[:, blk * T:end], ref[:, blk * T:end], rtol=1e-12, atol=1e-15)


def test_token_causal_matches_cumulative_sums():
    """T = 1: out_n = (sum_{j<=n} w_nj v_j) / (sum_{j<=n} w_nj + eps), evaluated with running
    (cumulative) sums of the outer products relu(k_j) v_j^T, a route independent of the
    oracle's masked weight matrix."""
    B, N, H, d = 1, 19, 1, 32
    _, bits = seeded(B, N, H, d, 25)
    q, k, v = qkv_arrays(bits, B, N, H, d)
    pq, pk, vv = np.maximum(q[0, :, 0], 0), np.maximum(k[0, :, 0], 0), v[0, :, 0]
    Scum = np.cumsum(pk[:, :, None] * vv[:, None, :], axis=0)     # [N, c, r]
    zcum = np.cumsum(pk, axis=0)                                  # [N, c]
    num = np.einsum("nc,ncr->nr", pq, Scum)
    den = np.einsum("nc,nc->n", pq, zcum)[:, None]
    np.testing.assert_allclose(lite_la_block_causal_fwd(bits, B, N, H, d, EPS, 1)[0, :, 0],
                               num / (den + EPS), rtol=1e-12, atol=1e-15)


def test_visible_key_count():
    n = np.arange(10)
    assert list(visible_key_count(n, 10, None)) == [10] * 10
    assert list(visible_key_count(n, 10, 1)) == list(range(1, 11))
    assert list(visible_key_count(n, 10, 4)) == [4, 4, 4, 4, 8, 8, 8, 8, 10, 10]
    assert list(visible_key_count(n, 10, 10)) == [10] * 10
    with pytest.raises(ValueError):
        visible_key_count(n, 10, 0)


def test_row_sampling_matches_full_evaluation():
    B, N, H, d = 2, 50, 2, 32
    _, bits = seeded(B, N, H, d, 26)
    rows = np.array([0, 3, 17, 49])
    np.testing.assert_array_equal(lite_la_fwd(bits, B, N, H, d, EPS, rows=rows),
                                  lite_la_fwd(bits, B, N, H, d, EPS)[:, rows])
    np.testing.assert_array_equal(lite_la_block_causal_fwd(bits, B, N, H, d, EPS, 8, rows=rows),
                                  lite_la_block_causal_fwd(bits, B, N, H, d, EPS, 8)[:, rows])


def test_mostly_negative_input_has_sparse_relu_and_small_denominators():
    """The shifted input (q, k ~ N(-1.5, 1)) keeps results finite and in the value hull,
    zero exactly where a query has no positive channel."""
    B, N, H, d = 1, 64, 2, 32
    _, bits = seeded(B, N, H, d, 27, shift=-1.5)
    q, _, v = qkv_arrays(bits, B, N, H, d)
    got = lite_la_fwd(bits, B, N, H, d, EPS)
    assert np.all(np.isfinite(got))
    dead = (q <= 0).all(axis=-1)
    assert np.all(got[dead] == 0)
