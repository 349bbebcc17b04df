"""Pins for the fp64 oracle of the ELU+1 variant (oracle/litela_elu_oracle.py), CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_attention_diffusion_litela_b200.inputs import to_bits

D = 32


def test_phi_closed_forms_and_torch_elu():
    x = np.array([-30.0, -2.0, -1e-3, 0.0, 1e-3, 0.5, 3.0])
    want = [math.exp(-30.0), math.exp(-2.0), math.exp(-1e-3), 1.0, 1.001, 1.5, 4.0]
    np.testing.assert_allclose(oracle.phi_elu1(x), want, rtol=1e-15)
    t = torch.tensor(x, dtype=torch.float64)
    # torch forms elu(x) + 1 as expm1(x) + 1, which cancels for very negative x: absolute check
    np.testing.assert_allclose(oracle.phi_elu1(x), (torch.nn.functional.elu(t) + 1).numpy(), rtol=1e-15, atol=1e-15)
    assert np.all(oracle.phi_elu1(np.linspace(-50, 50, 1001)) > 0)


def context_route(q, k, v, clamp, T=None):
    """The page's context route (phi(K)^T V and the key sum), an independent evaluation."""
    N, d = q.shape
    pq = oracle.phi_elu1(q) / math.sqrt(d)
    pk = oracle.phi_elu1(k)
    out = np.empty_like(q)
    for i in range(N):
        n = N if T is None else min((i // T + 1) * T, N)
        ctx = pk[:n].T @ v[:n]                       # [d, d]
        ksum = pk[:n].sum(axis=0)                    # [d]
        out[i] = (pq[i] @ ctx) / max(pq[i] @ ksum, clamp)
    return out


@pytest.mark.parametrize("N,T", [(1, None), (5, None), (33, None), (9, 1), (20, 4), (17, 100)])
def test_quadratic_form_equals_the_context_route(N, T):
    rng = np.random.default_rng(N + (T or 0))
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    nv = None if T is None else oracle.visible_key_count(np.arange(N), N, T)
    got = oracle.elu1_rows(q, k, v, 1e-6, nv)
    np.testing.assert_allclose(got, context_route(q, k, v, 1e-6, T), rtol=1e-12, atol=1e-14)


def test_invariants_and_the_clamp_branch():
    rng = np.random.default_rng(3)
    N = 40
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    base = oracle.elu1_rows(q, k, v, 1e-6)
    perm = rng.permutation(N)
    np.testing.assert_allclose(oracle.elu1_rows(q, k[perm], v[perm], 1e-6), base, rtol=1e-12)
    # constant values: every weight is positive, so out = c exactly up to rounding
    np.testing.assert_allclose(oracle.elu1_rows(q, k, np.full((N, D), 2.5), 1e-6), 2.5, rtol=1e-13)
    # outputs are convex combinations of the values
    assert np.all(base <= v.max(axis=0) + 1e-12) and np.all(base >= v.min(axis=0) - 1e-12)
    # the clamp: very negative q and k make the key sum tiny, then out = num / clamp
    qs, ks = q - 30.0, k - 30.0
    w = (oracle.phi_elu1(qs) / math.sqrt(D)) @ oracle.phi_elu1(ks).T
    assert w.sum(axis=1).max() < 1e-6
    np.testing.assert_allclose(oracle.elu1_rows(qs, ks, v, 1e-6), (w @ v) / 1e-6, rtol=1e-12)
    # away from the clamp the 1/sqrt(d) scale cancels: an unscaled, unclamped evaluation agrees
    pq, pk = oracle.phi_elu1(q), oracle.phi_elu1(k)
    w2 = pq @ pk.T
    np.testing.assert_allclose(base, (w2 @ v) / w2.sum(axis=1, keepdims=True), rtol=1e-12)


def test_packed_entry_point_and_rows():
    rng = np.random.default_rng(4)
    B, N, H = 2, 30, 3
    bits = to_bits(torch.from_numpy(rng.standard_normal((B, N, 3 * H * D)).astype(np.float32)).to(torch.bfloat16))
    x = oracle.decode_bf16(bits).reshape(B, N, 3 * H * D)
    q, k, v = oracle.unpack_qkv(x, H, D)
    for T in (None, 7):
        full = oracle.elu1_fwd(bits, B, N, H, D, 1e-6, T)
        for b in range(B):
            for h in range(H):
                nv = None if T is None else oracle.visible_key_count(np.arange(N), N, T)
                np.testing.assert_array_equal(full[b, :, h], oracle.elu1_rows(q[b, :, h], k[b, :, h], v[b, :, h], 1e-6, nv))
        rows = np.array([0, 13, 29])
        np.testing.assert_allclose(oracle.elu1_fwd(bits, B, N, H, D, 1e-6, T, rows=rows), full[:, rows], rtol=1e-13)
    with pytest.raises(ValueError):
        oracle.elu1_fwd(bits, B, N, H, D, 1e-6, 0)
