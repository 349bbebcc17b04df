"""Oracle pinned to the hand-worked example in tests/golden/litela_worked_example.txt."""
import os
from fractions import Fraction

import numpy as np
import pytest

from linear_attention_diffusion_litela_b200.inputs import pack_qkv, to_bits
from oracle import lite_la_block_causal_fwd, lite_la_fwd
from tests.exact_state_form import lite_la_exact, state_of

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "litela_worked_example.txt")
EPS = 1e-15


def load_golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            out[key] = [[Fraction(x.strip()) for x in row.split(",")] for row in val.split(";")]
    return out


def golden_qkv_bits(g):
    q = np.array(g["q"], dtype=np.float64)[None, :, None, :]
    k = np.array(g["k"], dtype=np.float64)[None, :, None, :]
    v = np.array(g["v"], dtype=np.float64)[None, :, None, :]
    return to_bits(pack_qkv(q, k, v))


def as_float(rows):
    return np.array([[float(x) for x in r] for r in rows])


def test_golden_inputs_roundtrip_exactly():
    g = load_golden()
    from oracle import decode_bf16, unpack_qkv
    x = decode_bf16(golden_qkv_bits(g)).reshape(1, 3, 3 * 1 * 2)
    q, k, v = unpack_qkv(x, 1, 2)
    assert np.array_equal(q[0, :, 0], as_float(g["q"]))
    assert np.array_equal(k[0, :, 0], as_float(g["k"]))
    assert np.array_equal(v[0, :, 0], as_float(g["v"]))


@pytest.mark.parametrize("key,T", [("out_noncausal", None), ("out_block_T1", 1), ("out_block_T2", 2)])
def test_oracle_matches_hand_worked_values(key, T):
    g = load_golden()
    bits = golden_qkv_bits(g)
    if T is None:
        got = lite_la_fwd(bits, 1, 3, 1, 2, EPS)[0, :, 0, :]
    else:
        got = lite_la_block_causal_fwd(bits, 1, 3, 1, 2, EPS, T)[0, :, 0, :]
    np.testing.assert_allclose(got, as_float(g[key]), rtol=1e-13, atol=0)


@pytest.mark.parametrize("key,T", [("out_noncausal", None), ("out_block_T1", 1), ("out_block_T2", 2)])
def test_exact_state_route_matches_hand_worked_values(key, T):
    g = load_golden()
    got = lite_la_exact(g["q"], g["k"], g["v"], 0, T)
    assert got == g[key]


def test_hand_worked_states():
    g = load_golden()
    assert state_of(g["k"], g["v"]) == g["state"]
    assert state_of(g["k"][:2], g["v"][:2]) == g["state_block0_T2"]
