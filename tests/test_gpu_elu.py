"""GPU parity of the ELU+1 variant (lite_la_elu1_fwd) against its fp64 oracle.

Tolerance as for LiteLA: bf16 output |gpu - o| <= 1e-3 + 8e-3 |o|; fp32 output
|gpu - o| <= 1e-5 + 1e-4 |o| (phi is formed in fp32 with expf and enters the tensor cores as a
bf16 hi + lo pair, 2^-17 relative).  In the clamp branch every output is ~1e-17, so there the
absolute term is taken relative to the largest output instead.
"""
import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import WORKLOADS, make_qkv, to_bits
import oracle

pytestmark = pytest.mark.gpu

TOL = {"bf16": (1e-3, 8e-3), "f32": (1e-5, 1e-4)}
D = 32


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_diffusion_litela_b200.build import build
    build()
    ll.lib()


def run(qkv, H, T, mode, clamp=1e-6):
    out = ll.lite_la_elu1_fwd(qkv, H, tokens_per_block=T or 0, clamp_min=clamp,
                              out_dtype=torch.bfloat16 if mode == "bf16" else torch.float32)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    B, N = qkv.shape[:2]
    return out.view(B, N, H, D).double().cpu().numpy()


def check(got, want, mode, atol=None):
    a, r = TOL[mode]
    a = a if atol is None else atol
    err = np.abs(got - want)
    bound = a + r * np.abs(want)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError("%d of %d out of tolerance; worst at %s: gpu=%r oracle=%r" % (bad.sum(), bad.size, i, got[i], want[i]))


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H,T", [(1, 1, 1, None), (1, 7, 3, None), (2, 300, 5, None), (1, 1000, 7, None),
                                     (3, 257, 4, None), (1, 100, 2, 7), (2, 300, 3, 128), (1, 1000, 5, 100),
                                     (1, 40, 2, 1)])
def test_elu1_small_shapes_every_element(B, N, H, T, mode):
    qkv = make_qkv(B, N, H, D, seed=8000 + B * 101 + N + H + (T or 0), device="cuda")
    want = oracle.elu1_fwd(to_bits(qkv), B, N, H, D, 1e-6, T)
    check(run(qkv, H, T, mode), want, mode)


def test_elu1_clamp_branch():
    """q and k far below 0: phi ~ exp(-30), every key sum is below the clamp."""
    B, N, H = 1, 200, 2
    qkv = make_qkv(B, N, H, D, seed=8100, device="cuda")
    x = qkv.view(B, N, 3, H, D)
    x[:, :, :2] -= 30.0
    want = oracle.elu1_fwd(to_bits(qkv), B, N, H, D, 1e-6)
    got = run(qkv, H, None, "f32")
    check(got, want, "f32", atol=1e-4 * np.abs(want).max())


def test_elu1_4096px_sampled():
    w = WORKLOADS["sana4800m_4096px"]
    B, N, H = w["B"], w["N"], w["H"]
    qkv = make_qkv(B, N, H, D, seed=4000, device="cuda")
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 64, replace=False)]))
    want = oracle.elu1_fwd(to_bits(qkv), B, N, H, D, 1e-6, rows=rows)
    got = run(qkv, H, None, "bf16")[:, rows]
    check(got, want, "bf16")


def test_elu1_is_deterministic_and_differs_from_litela():
    B, N, H = 2, 3000, 9
    qkv = make_qkv(B, N, H, D, seed=8200, device="cuda")
    a = ll.lite_la_elu1_fwd(qkv, H)
    b = ll.lite_la_elu1_fwd(qkv, H)
    c = ll.lite_la_fwd(qkv, H)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and not torch.equal(a, c)


def test_elu1_more_head_quads_than_sms_takes_the_three_kernel_path():
    """Non-causal ELU + 1 calls take the fused single kernel while B * ceil(H/4) fits the SMs;
    with 160 head quads they take the reduction, the scan and the apply: both match the oracle."""
    B, N, H = 8, 512, 80
    assert ll.lib().lite_la_kernels_per_call(B, N, H, D, 0) == 3
    assert ll.lib().lite_la_kernels_per_call(2, 4096, 70, D, 0) == 1
    qkv = make_qkv(B, N, H, D, seed=8300, device="cuda")
    want = oracle.elu1_fwd(to_bits(qkv), B, N, H, D, 1e-6)
    check(run(qkv, H, None, "bf16"), want, "bf16")
