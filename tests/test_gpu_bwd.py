"""GPU parity of the LiteLA backward (through the C ABI) against the fp64 backward oracle.

Tolerance, per element of dq, dk or dv (o = oracle value, M = the oracle's error magnitude of
that element: the same sums over absolute values, see oracle/litela_bwd_oracle.py):
  bf16 output: |gpu - o| <= 8e-3 * |o| + 3e-5 * M
  fp32 output: |gpu - o| <= 1e-5 * |o| + 3e-5 * M
The relative term covers the output rounding (bf16: 2^-9).  The M term covers the arithmetic:
a gradient element is a sum of terms of both signs that may cancel far below their size (for
N = 1, dq is eps-small), and the kernels form it from fp32 operands held as bf16 hi + lo pairs
(2^-18 relative each: S, dS, dout/den, h) with fp32 accumulation (~1e-6 relative to the terms
for the token counts here), so its error scales with M, not with the element.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import WORKLOADS, make_qkv, to_bits
import oracle

pytestmark = pytest.mark.gpu

EPS = 1e-15
TOL = {"bf16": (8e-3, 3e-5), "f32": (1e-5, 3e-5)}
D = 32


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_diffusion_litela_b200.build import build
    build()
    ll.lib()


def make_dout(B, N, H, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn((B, N, H * D), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


def gpu_bwd(qkv, dout, H, T=None, mode="bf16"):
    dt = torch.bfloat16 if mode == "bf16" else torch.float32
    dqkv = ll.lite_la_bwd(qkv, dout, H, tokens_per_block=T or 0, eps=EPS, out_dtype=dt)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    B, N = qkv.shape[:2]
    x = dqkv.view(B, N, 3, H, D).to(torch.float64).cpu().numpy()
    return x[:, :, 0], x[:, :, 1], x[:, :, 2]


def oracle_bwd(qkv, dout, H, T=None, rows=None, heads=None):
    """(dq, dk, dv, M(dq), M(dk), M(dv)) from the oracle, each [B, R, H, d]."""
    B, N = qkv.shape[:2]
    qb, gb = to_bits(qkv), to_bits(dout)
    if T is None:
        return oracle.lite_la_bwd(qb, gb, B, N, H, D, EPS, rows=rows, heads=heads, magnitudes=True)
    return oracle.lite_la_block_causal_bwd(qb, gb, B, N, H, D, EPS, T, rows=rows, heads=heads, magnitudes=True)


WORST = {}


def assert_grad_close(got, want, mag, mode, name, heads=None):
    """got, want, mag: [B, R, H, d]; compares the (b, h) in `heads` (all when None)."""
    rtol, atol = TOL[mode]
    B, _, H, _ = want.shape
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for (b, h) in heads:
        w, g, m = want[b, :, h], got[b, :, h], mag[b, :, h]
        err = np.abs(g - w)
        bound = rtol * np.abs(w) + atol * m
        bad = err > bound
        if bad.any():
            i = np.unravel_index(np.argmax(err - bound), err.shape)
            raise AssertionError("%s (b=%d, h=%d): %d of %d elements out of tolerance; worst at %s: gpu=%r "
                                 "oracle=%r (M=%r)" % (name, b, h, bad.sum(), bad.size, i, g[i], w[i], m[i]))
        # largest error beyond the output rounding, in units of M (reported, not asserted)
        excess = np.maximum(err - rtol * np.abs(w), 0.0) / np.maximum(m, 1e-300)
        WORST[(mode, name)] = max(WORST.get((mode, name), 0.0), float(excess.max()))


def check_all(qkv, dout, H, T, mode):
    got = gpu_bwd(qkv, dout, H, T, mode)
    want = oracle_bwd(qkv, dout, H, T)
    for name, g, w, m in zip(("dq", "dk", "dv"), got, want[:3], want[3:]):
        assert_grad_close(g, w, m, mode, name)


SMALL = [  # (B, N, H): one token, ragged tiles, heads that do not fill a quad, several tiles
    (1, 1, 1), (1, 7, 3), (2, 100, 2), (1, 129, 5), (2, 300, 4), (1, 1000, 7), (3, 257, 6),
]


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H", SMALL)
def test_bwd_small_shapes_every_element(B, N, H, mode):
    qkv = make_qkv(B, N, H, D, seed=7000 + B * 1009 + N * 31 + H, device="cuda")
    dout = make_dout(B, N, H, seed=7100 + N + H)
    check_all(qkv, dout, H, None, mode)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H,T", [(1, 7, 2, 1), (2, 40, 3, 1), (1, 100, 2, 7), (2, 300, 3, 128),
                                     (1, 1000, 5, 100), (1, 700, 4, 256), (2, 513, 6, 64), (1, 300, 2, 300)])
def test_bwd_block_causal_small_shapes_every_element(B, N, H, T, mode):
    qkv = make_qkv(B, N, H, D, seed=7200 + B * 1009 + N * 31 + H + T, device="cuda")
    dout = make_dout(B, N, H, seed=7300 + N + T)
    check_all(qkv, dout, H, T, mode)


def test_bwd_1024px_every_element():
    w = WORKLOADS["sana1600m_1024px"]
    B, N, H = w["B"], w["N"], w["H"]
    qkv = make_qkv(B, N, H, D, seed=1001, device="cuda")
    dout = make_dout(B, N, H, seed=7401)
    check_all(qkv, dout, H, None, "bf16")


def sampled(N, T=None, k=48, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, N // 2, N - 2, N - 1]
    if T:
        fixed += [T - 1, T, min(N - 1, 2 * T)]
    return np.unique(np.concatenate([fixed, rng.choice(N, size=k, replace=False)])).astype(np.int64)


def full_size_check(qkv, dout, H, T, heads, rows, mode):
    got = gpu_bwd(qkv, dout, H, T, mode)
    want = oracle_bwd(qkv, dout, H, T, rows=rows, heads=heads)
    for name, g, w, m in zip(("dq", "dk", "dv"), got, want[:3], want[3:]):
        assert_grad_close(g[:, rows], w, m, mode, name, heads=heads)


def test_bwd_4096px_sampled():
    """Full Sana 4096px size (B=2, N=16384, H=70), sampled rows of heads at quad edges."""
    w = WORKLOADS["sana4800m_4096px"]
    B, N, H = w["B"], w["N"], w["H"]
    qkv = make_qkv(B, N, H, D, seed=4000, device="cuda")
    dout = make_dout(B, N, H, seed=7500)
    heads = [(0, 0), (0, 3), (0, 4), (1, 37), (1, 68), (1, 69)]
    full_size_check(qkv, dout, H, None, heads, sampled(N, seed=1), "bf16")


def test_bwd_block_causal_workload_sampled():
    w = WORKLOADS["block_causal_16x1024"]
    B, N, H, T = w["B"], w["N"], w["H"], w["tokens_per_block"]
    qkv = make_qkv(B, N, H, D, seed=1004, device="cuda")
    dout = make_dout(B, N, H, seed=7600)
    heads = [(0, 0), (0, 5), (0, 69)]
    full_size_check(qkv, dout, H, T, heads, sampled(N, T, seed=2), "bf16")


@pytest.mark.parametrize("H,T", [(9, 0), (7, 0), (5, 1024)])
def test_bwd_many_tiles_per_cta_with_a_lone_last_head(H, T):
    """An odd head count leaves the last head pair (and, for H % 4 == 1, the last quad) with one
    head, so one epilogue group of the CTA has no head; with many tiles per CTA that group must
    still keep step with the other.  Sampled rows of the lone head and two others."""
    B, N = 2, 16384
    qkv = make_qkv(B, N, H, D, seed=7650 + H + T, device="cuda")
    dout = make_dout(B, N, H, seed=7660 + H + T)
    heads = [(0, 0), (1, H - 2), (0, H - 1), (1, H - 1)]
    full_size_check(qkv, dout, H, T or None, heads, sampled(N, T or None, seed=3), "bf16")


@pytest.mark.parametrize("H,T", [(9, 0), (8, 0), (5, 512)])
def test_bwd_is_bitwise_deterministic_and_matches_the_phase_timed_call(H, T):
    B, N = 2, 3000
    qkv = make_qkv(B, N, H, D, seed=7700, device="cuda")
    dout = make_dout(B, N, H, seed=7701)
    a = ll.lite_la_bwd(qkv, dout, H, tokens_per_block=T)
    b = ll.lite_la_bwd(qkv, dout, H, tokens_per_block=T)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    stream = torch.cuda.current_stream()
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    c = torch.empty_like(a)
    handles = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in evs])
    s = ll.lib().lite_la_bwd_events(qkv.data_ptr(), dout.data_ptr(), c.data_ptr(), B, N, H, D, EPS, T,
                                    ctypes.c_void_p(stream.cuda_stream), handles)
    assert s == 0, ll.lib().lite_la_last_error().decode()
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    assert torch.equal(a, b) and torch.equal(a, c)
    assert all(evs[i].elapsed_time(evs[i + 1]) >= 0.0 for i in range(3))


def test_bwd_all_negative_query_row_and_interleaved_forward_calls():
    """A query that sees nothing (relu(q) = 0) gets dq = 0 and passes no gradient to k, v;
    forward and backward calls on one stream share the workspace."""
    B, N, H = 1, 600, 5
    qkv = make_qkv(B, N, H, D, seed=7800, device="cuda")
    x = qkv.view(B, N, 3, H, D)
    x[0, 17, 0] = -x[0, 17, 0].abs() - 0.5
    dout = make_dout(B, N, H, seed=7801)
    out1 = ll.lite_la_fwd(qkv, H)
    got = gpu_bwd(qkv, dout, H)
    out2 = ll.lite_la_fwd(qkv, H)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    assert np.all(got[0][0, 17] == 0.0)
    want = oracle_bwd(qkv, dout, H)
    for name, g, w, m in zip(("dq", "dk", "dv"), got, want[:3], want[3:]):
        assert_grad_close(g, w, m, "bf16", name)


def test_bwd_rejects_overlapping_or_misaligned_buffers():
    B, N, H = 1, 64, 2
    qkv = make_qkv(B, N, H, D, seed=7900, device="cuda")
    dout = make_dout(B, N, H, seed=7901)
    lib = ll.lib()
    sh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # dqkv on top of qkv, or of dout
    assert lib.lite_la_bwd(qkv.data_ptr(), dout.data_ptr(), qkv.data_ptr(), B, N, H, D, EPS, sh) == 1
    big = torch.empty(B * N * 3 * H * D + 64, dtype=torch.bfloat16, device="cuda")
    assert lib.lite_la_bwd(qkv.data_ptr(), dout.data_ptr(), big.data_ptr() + 2, B, N, H, D, EPS, sh) == 1
    assert lib.lite_la_block_causal_bwd(qkv.data_ptr(), dout.data_ptr(), big.data_ptr(), B, N, H, D, EPS, 0, sh) == 1
    assert lib.lite_la_bwd(qkv.data_ptr(), dout.data_ptr(), big.data_ptr(), B, N, H, 64, EPS, sh) == 2
    torch.cuda.synchronize()


def test_zz_report_worst_errors():
    """Prints the largest error beyond the output rounding seen above, in units of M."""
    for k in sorted(WORST):
        print("worst excess error / M  %-5s %-3s %.3g" % (k[0], k[1], WORST[k]))


@pytest.mark.parametrize("B,N,H,T,min_chunk", [(2, 1500, 9, 0, 0), (1, 700, 600, 0, 0), (1, 2000, 5, 256, 0),
                                               (2, 300, 3, 1, 0), (2, 2100, 7, 0, 64), (1, 1300, 60, 128, 64)])
def test_forward_saves_the_state_and_the_backward_uses_it(B, N, H, T, min_chunk, paired_min_chunk):
    """lite_la_fwd_save_state: bitwise the plain forward's output, states equal to their
    definition; lite_la_bwd_from_state: the backward within tolerance of the oracle.  The last
    two cases take the paired fused forms, which write the states from their merge warps."""
    from tests.test_gpu_parity import state_reference
    if min_chunk:
        paired_min_chunk(min_chunk)
        assert ll.lite_la_forward_form(B, N, H, D, T) == ("fused_paired_causal" if T else "fused_paired")
    qkv = make_qkv(B, N, H, D, seed=7950 + N + H + T, device="cuda")
    dout = make_dout(B, N, H, seed=7951 + N)
    out, states = ll.lite_la_fwd_save_state(qkv, H, tokens_per_block=T, eps=EPS)
    plain = ll.lite_la_fwd(qkv, H, eps=EPS) if T == 0 else ll.lite_la_block_causal_fwd(qkv, H, T, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
    want_states = state_reference(to_bits(qkv), B, N, H, T)
    got_states = states.double().cpu().numpy()
    err = np.abs(got_states - want_states)
    assert np.all(err <= 1e-6 * (np.abs(want_states) + 1.0) * max(1.0, np.sqrt(N)))
    dqkv = ll.lite_la_bwd_from_state(qkv, dout, states, H, tokens_per_block=T, eps=EPS)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    x = dqkv.view(B, N, 3, H, D).to(torch.float64).cpu().numpy()
    want = oracle_bwd(qkv, dout, H, T or None)
    for i, name in enumerate(("dq", "dk", "dv")):
        assert_grad_close(x[:, :, i], want[i], want[3 + i], "bf16", name)


@pytest.mark.parametrize("T", [0, 128])
def test_autograd_function_matches_the_oracle(T):
    """lite_la as a torch.autograd.Function: gradients of a downstream fp32 loss reach qkv
    through the saved-state backward and match the oracle's."""
    B, N, H = 2, 300, 3
    qkv = make_qkv(B, N, H, D, seed=7900 + T, device="cuda").requires_grad_(True)
    dout = make_dout(B, N, H, seed=7901 + T)
    out = ll.lite_la(qkv, H, tokens_per_block=T, eps=EPS)
    assert out.dtype == torch.bfloat16 and out.requires_grad
    (out.float() * dout.float()).sum().backward()
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    got = qkv.grad.view(B, N, 3, H, D).to(torch.float64).cpu().numpy()
    want = oracle_bwd(qkv.detach(), dout, H, T or None)
    for i, name in enumerate(("dq", "dk", "dv")):
        assert_grad_close(got[:, :, i], want[i], want[3 + i], "bf16", name)
