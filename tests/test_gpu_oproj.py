"""GPU parity of LiteLA + output projection (lite_la_fwd_oproj: the apply inside the projection
GEMM) and of the projection alone (lite_la_out_proj), through the C ABI, against the fp64
oracle (oracle/litela_oproj_oracle.py).

Tolerances, per output element n, derived from the arithmetic (x = the exact attention output
or the given input, W the weights, |.| elementwise, @ a matrix product):
  projection alone: products of bf16 values are exact in fp32; the fp32 accumulation of K
    terms errs by at most about K * 2^-23 of sum_k |x_k W_nk| (3e-4 covers K = 2240), and the
    bf16 output rounding by 2^-9 |y|:
        |y - y_ref| <= 2^-8 |y_ref| + 3e-4 (|x| @ |W|^T)_n + 1e-6
  fused: each A_k (LiteLA's output as the GEMM takes it) is the fp32 apply, accurate to the
    fp32-output bar 1e-5 + 1e-4 |x_k| of LiteLA's own tests, rounded to bf16 (2^-9 |x_k|), so
    |A_k - x_k| <= 1.1e-5 + 2.1e-3 |x_k|, and
        |y - y_ref| <= ((1.1e-5 + 2.1e-3 |x|) @ |W|^T)_n + 3e-4 (|x| @ |W|^T)_n + 2^-8 |y_ref| + 1e-6
  identity and signed power-of-two selection weights make the projection exact, so there the
  fused output must meet LiteLA's own bf16 bar, 1e-3 + 8e-3 |x|, element by element (scaled by
  the selection's power of two).
Small shapes are compared on every element; the 4096px shape on sampled token rows.
"""
import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import make_qkv, to_bits
import oracle

pytestmark = pytest.mark.gpu
EPS = 1e-15
D = 32


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_diffusion_litela_b200.build import build
    build()
    ll.lib()


def make_weight(C_out, C_in, seed):
    """nn.Linear-like weight U(-1/sqrt(C_in), 1/sqrt(C_in)) in bf16, and a small fp32 bias."""
    g = torch.Generator().manual_seed(seed)
    w = ((torch.rand((C_out, C_in), generator=g) * 2 - 1) / np.sqrt(C_in)).to(torch.bfloat16)
    b = (torch.randn((C_out,), generator=g) * 0.02).to(torch.float32)
    return w, b


def dec(t):
    return oracle.decode_bf16(to_bits(t.cpu()))


def attention(qkv, H, T=None, rows=None):
    B, N = qkv.shape[:2]
    bits = to_bits(qkv)
    x = (oracle.lite_la_block_causal_fwd(bits, B, N, H, D, EPS, T, rows=rows) if T else
         oracle.lite_la_fwd(bits, B, N, H, D, EPS, rows=rows))
    return x.reshape(B, x.shape[1], H * D)


def check(got, want, tol, what):
    err = np.abs(got - want)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError("%s: %d of %d elements out of tolerance; worst at %s: gpu=%r ref=%r tol=%r"
                             % (what, bad.sum(), bad.size, i, got[i], want[i], tol[i]))


def fused_tol(x, wd, y_ref):
    ax, aw = np.abs(x), np.abs(wd)
    return (1.1e-5 + 2.1e-3 * ax) @ aw.T + 3e-4 * (ax @ aw.T) + 2.0 ** -8 * np.abs(y_ref) + 1e-6


def run_fused(qkv, H, w, bias, T=0):
    y = ll.lite_la_fwd_oproj(qkv, H, w, bias, tokens_per_block=T or 0, eps=EPS)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    return y


FUSED = [  # (B, N, H, C_out, T): ragged token tiles, a lone last head (H odd), C_out below and
           # above one 224-column tile and not a multiple of it, block-causal, T >= N
    (1, 1, 1, 8, None), (1, 7, 3, 40, None), (2, 300, 5, 232, None), (1, 1000, 7, 456, None),
    (2, 256, 4, 224, 128), (1, 640, 2, 64, 256), (1, 300, 3, 96, 1000), (2, 129, 70, 2240, None),
]


@pytest.mark.parametrize("B,N,H,C_out,T", FUSED)
@pytest.mark.parametrize("with_bias", [True, False])
def test_fused_matches_the_oracle_every_element(B, N, H, C_out, T, with_bias):
    qkv = make_qkv(B, N, H, D, seed=500 + 7 * N + H, device="cuda")
    w, b = make_weight(C_out, H * D, seed=C_out + H)
    bias = b.cuda() if with_bias else None
    y = run_fused(qkv, H, w.cuda(), bias, T)
    x = attention(qkv, H, T)
    wd = dec(w)
    y_ref = oracle.linear(x, to_bits(w), C_out, H * D, b.numpy() if with_bias else None)
    check(dec(y), y_ref, fused_tol(x, wd, y_ref), "fused vs oracle")


@pytest.mark.parametrize("B,N,H,T", [(2, 300, 5, None), (1, 129, 70, None), (1, 384, 3, 128)])
def test_fused_with_exact_projections_meets_lite_la_bf16_bar(B, N, H, T):
    """W = I gives LiteLA's own output; a signed power-of-two selection (with repeats, fewer
    outputs than inputs) gives exactly that multiple of chosen channels."""
    qkv = make_qkv(B, N, H, D, seed=900 + N + H, device="cuda")
    C = H * D
    x = attention(qkv, H, T)
    y = dec(run_fused(qkv, H, torch.eye(C, dtype=torch.bfloat16, device="cuda"), None, T))
    check(y, x, 1e-3 + 8e-3 * np.abs(x), "identity projection")
    rng = np.random.default_rng(N)
    C_out = max(8, (C // 2) // 8 * 8)
    pick = rng.integers(0, C, C_out)
    scale = rng.choice([-4.0, -0.5, 0.25, 1.0, 2.0], C_out)
    sel = np.zeros((C_out, C), dtype=np.float32)
    sel[np.arange(C_out), pick] = scale
    y = dec(run_fused(qkv, H, torch.from_numpy(sel).to(torch.bfloat16).cuda(), None, T))
    want = x[:, :, pick] * scale
    check(y, want, np.abs(scale) * (1e-3 + 8e-3 * np.abs(x[:, :, pick])), "selection projection")


@pytest.mark.parametrize("B,N,C_in,C_out", [(1, 1, 8, 8), (2, 300, 96, 232), (1, 1000, 2240, 456),
                                            (2, 130, 2240, 2240), (1, 257, 72, 40)])
def test_projection_alone_matches_the_oracle(B, N, C_in, C_out):
    g = torch.Generator().manual_seed(C_in + C_out)
    x = torch.randn((B, N, C_in), generator=g).to(torch.bfloat16)
    w, b = make_weight(C_out, C_in, seed=C_in)
    y = ll.lite_la_out_proj(x.cuda(), w.cuda(), b.cuda())
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    xd, wd = dec(x), dec(w)
    y_ref = oracle.linear(to_bits(x), to_bits(w), C_out, C_in, b.numpy())
    tol = 2.0 ** -8 * np.abs(y_ref) + 3e-4 * (np.abs(xd) @ np.abs(wd).T) + 1e-6
    check(dec(y), y_ref, tol, "projection vs oracle")


def test_fused_agrees_with_the_unfused_chain_and_is_deterministic():
    """lite_la_fwd followed by lite_la_out_proj takes the same GEMM over the same bf16 x up to
    one bf16 unit in the last place of some x elements (the apply's two fp32 routes round
    differently): |y_fused - y_unfused| <= 2^-7 (|x| @ |W|^T) + 2^-8 |y|."""
    B, N, H, C_out = 2, 700, 70, 2240
    qkv = make_qkv(B, N, H, D, seed=4242, device="cuda")
    w, b = make_weight(C_out, H * D, seed=77)
    w, b = w.cuda(), b.cuda()
    y1 = run_fused(qkv, H, w, b)
    y2 = run_fused(qkv, H, w, b)
    assert torch.equal(y1, y2)
    x = ll.lite_la_fwd(qkv, H, eps=EPS)
    yu = ll.lite_la_out_proj(x, w, b)
    torch.cuda.synchronize()
    xd, wd, yud = dec(x), dec(w), dec(yu)
    check(dec(y1), yud, 2.0 ** -7 * (np.abs(xd) @ np.abs(wd).T) + 2.0 ** -8 * np.abs(yud) + 1e-6, "fused vs unfused")


def test_fused_1024px_every_element():
    """The Sana-1600M 1024px shape (B = 2 CFG pair, N = 32 x 32, H = 70, C_out = 2240), every
    output element, with bias."""
    B, N, H, C_out = 2, 1024, 70, 2240
    qkv = make_qkv(B, N, H, D, seed=1001, device="cuda")
    w, b = make_weight(C_out, H * D, seed=1024)
    y = run_fused(qkv, H, w.cuda(), b.cuda())
    y2 = run_fused(qkv, H, w.cuda(), b.cuda())
    assert torch.equal(y, y2)
    x = attention(qkv, H)
    y_ref = oracle.linear(x, to_bits(w), C_out, H * D, b.numpy())
    check(dec(y), y_ref, fused_tol(x, dec(w), y_ref), "fused 1024px vs oracle")


def test_fused_full_size_4096px_sampled_rows():
    B, N, H, C_out = 2, 16384, 70, 2240
    qkv = make_qkv(B, N, H, D, seed=4000, device="cuda")
    w, b = make_weight(C_out, H * D, seed=4096)
    y = dec(run_fused(qkv, H, w.cuda(), b.cuda()))
    rng = np.random.default_rng(4096)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, 255, 8191, 8192, N - 129, N - 128, N - 1],
                                     rng.integers(0, N, 13)]))
    x = attention(qkv, H, rows=rows)
    y_ref = oracle.linear(x, to_bits(w), C_out, H * D, b.numpy())
    check(y[:, rows], y_ref, fused_tol(x, dec(w), y_ref), "fused 4096px vs oracle")
