"""lite_la_fwd_noalloc: the entry point for callers that cannot let the library allocate.

Some hosts own every byte of device memory through their own pool and give an op only its
input and output buffers; others run a latency-bound loop where a first-use cudaMalloc (and
the device synchronisation it can bring) is not acceptable.  lite_la_fwd_noalloc serves them
from one fixed, statically defined device array instead of the library's allocated workspace.

These tests call it through the C ABI, on two calls in a row with different shapes (so that
contents the first call left in the shared array could show up in the second's result), and
check each result three ways:
  * against the fp64 oracle, element by element, at the bf16 tolerance 1e-3 + 8e-3 |o|;
  * bitwise against lite_la_fwd: both run the same deterministic kernels with a fixed merge
    order, so any difference would come from the scratch (a stale value, a wrong offset);
  * through lite_la_device_status, which reads the array's error word (a bounded wait that
    timed out would otherwise show only as wrong output).
All of the entry point's paths are covered: the single fused kernel (B * ceil(H/4) <= 148), its
paired form (chunks of at least the paired minimum: the 4096px call) and the three-kernel path
(more head quads than SMs).  A problem too large for the array is
refused before anything runs.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import make_qkv, to_bits
import oracle

pytestmark = pytest.mark.gpu
EPS = 1e-15


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_diffusion_litela_b200.build import build
    build()
    return ll.lib()


def noalloc(lib, qkv, H):
    B, N = qkv.shape[:2]
    out = torch.empty((B, N, H * 32), dtype=torch.bfloat16, device=qkv.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.lite_la_fwd_noalloc(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, stream)
    assert st == 0, lib.lite_la_last_error().decode()
    return out


def assert_matches_oracle(got, qkv, H, rows=None):
    B, N = qkv.shape[:2]
    want = oracle.lite_la_fwd(to_bits(qkv), B, N, H, 32, EPS, rows=rows)
    g = got.view(B, N, H, 32).double().cpu().numpy()
    if rows is not None:
        g = g[:, rows]
    err = np.abs(g - want)
    bound = 1e-3 + 8e-3 * np.abs(want)
    assert np.all(err <= bound), "%d elements out of tolerance" % int((err > bound).sum())


def test_noalloc_matches_the_oracle_and_lite_la_fwd_on_two_calls_in_a_row(lib):
    # (B, N, H, seed): the first takes the fused kernel; the second, with 160 head quads, the
    # three-kernel path (its partial states and state images fill about 6 MB of the array);
    # the third is the fused kernel again, after the three-kernel call left its contents
    cases = [(2, 1000, 5, 11), (8, 512, 80, 13), (1, 333, 3, 12)]
    assert lib.lite_la_kernels_per_call(8, 512, 80, 32, 0) == 3
    assert lib.lite_la_kernels_per_call(2, 1000, 5, 32, 0) == 1
    results = []
    for B, N, H, seed in cases:
        qkv = make_qkv(B, N, H, 32, seed=seed, device="cuda")
        got = noalloc(lib, qkv, H)
        ll.lite_la_device_status()
        ref = ll.lite_la_fwd(qkv, H, eps=EPS)
        ll.lite_la_device_status()
        results.append((qkv, H, got, ref))
    for qkv, H, got, ref in results:
        assert torch.equal(got, ref)
        assert_matches_oracle(got, qkv, H)


def test_noalloc_full_size_4096px_call(lib):
    B, N, H = 2, 16384, 70
    assert ll.lite_la_forward_form(B, N, H) == "fused_paired"
    qkv = make_qkv(B, N, H, 32, seed=4000, device="cuda")
    got = noalloc(lib, qkv, H)
    ll.lite_la_device_status()
    ref = ll.lite_la_fwd(qkv, H, eps=EPS)
    ll.lite_la_device_status()
    assert torch.equal(got, ref)
    rng = np.random.default_rng(77)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, N - 1], rng.integers(0, N, 24)]))
    assert_matches_oracle(got, qkv, H, rows)


def test_noalloc_rejects_a_problem_larger_than_its_scratch(lib):
    B, N, H = 1, 1, 4000            # 4000 heads: partial states alone exceed the fixed array
    qkv = torch.zeros((B, N, 3 * H * 32), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, N, H * 32), dtype=torch.bfloat16, device="cuda")
    st = lib.lite_la_fwd_noalloc(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, None)
    assert st == 1
    assert "scratch" in lib.lite_la_last_error().decode()
