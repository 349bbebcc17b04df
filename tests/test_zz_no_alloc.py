"""lite_la_fwd_noalloc: the entry point for callers that cannot let the library allocate.

Some hosts own every byte of device memory through their own pool and give an op only its
input and output buffers; others run a latency-bound loop where a first-use cudaMalloc (and
the device synchronisation it can bring) is not acceptable.  lite_la_fwd_noalloc serves them
from one fixed, statically defined device array instead of the library's allocated workspace.
These tests call it through the C ABI and check it against lite_la_fwd on two calls in a row
(the second with another shape, so that contents the first call left in the shared array
cannot leak into its result), and check that a problem too large for the array is refused.
This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import make_qkv

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


def test_noalloc_matches_lite_la_fwd_on_two_calls_in_a_row(lib):
    cases = [(2, 1000, 5, 11), (1, 333, 3, 12)]
    outs = []
    for B, N, H, seed in cases:
        qkv = make_qkv(B, N, H, 32, seed=seed, device="cuda")
        outs.append((noalloc(lib, qkv, H), ll.lite_la_fwd(qkv, H, eps=EPS)))
    torch.cuda.synchronize()
    for got, ref in outs:
        g = got.double().cpu().numpy()
        r = ref.double().cpu().numpy()
        assert np.all(np.abs(g - r) <= 1e-3 + 8e-3 * np.abs(r))


def test_noalloc_full_size_4096px_call(lib):
    B, N, H = 2, 16384, 70
    qkv = make_qkv(B, N, H, 32, seed=4000, device="cuda")
    got = noalloc(lib, qkv, H)
    ref = ll.lite_la_fwd(qkv, H, eps=EPS)
    torch.cuda.synchronize()
    g, r = got.double().cpu().numpy(), ref.double().cpu().numpy()
    assert np.all(np.abs(g - r) <= 1e-3 + 8e-3 * np.abs(r))


def test_noalloc_rejects_a_problem_larger_than_its_scratch(lib):
    B, N, H = 1, 1, 4000            # 4000 heads: partial states alone exceed the fixed array
    qkv = torch.zeros((B, N, 3 * H * 32), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, N, H * 32), dtype=torch.bfloat16, device="cuda")
    st = lib.lite_la_fwd_noalloc(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, None)
    assert st == 1
    assert "scratch" in lib.lite_la_last_error().decode()
