"""CPU-only checks of the C ABI: the library loads, exports every symbol include/litela.h
declares, and its host-side logic (status strings, argument validation, workspace sizing)
behaves as documented.  Nothing here launches a kernel."""
import ctypes
import os
import re

import pytest

import linear_attention_diffusion_litela_b200 as ll

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "litela.h")


@pytest.fixture(scope="module")
def lib():
    from linear_attention_diffusion_litela_b200.build import build
    build()
    return ll.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lite_la_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for required in ("lite_la_fwd", "lite_la_block_causal_fwd", "lite_la_fwd_f32out",
                     "lite_la_block_causal_fwd_f32out", "lite_la_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_binding_covers_every_declared_symbol():
    assert sorted(ll.EXPORTED_SYMBOLS) == declared_functions()


def test_status_strings(lib):
    for code, name in ll.STATUS.items():
        assert lib.lite_la_status_string(code).decode() == name
    assert lib.lite_la_status_string(99).decode() == "LITELA_UNKNOWN_STATUS"


# Argument validation happens on the host, before any CUDA call.
BAD_ARGS = [
    # (B, N, H, d, eps, expected status)
    (-1, 4, 1, 32, 1e-15, 1),
    (1, -4, 1, 32, 1e-15, 1),
    (1, 4, -1, 32, 1e-15, 1),
    (1, 4, 1, 0, 1e-15, 1),
    (1, 4, 1, 64, 1e-15, 2),
    (1, 4, 1, 16, 1e-15, 2),
    (1, 4, 1, 32, -1.0, 1),
    (1, 4, 1, 32, float("nan"), 1),
    (1, 4, 1, 32, float("inf"), 1),
    (70000, 4, 1, 32, 1e-15, 1),
]


@pytest.mark.parametrize("B,N,H,d,eps,want", BAD_ARGS)
def test_invalid_arguments_are_rejected_on_the_host(lib, B, N, H, d, eps, want):
    fake_in, fake_out = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 30)
    assert lib.lite_la_fwd(fake_in, fake_out, B, N, H, d, eps, None) == want
    assert lib.lite_la_last_error().decode() != ""
    assert lib.lite_la_fwd_f32out(fake_in, fake_out, B, N, H, d, eps, None) == want
    assert lib.lite_la_block_causal_fwd(fake_in, fake_out, B, N, H, d, eps, 16, None) == want


def test_null_misaligned_and_overlapping_buffers_are_rejected(lib):
    a, b = 1 << 20, 1 << 30
    assert lib.lite_la_fwd(None, ctypes.c_void_p(b), 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_fwd(ctypes.c_void_p(a), None, 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_fwd(ctypes.c_void_p(a + 2), ctypes.c_void_p(b), 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_fwd(ctypes.c_void_p(a), ctypes.c_void_p(b + 8), 1, 4, 1, 32, 1e-15, None) == 1
    # out starts inside qkv (qkv is 4 tokens * 96 channels * 2 bytes = 768 bytes)
    assert lib.lite_la_fwd(ctypes.c_void_p(a), ctypes.c_void_p(a + 256), 1, 4, 1, 32, 1e-15, None) == 1
    assert "overlap" in lib.lite_la_last_error().decode()


@pytest.mark.parametrize("T", [0, -3])
def test_block_size_must_be_positive(lib, T):
    a, b = 1 << 20, 1 << 30
    assert lib.lite_la_block_causal_fwd(ctypes.c_void_p(a), ctypes.c_void_p(b), 1, 4, 1, 32, 1e-15, T, None) == 1


@pytest.mark.parametrize("B,N,H", [(0, 4, 1), (1, 0, 1), (1, 4, 0), (0, 0, 0)])
def test_empty_problem_is_a_no_op(lib, B, N, H):
    # null pointers are fine for an empty problem: nothing is read or written
    assert lib.lite_la_fwd(None, None, B, N, H, 32, 1e-15, None) == 0
    assert lib.lite_la_block_causal_fwd(None, None, B, N, H, 32, 1e-15, 4, None) == 0


def test_workspace_bytes(lib):
    state = 33 * 32 * 4
    assert ll.lite_la_workspace_bytes(0, 16, 1) == 0
    assert ll.lite_la_workspace_bytes(1, 16, 1, d=64) == 0
    for (B, N, H, T) in [(1, 1, 1, 0), (2, 1024, 70, 0), (2, 16384, 70, 0), (1, 16384, 70, 1024),
                         (1, 100, 3, 7)]:
        nblk = 1 if T <= 0 else -(-N // T)
        got = ll.lite_la_workspace_bytes(B, N, H, 32, T)
        # at least one partial state per (batch, head, block)
        assert got >= B * H * nblk * state
        assert got % 4 == 0
    # a causal block at least as long as N is the non-causal problem
    assert ll.lite_la_workspace_bytes(2, 500, 3, 32, 500) == ll.lite_la_workspace_bytes(2, 500, 3, 32, 0)
    assert ll.lite_la_workspace_bytes(2, 500, 3, 32, 10**6) == ll.lite_la_workspace_bytes(2, 500, 3, 32, 0)


def test_ffma_peak_library_exports_its_header_and_counts_flops():
    from linear_attention_diffusion_litela_b200.build import build
    build()
    text = open(os.path.join(ROOT, "include", "litela_ffma_peak.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = sorted(set(re.findall(r"\b(litela_ffma_\w+)\s*\(", text)))
    assert names == ["litela_ffma_flops", "litela_ffma_launch"]
    h = ll.ffma_peak_lib()
    for n in names:
        assert hasattr(h, n)
    # 2 FLOPs per multiply-add, 8 chains x 16 unrolled rounds per iteration per thread
    assert h.litela_ffma_flops(148, 512, 10) == 2 * 148 * 512 * 10 * 128
    assert h.litela_ffma_flops(0, 512, 10) == 0
    # invalid launch arguments are rejected before anything is launched
    assert h.litela_ffma_launch(None, 1, 32, 1, None) == 1
    assert h.litela_ffma_launch(ctypes.c_void_p(1 << 20), 1, 48, 1, None) == 1
    assert h.litela_ffma_launch(ctypes.c_void_p(1 << 20), 1, 1024, 1, None) == 1


def test_backward_arguments_are_validated_on_the_host(lib):
    a, g, o = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24), ctypes.c_void_p(1 << 30)
    # qkv is 4 tokens x 96 channels x 2 bytes = 768 bytes, dout 256 bytes
    for B, N, H, d, eps, want in BAD_ARGS:
        assert lib.lite_la_bwd(a, g, o, B, N, H, d, eps, None) == want
        assert lib.lite_la_bwd_f32out(a, g, o, B, N, H, d, eps, None) == want
        assert lib.lite_la_block_causal_bwd(a, g, o, B, N, H, d, eps, 16, None) == want
    assert lib.lite_la_bwd(None, g, o, 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_bwd(a, None, o, 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_bwd(a, g, None, 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_bwd(a, g, ctypes.c_void_p((1 << 30) + 4), 1, 4, 1, 32, 1e-15, None) == 1
    # dqkv overlapping qkv or dout
    assert lib.lite_la_bwd(a, g, ctypes.c_void_p((1 << 20) + 512), 1, 4, 1, 32, 1e-15, None) == 1
    assert "overlap" in lib.lite_la_last_error().decode()
    assert lib.lite_la_bwd(a, g, ctypes.c_void_p((1 << 24) - 512), 1, 4, 1, 32, 1e-15, None) == 1
    assert lib.lite_la_block_causal_bwd(a, g, o, 1, 4, 1, 32, 1e-15, 0, None) == 1
    # an empty problem is a no-op; events are required for the timed variant
    assert lib.lite_la_bwd(None, None, None, 0, 4, 1, 32, 1e-15, None) == 0
    null = (ctypes.c_void_p * 4)(None, None, None, None)
    assert lib.lite_la_bwd_events(a, g, o, 1, 4, 1, 32, 1e-15, 0, None, null) == 1


def test_backward_workspace_bytes(lib):
    state = 33 * 32 * 4
    assert ll.lib().lite_la_bwd_workspace_bytes(0, 16, 1, 32, 0) == 0
    assert ll.lib().lite_la_bwd_workspace_bytes(1, 16, 1, 64, 0) == 0
    for (B, N, H, T) in [(1, 1, 1, 0), (2, 16384, 70, 0), (1, 16384, 70, 1024), (1, 100, 3, 7)]:
        nblk = 1 if T <= 0 else -(-N // T)
        got = ll.lib().lite_la_bwd_workspace_bytes(B, N, H, 32, T)
        # the forward's partials, S images (5120 B), S^T images (4096 B), dS partials, dS and dS^T
        # images (4096 B each) and dS ones rows (128 B)
        assert got >= B * H * nblk * (2 * state + 5120 + 3 * 4096 + 128)
        assert got >= ll.lite_la_workspace_bytes(B, N, H, 32, T) - 64 * 4


def test_saved_state_entry_points_validate_on_the_host(lib):
    a, g, o, st = (ctypes.c_void_p(1 << k) for k in (20, 24, 30, 34))
    assert lib.lite_la_fwd_save_state(a, o, None, 1, 4, 1, 32, 1e-15, 0, None) == 1
    assert lib.lite_la_fwd_save_state(a, o, ctypes.c_void_p((1 << 34) + 4), 1, 4, 1, 32, 1e-15, 0, None) == 1
    assert lib.lite_la_bwd_from_state(a, g, None, o, 1, 4, 1, 32, 1e-15, 0, None) == 1
    assert lib.lite_la_bwd_from_state(a, g, ctypes.c_void_p((1 << 34) + 8), o, 1, 4, 1, 32, 1e-15, 0, None) == 1
    assert lib.lite_la_fwd_save_state(None, None, None, 0, 4, 1, 32, 1e-15, 0, None) == 0
    assert lib.lite_la_bwd_from_state(a, g, st, o, 1, 4, 1, 64, 1e-15, 0, None) == 2


def test_elu1_entry_points_validate_on_the_host(lib):
    """The ELU+1 variant shares the forward's checks: clamp_min takes eps's place (finite, >= 0);
    tokens_per_block <= 0 selects the non-causal form rather than being an error."""
    a, o = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 30)
    for B, N, H, d, clamp, want in BAD_ARGS:
        assert lib.lite_la_elu1_fwd(a, o, B, N, H, d, clamp, 0, None) == want
        assert lib.lite_la_elu1_fwd_f32out(a, o, B, N, H, d, clamp, 16, None) == want
    assert lib.lite_la_elu1_fwd(None, o, 1, 4, 1, 32, 1e-6, 0, None) == 1
    assert lib.lite_la_elu1_fwd(a, ctypes.c_void_p((1 << 30) + 8), 1, 4, 1, 32, 1e-6, 0, None) == 1
    assert lib.lite_la_elu1_fwd(a, ctypes.c_void_p((1 << 20) + 256), 1, 4, 1, 32, 1e-6, 0, None) == 1
    assert "overlap" in lib.lite_la_last_error().decode()
    assert lib.lite_la_elu1_fwd(None, None, 0, 4, 1, 32, 1e-6, 0, None) == 0
    null = (ctypes.c_void_p * 3)(None, None, None)
    assert lib.lite_la_elu1_fwd_events(a, o, 1, 4, 1, 32, 1e-6, 0, None, null) == 1


def test_autograd_entry_point_rejects_host_tensors():
    import torch
    qkv = torch.zeros((1, 4, 96), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        ll.lite_la(qkv, 1)


def test_output_projection_entry_points_validate_on_the_host(lib):
    """lite_la_fwd_oproj and lite_la_out_proj check every buffer and size before any CUDA call:
    C_in and C_out multiples of 8 (16-byte rows), 16-byte aligned weight and output, a 4-byte
    aligned bias (or none), no output overlapping an input, a block size that is a multiple of
    128 tokens for the block-causal form; empty problems are no-ops."""
    a, w, y, b = (ctypes.c_void_p(1 << k) for k in (20, 24, 30, 34))
    f, lin = lib.lite_la_fwd_oproj, lib.lite_la_out_proj
    for B, N, H, d, eps, want in BAD_ARGS:
        assert f(a, w, None, y, B, N, H, d, 64, eps, 0, None) == want
    assert f(a, w, None, y, 1, 4, 1, 32, 36, 1e-15, 0, None) == 1                    # C_out % 8
    assert f(a, w, None, y, 1, 4, 1, 32, -8, 1e-15, 0, None) == 1
    assert f(a, ctypes.c_void_p((1 << 24) + 8), None, y, 1, 4, 1, 32, 64, 1e-15, 0, None) == 1
    assert f(a, w, ctypes.c_void_p((1 << 34) + 2), y, 1, 4, 1, 32, 64, 1e-15, 0, None) == 1
    assert f(a, None, None, y, 1, 4, 1, 32, 64, 1e-15, 0, None) == 1
    assert f(a, w, None, ctypes.c_void_p((1 << 20) + 256), 1, 4, 1, 32, 64, 1e-15, 0, None) == 1
    assert "overlap" in lib.lite_la_last_error().decode()
    assert f(a, w, None, y, 1, 300, 1, 32, 64, 1e-15, 100, None) == 2              # block of 100 tokens
    assert f(a, w, None, y, 1, 4, 1, 64, 64, 1e-15, 0, None) == 2                   # d != 32
    assert f(None, None, None, None, 0, 4, 1, 32, 64, 1e-15, 0, None) == 0          # empty
    assert f(a, None, None, y, 1, 4, 1, 32, 0, 1e-15, 0, None) == 0                 # C_out = 0
    null = (ctypes.c_void_p * 3)(None, None, None)
    assert lib.lite_la_fwd_oproj_events(a, w, None, y, 1, 4, 1, 32, 64, 1e-15, 0, None, null) == 1
    assert lin(a, w, None, y, 1, 4, 60, 64, None) == 1                              # C_in % 8
    assert lin(ctypes.c_void_p((1 << 20) + 8), w, None, y, 1, 4, 64, 64, None) == 1
    assert lin(None, w, None, y, 1, 4, 64, 64, None) == 1
    assert lin(a, w, None, ctypes.c_void_p((1 << 20) + 64), 1, 4, 64, 64, None) == 1
    assert lin(a, w, None, y, -1, 4, 64, 64, None) == 1
    assert lin(None, None, None, None, 0, 4, 64, 64, None) == 0


def test_forward_form_and_the_paired_minimum(lib):
    """The form query needs no GPU; the paired minimum is process-wide, returns the previous
    value and falls back to its default (1024 tokens) for values <= 0."""
    assert lib.lite_la_forward_form(0, 16, 1, 32, 0) == -1
    assert lib.lite_la_forward_form(1, 16, 1, 64, 0) == -1
    assert ll.lite_la_forward_form(2, 16384, 70) == "fused_paired"       # chunks of 2048 tokens
    assert ll.lite_la_forward_form(2, 4096, 70) == "fused"               # chunks of 512
    assert ll.lite_la_forward_form(1, 16384, 70, 32, 1024) == "fused_paired_causal"   # 18 quads x 8 block pairs
    assert ll.lite_la_forward_form(2, 16384, 70, 32, 1024) == "three_kernel"          # 36 x 8 > 148, 4 blocks a CTA
    assert ll.lite_la_forward_form(1, 4096, 70, 32, 512) == "fused_causal"            # blocks < 1024 tokens
    assert ll.lite_la_forward_form(8, 512, 80) == "three_kernel"         # 160 head quads
    prev = ll.lite_la_set_paired_min_chunk(512)
    try:
        assert prev == 1024
        assert ll.lite_la_forward_form(2, 4096, 70) == "fused_paired"
        assert ll.lite_la_forward_form(1, 4096, 4) == "fused"            # one quad: nothing to pair
        assert ll.lite_la_set_paired_min_chunk(-5) == 512
        assert ll.lite_la_set_paired_min_chunk(0) == 1024
    finally:
        ll.lite_la_set_paired_min_chunk(prev)
    # the workspace query follows the form: 8 siblings' partial states per quad when paired
    assert ll.lite_la_workspace_bytes(2, 16384, 70) >= 36 * 8 * 4 * 33 * 32 * 4


def test_backward_kernel_count(lib):
    """With one block per sequence the backward is three kernels (the dq and dk/dv kernels sum
    the partial states into their images themselves); with more blocks it keeps the two scans
    (one of them from saved states).  The query needs no GPU."""
    f = lib.lite_la_bwd_kernels_per_call
    assert f(2, 16384, 70, 32, 0, 0) == 3 and f(2, 16384, 70, 32, 0, 1) == 3
    assert f(1, 3000, 9, 32, 3000, 0) == 3 and f(1, 3000, 9, 32, 5000, 1) == 3   # T >= N: one block
    assert f(1, 16384, 70, 32, 1024, 0) == 5 and f(1, 16384, 70, 32, 1024, 1) == 4
    assert f(0, 16, 1, 32, 0, 0) == 0 and f(1, 16, 1, 64, 0, 0) == 0
