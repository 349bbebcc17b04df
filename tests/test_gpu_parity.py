"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances (per element, o = oracle value):
  bf16 output: |gpu - o| <= 1e-3 + 8e-3 * |o|
  fp32 output: |gpu - o| <= 1e-5 + 1e-4 * |o|
Small and medium shapes are compared on every output; the full-size workloads are compared
on sampled query rows (first, last, block edges and a seeded random set), which the oracle
evaluates one by one.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_diffusion_litela_b200 as ll
from linear_attention_diffusion_litela_b200.inputs import WORKLOADS, make_qkv, pack_qkv, to_bits
import oracle

pytestmark = pytest.mark.gpu

EPS = 1e-15
TOL = {"bf16": (1e-3, 8e-3), "f32": (1e-5, 1e-4)}


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_diffusion_litela_b200.build import build
    build()
    ll.lib()


def gpu_run(qkv, H, T=None, mode="bf16"):
    dt = torch.bfloat16 if mode == "bf16" else torch.float32
    if T is None:
        out = ll.lite_la_fwd(qkv, H, eps=EPS, out_dtype=dt)
    else:
        out = ll.lite_la_block_causal_fwd(qkv, H, T, eps=EPS, out_dtype=dt)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    B, N = qkv.shape[:2]
    return out.view(B, N, H, 32).to(torch.float64).cpu().numpy()


def oracle_run(qkv, H, T=None, rows=None):
    B, N = qkv.shape[:2]
    bits = to_bits(qkv)
    if T is None:
        return oracle.lite_la_fwd(bits, B, N, H, 32, EPS, rows=rows)
    return oracle.lite_la_block_causal_fwd(bits, B, N, H, 32, EPS, T, rows=rows)


def assert_close(got, want, mode):
    atol, rtol = TOL[mode]
    err = np.abs(got - want)
    bound = atol + rtol * np.abs(want)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError("%d of %d elements out of tolerance; worst at %s: gpu=%r oracle=%r"
                             % (bad.sum(), bad.size, i, got[i], want[i]))


SMALL = [  # (B, N, H): several tiles, ragged tails, tiny cases
    (1, 1, 1), (1, 2, 1), (1, 7, 3), (2, 31, 2), (1, 33, 5), (2, 300, 5), (1, 1000, 7),
    (3, 257, 4), (1, 2049, 2),
]


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H", SMALL)
def test_small_shapes_every_element(B, N, H, mode):
    qkv = make_qkv(B, N, H, 32, seed=B * 100003 + N * 31 + H, device="cuda")
    assert_close(gpu_run(qkv, H, mode=mode), oracle_run(qkv, H), mode)


PAIRED = [  # the paired fused form (N >= 2048, two or more head quads; each CTA of a sibling
            # group works on two quads): an odd quad count (a group with one quad), quads of 1 to
            # 3 heads, a ragged last chunk, quads whose head pair count changes between a CTA's
            # two quads, many siblings of one 64-token tile each
    (1, 2048, 8), (1, 2100, 5), (2, 2048, 7), (1, 4097, 12), (2, 3000, 9), (4, 2500, 36), (3, 2048, 10),
]


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H", PAIRED)
def test_paired_fused_shapes_every_element(B, N, H, mode, paired_min_chunk):
    paired_min_chunk(64)   # chunks of 64 tokens and more take the paired form
    assert ll.lite_la_forward_form(B, N, H) == "fused_paired"
    qkv = make_qkv(B, N, H, 32, seed=B * 7919 + N * 13 + H, device="cuda")
    assert_close(gpu_run(qkv, H, mode=mode), oracle_run(qkv, H), mode)


PAIRED_CAUSAL = [  # the paired block-causal form (sibling r owns blocks r and r + ceil(nblk/2) of a
                   # quad; taken where the plain form gives a CTA two blocks): an odd block count
                   # (the last sibling has one block), a ragged last block, quads of 2 heads
    (1, 2048, 40, 128), (1, 2100, 40, 128), (3, 1024, 30, 128), (2, 700, 70, 128), (2, 640, 66, 128),
]


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H,T", PAIRED_CAUSAL)
def test_paired_block_causal_shapes_every_element(B, N, H, T, mode, paired_min_chunk):
    paired_min_chunk(128)
    assert ll.lite_la_forward_form(B, N, H, 32, T) == "fused_paired_causal"
    qkv = make_qkv(B, N, H, 32, seed=B * 31337 + N + H * 7 + T, device="cuda")
    assert_close(gpu_run(qkv, H, T=T, mode=mode), oracle_run(qkv, H, T=T), mode)


def test_paired_and_plain_fused_forms_agree_and_are_deterministic(paired_min_chunk):
    """Both fused forms of the 2048px call: each bitwise repeatable, the two within the bf16
    rounding of each other (their fp32 partial states are summed over different chunks)."""
    w = WORKLOADS["sana1600m_2048px"]
    qkv = make_qkv(w["B"], w["N"], w["H"], 32, seed=2222, device="cuda")
    assert ll.lite_la_forward_form(w["B"], w["N"], w["H"]) == "fused"
    plain = [gpu_run(qkv, w["H"]) for _ in range(2)]
    paired_min_chunk(64)
    assert ll.lite_la_forward_form(w["B"], w["N"], w["H"]) == "fused_paired"
    paired = [gpu_run(qkv, w["H"]) for _ in range(2)]
    assert np.array_equal(plain[0], plain[1]) and np.array_equal(paired[0], paired[1])
    assert np.all(np.abs(paired[0] - plain[0]) <= 2.0 ** -7 * np.abs(plain[0]) + 1e-6)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H,T", [(1, 7, 2, 1), (2, 40, 3, 1), (1, 100, 2, 7), (2, 300, 3, 128),
                                     (1, 1000, 4, 256), (1, 1000, 2, 300), (1, 513, 3, 512),
                                     (2, 64, 2, 64), (1, 50, 2, 1000), (1, 2500, 2, 1024)])
def test_block_causal_small_shapes_every_element(B, N, H, T, mode):
    qkv = make_qkv(B, N, H, 32, seed=7 * N + T + H, device="cuda")
    assert_close(gpu_run(qkv, H, T=T, mode=mode), oracle_run(qkv, H, T=T), mode)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("name", ["sana600m_512px", "sana1600m_1024px"])
def test_small_workloads_every_element(name, mode):
    w = WORKLOADS[name]
    qkv = make_qkv(w["B"], w["N"], w["H"], 32, seed=1000 + list(WORKLOADS).index(name), device="cuda")
    assert_close(gpu_run(qkv, w["H"], mode=mode), oracle_run(qkv, w["H"]), mode)


def sample_rows(N, T=None, k=192, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, 1, N - 2, N - 1}
    if T is not None:
        for b0 in range(0, N, T):
            rows.update({b0, max(b0 - 1, 0), min(b0 + T - 1, N - 1)})
    rows.update(rng.choice(N, size=min(k, N), replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("shift", [0.0, -1.5])
def test_2048px_sampled(shift, mode):
    w = WORKLOADS["sana1600m_2048px"]
    seed = 1002 if shift == 0.0 else 3001
    qkv = make_qkv(w["B"], w["N"], w["H"], 32, seed=seed, device="cuda", qk_shift=shift)
    rows = sample_rows(w["N"], seed=seed)
    got = gpu_run(qkv, w["H"], mode=mode)[:, rows]
    assert_close(got, oracle_run(qkv, w["H"], rows=rows), mode)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_4096px_sampled(mode):
    w = WORKLOADS["sana4800m_4096px"]
    assert ll.lite_la_forward_form(w["B"], w["N"], w["H"]) == "fused_paired"
    qkv = make_qkv(w["B"], w["N"], w["H"], 32, seed=4000, device="cuda")
    rows = sample_rows(w["N"], k=96, seed=4)
    got = gpu_run(qkv, w["H"], mode=mode)[:, rows]
    assert_close(got, oracle_run(qkv, w["H"], rows=rows), mode)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_block_causal_workload_sampled(mode):
    w = WORKLOADS["block_causal_16x1024"]
    T = w["tokens_per_block"]
    assert ll.lite_la_forward_form(w["B"], w["N"], w["H"], 32, T) == "fused_paired_causal"
    qkv = make_qkv(w["B"], w["N"], w["H"], 32, seed=1004, device="cuda")
    rows = sample_rows(w["N"], T=T, k=64, seed=5)
    got = gpu_run(qkv, w["H"], T=T, mode=mode)[:, rows]
    assert_close(got, oracle_run(qkv, w["H"], T=T, rows=rows), mode)


@pytest.mark.parametrize("T", [512, 256])
@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_block_causal_short_blocks_sampled(T, mode):
    """Short blocks at the 4096px token count (N = 16384, H = 70): more blocks than the
    reduction has CTAs, so each reduction CTA walks several consecutive blocks (three-kernel
    path); sampled rows, block edges among them, against the oracle."""
    B, N, H = 1, 16384, 70
    assert ll.lite_la_forward_form(B, N, H, 32, T) == "three_kernel"
    qkv = make_qkv(B, N, H, 32, seed=1005 + T, device="cuda")
    rows = sample_rows(N, T=T, k=48, seed=7)
    got = gpu_run(qkv, H, T=T, mode=mode)[:, rows]
    assert_close(got, oracle_run(qkv, H, T=T, rows=rows), mode)


def test_hand_worked_example_padded_to_d32():
    """The golden d=2 example embedded in channels 0..1 of a d=32 head (other channels 0)."""
    from tests.test_golden import as_float, load_golden
    g = load_golden()
    q, k, v = (np.zeros((1, 3, 1, 32)) for _ in range(3))
    q[0, :, 0, :2], k[0, :, 0, :2], v[0, :, 0, :2] = as_float(g["q"]), as_float(g["k"]), as_float(g["v"])
    qkv = pack_qkv(q, k, v).cuda()
    for key, T in (("out_noncausal", None), ("out_block_T1", 1), ("out_block_T2", 2)):
        got = gpu_run(qkv, 1, T=T, mode="f32")[0, :, 0]
        np.testing.assert_allclose(got[:, :2], as_float(g[key]), rtol=1e-6, atol=1e-7)
        assert np.all(got[:, 2:] == 0)


def test_bitwise_deterministic():
    qkv = make_qkv(2, 3000, 7, 32, seed=77, device="cuda")
    a = gpu_run(qkv, 7, mode="f32")
    b = gpu_run(qkv, 7, mode="f32")
    assert np.array_equal(a, b)
    c = gpu_run(qkv, 7, T=500, mode="f32")
    d = gpu_run(qkv, 7, T=500, mode="f32")
    assert np.array_equal(c, d)


def test_all_negative_query_row_is_exactly_zero_and_q_scaling_is_bitwise_invariant():
    B, N, H = 1, 700, 3
    qkv = make_qkv(B, N, H, 32, seed=91, device="cuda")
    x = qkv.view(B, N, 3, H, 32)
    x[0, 10, 0, 1] = -x[0, 10, 0, 1].abs() - 0.5
    out = gpu_run(qkv, H, mode="f32")
    assert np.all(out[0, 10, 1] == 0.0)
    y = qkv.clone().view(B, N, 3, H, 32)
    y[:, :, 0] *= 4.0
    out2 = gpu_run(y.view(B, N, -1), H, mode="f32")
    assert np.array_equal(out, out2)


def test_non_default_stream_and_empty_problem():
    qkv = make_qkv(1, 129, 2, 32, seed=5, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = ll.lite_la_fwd(qkv, 2, eps=EPS, out_dtype=torch.float32, stream=s)
    s.synchronize()
    got = out.view(1, 129, 2, 32).double().cpu().numpy()
    assert_close(got, oracle_run(qkv, 2), "f32")
    empty = torch.empty((1, 0, 3 * 2 * 32), dtype=torch.bfloat16, device="cuda")
    assert ll.lite_la_fwd(empty, 2).shape == (1, 0, 64)


def test_rejects_bad_arguments_without_launching():
    qkv = make_qkv(1, 16, 1, 32, seed=1, device="cuda")
    out = torch.empty((1, 16, 32), dtype=torch.bfloat16, device="cuda")
    lib = ll.lib()
    assert lib.lite_la_fwd(qkv.data_ptr() + 2, out.data_ptr(), 1, 15, 1, 32, EPS, None) == 1
    assert lib.lite_la_fwd(qkv.data_ptr(), qkv.data_ptr(), 1, 16, 1, 32, EPS, None) == 1
    assert lib.lite_la_fwd(qkv.data_ptr(), out.data_ptr(), 1, 16, 1, 16, EPS, None) == 2


def test_workspace_allocation_failure_is_reported(monkeypatch):
    qkv = make_qkv(1, 64, 1, 32, seed=2, device="cuda")
    s = torch.cuda.Stream()                      # fresh stream: forces a new workspace
    monkeypatch.setenv("LITELA_FAIL_ALLOC", "1")
    with pytest.raises(ll.LiteLAError) as ei:
        ll.lite_la_fwd(qkv, 1, stream=s)
    assert ei.value.status == 3
    monkeypatch.delenv("LITELA_FAIL_ALLOC")
    out = ll.lite_la_fwd(qkv, 1, stream=s, out_dtype=torch.float32)
    s.synchronize()
    assert_close(out.view(1, 64, 1, 32).double().cpu().numpy(), oracle_run(qkv, 1), "f32")


def state_reference(bits, B, N, H, T):
    """[V;1]^T . relu(K) per (batch, head), summed over blocks 0..k (fp64, from the decoded
    bf16 inputs): the state the pages define, used to check lite_la_state_fwd."""
    x = oracle.decode_bf16(bits).reshape(B, N, 3 * H * 32)
    _, k, v = oracle.unpack_qkv(x, H, 32)
    T = T if 0 < T < N else N
    nblk = -(-N // T)
    out = np.zeros((B, H, nblk, 33, 32))
    for b in range(B):
        for h in range(H):
            run = np.zeros((33, 32))
            for blk in range(nblk):
                kk = np.maximum(k[b, blk * T:(blk + 1) * T, h], 0.0)
                vv = np.concatenate([v[b, blk * T:(blk + 1) * T, h], np.ones((kk.shape[0], 1))], axis=1)
                run = run + vv.T @ kk
                out[b, h, blk] = run
    return out


@pytest.mark.parametrize("B,N,H,T", [(1, 1, 1, 0), (1, 65, 3, 0), (2, 1000, 5, 0), (1, 300, 4, 128),
                                     (2, 100, 2, 7), (1, 4096, 70, 1024)])
def test_state_fwd_matches_padded_state_definition(B, N, H, T):
    qkv = make_qkv(B, N, H, 32, seed=3 * N + H + T, device="cuda")
    st = ll.lite_la_state_fwd(qkv, H, T)
    ll.lite_la_device_status()
    ref = state_reference(to_bits(qkv), B, N, H, T)
    got = st.double().cpu().numpy()
    # fp32 sums of exact bf16 products: relative error ~ sqrt(N) * 2^-24 of the magnitudes
    scale = np.abs(ref).max(axis=(-1, -2), keepdims=True) + 1e-30
    assert np.all(np.abs(got - ref) <= 1e-5 * scale + 1e-6)


def test_bounded_wait_timeout_is_reported_and_the_context_stays_usable():
    """A kernel whose barrier never completes gives up after its wait limit, records an error
    code that lite_la_device_status turns into LITELA_ERR_DEVICE_TIMEOUT, and the stream keeps
    working (nothing faults, nothing hangs)."""
    s = torch.cuda.Stream()
    lib = ll.lib()
    assert lib.lite_la_selftest_timeout(ctypes.c_void_p(s.cuda_stream)) == 0
    with pytest.raises(ll.LiteLAError) as ei:
        ll.lite_la_device_status(s)
    assert ei.value.status == 5 and "0x3f0" in str(ei.value)
    ll.lite_la_device_status(s)                       # the error word was cleared
    qkv = make_qkv(1, 300, 3, 32, seed=9, device="cuda")
    out = ll.lite_la_fwd(qkv, 3, eps=EPS, out_dtype=torch.float32, stream=s)
    s.synchronize()
    ll.lite_la_device_status(s)
    assert_close(out.view(1, 300, 3, 32).double().cpu().numpy(), oracle_run(qkv, 3), "f32")


@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_more_head_quads_than_sms(mode):
    """H = 600 gives 150 head quads (more than the 148 SMs): the apply takes the general,
    non quad-major work order."""
    B, N, H = 1, 96, 600
    qkv = make_qkv(B, N, H, 32, seed=600, device="cuda")
    assert_close(gpu_run(qkv, H, mode=mode), oracle_run(qkv, H), mode)


def test_interleaved_shapes_reuse_and_grow_the_workspace():
    """Calls of different sizes back to back on one stream (the workspace grows while earlier
    kernels may still be queued), without synchronising in between."""
    shapes = [(1, 200, 3), (2, 3000, 9), (1, 50, 2), (2, 4100, 17), (1, 700, 5)]
    qkvs = [make_qkv(B, N, H, 32, seed=B + N + H, device="cuda") for B, N, H in shapes]
    outs = [ll.lite_la_fwd(q, H, eps=EPS, out_dtype=torch.float32) for q, (B, N, H) in zip(qkvs, shapes)]
    outs += [ll.lite_la_block_causal_fwd(q, H, 128, eps=EPS, out_dtype=torch.float32)
             for q, (B, N, H) in zip(qkvs, shapes)]
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    for i, (q, (B, N, H)) in enumerate(zip(qkvs, shapes)):
        rows = sample_rows(N, T=128, k=64, seed=i)
        got = outs[i].view(B, N, H, 32).double().cpu().numpy()[:, rows]
        assert_close(got, oracle_run(q, H, rows=rows), "f32")
        got_c = outs[len(shapes) + i].view(B, N, H, 32).double().cpu().numpy()[:, rows]
        assert_close(got_c, oracle_run(q, H, T=128, rows=rows), "f32")


def test_eps_zero_and_a_head_with_only_negative_keys():
    B, N, H = 2, 500, 6
    qkv = make_qkv(B, N, H, 32, seed=31, device="cuda")
    x = qkv.view(B, N, 3, H, 32)
    x[1, :, 1, 4] = -x[1, :, 1, 4].abs() - 0.125          # batch 1, head 4: every key < 0
    out = ll.lite_la_fwd(qkv, H, eps=0.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    got = out.view(B, N, H, 32).double().cpu().numpy()
    bits = to_bits(qkv)
    want = oracle.lite_la_fwd(bits, B, N, H, 32, 0.0)
    dead = np.zeros(want.shape, dtype=bool)
    dead[1, :, 4] = True                                   # 0 / 0 there: undefined, checked below
    assert_close(got[~dead].reshape(-1), want[~dead].reshape(-1), "f32")
    with_eps = gpu_run(qkv, H, mode="f32")                 # with eps the dead head is exactly 0
    assert np.all(with_eps[1, :, 4] == 0.0)


@pytest.mark.parametrize("mode", ["bf16", "f32"])
@pytest.mark.parametrize("B,H,T,chunks", [(1, 3, 128, [256, 384, 100]), (2, 5, 64, [64, 64, 128, 7]),
                                          (1, 70, 1024, [4096, 4096])])
def test_state_carry_over_chunks_equals_the_whole_sequence(B, H, T, chunks, mode):
    """Chunked block-causal calls that carry the state (chunk lengths multiples of T) give the
    block-causal result of the whole sequence, and the final carried state is the state of all
    tokens."""
    N = sum(chunks)
    dt = torch.bfloat16 if mode == "bf16" else torch.float32
    qkv = make_qkv(B, N, H, 32, seed=17 * N + H + T, device="cuda")
    state, outs, n0 = None, [], 0
    for i, c in enumerate(chunks):
        part = qkv[:, n0:n0 + c].contiguous()
        # alternate between a fresh output state and updating the carried state in place
        out, state = ll.lite_la_block_causal_fwd_carry(part, H, T, state_in=state,
                                                       state_out=state if (i % 2 and state is not None) else None,
                                                       eps=EPS, out_dtype=dt)
        outs.append(out)
        n0 += c
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    got = torch.cat(outs, dim=1).view(B, N, H, 32).double().cpu().numpy()
    rows = np.arange(N) if N <= 2048 else sample_rows(N, T=T, k=96, seed=3)
    assert_close(got[:, rows], oracle_run(qkv, H, T=T, rows=rows), mode)
    full = state_reference(to_bits(qkv), B, N, H, 0)[:, :, 0]
    scale = np.abs(full).max(axis=(-1, -2), keepdims=True) + 1e-30
    assert np.all(np.abs(state.double().cpu().numpy() - full) <= 1e-5 * scale + 1e-6)


def test_state_carry_without_state_in_is_the_plain_block_causal_call():
    B, N, H, T = 1, 700, 4, 128
    qkv = make_qkv(B, N, H, 32, seed=77, device="cuda")
    out, st = ll.lite_la_block_causal_fwd_carry(qkv, H, T, eps=EPS, out_dtype=torch.float32)
    ref = ll.lite_la_block_causal_fwd(qkv, H, T, eps=EPS, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # the plain call may take the fused block-causal kernel, which sums the block states in
    # another (fixed) order than the carry path's scan: equal to fp32 rounding, not bitwise
    assert torch.allclose(out, ref, rtol=1e-5, atol=1e-6)
    full = ll.lite_la_state_fwd(qkv, H, 0)
    torch.cuda.synchronize()
    assert torch.allclose(st, full[:, :, 0], rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("B,N,H,T", [(2, 3000, 9, 0), (2, 1000, 600, 0), (1, 4000, 7, 512), (2, 700, 5, 700)])
def test_phase_timed_calls_give_the_plain_calls_result(B, N, H, T):
    """lite_la_fwd_events / lite_la_block_causal_fwd_events run the same kernels with events
    between the phases: bitwise the plain call's output, events complete and in order."""
    lib = ll.lib()
    qkv = make_qkv(B, N, H, 32, seed=9000 + N + H, device="cuda")
    want = ll.lite_la_fwd(qkv, H, eps=EPS) if T == 0 else ll.lite_la_block_causal_fwd(qkv, H, T, eps=EPS)
    out = torch.empty_like(want)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    stream = torch.cuda.current_stream()
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    handles = (ctypes.c_void_p * 3)(*[ctypes.c_void_p(e.cuda_event) for e in evs])
    sh = ctypes.c_void_p(stream.cuda_stream)
    if T == 0:
        s = lib.lite_la_fwd_events(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, sh, handles)
    else:
        s = lib.lite_la_block_causal_fwd_events(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, T, sh, handles)
    assert s == 0, lib.lite_la_last_error().decode()
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    assert torch.equal(out, want)
    assert evs[0].elapsed_time(evs[1]) >= 0.0 and evs[1].elapsed_time(evs[2]) >= 0.0
    assert evs[0].elapsed_time(evs[2]) > 0.0
    null = (ctypes.c_void_p * 3)(None, None, None)
    assert lib.lite_la_fwd_events(qkv.data_ptr(), out.data_ptr(), B, N, H, 32, EPS, sh, null) == 1


# one shape per fused form: paired, plain, paired block-causal, plain block-causal
FUSED_FORMS = [((2, 8192, 70, 0), "fused_paired"), ((2, 4096, 70, 0), "fused"),
               ((1, 16384, 70, 1024), "fused_paired_causal"), ((1, 8192, 70, 1024), "fused_causal")]


@pytest.mark.parametrize("shape,form", FUSED_FORMS)
def test_concurrent_fused_calls_on_two_streams(shape, form):
    """Two fused calls at once on two streams: each grid alone fills the SMs, so only part of
    each can be resident; CTAs take their roles by ticket in arrival order, so both complete.
    The results equal the single-stream ones bitwise and no wait times out."""
    B, N, H, T = shape
    assert ll.lite_la_forward_form(B, N, H, 32, T) == form
    xa = make_qkv(B, N, H, 32, seed=6100 + T, device="cuda")
    xb = make_qkv(B, N, H, 32, seed=6200 + T, device="cuda")
    run = (lambda x, **kw: ll.lite_la_fwd(x, H, eps=EPS, **kw)) if T == 0 else \
        (lambda x, **kw: ll.lite_la_block_causal_fwd(x, H, T, eps=EPS, **kw))
    assert ll.lib().lite_la_kernels_per_call(B, N, H, 32, T) == 1
    ra, rb = run(xa), run(xb)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(5):
        with torch.cuda.stream(sa):
            oa = run(xa, stream=sa)
        with torch.cuda.stream(sb):
            ob = run(xb, stream=sb)
        torch.cuda.synchronize()
        ll.lite_la_device_status(sa)
        ll.lite_la_device_status(sb)
        assert torch.equal(oa, ra) and torch.equal(ob, rb)


@pytest.mark.parametrize("shape,form", FUSED_FORMS)
def test_fused_call_replayed_from_a_captured_graph(shape, form):
    """One fused call captured into a CUDA graph and replayed several times, interleaved with
    eager calls on the same stream: the kernel's control words are left clean by the last CTA
    of every call, so each replay and each eager call gives the eager result bitwise."""
    B, N, H, T = shape
    assert ll.lite_la_forward_form(B, N, H, 32, T) == form
    x = make_qkv(B, N, H, 32, seed=6300 + T, device="cuda")
    run = (lambda **kw: ll.lite_la_fwd(x, H, eps=EPS, **kw)) if T == 0 else \
        (lambda **kw: ll.lite_la_block_causal_fwd(x, H, T, eps=EPS, **kw))
    assert ll.lib().lite_la_kernels_per_call(B, N, H, 32, T) == 1
    ref = run()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    og = torch.empty_like(ref)
    oe = torch.empty_like(ref)
    with torch.cuda.stream(s):
        run(out=og, stream=s)          # the stream's workspace exists before the capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(out=og, stream=s)
    for _ in range(4):
        og.zero_()
        oe.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            g.replay()
            run(out=oe, stream=s)
            g.replay()
        s.synchronize()
        ll.lite_la_device_status(s)
        assert torch.equal(og, ref) and torch.equal(oe, ref)
    del g


def test_head_shards_of_one_problem_match_the_full_call():
    """Tensor-parallel use: each of 3 ranks gets its heads' packed qkv (pack_head_shard) and calls
    lite_la_fwd with its own head count; the shards' outputs are the full call's heads, to the
    oracle's bf16 tolerance (heads are independent; the shards group heads into other quads)."""
    from linear_attention_diffusion_litela_b200.dist import pack_head_shard, shard_heads
    B, N, H = 2, 700, 70
    qkv = make_qkv(B, N, H, 32, seed=7070, device="cuda")
    want = oracle_run(qkv, H)
    full = gpu_run(qkv, H)
    assert_close(full, want, "bf16")
    for rank in range(3):
        h0, h1 = shard_heads(H, 3, rank)
        sub = pack_head_shard(qkv, H, h0, h1)
        got = gpu_run(sub, h1 - h0)
        assert_close(got, want[:, :, h0:h1], "bf16")


@pytest.mark.parametrize("shape,form", FUSED_FORMS + [((2, 300, 600, 0), "three_kernel")])
def test_input_rewritten_by_the_previous_kernel_is_the_one_read(shape, form):
    """Every fused form prefetches its CTA's first input tiles into L2 before it waits for the
    previous kernel in the stream (programmatic dependent launch).  Here that previous kernel
    rewrites the very qkv buffer in place; the call must see the new values, bitwise as a call
    on a fresh buffer, in both directions of the rewrite and back to back."""
    B, N, H, T = shape
    assert ll.lite_la_forward_form(B, N, H, 32, T) == form
    xa = make_qkv(B, N, H, 32, seed=7100 + N, device="cuda")
    xb = make_qkv(B, N, H, 32, seed=7200 + N, device="cuda")
    run = (lambda x: ll.lite_la_fwd(x, H, eps=EPS)) if T == 0 else \
        (lambda x: ll.lite_la_block_causal_fwd(x, H, T, eps=EPS))
    ra, rb = run(xa), run(xb)
    torch.cuda.synchronize()
    buf = xa.clone()
    outs = []
    for i in range(6):
        outs.append(run(buf))
        src = xb if i % 2 == 0 else xa
        torch.mul(src, 1.0, out=buf)   # an elementwise kernel rewrites the input in place
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    for i, o in enumerate(outs):
        assert torch.equal(o, ra if i % 2 == 0 else rb), i


def test_backward_input_rewritten_by_the_previous_kernel_is_the_one_read():
    """The backward's state reduction prefetches k and v before its dependency wait: a qkv
    rewritten in place by the kernel just before must be the one the backward reads."""
    B, N, H = 2, 2048, 70
    xa = make_qkv(B, N, H, 32, seed=7300, device="cuda")
    xb = make_qkv(B, N, H, 32, seed=7301, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7302)
    dout = torch.randn((B, N, H * 32), generator=g, device="cuda").to(torch.bfloat16)
    ra, rb = ll.lite_la_bwd(xa, dout, H, eps=EPS), ll.lite_la_bwd(xb, dout, H, eps=EPS)
    torch.cuda.synchronize()
    buf = xa.clone()
    outs = []
    for i in range(4):
        outs.append(ll.lite_la_bwd(buf, dout, H, eps=EPS))
        torch.mul(xb if i % 2 == 0 else xa, 1.0, out=buf)
    torch.cuda.synchronize()
    ll.lite_la_device_status()
    for i, o in enumerate(outs):
        assert torch.equal(o, ra if i % 2 == 0 else rb), i
