#!/usr/bin/env python
"""LiteLA forward benchmark on B200 (one JSON line on stdout, rank 0).

Workload (default): Sana 4096px LiteLA forward, B=2, N=128*128=16384 tokens, H=70 heads of
d=32, packed bf16 qkv drawn i.i.d. N(0,1) from seeds 4000..4059, eps=1e-15.  One step is 60
back-to-back calls on 60 distinct input buffers (the 60 self-attention layers of the 4.8B
model per sampling step).  Every call's input (440 MB) is larger than the 126 MB L2, so no
flush is needed between calls.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 it runs under torch.distributed.run, one rank per GPU, each rank doing the same
per-GPU workload (weak scaling; the calls are independent, there is no data-path
collective).  Timing: CUDA events on the launching stream, barrier + synchronize on both
sides, max over ranks.  `--impl reference` times the fp64 CPU oracle (the only reference
this method has) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS_BENCH = {
    # name: (B, N, H, calls per step, seed base, tokens per causal block or 0)
    "sana4800m_4096px_x60": (2, 128 * 128, 70, 60, 4000, 0),
    # one 4096px call per step on one buffer: the small case for detailed ncu captures
    "sana4800m_4096px_x1": (2, 128 * 128, 70, 1, 4000, 0),
    # 512px: far below a launch's latency; 64 buffers so that the rotation exceeds L2 (151 MB)
    "sana600m_512px": (1, 16 * 16, 36, 64, 1000, 0),
    "sana1600m_1024px": (2, 32 * 32, 70, 20, 1001, 0),
    "sana1600m_2048px": (2, 64 * 64, 70, 20, 1002, 0),
    # the 2048px shape with q and k shifted by -1.5 before the bf16 cast (mostly negative:
    # sparse ReLU, tiny denominators)
    "sana1600m_2048px_mostly_negative": (2, 64 * 64, 70, 20, 3001, 0),
    # video-style block-causal call: 16 blocks of 1024 tokens, 20 distinct buffers per step
    "block_causal_16x1024": (1, 16 * 1024, 70, 20, 1004, 1024),
    "block_causal_16x1024_x1": (1, 16 * 1024, 70, 1, 1004, 1024),
}
QK_SHIFT = {"sana1600m_2048px_mostly_negative": -1.5}
# the configs timed beside the headline in the default run (the `workloads` record)
RECORD_WORKLOADS = ("sana600m_512px", "sana1600m_1024px", "sana1600m_2048px", "sana1600m_2048px_mostly_negative",
                    "block_causal_16x1024")
D = 32
EPS = 1e-15
METRIC = "LiteLA fwd tokens·heads/s and µs/call at 4096px; % of HBM/FMA roofline"
METRIC_BWD = "LiteLA bwd tokens·heads/s and µs/call at 4096px; % of HBM roofline"
UNIT = "tokens·heads/s"
FP32_LANES_PER_SM = 128          # B200: 4 SM sub-partitions x 32 fp32 lanes
NUM_SMS = 148
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}
FORMS_PAIRED = (2, 4)            # lite_la_forward_form: the paired fused forms (non-causal, block-causal)
# The library runs a non-causal call as one fused kernel when B * ceil(H/4) fits the SMs
# (lite_la_kernels_per_call == 1), else as three (reduction, scan, apply); lite_la_fwd_events
# brackets the phases.  Per path: the timed phases and their algorithmic bytes (in units of
# E = B*N*H*d elements).
PATHS = {
    # backward (--direction bwd) with more than one block per sequence: five kernels in three
    # timed phases; 18 bytes per element
    # (k, v read for the state; q, dout read and dq written; k, v read and dk, dv written)
    5: {"phases": ("litela_reduce_tc+litela_state_scan", "litela_bwd_q_tc", "litela_state_scan+litela_bwd_kv_tc"),
        "alg_bytes_E": {"litela_reduce_tc+litela_state_scan": 4, "litela_bwd_q_tc": 6,
                        "litela_state_scan+litela_bwd_kv_tc": 8}},
    # the backward with one block per sequence (lite_la_bwd_kernels_per_call == 3): the dq and
    # dk/dv kernels sum the partial states into their images themselves, no scan launches
    "bwd3": {"phases": ("litela_reduce_tc", "litela_bwd_q_tc", "litela_bwd_kv_tc"),
             "alg_bytes_E": {"litela_reduce_tc": 4, "litela_bwd_q_tc": 6, "litela_bwd_kv_tc": 8}},
    1: {"phases": ("litela_fused_tc",), "alg_bytes_E": {"litela_fused_tc": 8}},
    # the fused kernel's paired form (lite_la_forward_form == LITELA_FORM_FUSED_PAIRED)
    "paired": {"phases": ("litela_paired_tc",), "alg_bytes_E": {"litela_paired_tc": 8}},
    3: {"phases": ("litela_reduce_tc+litela_state_scan", "litela_apply_tc"),
        "alg_bytes_E": {"litela_reduce_tc+litela_state_scan": 4, "litela_apply_tc": 4}},
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["_source"] = "fallback"
    return d


def fp32_fma_peak_tflops(mhz):
    return NUM_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during a timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid, self.proc, self.path = gpu_uuid, None, None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        power = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def clocks_rejected(c):
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    if bad & set(c.get("reasons", [])):
        return True
    if c.get("sm_mhz") and c.get("sm_max_mhz") and c["sm_mhz"] < 0.5 * c["sm_max_mhz"] \
            and "sw_power_cap" not in c.get("reasons", []):
        return True
    return False


def measure_ffma_peak(ll, dev, stream, seconds):
    """fp32 FMA peak of this GPU: the FMA loop of liblitela_ffma_peak on every SM (4 CTAs of
    512 threads per SM), sized to run about `seconds`, timed with CUDA events on `stream`, with
    the clocks it ran at."""
    import ctypes
    import torch
    h = ll.ffma_peak_lib()
    props = torch.cuda.get_device_properties(dev)
    blocks, threads = props.multi_processor_count * 4, 512
    sink = torch.empty(blocks * threads, dtype=torch.float32, device=dev)
    sh = ctypes.c_void_p(stream.cuda_stream)

    def run(iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if h.litela_ffma_launch(sink.data_ptr(), blocks, threads, iters, sh) != 0:
            raise RuntimeError("litela_ffma_launch failed")
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    iters = 2000
    ms = run(iters)
    iters = max(iters, int(iters * seconds * 1e3 / max(ms, 1e-3)))
    uuid = "GPU-" + str(props.uuid)
    with ClockSampler(uuid) as cs:
        ms = run(iters)
    flops = h.litela_ffma_flops(blocks, threads, iters)
    return {"tflops": flops / (ms * 1e-3) / 1e12, "seconds": ms * 1e-3, "blocks": blocks, "threads": threads,
            "clocks": cs.summary(), "how": "8 independent fp32 FMA chains per thread, 2048 threads per SM, "
                                           "CUDA events on the launching stream"}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def single_thread_rate(fn, seconds):
    """fn(seconds) with numpy's BLAS limited to one thread (None if that cannot be set)."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    with threadpool_limits(limits=1):
        return fn(seconds)


def one_head_bits(qkv_bits, B, N, H, b, h):
    """Packed [1, N, 3*d] bits of head h of batch b (input re-packing only)."""
    import numpy as np
    x = qkv_bits.reshape(B, N, 3, H, D)[b, :, :, h, :]
    return np.ascontiguousarray(x.reshape(1, N, 3 * D))


def oracle_head(oracle, head_bits, N, T, dout_bits=None, variant="litela"):
    """The oracle on one whole (batch, head): non-causal when T == 0; the backward (all N
    tokens' dq, dk, dv) when dout_bits [1, N, d] is given; the ELU+1 forward for elu1."""
    if variant == "elu1":
        return oracle.elu1_fwd(head_bits, 1, N, 1, D, 1e-6, T or None)
    if dout_bits is not None:
        if T:
            return oracle.lite_la_block_causal_bwd(head_bits, dout_bits, 1, N, 1, D, EPS, T)
        return oracle.lite_la_bwd(head_bits, dout_bits, 1, N, 1, D, EPS)
    if T:
        return oracle.lite_la_block_causal_fwd(head_bits, 1, N, 1, D, EPS, T)
    return oracle.lite_la_fwd(head_bits, 1, N, 1, D, EPS)


def one_head_dout_bits(dout_bits, B, N, H, b, h):
    """[1, N, d] bits of head h of batch b of an incoming gradient [B, N, H*d]."""
    import numpy as np
    return np.ascontiguousarray(dout_bits.reshape(B, N, H, D)[b, :, h, :].reshape(1, N, D))


def oracle_head_rate(qkv_bits, B, N, H, T, seconds, max_heads=None, dout_bits=None, variant="litela"):
    """Times the fp64 oracle on whole heads (all N queries of one (batch, head)) until
    `seconds` have passed; returns (tokens*heads per second, heads done, elapsed)."""
    import oracle
    heads, t0 = 0, time.perf_counter()
    while True:
        b, h = divmod(heads % (B * H), H)
        g = None if dout_bits is None else one_head_dout_bits(dout_bits, B, N, H, b, h)
        oracle_head(oracle, one_head_bits(qkv_bits, B, N, H, b, h), N, T, g, variant)
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_heads and heads >= max_heads):
            return heads * N / el, heads, el


def workload_seeds(wl, calls):
    """Seeds of a workload's distinct input buffers (the 4096px ones are 4000 + i)."""
    seed0 = WORKLOADS_BENCH[wl][4]
    return [seed0 + i for i in range(calls)] if wl.startswith("sana4800m") else [seed0 * 10 + i for i in range(calls)]


def call_bounds_us(B, N, H, peaks, ffma_tflops=None):
    """The workload definition's roofline of one forward call: 8 bytes per (token, head,
    channel) at the copy bandwidth, and 4*B*H*N*d*(d+1) FLOPs at the fp32 FMA peak (from the
    unit counts at the maximum clock, and as measured when given)."""
    E = B * N * H * D
    t_hbm = 8 * E / (peaks["hbm_gbs"] * 1e9) * 1e6
    flops = 4 * B * H * N * D * (D + 1)
    t_fma = flops / (fp32_fma_peak_tflops(peaks.get("sm_max_mhz", 1965.0)) * 1e12) * 1e6
    t_fma_meas = flops / (ffma_tflops * 1e12) * 1e6 if ffma_tflops else None
    return t_hbm, t_fma, t_fma_meas


def time_record_workload(ll, lib, dev, stream, wl, peaks, ffma_tflops=None, reps=5, min_ms=25.0):
    """One entry of the `workloads` record: the workload's calls on its distinct buffers,
    back to back, timed with CUDA events on the launching stream; `reps` repetitions of K
    steps (K sized so one repetition lasts at least `min_ms`), median reported."""
    import ctypes
    import torch
    from linear_attention_diffusion_litela_b200.inputs import make_qkv
    B, N, H, calls, _seed0, T = WORKLOADS_BENCH[wl]
    ins = [make_qkv(B, N, H, D, seed=s, device=dev, qk_shift=QK_SHIFT.get(wl, 0.0)) for s in workload_seeds(wl, calls)]
    outs = [torch.empty((B, N, H * D), dtype=torch.bfloat16, device=dev) for _ in range(calls)]
    sh = ctypes.c_void_p(stream.cuda_stream)
    in_p, out_p = [t.data_ptr() for t in ins], [t.data_ptr() for t in outs]

    def step():
        for i in range(calls):
            s = (lib.lite_la_block_causal_fwd(in_p[i], out_p[i], B, N, H, D, EPS, T, sh) if T else
                 lib.lite_la_fwd(in_p[i], out_p[i], B, N, H, D, EPS, sh))
            if s != 0:
                raise ll.LiteLAError(s, lib.lite_la_last_error().decode())

    def run(K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    run(3)                                   # warm-up
    K = max(3, int(min_ms / max(run(3) / 3, 1e-3)) + 1)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    with ClockSampler(uuid) as cs:
        us = [1e3 * run(K) / (K * calls) for _ in range(reps)]
    clocks = cs.summary()
    ll.lite_la_device_status(stream)
    del ins, outs
    us_call = statistics.median(us)
    t_hbm, t_fma, t_fma_meas = call_bounds_us(B, N, H, peaks, ffma_tflops)
    rec = {"workload": wl, "B": B, "N": N, "H": H, "tokens_per_block": T or None,
           "qk_shift": QK_SHIFT.get(wl), "calls_per_step": calls, "steps_per_rep": K, "reps": reps,
           "us_per_call": us_call, "us_per_call_reps": us, "tokens_heads_per_s": B * N * H / (us_call * 1e-6),
           "kernels_per_call": int(lib.lite_la_kernels_per_call(B, N, H, D, T)),
           "form": ll.FORMS.get(int(lib.lite_la_forward_form(B, N, H, D, T))),
           "t_hbm_us": t_hbm, "hbm_frac": t_hbm / us_call, "t_fma_us": t_fma,
           "t_roof_us": max(t_hbm, t_fma), "roof_frac": max(t_hbm, t_fma) / us_call,
           "l2": l2_note(B, N, H, calls), "clocks": clocks}
    if t_fma_meas:
        rec["frac_vs_measured_fma_peak"] = max(t_hbm, t_fma_meas) / us_call
    return rec


def emit(line):
    print(json.dumps(line), flush=True)


def run_reference(args, wl):
    """Reference arm: the fp64 oracle on the host cores, one whole head per step."""
    import numpy as np
    import torch
    from linear_attention_diffusion_litela_b200.inputs import make_qkv, to_bits
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    B, N, H, calls, seed, T = WORKLOADS_BENCH[wl]
    bits = to_bits(make_qkv(B, N, H, D, seed=seed, device="cpu", qk_shift=QK_SHIFT.get(wl, 0.0)))
    if args.variant == "fused_oproj":
        return run_reference_oproj(args, wl, bits)
    bwd = args.direction == "bwd"
    gbits = to_bits(make_dout(B, N, H, seed + 500, "cpu")) if bwd else None
    import oracle
    heads = [(i // H % B, i % H) for i in range(args.warmup + args.steps)]

    def head_dout(b, h):
        return None if gbits is None else one_head_dout_bits(gbits, B, N, H, b, h)

    for i in range(args.warmup):
        oracle_head(oracle, one_head_bits(bits, B, N, H, *heads[i]), N, T, head_dout(*heads[i]), args.variant)
    times = []
    for i in range(args.steps):
        hb = one_head_bits(bits, B, N, H, *heads[args.warmup + i])
        gb = head_dout(*heads[args.warmup + i])
        t0 = time.perf_counter()
        oracle_head(oracle, hb, N, T, gb, args.variant)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    value = N / (ms / 1e3)
    sample = ("one whole (batch, head) per step: all %d queries against all %d keys" % (N, N) if not T else
              "one whole (batch, head) per step: %d queries, blocks of %d tokens" % (N, T))
    emit({"impl": "reference", "metric": METRIC_BWD if bwd else METRIC, "value": value, "unit": UNIT,
          "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
          "data": "synthetic: i.i.d. N(0,1) bf16 qkv, seed %d" % seed,
          "config": config_of(wl, args.direction, args.variant),
          "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                           "sample": sample},
          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
    return 0


def run_reference_oproj(args, wl, bits):
    """Reference arm of --variant fused_oproj: the fp64 oracle of LiteLA + projection, 16 query
    rows of batch 0 per step (all heads against all keys, then the projection)."""
    import numpy as np
    import oracle
    from linear_attention_diffusion_litela_b200.inputs import to_bits
    B, N, H, calls, seed, T = WORKLOADS_BENCH[wl]
    C = H * D
    w, b = make_proj_weight(C, C, seed + 7000, "cpu")
    wbits, bias = to_bits(w), b.numpy()
    bits0 = np.ascontiguousarray(bits.reshape(B, N, 3 * C)[:1])
    times = []
    for i in range(args.warmup + args.steps):
        rows = (i + np.arange(16) * 1021) % N
        t0 = time.perf_counter()
        oracle.lite_la_oproj(bits0, wbits, 1, N, H, D, C, EPS, bias, T or None, rows=rows)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    value = 16 * H / (ms / 1e3)
    cfg = config_of(wl)
    cfg.update({"workload": wl + "_fused_oproj", "variant": "fused_oproj", "C_out": C})
    emit({"impl": "reference", "metric": METRIC_OPROJ, "value": value, "unit": UNIT, "n_gpus": args.gpus,
          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
          "scaling": "weak", "vs_baseline": None, "dtype": "f64",
          "data": "synthetic: i.i.d. N(0,1) bf16 qkv, seed %d; seeded projection weight" % seed, "config": cfg,
          "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                           "sample": "16 query rows of batch 0 per step: all %d heads against all %d keys, then "
                                     "the %d x %d projection" % (H, N, C, C)},
          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
    return 0


def make_dout(B, N, H, seed, device):
    """Incoming gradient for the backward: bf16 [B, N, H*d], i.i.d. N(0,1) from a seeded generator."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((B, N, H * D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def config_of(wl, direction="fwd", variant="litela", from_state=False):
    B, N, H, calls, seed, T = WORKLOADS_BENCH[wl]
    return {"workload": wl + ("_bwd" if direction == "bwd" else "") + ("_elu1" if variant == "elu1" else "")
            + ("_from_state" if from_state else ""),
            "direction": direction, "feature_map": "relu" if variant == "litela" else "elu+1 (clamp 1e-6)",
            "B": B, "N": N, "H": H, "d": D, "tokens_per_block": T or None, "calls_per_step": calls,
            "distinct_input_buffers": calls, "eps": EPS, "layout": "qkv bf16 [B,N,3*H*d], out bf16 [B,N,H*d]",
            "l2": l2_note(B, N, H, calls, direction)}


def l2_note(B, N, H, calls, direction="fwd"):
    """How the timed region avoids L2 reuse: the bytes one step touches (its distinct buffers)
    against the 126 MB L2."""
    E = B * N * H * D
    per_call = (3 * E + E + (E + 3 * E) if direction == "bwd" else 3 * E + E) * 2   # bf16 bytes
    ws = calls * per_call
    if ws > 126e6:
        return ("%d distinct buffer sets rotate, %.0f MB per step (%.0f MB per call) against a 126 MB L2: "
                "no flush needed" % (calls, ws / 1e6, per_call / 1e6))
    return "%d buffer sets, %.0f MB per step: SMALLER than the 126 MB L2 (warm-L2 figure)" % (calls, ws / 1e6)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)   # 50 x 60 calls: ~0.33 s timed at 4096px
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS_BENCH), default="sana4800m_4096px_x60")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffma-seconds", type=float, default=2.0,
                    help="duration of the fp32 FMA peak measurement (0 skips it)")
    ap.add_argument("--direction", choices=["fwd", "bwd"], default="fwd",
                    help="bwd times the backward (dq, dk, dv of a seeded incoming gradient)")
    ap.add_argument("--bwd-from-state", action="store_true",
                    help="with --direction bwd: the backward given the forward's saved states "
                         "(lite_la_bwd_from_state; the states are made once before timing)")
    ap.add_argument("--variant", choices=["litela", "elu1", "fused_oproj"], default="litela",
                    help="elu1 times the ELU+1 feature-map variant of the forward (clamp 1e-6); fused_oproj "
                         "LiteLA with the output projection fused (and the unfused chain beside it)")
    ap.add_argument("--shard-heads", action="store_true",
                    help="strong scaling: the ranks split the workload's heads (each rank runs its own head shard "
                         "of every call, as after a tensor-parallel qkv projection) instead of each running the "
                         "whole workload")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the `workloads` record (the other configs, timed after the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, args.workload)
    if args.variant == "fused_oproj":
        if args.direction == "bwd":
            ap.error("--variant fused_oproj has no backward")
        return main_oproj(args)

    import ctypes

    import numpy as np
    import torch
    import linear_attention_diffusion_litela_b200 as ll
    from linear_attention_diffusion_litela_b200.dist import aggregate_rate, rank_seeds, world_info
    from linear_attention_diffusion_litela_b200.dist import max_over_ranks as _max_over_ranks
    from linear_attention_diffusion_litela_b200.inputs import make_qkv, to_bits

    world, rank, local_rank = world_info()
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d (launch N>1 with torch.distributed.run)" % (args.gpus, world))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        return _max_over_ranks(x, device=dev)

    lib = ll.lib()
    B, N, H, calls, seed0, T = WORKLOADS_BENCH[args.workload]
    H_total = H
    if args.shard_heads:   # this rank's heads of every call (strong scaling)
        from linear_attention_diffusion_litela_b200.dist import shard_heads
        h0, h1 = shard_heads(H, world, rank)
        H = h1 - h0
    bwd = args.direction == "bwd"
    qkv_bytes, out_bytes = B * N * 3 * H * D * 2, B * N * H * D * 2
    free, _ = torch.cuda.mem_get_info(dev)
    need = calls * (qkv_bytes + out_bytes + (qkv_bytes if bwd else 0)) + (2 << 30)
    if free < need:
        raise SystemExit("not enough free GPU memory: need %.1f GB, free %.1f GB" % (need / 1e9, free / 1e9))
    seeds = rank_seeds(workload_seeds(args.workload, calls), 0 if args.shard_heads else rank)
    ins = [make_qkv(B, N, H, D, seed=s + (7919 * rank if args.shard_heads else 0), device=dev,
                    qk_shift=QK_SHIFT.get(args.workload, 0.0)) for s in seeds]
    outs = [torch.empty((B, N, H * D), dtype=torch.bfloat16, device=dev) for _ in range(calls)]
    if bwd:   # the backward reads an incoming gradient (in `outs`) and writes dqkv
        outs = [make_dout(B, N, H, s + 500, dev) for s in seeds]
        grads = [torch.empty((B, N, 3 * H * D), dtype=torch.bfloat16, device=dev) for _ in range(calls)]
        grad_p = [t.data_ptr() for t in grads]
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    in_p = [t.data_ptr() for t in ins]
    out_p = [t.data_ptr() for t in outs]
    if args.variant == "elu1":
        if bwd:
            raise SystemExit("--variant elu1 has no backward")

        def fwd(qkv, out, B, N, H, d, eps, stream):
            return lib.lite_la_elu1_fwd(qkv, out, B, N, H, d, 1e-6, T, stream)

        def fwd_events(qkv, out, B, N, H, d, eps, stream, evs):
            return lib.lite_la_elu1_fwd_events(qkv, out, B, N, H, d, 1e-6, T, stream, evs)
    elif bwd:   # fwd(i, ...) runs call i: here the backward of buffer i
        dq_of = {p_: g_ for p_, g_ in zip(in_p, grad_p)}
        if args.bwd_from_state:   # the forward's states of every buffer, made before timing
            nblk = -(-N // T) if T else 1
            st_bufs = [torch.empty((B, H, nblk, D + 1, D), dtype=torch.float32, device=dev) for _ in range(calls)]
            tmp = torch.empty((B, N, H * D), dtype=torch.bfloat16, device=dev)
            for p_, st in zip(in_p, st_bufs):
                if lib.lite_la_fwd_save_state(p_, tmp.data_ptr(), st.data_ptr(), B, N, H, D, EPS, T, sh) != 0:
                    raise ll.LiteLAError(1, lib.lite_la_last_error().decode())
            torch.cuda.synchronize(dev)
            st_of = {p_: st.data_ptr() for p_, st in zip(in_p, st_bufs)}

            def fwd(qkv, out, B, N, H, d, eps, stream):
                return lib.lite_la_bwd_from_state(qkv, out, st_of[qkv], dq_of[qkv], B, N, H, d, eps, T, stream)
        else:
            def fwd(qkv, out, B, N, H, d, eps, stream):
                if T:
                    return lib.lite_la_block_causal_bwd(qkv, out, dq_of[qkv], B, N, H, d, eps, T, stream)
                return lib.lite_la_bwd(qkv, out, dq_of[qkv], B, N, H, d, eps, stream)

        def fwd_events(qkv, out, B, N, H, d, eps, stream, evs):
            return lib.lite_la_bwd_events(qkv, out, dq_of[qkv], B, N, H, d, eps, T, stream, evs)
    elif T:
        def fwd(qkv, out, B, N, H, d, eps, stream):
            return lib.lite_la_block_causal_fwd(qkv, out, B, N, H, d, eps, T, stream)

        def fwd_events(qkv, out, B, N, H, d, eps, stream, evs):
            return lib.lite_la_block_causal_fwd_events(qkv, out, B, N, H, d, eps, T, stream, evs)
    else:
        fwd, fwd_events = lib.lite_la_fwd, lib.lite_la_fwd_events

    def step():
        for i in range(calls):
            s = fwd(in_p[i], out_p[i], B, N, H, D, EPS, sh)
            if s != 0:
                raise ll.LiteLAError(s, lib.lite_la_last_error().decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)

    def timed(fn, K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(uuid) as cs:
            e0.record(stream)
            for _ in range(K):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        return e0.elapsed_time(e1), cs.summary()

    ms_total, clocks = timed(step, args.steps)
    rejected = None
    # every rank re-measures if any rank's clocks were rejected (same collective steps on all)
    if max_over_ranks(1.0 if clocks_rejected(clocks) else 0.0) > 0.0:
        rejected = clocks
        ms_total, clocks = timed(step, args.steps)
    ms_total = max_over_ranks(ms_total)
    ms_step = ms_total / args.steps
    us_call = 1e3 * ms_step / calls
    # weak scaling: every rank processes the whole workload; strong: the ranks share its heads
    value = (B * N * H_total * calls * args.steps / (ms_total / 1e3) if args.shard_heads else
             aggregate_rate(B * N * H * calls * args.steps, world, ms_total))

    # per-kernel durations: the same calls through the phase-timed entry points (3 events per
    # forward call, 4 per backward call)
    nev = 4 if bwd else 3
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(calls)]
    for trip in evs:                      # recording once creates the underlying CUDA events
        for e in trip:
            e.record(stream)
    torch.cuda.synchronize(dev)
    ev_handles = [(ctypes.c_void_p * nev)(*[ctypes.c_void_p(e.cuda_event) for e in trip]) for trip in evs]
    # the ELU + 1 variant's block-causal form always takes the three-kernel path
    nk = 5 if bwd else (3 if args.variant == "elu1" and T else int(lib.lite_la_kernels_per_call(B, N, H, D, T)))
    # kernels per timed call (the saved-state backward: its own count)
    launches_per_call = (int(lib.lite_la_bwd_kernels_per_call(B, N, H, D, T, 1 if args.bwd_from_state else 0))
                         if bwd else nk)
    # the ELU + 1 variant never takes the paired form
    if bwd:   # the phases are timed on the recomputing backward
        path = PATHS["bwd3"] if int(lib.lite_la_bwd_kernels_per_call(B, N, H, D, T, 0)) == 3 else PATHS[5]
    else:
        path = PATHS["paired"] if (nk == 1 and args.variant == "litela" and
                                   int(lib.lite_la_forward_form(B, N, H, D, T)) in FORMS_PAIRED) else PATHS[nk]
    phases = path["phases"]
    kern_ms = {k: 0.0 for k in phases}
    nlaunch = 0
    for _ in range(args.steps):
        for i in range(calls):
            s = fwd_events(in_p[i], out_p[i], B, N, H, D, EPS, sh, ev_handles[i])
            if s != 0:
                raise ll.LiteLAError(s, lib.lite_la_last_error().decode())
        torch.cuda.synchronize(dev)
        for trip in evs:
            if nk == 1:
                kern_ms[phases[0]] += trip[0].elapsed_time(trip[2])
            else:
                for k in range(len(phases)):
                    kern_ms[phases[k]] += trip[k].elapsed_time(trip[k + 1])
        nlaunch += calls
    kern_us = {k: 1e3 * v / nlaunch for k, v in kern_ms.items()}
    kern_us_isolated = dict(kern_us)
    if nk == 1:
        # one kernel per call: its average launch duration over the timed region is the period
        # of the back-to-back calls (launches overlap only through programmatic dependent launch:
        # a kernel's set-up runs while its predecessor drains, its memory traffic after it)
        kern_us = {phases[0]: us_call}
    E = B * N * H * D
    # algorithmic FLOPs (2 per multiply-add): forward, the state (d+1) and the apply (d+1) per
    # element; backward, the state (d+1), y (d+1), S^T g (d), dS (d+1), dk (d), dv (d)
    flops_per_call = 2 * E * ((D + 1) + (D + 1) + D + (D + 1) + D + D) if bwd else 4 * B * H * N * D * (D + 1)
    phase_bytes_E = 18 if bwd else 8   # the phases are timed on the recomputing call
    # the call itself: the saved-state backward skips the state (k and v read, d+1 MACs per
    # element), 14 bytes per element instead of 18
    call_bytes_E = (14 if args.bwd_from_state else 18) if bwd else 8
    call_flops = flops_per_call - (2 * E * (D + 1) if bwd and args.bwd_from_state else 0)
    alg_bytes = {k: path["alg_bytes_E"][k] * E for k in phases}
    peaks = load_peaks()
    dom = max(kern_us, key=kern_us.get)
    traffic = load_traffic(dom, B, N, H, T, "bwd" if bwd else ("elu1_fwd" if args.variant == "elu1" else "fwd"))
    achieved = alg_bytes[dom] / (kern_us[dom] * 1e-6) / 1e9
    peak, unit = peaks["hbm_gbs"], "GB/s"
    peak_note = "%s copy bandwidth" % peaks["_source"]
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "kernel": dom, "kernel_us": kern_us[dom],
                "alg_bytes_per_launch": alg_bytes[dom],
                "alg_flops_per_launch": flops_per_call * alg_bytes[dom] // (phase_bytes_E * E),
                "peak_source": peak_note, "kernel_us_all": kern_us, "kernel_us_isolated": kern_us_isolated,
                "timing": ("average launch duration over the timed region: CUDA events around the back-to-back "
                           "calls on the launching stream, / launches" if nk == 1 else
                           "CUDA events on the launching stream around each phase (phase-timed entry points; "
                           "no programmatic overlap with the neighbouring kernels)")
                          + "; kernel_us_isolated: each call alone between events"
                          + ("; phases timed on the recomputing backward (the same dq and dk/dv kernels)"
                             if bwd and args.bwd_from_state else "")}
    # the call as a whole against the slower of the HBM and fp32-FMA bounds
    t_hbm = call_bytes_E * E / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_fma = call_flops / (fp32_fma_peak_tflops(peaks.get("sm_max_mhz", 1965.0)) * 1e12) * 1e6
    call_roof = {"t_hbm_us": t_hbm, "t_fma_us": t_fma, "t_roof_us": max(t_hbm, t_fma),
                 "us_per_call": us_call, "frac": max(t_hbm, t_fma) / us_call}
    if clocks.get("sm_mhz"):
        t_fma_clk = t_fma * peaks.get("sm_max_mhz", 1965.0) / clocks["sm_mhz"]
        call_roof["t_fma_us_at_measured_clock"] = t_fma_clk
        call_roof["frac_at_measured_clock"] = max(t_hbm, t_fma_clk) / us_call
    if args.ffma_seconds > 0:
        ffma = measure_ffma_peak(ll, dev, stream, args.ffma_seconds)
        t_fma_meas = call_flops / (ffma["tflops"] * 1e12) * 1e6
        call_roof["ffma_peak_measured"] = ffma
        call_roof["t_fma_us_measured_peak"] = t_fma_meas
        call_roof["frac_vs_measured_fma_peak"] = max(t_hbm, t_fma_meas) / us_call

    # end to end: pinned host input -> device, forward, device -> pinned host output, per call.
    # The copies run on their own streams so that the next call's upload and the previous
    # call's download overlap this call's kernels (PCIe is full duplex); events order them.
    e2e = None
    if args.e2e_steps > 0:
        nbuf = 3
        h_in = [torch.empty((B, N, 3 * H * D), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
        h_out = [torch.empty((B, N, H * D), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
        for j in range(nbuf):
            h_in[j].copy_(ins[j])
        if bwd:   # the backward uploads qkv and dout, and downloads dqkv
            h_g = [torch.empty((B, N, H * D), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
            h_out = [torch.empty((B, N, 3 * H * D), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
            for j in range(nbuf):
                h_g[j].copy_(outs[j])
        results = grads if bwd else outs
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(nbuf)]
        ev_fwd = [torch.cuda.Event() for _ in range(nbuf)]
        ev_down = [torch.cuda.Event() for _ in range(nbuf)]
        for j in range(nbuf):
            ev_down[j].record(down)

        def e2e_step():
            for i in range(calls):
                j = i % nbuf
                with torch.cuda.stream(up):
                    up.wait_event(ev_fwd[j])          # the forward that last read ins[j] is done
                    ins[j].copy_(h_in[j], non_blocking=True)
                    if bwd:
                        outs[j].copy_(h_g[j], non_blocking=True)
                    ev_up[j].record(up)
                stream.wait_event(ev_up[j])
                stream.wait_event(ev_down[j])         # outs[j] has been downloaded
                s = fwd(in_p[j], out_p[j], B, N, H, D, EPS, sh)
                if s != 0:
                    raise ll.LiteLAError(s, lib.lite_la_last_error().decode())
                ev_fwd[j].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(ev_fwd[j])
                    h_out[j].copy_(results[j], non_blocking=True)
                    ev_down[j].record(down)
            stream.wait_stream(down)                  # the step ends when the last result is on the host

        e2e_step()
        torch.cuda.synchronize(dev)
        e2e_ms, _ = timed(e2e_step, args.e2e_steps)
        e2e_ms = max_over_ranks(e2e_ms)
        e2e = {"value": (B * N * H_total * calls * args.e2e_steps / (e2e_ms / 1e3) if args.shard_heads else
                         aggregate_rate(B * N * H * calls * args.e2e_steps, world, e2e_ms)), "unit": UNIT,
               "h2d_bytes_per_step": calls * (qkv_bytes + (out_bytes if bwd else 0)),
               "d2h_bytes_per_step": calls * (qkv_bytes if bwd else out_bytes),
               "ms_per_step": e2e_ms / args.e2e_steps, "steps": args.e2e_steps,
               "how": ("per call: pinned host qkv and dout -> device (upload stream), lite_la_bwd (compute stream), "
                       "dqkv -> pinned host (download stream)" if bwd else
                       "per call: pinned host qkv -> device copy (upload stream), lite_la_fwd (compute stream), "
                       "device -> pinned host out copy (download stream)")
                      + "; 3 buffers in rotation, events order them"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        bits = to_bits(ins[0])
        gbits = to_bits(outs[0]) if bwd else None
        rate, heads, el = oracle_head_rate(bits, B, N, H, T, args.cpu_seconds, dout_bits=gbits, variant=args.variant)
        what = "dq, dk, dv" if bwd else "all queries x all keys"
        cpu = {"value": rate, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": "%d whole (batch, head) pairs of input buffer 0 (%s, all %d tokens), %.1f s"
                         % (heads, what, N, el)}
        single = single_thread_rate(lambda sec: oracle_head_rate(bits, B, N, H, T, sec, dout_bits=gbits,
                                                                 variant=args.variant), args.cpu_seconds / 2)
        if single is not None:
            r1, h1, e1 = single
            cpu["single_thread"] = {"value": r1, "unit": UNIT, "cores": 1,
                                    "sample": "%d whole (batch, head) pairs, %s, %.1f s" % (h1, what, e1)}

    # the other configs, timed in the same run on the same GPU (single-GPU runs of the
    # headline only: a few seconds in all)
    records = None
    if (rank == 0 and world == 1 and not args.no_workloads and not bwd and args.variant == "litela"
            and args.workload == "sana4800m_4096px_x60"):
        ffma_t = call_roof.get("ffma_peak_measured", {}).get("tflops")
        records = [time_record_workload(ll, lib, dev, stream, w, peaks, ffma_t) for w in RECORD_WORKLOADS]

    if rank == 0:
        line = {"metric": METRIC_BWD if bwd else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "us_per_call": us_call,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "math": "tensor-core bf16 x bf16 products with fp32 accumulation; fp32 state applied as bf16 hi + lo",
                "data": "synthetic: i.i.d. N(0,1) bf16 qkv from seeded torch generators",
                "config": config_of(args.workload, args.direction, args.variant, args.bwd_from_state),
                "roofline": roofline,
                "call_roofline": call_roof,
                "cpu_baseline": cpu, "e2e": e2e,
                # kernels the timed calls launch (lite_la_kernels_per_call,
                # lite_la_bwd_kernels_per_call)
                "gpu_launches": launches_per_call * calls * args.steps,
                "clocks": clocks, "gpu": torch.cuda.get_device_name(dev)}
        if world > 1:
            line["config"]["parallelism"] = "dp%d (independent calls per rank, no collective)" % world
        if args.shard_heads:
            from linear_attention_diffusion_litela_b200.dist import shard_heads
            line["scaling"] = "strong"
            line["config"]["parallelism"] = ("tp%d over heads: rank r runs heads shard_heads(%d, %d, r) of every call "
                                             "(no collective)" % (world, H_total, world))
            line["config"]["heads_per_rank"] = [shard_heads(H_total, world, r) for r in range(world)]
        if rejected is not None:
            line["clocks_rejected_first_run"] = rejected
        if records is not None:
            line["workloads"] = records
        emit(line)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


METRIC_OPROJ = "LiteLA fwd + output projection tokens·heads/s and µs/call at 4096px; % of tensor roofline"
PEAKS_BF16_FALLBACK = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def make_proj_weight(C_out, C_in, seed, device):
    """Synthetic projection weight (nn.Linear-like U(-1/sqrt(C_in), 1/sqrt(C_in)), bf16) and bias
    (N(0, 0.02), fp32), from a seeded generator: Sana's trained weights are not available."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = ((torch.rand((C_out, C_in), generator=g, device=device) * 2 - 1) / C_in ** 0.5).to(torch.bfloat16)
    b = torch.randn((C_out,), generator=g, device=device) * 0.02
    return w, b


def oracle_oproj_rate(qkv_bits, w_bits, bias, B, N, H, T, seconds):
    """The fp64 oracle of LiteLA + projection on batches of 16 query rows of batch 0 (each row:
    all heads against all keys, then the projection) until `seconds` have passed; returns
    (tokens*heads per second, rows done, elapsed)."""
    import numpy as np
    import oracle
    C = H * D
    rows_done, t0, r0 = 0, time.perf_counter(), 0
    bits0 = np.ascontiguousarray(qkv_bits.reshape(B, N, 3 * C)[:1])
    while True:
        rows = (r0 + np.arange(16) * 1021) % N
        oracle.lite_la_oproj(bits0, w_bits, 1, N, H, D, C, EPS, bias, T or None, rows=rows)
        rows_done += rows.size
        r0 += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return rows_done * H / el, rows_done, el


def main_oproj(args):
    """--variant fused_oproj: one step is `calls` back-to-back calls of LiteLA + output
    projection (each layer its own qkv buffer and its own 2240 x 2240 weight and bias),
    timed as the fused call (lite_la_fwd_oproj) and, in the same run, as the unfused chain
    (lite_la_fwd, then lite_la_out_proj on its output)."""
    import ctypes
    import numpy as np
    import torch
    import linear_attention_diffusion_litela_b200 as ll
    from linear_attention_diffusion_litela_b200.dist import aggregate_rate, rank_seeds, world_info
    from linear_attention_diffusion_litela_b200.dist import max_over_ranks as _max_over_ranks
    from linear_attention_diffusion_litela_b200.inputs import make_qkv, to_bits

    world, rank, local_rank = world_info()
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d (launch N>1 with torch.distributed.run)" % (args.gpus, world))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    lib = ll.lib()
    B, N, H, calls, _seed0, T = WORKLOADS_BENCH[args.workload]
    C = H * D
    E = B * N * H * D
    seeds = rank_seeds(workload_seeds(args.workload, calls), rank)
    free, _ = torch.cuda.mem_get_info(dev)
    need = calls * (6 * E + 2 * B * N * C + 2 * C * C) + 2 * E + (2 << 30)
    if free < need:
        raise SystemExit("not enough free GPU memory: need %.1f GB, free %.1f GB" % (need / 1e9, free / 1e9))
    ins = [make_qkv(B, N, H, D, seed=s, device=dev, qk_shift=QK_SHIFT.get(args.workload, 0.0)) for s in seeds]
    wts = [make_proj_weight(C, C, s + 7000, dev) for s in seeds]
    ys = [torch.empty((B, N, C), dtype=torch.bfloat16, device=dev) for _ in range(calls)]
    xbuf = torch.empty((B, N, C), dtype=torch.bfloat16, device=dev)    # the unfused chain's attention output
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    in_p, y_p = [t.data_ptr() for t in ins], [t.data_ptr() for t in ys]
    w_p, b_p = [w.data_ptr() for w, _ in wts], [b.data_ptr() for _, b in wts]

    def call_fused(i, qkv_ptr=None, y_ptr=None):
        s = lib.lite_la_fwd_oproj(qkv_ptr or in_p[i], w_p[i], b_p[i], y_ptr or y_p[i], B, N, H, D, C, EPS, T, sh)
        if s != 0:
            raise ll.LiteLAError(s, lib.lite_la_last_error().decode())

    def call_unfused(i):
        s = (lib.lite_la_block_causal_fwd(in_p[i], xbuf.data_ptr(), B, N, H, D, EPS, T, sh) if T else
             lib.lite_la_fwd(in_p[i], xbuf.data_ptr(), B, N, H, D, EPS, sh))
        if s == 0:
            s = lib.lite_la_out_proj(xbuf.data_ptr(), w_p[i], b_p[i], y_p[i], B, N, C, C, sh)
        if s != 0:
            raise ll.LiteLAError(s, lib.lite_la_last_error().decode())

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)

    def timed(fn, K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(uuid) as cs:
            e0.record(stream)
            for _ in range(K):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        return e0.elapsed_time(e1), cs.summary()

    def step_fused():
        for i in range(calls):
            call_fused(i)

    def step_unfused():
        for i in range(calls):
            call_unfused(i)

    for _ in range(args.warmup):
        step_fused()
        step_unfused()
    torch.cuda.synchronize(dev)
    ll.lite_la_device_status(stream)
    ms_total, clocks = timed(step_fused, args.steps)
    rejected = None
    if _max_over_ranks(1.0 if clocks_rejected(clocks) else 0.0, device=dev) > 0.0:
        rejected = clocks
        ms_total, clocks = timed(step_fused, args.steps)
    ms_total = _max_over_ranks(ms_total, device=dev)
    ms_unf, clocks_unf = timed(step_unfused, args.steps)
    ms_unf = _max_over_ranks(ms_unf, device=dev)
    ll.lite_la_device_status(stream)
    ms_step = ms_total / args.steps
    us_call = 1e3 * ms_step / calls
    us_unf = 1e3 * ms_unf / (args.steps * calls)
    value = aggregate_rate(B * N * H * calls * args.steps, world, ms_total)

    # phases of the fused call: the state (reduction + scan) and the apply + projection kernel
    nev = 3
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(calls)]
    for trip in evs:
        for e in trip:
            e.record(stream)
    torch.cuda.synchronize(dev)
    ev_h = [(ctypes.c_void_p * nev)(*[ctypes.c_void_p(e.cuda_event) for e in trip]) for trip in evs]
    ph = {"litela_reduce_tc+litela_state_scan": 0.0, "litela_oproj_tc": 0.0}
    for _ in range(args.steps):
        for i in range(calls):
            s = lib.lite_la_fwd_oproj_events(in_p[i], w_p[i], b_p[i], y_p[i], B, N, H, D, C, EPS, T, sh, ev_h[i])
            if s != 0:
                raise ll.LiteLAError(s, lib.lite_la_last_error().decode())
        torch.cuda.synchronize(dev)
        for trip in evs:
            ph["litela_reduce_tc+litela_state_scan"] += trip[0].elapsed_time(trip[1])
            ph["litela_oproj_tc"] += trip[1].elapsed_time(trip[2])
    ph_us = {k: 1e3 * v / (args.steps * calls) for k, v in ph.items()}
    peaks = load_peaks()
    bf16_sust = peaks.get("bf16_tflops_sustained") or PEAKS_BF16_FALLBACK["bf16_tflops_sustained"]
    bf16_src = "measured" if peaks.get("bf16_tflops_sustained") else "fallback"
    gemm_flops = 2 * B * N * C * C
    apply_flops = 2 * E * (D + 1)
    k_flops = gemm_flops + apply_flops
    achieved = k_flops / (ph_us["litela_oproj_tc"] * 1e-6) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": bf16_sust, "unit": "TFLOP/s",
                "frac": achieved / bf16_sust, "traffic": load_traffic("litela_oproj_tc", B, N, H, T, "oproj"),
                "kernel": "litela_oproj_tc",
                "kernel_us": ph_us["litela_oproj_tc"], "alg_flops_per_launch": k_flops,
                "alg_bytes_per_launch": 2 * E + 2 * C * C + 2 * B * N * C,
                "peak_source": "%s sustained dense bf16 (cuBLAS) throughput" % bf16_src, "kernel_us_all": ph_us,
                "timing": "CUDA events on the launching stream around each phase (phase-timed entry point; no "
                          "programmatic overlap with the neighbouring kernels)"}
    t_tensor = k_flops / (bf16_sust * 1e12) * 1e6
    t_hbm = (4 * E + 2 * E + 2 * C * C + 2 * B * N * C) / (peaks["hbm_gbs"] * 1e9) * 1e6
    call_roof = {"t_tensor_us": t_tensor, "t_hbm_us": t_hbm, "t_roof_us": max(t_tensor, t_hbm),
                 "us_per_call": us_call, "frac": max(t_tensor, t_hbm) / us_call,
                 "how": "the projection GEMM's FLOPs (2 B N C^2) plus the apply's at the sustained bf16 peak, "
                        "against k, v, q read once, W read once and y written once at the copy bandwidth"}

    e2e = None
    if args.e2e_steps > 0:
        nbuf = 3
        h_in = [torch.empty((B, N, 3 * C), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
        h_out = [torch.empty((B, N, C), dtype=torch.bfloat16, pin_memory=True) for _ in range(nbuf)]
        for j in range(nbuf):
            h_in[j].copy_(ins[j])
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(nbuf)]
        ev_fw = [torch.cuda.Event() for _ in range(nbuf)]
        ev_dn = [torch.cuda.Event() for _ in range(nbuf)]
        for j in range(nbuf):
            ev_dn[j].record(down)

        def e2e_step():
            for i in range(calls):
                j = i % nbuf
                with torch.cuda.stream(up):
                    up.wait_event(ev_fw[j])
                    ins[j].copy_(h_in[j], non_blocking=True)
                    ev_up[j].record(up)
                stream.wait_event(ev_up[j])
                stream.wait_event(ev_dn[j])
                s = lib.lite_la_fwd_oproj(in_p[j], w_p[i], b_p[i], y_p[j], B, N, H, D, C, EPS, T, sh)
                if s != 0:
                    raise ll.LiteLAError(s, lib.lite_la_last_error().decode())
                ev_fw[j].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(ev_fw[j])
                    h_out[j].copy_(ys[j], non_blocking=True)
                    ev_dn[j].record(down)
            stream.wait_stream(down)

        e2e_step()
        torch.cuda.synchronize(dev)
        e2e_ms, _ = timed(e2e_step, args.e2e_steps)
        e2e_ms = _max_over_ranks(e2e_ms, device=dev)
        e2e = {"value": aggregate_rate(B * N * H * calls * args.e2e_steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": calls * 6 * E, "d2h_bytes_per_step": calls * 2 * B * N * C,
               "ms_per_step": e2e_ms / args.e2e_steps, "steps": args.e2e_steps,
               "how": "per call: pinned host qkv -> device (upload stream), lite_la_fwd_oproj (compute stream, the "
                      "layer's resident weight), y -> pinned host (download stream); 3 buffers in rotation"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nrows, el = oracle_oproj_rate(to_bits(ins[0]), to_bits(wts[0][0]), wts[0][1].cpu().numpy(), B, N, H, T,
                                            args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": "%d query rows of batch 0 of input buffer 0 (all %d heads against all %d keys, then the "
                         "%d x %d projection), %.1f s" % (nrows, H, N, C, C, el)}

    if rank == 0:
        cfg = config_of(args.workload)
        cfg.update({"workload": args.workload + "_fused_oproj", "variant": "fused_oproj", "C_out": C,
                    "weights": "%d distinct %d x %d bf16 weights and fp32 biases, one per layer (synthetic, seeded)"
                               % (calls, C, C),
                    "layout": "qkv bf16 [B,N,3*H*d], W bf16 [C_out, H*d], bias fp32 [C_out], y bf16 [B,N,C_out]"})
        line = {"metric": METRIC_OPROJ, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "us_per_call": us_call,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "math": "tensor-core bf16 x bf16 products with fp32 accumulation; LiteLA's output rounded to bf16 "
                        "inside the GEMM's operand prologue",
                "data": "synthetic: i.i.d. N(0,1) bf16 qkv and seeded nn.Linear-like weights",
                "config": cfg, "roofline": roofline, "call_roofline": call_roof,
                "unfused_chain": {"us_per_call": us_unf, "speedup_fused": us_unf / us_call, "clocks": clocks_unf,
                                  "how": "lite_la_fwd then lite_la_out_proj (this library's tcgen05 GEMM, the same "
                                         "tiles) on the same buffers, back to back"},
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 3 * calls * args.steps,
                "clocks": clocks, "gpu": torch.cuda.get_device_name(dev)}
        if world > 1:
            line["config"]["parallelism"] = "dp%d (independent calls per rank, no collective)" % world
        if rejected is not None:
            line["clocks_rejected_first_run"] = rejected
        emit(line)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def load_traffic(kernel, B, N, H, T, call="fwd"):
    """DRAM bytes per launch of `kernel` (a phase name may join several kernels with '+') on a
    call of this kind ("fwd", "bwd", "elu1_fwd") and shape, from the committed ncu summaries;
    None when there is none or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    total = 0
    for k in kernel.split("+"):
        ent = [e for e in d.get("entries", []) if e["kernel"] == k and e.get("call", "fwd") == call
               and [e["B"], e["N"], e["H"], e["T"]] == [B, N, H, T]]
        if not ent or ent[0].get("sources_sha256") != sources_hash(ent[0].get("sources")):
            return None
        total += ent[0]["dram_bytes_per_launch"]
    return total


# the kernel sources each profiled kernel is built from (the ABI file sets its launch shape)
KERNEL_SOURCES = {
    "fwd": ["litela_abi.cu", "litela_fused.cuh", "litela_paired.cuh", "litela_plan.h", "litela_tc.cuh",
            "sm100_ptx.cuh"],
    "elu1_fwd": ["litela_abi.cu", "litela_fused.cuh", "litela_plan.h", "litela_tc.cuh", "sm100_ptx.cuh"],
    "bwd": ["litela_abi.cu", "litela_bwd.cuh", "litela_plan.h", "litela_tc.cuh", "sm100_ptx.cuh"],
    "oproj": ["litela_abi.cu", "litela_oproj.cuh", "litela_plan.h", "litela_tc.cuh", "sm100_ptx.cuh"],
}


def sources_hash(files=None):
    """sha256 over the named kernel source files (all of csrc/ when None)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_diffusion_litela_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


if __name__ == "__main__":
    sys.exit(main())
