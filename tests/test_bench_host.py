"""Host-side logic of bench.py (no GPU): the clock rule, the L2 working-set note, the keying of
the ncu traffic table to kernel source files, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("clocks,rejected", [
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, False),
    ({"sm_mhz": 1300, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}, False),   # kept and noted
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]}, True),
    ({"sm_mhz": 1800, "sm_max_mhz": 1965, "reasons": ["sw_thermal_slowdown"]}, True),
    ({"sm_mhz": 1800, "sm_max_mhz": 1965, "reasons": ["hw_thermal_slowdown", "sw_power_cap"]}, True),
    ({"sm_mhz": 600, "sm_max_mhz": 1965, "reasons": []}, True),                  # a leftover clock lock
    ({}, False),                                                                   # no samples
])
def test_clock_rule(clocks, rejected):
    assert bench.clocks_rejected(clocks) is rejected


def test_every_bench_workload_rotates_more_bytes_than_l2():
    for wl, (B, N, H, calls, _seed, _T) in bench.WORKLOADS_BENCH.items():
        for direction in ("fwd", "bwd"):
            note = bench.l2_note(B, N, H, calls, direction)
            assert "no flush needed" in note, (wl, direction, note)
    # a rotation that fits in L2 is called out as such
    assert "SMALLER" in bench.l2_note(1, 256, 36, 20)


def test_config_names_the_workload_and_its_variant():
    assert bench.config_of("sana4800m_4096px_x60")["workload"] == "sana4800m_4096px_x60"
    c = bench.config_of("block_causal_16x1024", "bwd", "litela", True)
    assert c["workload"] == "block_causal_16x1024_bwd_from_state" and c["tokens_per_block"] == 1024
    assert bench.config_of("sana1600m_2048px", variant="elu1")["feature_map"].startswith("elu+1")


def test_traffic_entries_follow_their_own_kernel_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "linear_attention_diffusion_litela_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    for name, text in (("a.cuh", "kernel a"), ("b.cuh", "kernel b"), ("common.h", "shared")):
        (csrc / name).write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))

    def entry(kernel, call, files, nbytes):
        return {"kernel": kernel, "call": call, "B": 2, "N": 8, "H": 4, "T": 0, "dram_bytes_per_launch": nbytes,
                "sources": files, "sources_sha256": bench.sources_hash(files)}

    table = {"entries": [entry("ka", "fwd", ["a.cuh", "common.h"], 100),
                         entry("kb", "fwd", ["b.cuh", "common.h"], 20),
                         entry("ka", "bwd", ["a.cuh", "common.h"], 7)]}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(table))
    assert bench.load_traffic("ka", 2, 8, 4, 0) == 100
    assert bench.load_traffic("ka", 2, 8, 4, 0, "bwd") == 7             # keyed by the call kind
    assert bench.load_traffic("ka+kb", 2, 8, 4, 0) == 120                # a phase sums its kernels
    assert bench.load_traffic("ka", 2, 8, 4, 64) is None                 # another shape
    assert bench.load_traffic("kc", 2, 8, 4, 0) is None                  # no capture
    (csrc / "b.cuh").write_text("kernel b, changed")
    assert bench.load_traffic("ka", 2, 8, 4, 0) == 100                   # a's files did not change
    assert bench.load_traffic("kb", 2, 8, 4, 0) is None                  # b's did: its entry lapses
    assert bench.load_traffic("ka+kb", 2, 8, 4, 0) is None
    (csrc / "common.h").write_text("shared, changed")
    assert bench.load_traffic("ka", 2, 8, 4, 0) is None


def test_committed_traffic_entries_name_existing_sources():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        table = json.load(f)
    csrc = os.path.join(ROOT, "linear_attention_diffusion_litela_b200", "csrc")
    for e in table["entries"]:
        assert e["sources"] == bench.KERNEL_SOURCES[e["call"]]
        assert all(os.path.exists(os.path.join(csrc, f)) for f in e["sources"])
        assert os.path.exists(os.path.join(ROOT, "profiles", e["profile"]))


def test_reference_arm_prints_its_line_on_the_host_cores():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "sana600m_512px", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "sana600m_512px"


def test_the_workloads_record_covers_every_other_config_with_its_bounds():
    """The default run times the other configs of the workload definition beside the headline:
    512px, 1024px, 2048px (and its mostly-negative input) and the block-causal call; each bound
    follows from the unit counts (8 bytes per element at the copy peak; 4*B*H*N*d*(d+1) FLOPs at
    148 SMs x 128 lanes x 2 x the clock)."""
    assert set(bench.RECORD_WORKLOADS) == {"sana600m_512px", "sana1600m_1024px", "sana1600m_2048px",
                                           "sana1600m_2048px_mostly_negative", "block_causal_16x1024"}
    assert bench.QK_SHIFT["sana1600m_2048px_mostly_negative"] == -1.5
    peaks = {"hbm_gbs": 6543.4, "sm_max_mhz": 1965.0}
    t_hbm, t_fma, t_meas = bench.call_bounds_us(2, 16384, 70, peaks, 71.48)
    assert abs(t_hbm - 89.74) < 0.01 and abs(t_fma - 130.14) < 0.01 and abs(t_meas - 135.54) < 0.01
    t_hbm, t_fma, t_meas = bench.call_bounds_us(2, 1024, 70, peaks)
    assert abs(t_hbm - 5.61) < 0.01 and abs(t_fma - 8.13) < 0.01 and t_meas is None
    assert bench.workload_seeds("sana4800m_4096px_x60", 3) == [4000, 4001, 4002]
    assert bench.workload_seeds("sana1600m_2048px_mostly_negative", 2) == [30010, 30011]
