"""Host-side checks of the forward's partition (litela_plan.h compiled with g++; no GPU).

The paired fused form (fused_paired: every CTA of a sibling group works on two head quads) must
reduce every (quad, token) exactly once and apply every (quad, 128-token tile) exactly once,
with at most one CTA per SM; the index arithmetic below restates the kernel's role decode
(ticket -> sibling r of group g, units g and g + ceil(nq / 2), token chunk r, tiles
[r*nt/S, (r+1)*nt/S)).
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_attention_diffusion_litela_b200", "csrc")

SHAPES = [(2, 16384, 70), (2, 4096, 70), (2, 1024, 70), (1, 256, 36), (1, 2048, 8), (1, 2100, 5),
          (2, 2048, 7), (3, 4096, 6), (1, 4097, 12), (2, 3000, 9), (4, 2500, 36), (1, 8192, 140),
          (1, 2049, 2), (1, 5000, 4), (40, 2048, 32)]
# block-causal (B, N, H, T)
CAUSAL = [(1, 16384, 70, 1024), (2, 16384, 70, 1024), (1, 8192, 70, 1024), (1, 2048, 40, 128), (1, 2100, 40, 128),
          (3, 1024, 30, 128), (2, 700, 70, 128), (2, 640, 66, 128), (1, 1000, 8, 128), (1, 16384, 70, 512),
          (1, 4096, 70, 512), (1, 300, 8, 100), (2, 8192, 36, 1024), (1, 16384, 70, 256), (1, 300, 5, 1)]

DRIVER = r"""
#include <cstdio>
#include "litela_plan.h"
int main(int argc, char** argv) {
  const int min_chunk = atoi(argv[1]);
  for (int i = 2; i + 3 < argc; i += 4) {
    litela::Plan p;
    litela::make_plan(atoi(argv[i]), atoi(argv[i + 1]), atoi(argv[i + 2]), atoi(argv[i + 3]), 148, &p, min_chunk);
    printf("{\"fused\": %d, \"paired\": %d, \"causal\": %d, \"nquads\": %d, \"ntiles\": %d, \"S\": %d, "
           "\"chunk\": %d, \"bytes\": %zu, \"counters\": %zu, \"cpb\": %d, \"bpc\": %d, \"nblk\": %d, "
           "\"red_cpb\": %d, \"red_bpc\": %d, \"ngroups\": %d}\n",
           p.fused, p.fused_paired, p.fused_causal, p.nquads, p.fused_ntiles, p.paired_cpb, p.paired_chunk,
           p.paired_bytes, p.counters, p.fused_cpb, p.fused_bpc, p.nblk, p.chunks_per_block, p.red_bpc, p.ngroups);
  }
  return 0;
}
"""


@pytest.fixture(scope="module", params=[1024, 64], ids=["default_min_chunk", "min_chunk_64"])
def plans(tmp_path_factory, request):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("plan")
    src = d / "plan_driver.cpp"
    src.write_text("#include <cstdlib>\n" + DRIVER)
    exe = d / "plan_driver"
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    keys = [s + (0,) for s in SHAPES] + CAUSAL
    args = [str(x) for k in keys for x in k]
    out = subprocess.run([str(exe), str(request.param), *args], check=True, capture_output=True, text=True).stdout
    res = dict(zip(keys, (json.loads(l) for l in out.splitlines())))
    return request.param, {k[:3]: v for k, v in res.items() if k[3] == 0}, {k: v for k, v in res.items() if k[3]}


def test_paired_form_is_chosen_for_chunks_of_the_paired_minimum(plans):
    min_chunk, plans, _ = plans
    for (B, N, H), p in plans.items():
        nq = B * ((H + 3) // 4)
        assert p["fused"] == (nq <= 148)
        # the paired form's chunk: 148 // ceil(nq / 2) siblings per quad (at most one per apply
        # tile), tokens split evenly and rounded up to 64
        S = max(1, min(148 // ((nq + 1) // 2), -(-N // 128)))
        chunk = -(-(-(-N // S)) // 64) * 64
        assert p["paired"] == (p["fused"] == 1 and nq >= 2 and chunk >= min_chunk), (B, N, H, p)
        if p["paired"]:
            assert p["chunk"] == chunk
    # the Sana 4096px call: 18 sibling groups of 8 CTAs (144 CTAs), chunks of 2048 tokens; the
    # 2048px call (chunks of 512) takes the plain fused form unless the minimum is lowered
    p = plans[(2, 16384, 70)]
    assert p["paired"] and p["S"] == 8 and p["chunk"] == 2048
    assert plans[(2, 4096, 70)]["paired"] == (min_chunk <= 512)


@pytest.mark.parametrize("shape", [s for s in SHAPES])
def test_paired_partition_covers_every_token_and_tile_once(plans, shape):
    B, N, H = shape
    p = plans[1][shape]
    assert not p["causal"]
    if not p["paired"]:
        return
    nq = B * p["nquads"]
    S, chunk, nt = p["S"], p["chunk"], p["ntiles"]
    grid = (nq + 1) // 2 * S
    assert grid <= 148 and chunk % 64 == 0 and (S - 1) * chunk < N <= S * chunk
    assert p["bytes"] >= nq * S * 4 * 33 * 32 * 4 and p["counters"] == nq + 2
    red = [[0] * N for _ in range(nq)]
    app = [[0] * nt for _ in range(nq)]
    for ticket in range(grid):
        r, g = ticket % S, ticket // S
        units = [c for c in (g, g + (nq + 1) // 2) if c < nq]
        n0, n1 = r * chunk, min(r * chunk + chunk, N)
        t0, t1 = r * nt // S, (r + 1) * nt // S
        for c in units:
            for t in range(n0, n1):
                red[c][t] += 1
            for tl in range(t0, t1):
                app[c][tl] += 1
    assert all(x == 1 for row in red for x in row)
    assert all(x == 1 for row in app for x in row)


def test_paired_block_causal_form_and_its_partition(plans):
    """Block-causal calls take the paired form when every (quad, pair of blocks) has a CTA and
    blocks have at least the paired minimum of tokens.  Sibling r of quad c then owns blocks r and
    r + S (S = ceil(nblk / 2)): every (quad, token) is reduced once and every (quad, tile) applied
    once, each tile inside its block; block r's prefix needs only blocks 0..r, which are all first
    halves, and block r + S's adds blocks r + 1..r + S."""
    min_chunk, _, causal = plans
    for (B, N, H, T), p in causal.items():
        nq, nblk = B * ((H + 3) // 4), -(-N // T)
        S = (nblk + 1) // 2
        # the plain form's blocks per CTA: 148 // nq CTAs per quad at most, one per block
        bpc = -(-nblk // max(1, min(148 // nq, nblk))) if nq <= 148 else 0
        want = 1 < nblk and nq <= 148 and T % 128 == 0 and bpc == 2 and T >= min_chunk
        assert p["paired"] == want, (B, N, H, T, p)
        assert nq * S <= 148 or not want
        if not want:
            continue
        assert p["causal"] and p["S"] == S and p["chunk"] == T and p["counters"] == nq * nblk + 2
        assert p["bytes"] >= nq * nblk * 4 * 33 * 32 * 4
        nt = -(-N // 128)
        red = [[0] * N for _ in range(nq)]
        app = [[0] * nt for _ in range(nq)]
        for ticket in range(nq * S):
            r, c = ticket % S, ticket // S
            for blk in (r, r + S):
                if blk >= nblk:
                    continue
                n0, n1 = blk * T, min(blk * T + T, N)
                for t in range(n0, n1):
                    red[c][t] += 1
                for tl in range(n0 // 128, -(-n1 // 128)):
                    assert tl * 128 >= n0 and min(tl * 128 + 128, N) <= n1   # the tile lies in the block
                    app[c][tl] += 1
            assert r < S and r + 1 <= S   # block r's prefix: blocks 0..r, all owned as first halves
        assert all(x == 1 for row in red for x in row)
        assert all(x == 1 for row in app for x in row)
    assert causal[(1, 16384, 70, 1024)]["paired"]   # the 16 x 1024 workload: 18 quads x 8 siblings


def test_reduction_walks_several_blocks_per_cta_when_blocks_are_short(plans):
    """With one chunk per block and more (batch, group, block) units than two CTAs per SM, a
    reduction CTA walks red_bpc consecutive blocks: the grid is at most one wave and covers
    every block of every (batch, group) once."""
    _, _, causal = plans
    seen_multi = False
    for (B, N, H, T), p in causal.items():
        units = B * p["ngroups"] * p["nblk"]
        if p["red_bpc"] == 1:
            assert p["red_cpb"] > 1 or units <= 2 * 148 or p["nblk"] <= (2 * 148) // (B * p["ngroups"])
            continue
        seen_multi = True
        assert p["red_cpb"] == 1
        per_group = -(-p["nblk"] // p["red_bpc"])
        assert B * p["ngroups"] * per_group <= 2 * 148
        cover = [0] * p["nblk"]
        for x in range(per_group):
            for k in range(x * p["red_bpc"], min((x + 1) * p["red_bpc"], p["nblk"])):
                cover[k] += 1
        assert all(c == 1 for c in cover), (B, N, H, T)
    assert seen_multi
