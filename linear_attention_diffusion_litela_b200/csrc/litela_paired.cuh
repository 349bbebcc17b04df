// LiteLA forward (non-causal) as one persistent kernel in which every CTA works on two head
// quads, so that the wait for a quad's sibling CTAs and the merge of their partial states run
// while the CTA streams the other quad's tokens: HBM does not idle between the state
// reduction and the apply.
//
// Method: see litela_tc.cuh.  The nq quads are indexed c = b * nquads + q.  A sibling group g
// of S CTAs (S consecutive tickets) owns quads g and g + ceil(nq / 2) (its units 0 and 1; the
// last group may own one); sibling r takes token chunk r of both quads for the reduction and
// apply tiles [r * ntiles / S, (r + 1) * ntiles / S) of both.  One ring of 32 KB stages
// carries, in order,
//   unit 0's k|v tiles (64 tokens x 4 heads of k and of v), unit 1's k|v tiles   (6 stages),
//   unit 0's q tiles (128 tokens x 4 heads), unit 1's q tiles       (the first 4 stages),
// so the TMA producer streams without a break between the phases; once the reductions are
// over, the stages after the q stages hold the output staging and unit 1's state image.
// Before the programmatic-launch wait the producer prefetches its first k|v tiles into L2, so
// that the start of a call overlaps the end of the previous one.  Four ReLU warps clamp every
// stage in place (k of a k|v stage, all of a q stage).  One thread issues the MMAs in the same
// order: per 16 tokens of unit u's k|v, D_u[0:128, 0:128] += phi(K)^T . V and
// D_u[0:128, 128:144] += phi(K)^T . 1 into TMEM accumulator u; then, once unit 0's merged state
// is in shared memory, y = phi(Q) . [S_hi ; S_lo]^T per head of unit 0's q tiles (M = 128
// tokens, N = 80, one head pair per TMEM slot, three slots), then the same for unit 1.
// Four merge warps read accumulator u out as this CTA's partial state of quad c_u, publish it
// (a global write, then an arrival count), wait until the quad's S siblings have arrived, sum
// the S partials in fixed order r = 0..S-1 (deterministic), and write the state image (bf16
// hi + lo, the apply's B operand).  Unit 0's merge runs during unit 1's reduction; unit 1's
// during unit 0's apply.  Four epilogue warps read the apply's accumulators (thread = token),
// form y[r] / (y[d] + eps) and stage each head pair's output box, which is stored with TMA as
// soon as it is staged.
// Block-causal form (kCausal, blocks of T tokens, T a multiple of 128): group g is quad g alone
// and sibling r owns its blocks r and r + S (units 0 and 1; S = ceil(nblk / 2)).  Each sibling
// publishes its two block states, each with a flag of its own.  Block r's prefix (the sum of
// the states of blocks 0..r, in that order) needs only first-half blocks, which the siblings
// publish halfway through their reductions, so its merge runs during block r + S's reduction;
// block r + S's prefix continues the same running sum over blocks r + 1..r + S, during block r's
// apply.
// TMEM (512 columns): accumulator 0 in columns 0..143, under apply slot 0, which the MMAs use
// only after unit 0's merge (it follows the read-out); accumulator 1 in columns 320..463,
// under apply slot 2, which they use only after the merge warps release it.
// Cross-CTA control words, tickets and the programmatic-launch protocol are those of
// litela_fused_tc: every CTA takes its ticket before the programmatic-launch wait, siblings
// hold consecutive tickets, the arrival and finish counters are touched only after the
// previous kernel in the stream completed, and the CTA that counts itself out last zeroes
// them.  Every wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "litela_fused.cuh"
#include "litela_plan.h"
#include "litela_tc.cuh"
#include "sm100_ptx.cuh"

namespace litela {

enum : int {
  kErrPairProducer = 0x480, kErrPairMma = 0x490, kErrPairMap = 0x4a0, kErrPairMerge = 0x4b0,
  kErrPairEpi = 0x4c0, kErrPairSibling = 0x4d0, kErrPairTicket = 0x4e0,
};

template <typename OutT>
struct PairedCfg {
  // warps: 0 TMA, 1 MMA, 2..5 ReLU, 6..9 accumulator read-out and merges, 10..13 apply epilogue
  static constexpr int kThreads = 448;
  static constexpr int kMergeWarp0 = 6, kEpiWarp0 = 10;
  // 448 threads: a launch bound of 512 keeps ptxas at 128 registers (4 warps share an SM
  // sub-partition's 16K registers)
  static constexpr int kLaunchBound = 512;
  static constexpr uint32_t kStageBytes = kRedStageBytes;   // = one q tile of 2 x kQBoxBytes
  static constexpr int kBoxChannels = 128 / (int)sizeof(OutT);
  static constexpr int kOutBoxes = kApUnitHeads * kD / kBoxChannels;   // 2 (bf16) or 4 (fp32)
  static constexpr int kBoxesPerPair = kOutBoxes / 2;
  static constexpr uint32_t kOutBytes = kOutBoxes * kOutBoxBytes;    // one tile's output boxes
  // ring: 6 stages while the reductions stream (the loads in flight set their pace); then the
  // output boxes take the stages after the q stages and unit 1's image the last one
  static constexpr int kStages1 = 6;
  static constexpr int kOutStages = (int)(kOutBytes / kStageBytes);   // 1 (bf16) or 2 (fp32)
  static constexpr int kStages2 = kStages1 - kOutStages - 1;          // 4 (bf16) or 3 (fp32)
  static constexpr uint32_t kBarBytes = 512;
  static constexpr uint32_t kSmemBytes = kStages1 * kStageBytes + kApSbufBytes + 512 + kBarBytes + 1024;
  static constexpr uint32_t kAcc1Col = 2 * kApAccCols;
  // k|v tiles of unit 0 prefetched into L2 before the programmatic-launch wait (8 measured
  // 1-2 % faster than 12 with the evict-first inputs; 6 no better)
  static constexpr int kPrefetchTiles = 8;
};
static_assert(kRedStageBytes == 2 * kQBoxBytes, "a k|v stage and a q stage take the same ring slot");
// the ReLU role is warps 2..5 (128 threads: its loops and its barrier count), then 4 merge and 4
// epilogue warps (any 4 consecutive warps cover the four TMEM lane quarters)
static_assert(PairedCfg<__nv_bfloat16>::kMergeWarp0 == 6 && PairedCfg<__nv_bfloat16>::kEpiWarp0 == 10 &&
                  PairedCfg<__nv_bfloat16>::kThreads == 32 * 14 && PairedCfg<float>::kThreads == 32 * 14,
              "paired kernel warp roles");
static_assert(kApSbufBytes <= kRedStageBytes, "unit 1's image fits one stage");
static_assert(PairedCfg<__nv_bfloat16>::kAcc1Col + 144 <= kFuTmemCols, "TMEM columns");

template <typename OutT, bool kCausal = false>
__global__ void __launch_bounds__(PairedCfg<OutT>::kLaunchBound, 1)
litela_paired_tc(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_q,
                 const __grid_constant__ CUtensorMap tmap_out, float* __restrict__ partials,
                 unsigned* __restrict__ counters, int* __restrict__ err, FusedPlan p) {
  using namespace sm100;
  using Cfg = PairedCfg<OutT>;
  constexpr int R = Cfg::kStages1, R2 = Cfg::kStages2;
  constexpr uint32_t kStageBytes = Cfg::kStageBytes;
  constexpr int kChunksPerHead = kD * (int)sizeof(OutT) / 16;
  constexpr int kPartFloats = kRedHeads * kStateFloats;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* ring = smem;
  uint8_t* obuf = ring + R2 * kStageBytes;              // after the reductions
  uint8_t* sbuf1 = ring + (R - 1) * kStageBytes;        // after the reductions
  uint8_t* sbuf = ring + R * kStageBytes;               // unit 0's image
  uint8_t* ones = sbuf + kApSbufBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ones + 512);
  uint64_t* full = bars;              // ring: loads landed
  uint64_t* mapped = full + R;        // ring: ReLU done
  uint64_t* empty = mapped + R;       // ring: the MMAs reading the stage completed
  uint64_t* done = empty + R;         // [2] unit u's reduction MMAs completed
  uint64_t* sfull = done + 2;         // [2] unit u's state image written
  uint64_t* acc1_free = sfull + 2;    // accumulator 1 read out (apply slot 2 may be used)
  uint64_t* tfull = acc1_free + 1;    // [3] apply slot holds a head pair's result
  uint64_t* tempty = tfull + kApAccSlots;
  uint64_t* mma_idle = tempty + kApAccSlots;   // every MMA this CTA issued completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_idle + 1);
  static_assert((3 * R + 6 + 2 * kApAccSlots) * 8 + 3 * 4 <= Cfg::kBarBytes, "paired kernel: barrier area");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* ticket_slot = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // ticket in arrival order (see litela_fused_tc), before the programmatic-launch wait
    const unsigned tk = atomicAdd(&counters[p.counter_words - 1], 1u);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&mapped[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&done[u], 1);
      mbar_init(&sfull[u], 1);
    }
    mbar_init(acc1_free, 1);
    for (int s = 0; s < kApAccSlots; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 128);
    }
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    if (tk == gridDim.x - 1) {
      counters[p.counter_words - 1] = 0u;
      __threadfence();
    }
    *ticket_slot = (int)tk;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 128; i += Cfg::kThreads) reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_holder, kFuTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_kv);
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_out);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  auto count_out = [&]() {
    if (atomicAdd(&counters[p.counter_words - 2], 1u) == gridDim.x - 1)
      for (int i = 0; i < p.counter_words - 1; ++i) counters[i] = 0u;
  };
  auto leave = [&](bool mma_issued) {
    if (mma_issued && warp == 1 && lane == 0) mbar_drain(mma_idle, 0);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, kFuTmemCols);
    }
  };
  if (warp == 0 && lane == 0) {
    // while the previous call drains: warm L2 with this CTA's first k|v tiles (its ticket fixes
    // its units before the wait; a prefetch reads nothing into the CTA).  Measured at 4096px,
    // back to back: 119.8 us without, 114.1 us with 12 tiles (6 and 18: 116.2, 114.4; 24: 116.3,
    // the prefetches then evict more of what the previous call still uses)
    const int tk = *ticket_slot;
    if (tk >= 0 && tk < (int)gridDim.x) {
      const int rr = tk % p.cpb, c = tk / p.cpb;
      const int bb = c / p.nquads, qq = c - bb * p.nquads;
      const int y0 = rr * p.chunk, y1 = min(y0 + p.chunk, p.N);
      const int kx = p.H * kD + qq * (kRedHeads * kD), vx = 2 * p.H * kD + qq * (kRedHeads * kD);
      for (int i = 0; i < Cfg::kPrefetchTiles && y0 + i * kRedTile < y1; ++i) {
        const int y = y0 + i * kRedTile;
        tma_prefetch_3d(&tmap_kv, kx, y, bb);
        tma_prefetch_3d(&tmap_kv, kx + 64, y, bb);
        tma_prefetch_3d(&tmap_kv, vx, y, bb);
        tma_prefetch_3d(&tmap_kv, vx + 64, y, bb);
      }
    }
  }
  pdl_wait_primary();
  const int ticket = *ticket_slot;
  if (ticket < 0 || ticket >= (int)gridDim.x) {   // control words not clean: record it, do nothing
    if (threadIdx.x == 0) {
      atomicCAS(err, 0, kErrPairTicket);
      count_out();
    }
    leave(false);
    return;
  }
  const int S = p.cpb;
  const int r = ticket % S, g = ticket / S;
  // non-causal: units g and g + G of the nq quads (G = ceil(nq / 2) groups): at any time the CTAs
  // stream the quads of one contiguous range, so every DRAM page of a token row is read in one
  // pass; block-causal: blocks r and r + S of quad g
  const int nq = p.B * p.nquads, G = (nq + 1) / 2;
  const int c0 = g, c1 = kCausal ? g : g + G;
  const int blk0 = r, blk1 = r + S;   // block-causal
  const int nu = kCausal ? (blk1 < p.nblk ? 2 : 1) : (c1 < nq ? 2 : 1);
  const int b0 = c0 / p.nquads, q0 = c0 - b0 * p.nquads;
  const int b1 = c1 / p.nquads, q1 = c1 - b1 * p.nquads;
  // unit u's tokens: reduction tiles of 64 tokens in [n0_u, n1_u), apply tiles of 128 tokens
  // [t0_u, t1_u) (non-causal: chunk r of the quad and tiles [r * ntiles / S, (r + 1) * ntiles / S);
  // block-causal: the block and its tiles)
  const int n0a = kCausal ? blk0 * p.T : r * p.chunk;
  const int n1a = min(n0a + p.chunk, p.N);
  const int n0b = kCausal ? blk1 * p.T : n0a;
  const int n1b = nu == 2 ? min(n0b + p.chunk, p.N) : n0b;
  const int Pa = n1a > n0a ? (n1a - n0a + kRedTile - 1) / kRedTile : 0;
  const int Pb = n1b > n0b ? (n1b - n0b + kRedTile - 1) / kRedTile : 0;
  const int t0a = kCausal ? n0a / kApTile : (int)((long long)r * p.ntiles / S);
  const int t1a = kCausal ? (n1a + kApTile - 1) / kApTile : (int)((long long)(r + 1) * p.ntiles / S);
  const int t0b = kCausal ? n0b / kApTile : t0a;
  const int t1b = kCausal ? (n1b + kApTile - 1) / kApTile : (nu == 2 ? t1a : t0a);
  const int Qa = t1a - t0a, Qb = t1b - t0b;
  const int nP = Pa + Pb;
  const int nitems = nP + Qa + Qb;
  // per unit u: first reduction token, reduction end, reduction tiles, first apply tile, apply tiles
  auto N0 = [&](int u) { return u ? n0b : n0a; };
  auto N1 = [&](int u) { return u ? n1b : n1a; };
  auto P_ = [&](int u) { return u ? Pb : Pa; };
  auto T0 = [&](int u) { return u ? t0b : t0a; };
  auto Q_ = [&](int u) { return u ? Qb : Qa; };
  // item i's ring stage and how many earlier items used it: the reductions' items cycle
  // through R stages, the applies' through the first R2
  auto slot = [&](int i, int& s, int& use) {
    if (i < nP) {
      s = i % R;
      use = i / R;
    } else {
      const int k = i - nP;
      s = k % R2;
      use = (nP - s + R - 1) / R + k / R2;
    }
  };
  // the ring's items in order: (phase, unit, index within the unit's phase); a phase in which
  // the units have no items (a sibling past the end of the tokens) is skipped whole
  auto advance = [&](int& u, int& j, bool& ph2) {
    if (++j == (ph2 ? Q_(u) : P_(u))) {
      j = 0;
      if (++u == nu) {
        u = 0;
        ph2 = true;
      }
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // every input byte is read once: its L2 lines go first, ahead of the outputs still being
      // written back and of the next call's prefetched tiles
      const uint64_t pol = l2_policy_evict_first();
      int u = 0, j = 0, issued = 0;
      bool ph2 = nP == 0;
      for (int i = 0; i < nitems; ++i) {
        int s, use;
        slot(i, s, use);
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, abort_flag, err, kErrPairProducer | s)) break;
        uint8_t* st = ring + s * kStageBytes;
        const int b = u ? b1 : b0, q = u ? q1 : q0;
        if (!ph2) {
          const int kx = p.H * kD + q * (kRedHeads * kD), vx = 2 * p.H * kD + q * (kRedHeads * kD);
          const int y = N0(u) + j * kRedTile;
          mbar_arrive_expect_tx(&full[s], kRedStageBytes);
          tma_load_3d(st, &tmap_kv, &full[s], kx, y, b, pol);
          tma_load_3d(st + kRedBoxBytes, &tmap_kv, &full[s], kx + 64, y, b, pol);
          tma_load_3d(st + 2 * kRedBoxBytes, &tmap_kv, &full[s], vx, y, b, pol);
          tma_load_3d(st + 3 * kRedBoxBytes, &tmap_kv, &full[s], vx + 64, y, b, pol);
        } else {
          const int np = pair_heads_h(p.H, q, 1) > 0 ? 2 : 1;
          mbar_arrive_expect_tx(&full[s], np * kQBoxBytes);
          for (int h = 0; h < np; ++h)
            tma_load_3d(st + h * kQBoxBytes, &tmap_q, &full[s], q * kApUnitHeads * kD + h * kApHeads * kD,
                        (T0(u) + j) * kApTile, b, pol);
        }
        issued = i + 1;
        advance(u, j, ph2);
      }
      if (*abort_flag) {   // let this CTA's own loads land before it exits
        for (int i = (issued > R ? issued - R : 0); i < issued; ++i) {
          int s, use;
          slot(i, s, use);
          mbar_drain(&full[s], use & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_num = idesc_bf16_f32(128, 128, true, true);
      constexpr uint32_t idesc_den = idesc_bf16_f32(128, 16, true, false);
      constexpr uint32_t idesc_ap = idesc_bf16_f32(128, kImageRows, false, false);
      const uint64_t ones_desc = smem_desc(smem_u32(ones), 128, 256, kSwizzleNone);
      int u = 0, j = 0, pn = 0;
      bool ph2 = nP == 0, stop = false;
      for (int i = 0; i < nitems && !stop; ++i) {
        int s, use;
        slot(i, s, use);
        if (ph2 && j == 0 && !mbar_wait(&sfull[u], 0, abort_flag, err, kErrPairMma | 8 | u)) break;
        if (!mbar_wait(&mapped[s], use & 1, abort_flag, err, kErrPairMma | s)) break;
        tc_fence_after_sync();
        const uint32_t base = smem_u32(ring + s * kStageBytes);
        if (!ph2) {
          const uint32_t dacc = tmem + (u ? Cfg::kAcc1Col : 0u);
#pragma unroll
          for (int ks = 0; ks < kRedTile / 16; ++ks) {
            const uint64_t a = smem_desc(base + ks * 2048, kRedBoxBytes, 1024, kSwizzle128B);
            const uint64_t bv = smem_desc(base + 2 * kRedBoxBytes + ks * 2048, kRedBoxBytes, 1024, kSwizzle128B);
            const uint32_t acc = (j > 0 || ks > 0) ? 1u : 0u;
            umma_bf16(dacc, a, bv, idesc_num, acc);
            umma_bf16(dacc + 128, a, ones_desc, idesc_den, acc);
          }
          umma_commit(&empty[s]);
          if (j == P_(u) - 1) umma_commit(&done[u]);
        } else {
          const int q = u ? q1 : q0;
          const uint32_t saddr = smem_u32(u ? sbuf1 : sbuf);
          for (int h = 0; h < 2; ++h) {
            const int nh = pair_heads_h(p.H, q, h);
            if (nh == 0) break;
            const int a = pn % kApAccSlots;
            if (pn >= kApAccSlots &&
                !mbar_wait(&tempty[a], ((pn / kApAccSlots) - 1) & 1, abort_flag, err, kErrPairMma | 12 | a)) {
              stop = true;
              break;
            }
            // slot 2 lies over accumulator 1
            if (pn == 2 && !mbar_wait(acc1_free, 0, abort_flag, err, kErrPairMma | 11)) {
              stop = true;
              break;
            }
            tc_fence_after_sync();
            for (int jj = 0; jj < nh; ++jj) {
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                const uint64_t ad = smem_desc(base + h * kQBoxBytes + jj * 64 + ks * 32, 16, 1024, kSwizzle128B);
                const uint64_t bd =
                    smem_desc(saddr + (h * kApHeads + jj) * kImageBytes + ks * 256, 128, 512, kSwizzleNone);
                umma_bf16(tmem + a * kApAccCols + jj * kImageRows, ad, bd, idesc_ap, ks);
              }
            }
            umma_commit(&tfull[a]);
            ++pn;
          }
          if (stop) break;
          umma_commit(&empty[s]);
        }
        advance(u, j, ph2);
      }
      umma_commit(mma_idle);
    }
  } else if (warp < Cfg::kMergeWarp0) {
    // ------------------------------------------------------------------ ReLU of every stage
    const int t = threadIdx.x - 64;   // 0..127
    int u = 0, j = 0;
    bool ph2 = nP == 0;
    for (int i = 0; i < nitems; ++i) {
      int s, use;
      slot(i, s, use);
      if (!mbar_wait(&full[s], use & 1, abort_flag, err, kErrPairMap | s)) break;
      uint8_t* st = ring + s * kStageBytes;
      if (!ph2) {
        // k boxes in place; rows of tokens past the chunk are zeroed in k and v
        const int valid = min(kRedTile, N1(u) - (N0(u) + j * kRedTile));
#pragma unroll 4
        for (int c = t; c < 1024; c += 128) {
          uint4* w = reinterpret_cast<uint4*>(st + c * 16);
          const int row = (c >> 3) & (kRedTile - 1);
          *w = row < valid ? relu_bf16x8(*w) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (valid < kRedTile) {
          for (int c = t; c < 1024; c += 128) {
            const int row = (c >> 3) & (kRedTile - 1);
            if (row >= valid) *reinterpret_cast<uint4*>(st + 2 * kRedBoxBytes + c * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      } else {
        const int nchunks = (pair_heads_h(p.H, u ? q1 : q0, 1) > 0 ? 2 : 1) * (int)(kQBoxBytes / 16);
#pragma unroll 4
        for (int c = t; c < nchunks; c += 128) {
          uint4* w = reinterpret_cast<uint4*>(st + c * 16);
          *w = relu_bf16x8(*w);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&mapped[s]);
      advance(u, j, ph2);
    }
  } else if (warp < Cfg::kEpiWarp0) {
    // ------------------------------------------------------------------ read-out and merges
    const int hq = warp & 3;                           // TMEM lane quarter
    const int et = threadIdx.x - 32 * Cfg::kMergeWarp0;   // 0..127
    const bool leader = et == 0;
    constexpr int kUnits = kRedHeads * kRows * (kD / 8);   // (head, row, 8-column chunk)
    constexpr int kUPT = (kUnits + 127) / 128;
    int off[kUPT];   // the thread's units: float offsets in a partial
#pragma unroll
    for (int m = 0; m < kUPT; ++m) {
      const int un = et + m * 128;
      const int hl = un / (kRows * 4), rcc = un - hl * (kRows * 4);
      off[m] = hl * kStateFloats + (rcc >> 2) * kD + (rcc & 3) * 8;
    }
    bool ok = true;
    if (nu == 1 && leader) mbar_arrive(acc1_free);   // no second accumulator
    // the running sums (block-causal: unit 1 continues unit 0's prefix)
    float sum[kUPT][8];
#pragma unroll
    for (int m = 0; m < kUPT; ++m)
#pragma unroll
      for (int k = 0; k < 8; ++k) sum[m][k] = 0.f;
    for (int u = 0; u < nu; ++u) {
      const int c = u ? c1 : c0, b = u ? b1 : b0, q = u ? q1 : q0;
      const int blk = u ? blk1 : blk0;   // block-causal
      // (1) accumulator u -> this sibling's partial of quad c
      bool got = ok && P_(u) > 0;
      if (got) got = mbar_wait_long(&done[u], 0, abort_flag, err, kErrPairMerge | u);
      got = __all_sync(0xffffffffu, got);
      float sv[kRows];
      if (got) {
        tc_fence_after_sync();
        uint32_t rr[32], zr;
        const uint32_t ta = tmem + (static_cast<uint32_t>(hq * 32) << 16) + (u ? Cfg::kAcc1Col : 0u);
        tmem_ld_x32(ta + hq * 32, rr);
        tmem_ld_x1(ta + 128, zr);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) sv[k] = __uint_as_float(rr[k]);
        sv[32] = __uint_as_float(zr);
      } else {
#pragma unroll
        for (int k = 0; k < kRows; ++k) sv[k] = 0.f;
      }
      tc_fence_before_sync();
      // non-causal: partial r of quad c, [nq][S]; block-causal: the state of block blk, [nq][nblk]
      float* dst = partials + ((int64_t)c * (kCausal ? p.nblk : S) + (kCausal ? blk : r)) * kPartFloats +
                   hq * kStateFloats;
#pragma unroll
      for (int k = 0; k < kRows; ++k) dst[k * kD + lane] = sv[k];
      if (bar_any(3, 128, ok && P_(u) > 0 && !got)) ok = false;
      if (leader) {
        if (u == 1) mbar_arrive(acc1_free);
        // the arrival: the barrier orders the group's partial writes before the leader's fence,
        // which makes them visible at GPU scope before the count (one fence for the CTA: under
        // the streaming load a fence waits several microseconds for the stores to land)
        if (ok) {
          __threadfence();
          if (kCausal) atomicExch(&counters[c * p.nblk + blk], 1u);   // the block's flag
          else atomicAdd(&counters[c], 1u);
        }
      }
      // (2) wait for what this unit sums: non-causal, all S partials of quad c; block-causal,
      // the states of blocks [k0, k1) (unit 0: 0..r; unit 1: r + 1..r + S)
      const int k0 = kCausal && u ? r + 1 : 0;
      const int k1 = kCausal ? (u ? r + S + 1 : r + 1) : S;
      if (leader && ok) {
        const uint64_t tstart = globaltimer_ns();
        for (int w = (kCausal ? k0 : 0); ok && w < (kCausal ? k1 : 1); ++w) {
          volatile unsigned* arr = counters + (kCausal ? c * p.nblk + w : c);
          while (kCausal ? *arr == 0u : *arr < (unsigned)S) {
            if (*abort_flag) { ok = false; break; }
            if (globaltimer_ns() - tstart > kWaitLimitNs) {
              *abort_flag = 1;
              atomicCAS(err, 0, kErrPairSibling | u);
              ok = false;
              break;
            }
            __nanosleep(256);
          }
        }
        __threadfence();   // acquire: the siblings' partial writes precede their arrivals
      }
      if (bar_any(3, 128, !ok)) ok = false;
      if (!ok) break;
      // (3) the sum in fixed order: non-causal, partials 0..S-1; block-causal, block states
      // k0..k1-1 added to the running prefix
      if (!kCausal && u == 1) {
#pragma unroll
        for (int m = 0; m < kUPT; ++m)
#pragma unroll
          for (int k = 0; k < 8; ++k) sum[m][k] = 0.f;
      }
      const float* src = partials + ((int64_t)c * (kCausal ? p.nblk : S) + k0) * kPartFloats;
      for (int k = k0; k < k1; ++k, src += kPartFloats) {
        float4 x[kUPT][2];
#pragma unroll
        for (int m = 0; m < kUPT; ++m)
          if (et + m * 128 < kUnits) {
            const float4* a = reinterpret_cast<const float4*>(src + off[m]);
            x[m][0] = __ldcg(a);
            x[m][1] = __ldcg(a + 1);
          }
#pragma unroll
        for (int m = 0; m < kUPT; ++m)
          if (et + m * 128 < kUnits) {
            sum[m][0] += x[m][0].x; sum[m][1] += x[m][0].y; sum[m][2] += x[m][0].z; sum[m][3] += x[m][0].w;
            sum[m][4] += x[m][1].x; sum[m][5] += x[m][1].y; sum[m][6] += x[m][1].z; sum[m][7] += x[m][1].w;
          }
      }
      // (4) the image and the fp32 states (unit 1's image goes to the last ring stage, free once
      // accumulator 1 was complete: its MMAs were the last to read a reduction stage)
      uint8_t* ibuf = u ? sbuf1 : sbuf;
      const int heads = min(kApUnitHeads, p.H - q * kApUnitHeads);
#pragma unroll
      for (int m = 0; m < kUPT; ++m) {
        const int un = et + m * 128;
        if (un >= kUnits) break;
        const int hl = un / (kRows * 4), rcc = un - hl * (kRows * 4), rr = rcc >> 2, cc = rcc & 3;
        if (Q_(u) > 0) {
          float hi[8], lo[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float v = hl < heads ? sum[m][k] : 0.f;
            hi[k] = __bfloat162float(__float2bfloat16_rn(v));
            lo[k] = v - hi[k];
          }
          uint8_t* img = ibuf + hl * kImageBytes;
          *reinterpret_cast<uint4*>(img + image_offset(rr, cc * 8)) = pack_bf16x8(hi);
          *reinterpret_cast<uint4*>(img + image_offset(kImageLoRow + rr, cc * 8)) = pack_bf16x8(lo);
        }
        if (p.states != nullptr && (kCausal || r == 0) && hl < heads) {
          // the states the queries use, [B][H][nblk][33][32] (non-causal: nblk = 1)
          const int64_t st = ((int64_t)b * p.H + q * kApUnitHeads + hl) * (kCausal ? p.nblk : 1) + (kCausal ? blk : 0);
          float4* d4 = reinterpret_cast<float4*>(p.states + st * kStateFloats + rr * kD + cc * 8);
          d4[0] = make_float4(sum[m][0], sum[m][1], sum[m][2], sum[m][3]);
          d4[1] = make_float4(sum[m][4], sum[m][5], sum[m][6], sum[m][7]);
        }
      }
      if (Q_(u) > 0)
        for (int i = et; i < kRedHeads * 14 * 4; i += 128) {   // zero rows 33..39, 73..79
          const int hl = i / 56, k = i - hl * 56, zr = k >> 2, cc = k & 3;
          const int nrow = zr < 7 ? kRows + zr : kImageLoRow + kRows + (zr - 7);
          *reinterpret_cast<uint4*>(ibuf + hl * kImageBytes + image_offset(nrow, cc * 8)) = make_uint4(0u, 0u, 0u, 0u);
        }
      fence_proxy_async_smem();
      bar_sync(3, 128);
      if (leader) mbar_arrive(&sfull[u]);
    }
    // every CTA counts itself out once, after its last access to the arrival counters
    if (leader) {
      __threadfence();
      count_out();
    }
  } else {
    // ------------------------------------------------------------------ apply epilogue
    const int hq = warp & 3;
    const int et = threadIdx.x - 32 * Cfg::kEpiWarp0;   // 0..127
    const bool leader = et == 0;
    const int row = hq * 32 + lane;
    int pn = 0;
    bool ok = true;
    for (int u = 0; ok && u < nu; ++u) {
      const int b = u ? b1 : b0, q = u ? q1 : q0;
      const int np = pair_heads_h(p.H, q, 1) > 0 ? 2 : 1;
      for (int lu = 0; ok && lu < Q_(u); ++lu) {
        const int tok0 = (T0(u) + lu) * kApTile;   // the last tile is clipped to N by the TMA store
        for (int h = 0; h < np; ++h) {
          const int nh = pair_heads_h(p.H, q, h);
          const int a = pn % kApAccSlots;
          uint8_t* pbox = obuf + h * Cfg::kBoxesPerPair * kOutBoxBytes;
          // the pair's boxes were last stored one tile earlier: np - 1 stores were committed
          // after that one (all of them at a unit's first pair, where np may have changed)
          if (leader) {
            if (np == 2 && (lu > 0 || h > 0)) bulk_wait_group_read<1>();
            else bulk_wait_group_read<0>();
          }
          const bool okw = mbar_wait_long(&tfull[a], (pn / kApAccSlots) & 1, abort_flag, err, kErrPairEpi | a);
          if (bar_any(4, 128, !okw)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t ta = tmem + (static_cast<uint32_t>(hq * 32) << 16) + a * kApAccCols;
          for (int jj = 0; jj < nh; ++jj) {
            uint32_t v[kImageRows];
#pragma unroll
            for (int k = 0; k < kImageRows / 16; ++k) tmem_ld_x16(ta + jj * kImageRows + k * 16, v + k * 16);
            tmem_wait_ld();
            if (jj == nh - 1) {
              tc_fence_before_sync();
              mbar_arrive(&tempty[a]);
            }
            const float den = __uint_as_float(v[kD]) + __uint_as_float(v[kImageLoRow + kD]) + p.eps;
            const float inv = 1.0f / den;
            float o[kD];
#pragma unroll
            for (int k = 0; k < kD; ++k) o[k] = (__uint_as_float(v[k]) + __uint_as_float(v[kImageLoRow + k])) * inv;
            uint4 w[kChunksPerHead];
            pack_out(static_cast<OutT*>(nullptr), o, w);
#pragma unroll
            for (int k = 0; k < kChunksPerHead; ++k) {
              const int ck = jj * kChunksPerHead + k;   // 16-byte chunk within the pair's boxes
              uint8_t* box = pbox + (ck >> 3) * kOutBoxBytes;
              *reinterpret_cast<uint4*>(box + row * 128 + (((ck & 7) ^ (row & 7)) << 4)) = w[k];
            }
          }
          fence_proxy_async_smem();
          bar_sync(4, 128);
          if (leader) {
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxesPerPair; ++bx) {
              const int x = q * kApUnitHeads * kD + (h * Cfg::kBoxesPerPair + bx) * Cfg::kBoxChannels;
              if (x < p.H * kD) tma_store_3d(&tmap_out, pbox + bx * kOutBoxBytes, x, tok0, b);
            }
            bulk_commit_group();
          }
          ++pn;
        }
      }
    }
    if (leader) bulk_wait_group<0>();
  }

  leave(true);
}

}  // namespace litela
