// LiteLA followed by the attention block's output projection, y = x W^T (+ b), with the apply
// computed in the projection GEMM's operand prologue, so the attention output x never goes to
// HBM (Sana explainer, "What LiteLA actually computes": LiteLA sits between the qkv projection
// and the output projection; "Two levers": the ledger's 4 N d^2 projection multiply-adds).
//
// litela_oproj_tc<kFused>   persistent, one CTA per SM, 448 threads.
//   Tile = 128 tokens of one batch x 224 output columns (C_out = 2240 is 10 tiles); the GEMM
//   accumulator D[128][224] (fp32) lives in TMEM.  K is stepped one head pair (64 input
//   channels) per pipeline stage; a 4-stage ring holds { q (or A): 128 x 64 bf16, W: 224 x 64
//   bf16, the pair's two state images }: TMA boxes with 128B swizzle, bulk copies for images.
//   kFused: the intermediate operands never touch shared memory again after the loads:
//     - four ReLU warps (thread = token row) read the row's q from the stage, clamp it and
//       store it into a TMEM slot (two 32-column slots, alternating K steps);
//     - one thread issues, per head, y = relu(q) . [S_hi ; S_lo]^T as two tcgen05 MMAs with A in
//       TMEM (M = 128 tokens, N = 80 image rows, K = 16): columns r and 40 + r hold the products
//       with the hi and the lo halves of state row r (the tensor core pays per instruction, so
//       few wide products beat more narrow ones);
//     - an epilogue warpgroup (two, alternating K steps) reads them, forms (hi + lo)[r] /
//       ((hi + lo)[32] + eps) as the forward's apply does, rounds to bf16 and stores it with
//       tcgen05.st into an A slot: that is the GEMM's A operand;
//     - the same thread issues, in order, the GEMM step D += A . W^T of step G (A in TMEM, W
//       from shared memory, N = 224, K = 64) and then the apply of step G + 2, so that the
//       applies run two steps ahead of the GEMM.
//   plain: A is loaded by TMA from a bf16 [B, N, C_in] input into the stage and read from there
//   (the unfused chain's second step).
//   The ReLU warps also drain the accumulator at the end of a tile (+ bias, staged in shared
//   memory once per tile; bf16) straight to global memory while the next tile's first steps
//   already load and apply.
// Tensor memory: D 224 columns, one apply slot of 160 (2 heads x 80), 2 relu(q) slots and 2 A
// slots of 32 (64 bf16 per lane) = 512.  Shared memory: 4 x 54 KB of stages, the tile's bias,
// barriers.
// The state images are those litela_state_scan writes: per (batch, head, block) 80 rows x 32
// bf16 (rows 0..32 = S hi, rows 40..72 = S lo, the rest zero), K-major without swizzle.
// Every mbarrier wait is bounded (sm100::mbar_wait, or a polling loop with the same limit): on a
// time-out the kernel records an error code, stops its loops, waits (bounded) for its own
// copies, frees TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "litela_plan.h"
#include "litela_tc.cuh"
#include "sm100_ptx.cuh"

namespace litela {

struct OprojPlan {
  int B, N, H;          // batch, tokens, heads (kFused); H = 0 for the plain GEMM
  int C_in, C_out;      // input width (H * 32 when fused) and output width
  int T, nblk;          // causal block size (N when non-causal) and number of blocks (kFused)
  int ntn, ntt;         // output-column tiles, token tiles per batch
  int nsteps;           // K steps of 64 channels: ceil(C_in / 64)
  long long ntiles;     // B * ntt * ntn
  float eps;
};

enum : int { kErrOpProducer = 0x710, kErrOpMma = 0x720, kErrOpRelu = 0x730, kErrOpApply = 0x740, kErrOpOut = 0x750 };

constexpr int kOpTileM = 128;
constexpr int kOpTileN = 224;
constexpr int kOpK = 64;                                        // channels per stage (a head pair)
constexpr int kOpStages = 4;
constexpr int kOpThreads = 448;   // w0 TMA, w1 MMA, w2..5 ReLU + output, w6..9 / w10..13 apply epilogue
constexpr uint32_t kOpABytes = kOpTileM * kOpK * 2;              // 16 KB
constexpr uint32_t kOpWBytes = kOpTileN * kOpK * 2;              // 28 KB
constexpr uint32_t kOpImgBytes = 2 * kImageBytes;                // the pair's two state images
constexpr int kOpApplyN = kImageRows;                            // accumulator columns per head (hi | lo)
constexpr uint32_t kOpSlotCols = 2 * kOpApplyN;                  // one head pair
constexpr uint32_t kOpApplyCol0 = kOpTileN;                      // the apply slot after the GEMM accumulator
constexpr uint32_t kOpQCol0 = kOpApplyCol0 + kOpSlotCols;        // 2 relu(q) slots of 32 columns
constexpr uint32_t kOpACol0 = kOpQCol0 + 2 * 32;                 // 2 A slots of 32 columns
constexpr uint32_t kOpTmemCols = 512;
constexpr uint32_t kOpBiasBytes = 1024;
constexpr uint32_t kOpSmemBytes = kOpStages * (kOpABytes + kOpWBytes + kOpImgBytes) + kOpBiasBytes + 512 + 1024;
static_assert(kOpACol0 + 2 * 32 <= kOpTmemCols, "TMEM columns");
static_assert(kOpTileN * 4 <= kOpBiasBytes, "bias slice");
static_assert(kOpSmemBytes <= 232448, "shared memory");

template <bool kFused>
__global__ void __launch_bounds__(kOpThreads, 1)
litela_oproj_tc(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                const uint8_t* __restrict__ images, const float* __restrict__ bias,
                __nv_bfloat16* __restrict__ out, int* __restrict__ err, OprojPlan p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* abuf = smem;                                           // [kOpStages][16 KB]
  uint8_t* wbuf = abuf + kOpStages * kOpABytes;                   // [kOpStages][28 KB]
  uint8_t* ibuf = wbuf + kOpStages * kOpWBytes;                   // [kOpStages][10.5 KB]
  float* bias_s = reinterpret_cast<float*>(ibuf + kOpStages * kOpImgBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(bias_s) + kOpBiasBytes);
  uint64_t* full = bars;                      // the stage's loads landed                  (tx)
  uint64_t* empty = full + kOpStages;         // the GEMM step read the stage              (commit)
  uint64_t* qtm = empty + kOpStages;          // relu(q) is in its TMEM slot               (128) x2
  uint64_t* qfree = qtm + 2;                  // the apply read the relu(q) slot           (commit) x2
  uint64_t* afull = qfree + 2;                // the apply slot holds y, steps G % 2 == i  (commit) x2
  uint64_t* aempty = afull + 2;               // the epilogue read y                       (128)
  uint64_t* aready = aempty + 1;              // A is in its TMEM slot                     (128) x2
  uint64_t* afree = aready + 2;               // the GEMM step read the A slot             (commit) x2
  uint64_t* accfull = afree + 2;              // the tile's accumulator is complete        (commit)
  uint64_t* accempty = accfull + 1;           // the accumulator was read                  (128)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert((2 * kOpStages + 11 + 2) * 8 + 8 <= 512, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the TMEM lanes a warp may access: 32 * (warp % 4) ..; thread = token row of the tile
  const int row = (warp & 3) * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qtm[s], 128);
      mbar_init(&qfree[s], 1);
      mbar_init(&aready[s], 128);
      mbar_init(&afree[s], 1);
      mbar_init(&afull[s], 1);   // one per epilogue warpgroup: each waits parity 0 first
    }
    mbar_init(aempty, 128);
    mbar_init(accfull, 1);
    mbar_init(accempty, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kOpTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_w);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait_primary();   // every input may come from the previous kernels in the stream

  // This CTA's tiles are t = blockIdx.x + i * gridDim.x; its K steps G = i * nsteps + k run
  // through the stage ring and the TMEM slots in order.  Every role walks them with running
  // counters (a StepIter): no 64-bit division per step.
  const int ntl = p.ntiles > (long long)blockIdx.x ? (int)((p.ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
  struct StepIter {
    int i = 0, k = 0;              // tile of this CTA, K step within it
    long long G = 0;               // step counter
    int b = 0, tok0 = 0, n0 = 0;   // the tile's batch, first token, first output column
    int tn = 0, tt = 0;            // its column tile and token tile
  };
  // position of this CTA's first tile
  auto first_step = [&](StepIter& it) {
    const long long t = blockIdx.x;
    it.tn = (int)(t % p.ntn);
    const long long r = t / p.ntn;
    it.tt = (int)(r % p.ntt);
    it.b = (int)(r / p.ntt);
    it.tok0 = it.tt * kOpTileM;
    it.n0 = it.tn * kOpTileN;
  };
  // advance by one K step; moving to the next tile advances (tn, tt, b) by gridDim.x tiles
  const int dtn = (int)(gridDim.x % p.ntn), dr = (int)(gridDim.x / p.ntn);
  const int dtt = dr % p.ntt, db = dr / p.ntt;
  auto next_step = [&](StepIter& it) {
    ++it.G;
    if (++it.k < p.nsteps) return;
    it.k = 0;
    ++it.i;
    it.tn += dtn;
    int carry = 0;
    if (it.tn >= p.ntn) { it.tn -= p.ntn; carry = 1; }
    it.tt += dtt + carry;
    carry = 0;
    if (it.tt >= p.ntt) { it.tt -= p.ntt; carry = 1; }
    it.b += db + carry;
    it.tok0 = it.tt * kOpTileM;
    it.n0 = it.tn * kOpTileN;
  };
  // heads of K step k (fused): 2, or 1 for the last step when H is odd
  auto step_heads = [&](int k) { return min(2, p.H - 2 * k); };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      StepIter it;
      first_step(it);
      for (; it.i < ntl; next_step(it)) {
        const int s = (int)(it.G % kOpStages);
        if (it.G >= kOpStages &&
            !mbar_wait(&empty[s], (uint32_t)((it.G / kOpStages) - 1) & 1, abort_flag, err, kErrOpProducer | s))
          break;
        const int nh = kFused ? step_heads(it.k) : 0;
        mbar_arrive_expect_tx(&full[s], kOpABytes + kOpWBytes + nh * kImageBytes);
        // fused: the q columns of heads 2k, 2k + 1 (a lone last head's box also covers the first
        // k columns, which are never used); plain: input channels 64k ..
        tma_load_3d(abuf + s * kOpABytes, &tmap_a, &full[s], it.k * kOpK, it.tok0, it.b);
        tma_load_2d(wbuf + s * kOpWBytes, &tmap_w, &full[s], it.k * kOpK, it.n0);
        if (kFused) {
          const int blk = it.tok0 / p.T;
          for (int j = 0; j < nh; ++j)
            bulk_load(ibuf + s * kOpImgBytes + j * kImageBytes,
                      images + (((int64_t)it.b * p.H + 2 * it.k + j) * p.nblk + blk) * kImageBytes, kImageBytes,
                      &full[s]);
        }
      }
      if (*abort_flag) {   // let this CTA's own copies land before it leaves
        for (long long i = (it.G > kOpStages ? it.G - kOpStages : 0); i < it.G; ++i)
          mbar_drain(&full[i % kOpStages], (uint32_t)(i / kOpStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // In order, per step G: (fused) the apply of step G + 1, once relu(q) of that step is in
    // TMEM and the epilogue has read the apply slot's previous y; then the GEMM step G, once its
    // A operand (and, for a tile's first step, the drained accumulator) is there.  So the
    // epilogue of step G + 1 runs while the tensor core works on GEMM step G.
    if (lane == 0) {
      constexpr uint32_t idesc_gemm = idesc_bf16_f32(kOpTileM, kOpTileN, false, false);
      constexpr uint32_t idesc_apply = idesc_bf16_f32(kOpTileM, kOpApplyN, false, false);
      auto apply = [&](const StepIter& a) -> bool {
        if (!mbar_wait(&qtm[a.G & 1], (uint32_t)(a.G >> 1) & 1, abort_flag, err, kErrOpMma | 1)) return false;
        if (a.G > 0 && !mbar_wait(aempty, (uint32_t)(a.G - 1) & 1, abort_flag, err, kErrOpMma | 5)) return false;
        tc_fence_after_sync();
        const uint32_t i0 = smem_u32(ibuf + (int)(a.G % kOpStages) * kOpImgBytes);
        const uint32_t qa = tmem + kOpQCol0 + (uint32_t)(a.G & 1) * 32;
        const int nh = step_heads(a.k);
        for (int j = 0; j < nh; ++j) {
          // y = relu(q) . [S_hi ; S_lo]^T: columns r = S_hi row r, 40 + r = S_lo row r
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t bd = smem_desc(i0 + j * kImageBytes + ks * 256, 128, 512, kSwizzleNone);
            umma_bf16_ts(tmem + kOpApplyCol0 + j * kOpApplyN, qa + j * 16 + ks * 8, bd, idesc_apply, ks);
          }
        }
        umma_commit(&afull[a.G & 1]);
        umma_commit(&qfree[a.G & 1]);
        return true;
      };
      StepIter g, a;
      first_step(g);
      first_step(a);
      bool ok = true;
      if (kFused && a.i < ntl) {
        ok = apply(a);
        next_step(a);
      }
      for (; g.i < ntl && ok; next_step(g)) {
        if (kFused && a.i < ntl) {
          if (!(ok = apply(a))) break;
          next_step(a);
        }
        const int s = (int)(g.G % kOpStages);
        ok = kFused ? mbar_wait(&aready[g.G & 1], (uint32_t)(g.G >> 1) & 1, abort_flag, err, kErrOpMma | 2)
                    : mbar_wait(&full[s], (uint32_t)(g.G / kOpStages) & 1, abort_flag, err, kErrOpMma | 3);
        if (ok && g.k == 0 && g.i > 0) ok = mbar_wait(accempty, (uint32_t)(g.i - 1) & 1, abort_flag, err, kErrOpMma | 4);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t w0 = smem_u32(wbuf + s * kOpWBytes);
#pragma unroll
        for (int ks = 0; ks < kOpK / 16; ++ks) {
          const uint64_t wd = smem_desc(w0 + ks * 32, 16, 1024, kSwizzle128B);
          const uint32_t acc = (g.k > 0 || ks > 0) ? 1u : 0u;
          if (kFused)
            umma_bf16_ts(tmem, tmem + kOpACol0 + (uint32_t)(g.G & 1) * 32 + ks * 8, wd, idesc_gemm, acc);
          else
            umma_bf16(tmem, smem_desc(smem_u32(abuf + s * kOpABytes) + ks * 32, 16, 1024, kSwizzle128B), wd,
                      idesc_gemm, acc);
        }
        umma_commit(&empty[s]);
        if (kFused) umma_commit(&afree[g.G & 1]);
        if (g.k == p.nsteps - 1) umma_commit(accfull);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ ReLU(q) -> TMEM, output
    // (fused) relu(q) of every step into its TMEM slot.  At the end of every tile these warps
    // also drain the accumulator (+ bias, bf16) to global memory: right after the next tile's
    // first relu(q) (the MMA issues that step's apply before the tile's last GEMM step) or after
    // the last step.
    const int ot = threadIdx.x - 2 * 32;   // 0..127
    auto drain = [&](int i, int b, int tok0, int n0) -> bool {
      bar_sync(5, 128);   // the previous tile's bias slice is no longer read
      for (int c = ot; c < kOpTileN; c += 128)
        bias_s[c] = (bias != nullptr && n0 + c < p.C_out) ? bias[n0 + c] : 0.f;
      bar_sync(5, 128);
      const bool ok = mbar_wait(accfull, (uint32_t)i & 1, abort_flag, err, kErrOpOut);
      if (bar_any(5, 128, !ok)) return false;
      tc_fence_after_sync();
      const int tok = tok0 + row;
      __nv_bfloat16* dst = out + ((int64_t)b * p.N + tok) * p.C_out + n0;
#pragma unroll 1
      for (int c0 = 0; c0 < kOpTileN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_base + c0, v);
        tmem_wait_ld();
        if (c0 + 32 >= kOpTileN) {   // every column read: the MMA may start the next tile
          tc_fence_before_sync();
          mbar_arrive(accempty);
        }
        if (tok < p.N) {
          float o[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(v[c]) + bias_s[c0 + c];
          uint4 w[4];
          pack_out(static_cast<__nv_bfloat16*>(nullptr), o, w);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (n0 + c0 + 8 * j < p.C_out) *reinterpret_cast<uint4*>(dst + c0 + 8 * j) = w[j];
        }
      }
      return true;
    };
    StepIter it;
    first_step(it);
    int pb = it.b, ptok = it.tok0, pn = it.n0;   // the tile whose accumulator is drained next
    bool ok = true;
    for (; it.i < ntl; next_step(it)) {
      if (kFused) {
        const int s = (int)(it.G % kOpStages), slot = (int)(it.G & 1);
        ok = mbar_wait(&full[s], (uint32_t)(it.G / kOpStages) & 1, abort_flag, err, kErrOpRelu | s);
        // the slot's previous relu(q) has been read by its apply
        if (ok && it.G >= 2)
          ok = mbar_wait(&qfree[slot], (uint32_t)((it.G >> 1) - 1) & 1, abort_flag, err, kErrOpRelu | 8);
        if (bar_any(5, 128, !ok)) break;
        const uint8_t* q = abuf + s * kOpABytes + row * 128;
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = relu_bf16x8(*reinterpret_cast<const uint4*>(q + ((c ^ (row & 7)) << 4)));
          v[4 * c] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + lane_base + kOpQCol0 + slot * 32;
        tmem_st_x16(ta, v);
        tmem_st_x16(ta + 16, v + 16);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&qtm[slot]);
      }
      // the first step of tile i > 0 is prepared: drain tile i - 1
      if (it.k == 0 && it.i > 0) {
        if (!(ok = drain(it.i - 1, pb, ptok, pn))) break;
        pb = it.b; ptok = it.tok0; pn = it.n0;
      }
    }
    if (ok && ntl > 0) drain(ntl - 1, pb, ptok, pn);
  } else if (warp < 14) {
    // ------------------------------------------------------------------ apply epilogue (fused)
    if (kFused) {
      const int g = (warp - 6) >> 2;                      // warpgroup: steps G with G % 2 == g
      StepIter it;
      first_step(it);
      if (g == 1) next_step(it);
      for (; it.i < ntl; next_step(it), next_step(it)) {
        bool ok = mbar_wait(&afull[g], (uint32_t)(it.G >> 1) & 1, abort_flag, err, kErrOpApply | g);
        if (bar_any(3 + g, 128, !ok)) break;
        tc_fence_after_sync();
        const int nh = step_heads(it.k);
        // A = (y_hi + y_lo)[r] / ((y_hi + y_lo)[32] + eps) in bf16, the forward apply's arithmetic
        uint32_t w[2][16];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j < nh) {
            uint32_t v[kImageRows];
            const uint32_t ya = tmem + lane_base + kOpApplyCol0 + j * kOpApplyN;
            tmem_ld_x32(ya, v);
            tmem_ld_x1(ya + kD, v[kD]);
            tmem_ld_x32(ya + kImageLoRow, v + kImageLoRow);
            tmem_ld_x1(ya + kImageLoRow + kD, v[kImageLoRow + kD]);
            tmem_wait_ld();
            if (j == nh - 1) {   // the apply slot may take the next step's y
              tc_fence_before_sync();
              mbar_arrive(aempty);
            }
            const float den = (__uint_as_float(v[kD]) + __uint_as_float(v[kImageLoRow + kD])) + p.eps;
            const float inv = 1.0f / den;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              __nv_bfloat162 v2 = __floats2bfloat162_rn(
                  (__uint_as_float(v[2 * c]) + __uint_as_float(v[kImageLoRow + 2 * c])) * inv,
                  (__uint_as_float(v[2 * c + 1]) + __uint_as_float(v[kImageLoRow + 2 * c + 1])) * inv);
              w[j][c] = *reinterpret_cast<uint32_t*>(&v2);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) w[j][c] = 0u;
          }
        }
        // A goes into the step's A slot once its GEMM step G - 2 is done
        ok = it.G < 2 || mbar_wait(&afree[g], (uint32_t)((it.G >> 1) - 1) & 1, abort_flag, err, kErrOpApply | 4 | g);
        if (bar_any(3 + g, 128, !ok)) break;
        tc_fence_after_sync();
        const uint32_t ta = tmem + lane_base + kOpACol0 + g * 32;
        tmem_st_x16(ta, w[0]);
        tmem_st_x16(ta + 16, w[1]);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&aready[g]);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kOpTmemCols);
  }
}

}  // namespace litela
