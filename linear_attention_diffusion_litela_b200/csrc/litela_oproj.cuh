// LiteLA followed by the attention block's output projection, y = x W^T (+ b), with the apply
// computed in the projection GEMM's operand prologue, so the attention output x never goes to
// HBM (Sana explainer, "What LiteLA actually computes": LiteLA sits between the qkv projection
// and the output projection; "Two levers": the ledger's 4 N d^2 projection multiply-adds).
//
// litela_oproj_tc<kFused>   persistent, one CTA per SM, 512 threads.
//   Tile = 128 tokens of one batch x 224 output columns (C_out = 2240 is 10 tiles); the GEMM
//   accumulator D[128][224] (fp32) lives in TMEM.  K is stepped one head pair (64 input
//   channels) per pipeline stage, 4 stages of { A: 128 x 64 bf16, W: 224 x 64 bf16, the pair's
//   two state images }, all 128B-swizzled TMA boxes except the images (bulk copies).
//   kFused:  A starts as the q tile of the pair (TMA from the packed qkv); two ReLU warps clamp
//            it in place; one thread issues, per head, y = relu(q) . [S_hi ; S_lo]^T as four
//            tcgen05 MMAs (M = 128 tokens, N = 48, K = 16) that accumulate the hi and the lo
//            halves of the fp32 state into the same 48 columns (column r < 33 holds y[r]); an
//            epilogue warpgroup (two, alternating pairs) reads y, forms y[r] / (y[32] + eps),
//            rounds to bf16 and writes it over the q tile in the A layout; then the same thread
//            issues the GEMM step D += A . W^T (N = 224, K = 64).  The apply of pair p + 2 is
//            issued before the GEMM step of pair p, so the tensor pipe has the GEMM of one pair
//            to do while the epilogue prepares the next one's A.
//   plain:   A is loaded by TMA from a bf16 [B, N, C_in] input (the unfused chain's second step).
//   A third warpgroup drains the accumulator at the end of a tile (+ bias, bf16) straight to
//   global memory while the next tile's first pairs already load and apply.
// The state images are those litela_state_scan writes: per (batch, head, block) 80 rows x 32
// bf16 (rows 0..32 = S hi, rows 40..72 = S lo, the rest zero), K-major without swizzle.  Reading
// N = 48 rows from row 40 runs 8 rows past the lo half into the next image (or 512 bytes of
// padding after the last): those land in accumulator columns 40..47, which are never read.
// Every mbarrier wait is bounded (sm100::mbar_wait): on a time-out the kernel records an error
// code, stops its loops, waits (bounded) for its own copies, frees TMEM and returns.
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
constexpr int kOpThreads = 512;   // w0 TMA, w1 MMA, w2..3 ReLU, w4..7 / w8..11 apply epilogue, w12..15 output
constexpr uint32_t kOpABytes = kOpTileM * kOpK * 2;              // 16 KB
constexpr uint32_t kOpWBytes = kOpTileN * kOpK * 2;              // 28 KB
constexpr uint32_t kOpImgBytes = 2 * kImageBytes + 512;          // two images + the rows read past the last
constexpr int kOpApplyN = 48;                                    // accumulator columns per head
constexpr uint32_t kOpSlotCols = 2 * kOpApplyN;                  // one head pair
constexpr uint32_t kOpApplyCol0 = 256;                           // apply slots after the GEMM accumulator
constexpr uint32_t kOpTmemCols = 512;
constexpr uint32_t kOpSmemBytes = kOpStages * (kOpABytes + kOpWBytes + kOpImgBytes) + 512 + 1024;
static_assert(kOpApplyCol0 >= kOpTileN && kOpApplyCol0 + 2 * kOpSlotCols <= kOpTmemCols, "TMEM columns");
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(ibuf + kOpStages * kOpImgBytes);
  uint64_t* full = bars;                      // loads landed                       (tx)
  uint64_t* qrelu = full + kOpStages;         // ReLU of the q tile done            (64)
  uint64_t* aready = qrelu + kOpStages;       // the A tile is written              (128)
  uint64_t* empty = aready + kOpStages;       // the GEMM step read the stage       (commit)
  uint64_t* afull = empty + kOpStages;        // an apply slot holds y              (commit) x2
  uint64_t* aempty = afull + 2;               // an apply slot was read             (128) x2
  uint64_t* accfull = aempty + 2;             // the tile's accumulator is complete (commit)
  uint64_t* accempty = accfull + 1;           // the accumulator was read           (128)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert((4 * kOpStages + 6) * 8 + 8 <= 512, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&qrelu[s], 64);
      mbar_init(&aready[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&afull[g], 1);
      mbar_init(&aempty[g], 128);
    }
    mbar_init(accfull, 1);
    mbar_init(accempty, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the padding after each stage's second image is read by the lo product of the pair's second
  // head (columns that are never used); zero it once so that it holds finite values
  for (int i = threadIdx.x; i < kOpStages * 128; i += kOpThreads)
    reinterpret_cast<uint32_t*>(ibuf + (i >> 7) * kOpImgBytes + 2 * kImageBytes)[i & 127] = 0u;
  fence_proxy_async_smem();
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

  const long long t_first = blockIdx.x, t_step = gridDim.x;
  auto tile_of = [&](long long t, int& b, int& tok0, int& n0) {
    const int tn = (int)(t % p.ntn);
    const long long r = t / p.ntn;
    tok0 = (int)(r % p.ntt) * kOpTileM;
    b = (int)(r / p.ntt);
    n0 = tn * kOpTileN;
  };
  // heads of K step k (fused): 2, or 1 for the last step when H is odd
  auto step_heads = [&](int k) { return min(2, p.H - 2 * k); };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long gp = 0;   // pipeline steps issued by this CTA
      bool stop = false;
      for (long long t = t_first; t < p.ntiles && !stop; t += t_step) {
        int b, tok0, n0;
        tile_of(t, b, tok0, n0);
        const int blk = kFused ? tok0 / p.T : 0;
        for (int k = 0; k < p.nsteps; ++k, ++gp) {
          const int s = (int)(gp % kOpStages);
          if (gp >= kOpStages &&
              !mbar_wait(&empty[s], (uint32_t)((gp / kOpStages) - 1) & 1, abort_flag, err, kErrOpProducer | s)) {
            stop = true;
            break;
          }
          const int nh = kFused ? step_heads(k) : 0;
          mbar_arrive_expect_tx(&full[s], kOpABytes + kOpWBytes + nh * kImageBytes);
          // fused: the q columns of heads 2k, 2k + 1 (a lone last head's box also covers the
          // first k columns, which are never used); plain: input channels 64k ..
          tma_load_3d(abuf + s * kOpABytes, &tmap_a, &full[s], k * kOpK, tok0, b);
          tma_load_2d(wbuf + s * kOpWBytes, &tmap_w, &full[s], k * kOpK, n0);
          for (int j = 0; j < nh; ++j) {
            const int h = 2 * k + j;
            bulk_load(ibuf + s * kOpImgBytes + j * kImageBytes,
                      images + (((int64_t)b * p.H + h) * p.nblk + blk) * kImageBytes, kImageBytes, &full[s]);
          }
        }
      }
      if (*abort_flag) {   // let this CTA's own copies land before it leaves
        for (long long i = (gp > kOpStages ? gp - kOpStages : 0); i < gp; ++i)
          mbar_drain(&full[i % kOpStages], (uint32_t)(i / kOpStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_gemm = idesc_bf16_f32(kOpTileM, kOpTileN, false, false);
      constexpr uint32_t idesc_apply = idesc_bf16_f32(kOpTileM, kOpApplyN, false, false);
      long long gp = 0;        // steps of this CTA (stage ring position)
      long long slot_uses[2] = {0, 0};
      long long tiles_done = 0;
      bool stop = false;
      // the GEMM step of pipeline step `g` (stage g % kOpStages), K step k of its tile
      auto gemm_step = [&](long long g, int k) -> bool {
        const int s = (int)(g % kOpStages);
        // the tile's first step overwrites the accumulator: the previous tile's must be read
        if (k == 0 && tiles_done > 0 &&
            !mbar_wait(accempty, (uint32_t)(tiles_done - 1) & 1, abort_flag, err, kErrOpMma | 12))
          return false;
        if (kFused) {
          if (!mbar_wait(&aready[s], (uint32_t)(g / kOpStages) & 1, abort_flag, err, kErrOpMma | 4 | s)) return false;
        } else {
          if (!mbar_wait(&full[s], (uint32_t)(g / kOpStages) & 1, abort_flag, err, kErrOpMma | 8 | s)) return false;
        }
        tc_fence_after_sync();
        const uint32_t a0 = smem_u32(abuf + s * kOpABytes), w0 = smem_u32(wbuf + s * kOpWBytes);
#pragma unroll
        for (int ks = 0; ks < kOpK / 16; ++ks) {
          const uint64_t ad = smem_desc(a0 + ks * 32, 16, 1024, kSwizzle128B);
          const uint64_t wd = smem_desc(w0 + ks * 32, 16, 1024, kSwizzle128B);
          umma_bf16(tmem, ad, wd, idesc_gemm, (k > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        return true;
      };
      for (long long t = t_first; t < p.ntiles && !stop; t += t_step, ++tiles_done) {
        const long long g0 = gp;
        if (kFused) {
          for (int k = 0; k < p.nsteps; ++k, ++gp) {
            const int s = (int)(gp % kOpStages), slot = k & 1;
            if (!mbar_wait(&qrelu[s], (uint32_t)(gp / kOpStages) & 1, abort_flag, err, kErrOpMma | s)) {
              stop = true;
              break;
            }
            if (slot_uses[slot] > 0 &&
                !mbar_wait(&aempty[slot], (uint32_t)(slot_uses[slot] - 1) & 1, abort_flag, err, kErrOpMma | 13 | slot << 1)) {
              stop = true;
              break;
            }
            tc_fence_after_sync();
            const uint32_t q0 = smem_u32(abuf + s * kOpABytes), i0 = smem_u32(ibuf + s * kOpImgBytes);
            const int nh = step_heads(k);
            for (int j = 0; j < nh; ++j) {
              const uint32_t dacc = tmem + kOpApplyCol0 + slot * kOpSlotCols + j * kOpApplyN;
#pragma unroll
              for (int half = 0; half < 2; ++half) {     // S hi (rows 0..), then S lo (rows 40..)
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                  const uint64_t ad = smem_desc(q0 + j * 64 + ks * 32, 16, 1024, kSwizzle128B);
                  const uint64_t bd = smem_desc(i0 + j * kImageBytes + half * (kImageLoRow / 8) * 512 + ks * 256, 128,
                                                512, kSwizzleNone);
                  umma_bf16(dacc, ad, bd, idesc_apply, (half > 0 || ks > 0) ? 1u : 0u);
                }
              }
            }
            umma_commit(&afull[slot]);
            ++slot_uses[slot];
            // the GEMM step two K steps back (its A was prepared meanwhile)
            if (k >= 2 && !gemm_step(gp - 2, k - 2)) {
              stop = true;
              break;
            }
          }
          if (stop) break;
          for (int k = max(0, p.nsteps - 2); k < p.nsteps; ++k)
            if (!gemm_step(g0 + k, k)) {
              stop = true;
              break;
            }
          if (stop) break;
        } else {
          for (int k = 0; k < p.nsteps; ++k, ++gp)
            if (!gemm_step(gp, k)) {
              stop = true;
              break;
            }
          if (stop) break;
        }
        umma_commit(accfull);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ ReLU of q (fused)
    if (kFused) {
      const int t = threadIdx.x - 64;
      long long gp = 0;
      bool stop = false;
      for (long long tt = t_first; tt < p.ntiles && !stop; tt += t_step) {
        for (int k = 0; k < p.nsteps; ++k, ++gp) {
          const int s = (int)(gp % kOpStages);
          if (!mbar_wait(&full[s], (uint32_t)(gp / kOpStages) & 1, abort_flag, err, kErrOpRelu | s)) {
            stop = true;
            break;
          }
          uint8_t* st = abuf + s * kOpABytes;
#pragma unroll 4
          for (int j = t; j < (int)(kOpABytes / 16); j += 64) {
            uint4* c = reinterpret_cast<uint4*>(st + j * 16);
            *c = relu_bf16x8(*c);
          }
          fence_proxy_async_smem();
          mbar_arrive(&qrelu[s]);
        }
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------------ apply epilogue (fused)
    if (kFused) {
      const int g = (warp - 4) >> 2;                      // warpgroup: K steps k with k % 2 == g
      const int row = (warp & 3) * 32 + lane;             // token row of the tile = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      long long gp = 0, uses = 0;
      bool stop = false;
      for (long long t = t_first; t < p.ntiles && !stop; t += t_step) {
        for (int k = 0; k < p.nsteps; ++k, ++gp) {
          if ((k & 1) != g) continue;
          const int s = (int)(gp % kOpStages);
          const bool ok = mbar_wait(&afull[g], (uint32_t)uses & 1, abort_flag, err, kErrOpApply | g);
          if (bar_any(3 + g, 128, !ok)) {
            stop = true;
            break;
          }
          ++uses;
          tc_fence_after_sync();
          const int nh = step_heads(k);
          uint32_t y[2][33];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j < nh) {
              const uint32_t ta = tmem + lane_base + kOpApplyCol0 + g * kOpSlotCols + j * kOpApplyN;
              tmem_ld_x32(ta, y[j]);
              tmem_ld_x1(ta + 32, y[j][32]);
            }
          }
          tmem_wait_ld();
          tc_fence_before_sync();
          mbar_arrive(&aempty[g]);
          uint8_t* a = abuf + s * kOpABytes + row * 128;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint4 w[4];
            if (j < nh) {
              const float inv = 1.0f / (__uint_as_float(y[j][32]) + p.eps);
              float o[kD];
#pragma unroll
              for (int c = 0; c < kD; ++c) o[c] = __uint_as_float(y[j][c]) * inv;
              pack_out(static_cast<__nv_bfloat16*>(nullptr), o, w);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(a + ((((j * 4 + i) & 7) ^ (row & 7)) << 4)) = w[i];
          }
          fence_proxy_async_smem();
          mbar_arrive(&aready[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ output: D (+ bias) -> bf16
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    long long tiles_done = 0;
    for (long long t = t_first; t < p.ntiles; t += t_step, ++tiles_done) {
      int b, tok0, n0;
      tile_of(t, b, tok0, n0);
      const bool ok = mbar_wait(accfull, (uint32_t)tiles_done & 1, abort_flag, err, kErrOpOut);
      if (bar_any(5, 128, !ok)) break;
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
          for (int c = 0; c < 32; ++c) {
            const int n = n0 + c0 + c;
            o[c] = __uint_as_float(v[c]) + ((bias != nullptr && n < p.C_out) ? bias[n] : 0.f);
          }
          uint4 w[4];
          pack_out(static_cast<__nv_bfloat16*>(nullptr), o, w);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (n0 + c0 + 8 * i < p.C_out) *reinterpret_cast<uint4*>(dst + c0 + 8 * i) = w[i];
        }
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
