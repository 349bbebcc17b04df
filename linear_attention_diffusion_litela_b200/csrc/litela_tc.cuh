// LiteLA forward on the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA staging).
//
// Method (Sana explainer "Sana: the autoencoder does more of the work than the linear
// attention", section "What LiteLA actually computes"): phi = ReLU on q and k, V padded with a
// row of ones, state S = [V;1] . phi(K)^T (a (d+1) x d fp32 matrix per batch and head),
// y = S . phi(q), out = y[:d] / (y[d] + eps).  Block-causal variant (instagit page "How Linear
// Attention Improves Efficiency in DiT for High-Resolution Images", section "Video Generation
// and Constant-Memory KV Cache"): a query in block b uses the sum of the per-block states of
// blocks 0..b.
//
// litela_reduce_tc  (one CTA = 4 heads x one chunk of tokens inside one causal block)
//   TMA streams the chunk's k and v columns of the 4 heads (64 tokens x 128 channels each, 128B
//   swizzle) through a 3-stage ring.  Four ReLU warps clamp k in shared memory (and zero the
//   rows of tokens outside the chunk).  One thread issues, per 16 tokens,
//     D[0:128, 0:128]   += phi(K)^T . V     (M = 4 heads x 32 key channels, N = 4 x 32 values)
//     D[0:128, 128:144] += phi(K)^T . 1     (the ones pad: the denominator row)
//   with fp32 accumulators in TMEM; only the 4 diagonal 32 x 32 blocks of the first product
//   are used (the off-diagonal blocks pair different heads and are discarded: the tensor core
//   has 30x more throughput than this HBM-bound pass needs).  Products of bf16 values are exact
//   in fp32, so this is the fp32 state the method specifies.  The epilogue writes the chunk's
//   partial states [4][33][32] to the workspace; nothing else (no atomics, no merge tail).
//
// litela_state_scan  sums the partial states in fixed order into per-block prefix states.
//
// The kernels of a call, and consecutive calls, are chained with programmatic dependent launch:
// each kernel starts its private set-up while its predecessor drains and waits for it
// (griddepcontrol.wait) before touching global memory that the predecessor may still use.
//
// litela_apply_tc  (persistent, one CTA per SM; work unit = 4 heads x 128 tokens of a block)
//   Units span 4 heads so that every q row read and every output row written is a 256-byte
//   run: on B200, 128-byte runs at these row strides reach only about half the HBM bandwidth.
//   The producer bulk-copies each segment's state images (litela_state_scan's output: the
//   MMA's B operand, S split into bf16 hi + lo) into shared memory and streams q tiles
//   (128 tokens x 128 channels as two 128B-swizzled boxes) through a ring with TMA; two ReLU
//   warps clamp them in place; one thread issues
//   y = phi(Q) . [S_hi ; S_lo]^T per head (M = 128 tokens, N = 80, K = 32), one head pair at a
//   time into one of three TMEM accumulator slots; four epilogue warps read them back
//   (thread = token), form (y_hi + y_lo)[r] / ((y_hi + y_lo)[32] + eps), stage the unit's
//   output tile in shared memory and store it with TMA (partial tiles inside a causal block
//   are stored row by row).  The kernel is launched as a programmatic dependent of the scan:
//   its set-up and first q loads overlap the end of the preceding grids.
//
// Every mbarrier wait is bounded (sm100::mbar_wait): on a time-out the kernel records an
// error code in the workspace's error word, stops its loops, waits (bounded) for its own TMA
// copies, frees its TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "litela_plan.h"
#include "sm100_ptx.cuh"

namespace litela {

struct TcPlan {
  int B, N, H, T, nblk, ngroups, cpb, chunk, nquads, tpb;
  long long units;
  float eps;
  int bpc;   // consecutive blocks per reduction CTA (> 1 only with cpb == 1)
};

// error codes written to the workspace error word: 0x100 | role << 4 | stage
enum : int {
  kErrReduceProducer = 0x110, kErrReduceMma = 0x120, kErrReduceRelu = 0x130, kErrReduceEpi = 0x140,
  kErrApplyProducer = 0x210, kErrApplyMma = 0x220, kErrApplyRelu = 0x230, kErrApplyEpi = 0x240,
  kErrApplyMerge = 0x250,
  kErrSelfTest = 0x3f0,
};

// Self-test of the bounded-wait error path: one thread waits on an mbarrier that nothing ever
// arrives on; after the wait limit it records kErrSelfTest in *err and the kernel returns.
__global__ void litela_selftest_timeout(int* err) {
  using namespace sm100;
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, kErrSelfTest);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ReLU of 8 packed bf16 values (IEEE maxNum with +0: negative and -0 become +0)
__device__ __forceinline__ uint4 relu_bf16x8(uint4 w) {
  const __nv_bfloat162 z = __float2bfloat162_rn(0.f);
  uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&u[i]);
    x = __hmax2(x, z);
    u[i] = *reinterpret_cast<uint32_t*>(&x);
  }
  return w;
}

// byte offset of element (row n, column c) in a head's state image (the apply's B operand,
// K-major without swizzle: 8 x 8 core matrices of 128 B, K-direction stride 128 B, 8-row
// group stride 512 B)
__device__ __forceinline__ uint32_t image_offset(int n, int c) {
  return (uint32_t)((n >> 3) * 512 + (c >> 3) * 128 + (n & 7) * 16 + (c & 7) * 2);
}

// ---------------------------------------------------------------------------------------
// state reduction

constexpr int kRedStages = 3;
constexpr int kRedThreads = 192;                       // w0 TMA, w1 MMA, w2..5 ReLU + epilogue
constexpr uint32_t kRedBoxBytes = 64 * 2 * kRedTile;   // 64 channels x 64 tokens x bf16
constexpr uint32_t kRedStageBytes = 4 * kRedBoxBytes;  // k lo/hi channels, v lo/hi channels
constexpr uint32_t kRedTmemCols = 256;
constexpr uint32_t kRedSmemBytes = kRedStages * kRedStageBytes + 512 + 256 + 1024;
constexpr int kRedPrefetchTiles = 6;   // k|v tiles prefetched into L2 before the dependency wait

// Feature maps.  kMap 0: phi = ReLU (LiteLA), exact in bf16.  kMap 1: phi = ELU + 1 (the Sana
// tutorial page's linear-attention block: exp(x) for x <= 0, x + 1 above), formed in fp32 and
// entered into the tensor cores as a bf16 hi + lo pair (the lo halves in an extra buffer).
template <int kMap>
struct RedCfg {
  static constexpr uint32_t kStageBytes = (kMap ? 6 : 4) * kRedBoxBytes;   // + phi(k) lo boxes
  // ring depth: two CTAs per SM either way (the grid is one wave of two CTAs per SM), so the
  // ELU + 1 form, with 48 KB stages, keeps two of them
  static constexpr int kStages = kMap ? 2 : kRedStages;
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + 512 + 256 + 1024;
  // warps: 0 TMA, 1 MMA, 2.. feature map (4 for ReLU, 8 for ELU + 1); warps 2..5 also read the
  // accumulators at the end
  static constexpr int kMapWarps = kMap ? 8 : 4;
  static constexpr int kThreads = 32 * (2 + kMapWarps);
  // the read-out warps 2..5 cover the four TMEM lane quarters and are all map warps
  static_assert(kMapWarps >= 4, "reduction read-out warps");
};

// exp by the hardware approximation (__expf, ~2^-21 relative error here): far inside the
// tolerance of a bf16 or fp32 result, and cheap enough for an elementwise pass over q and k
__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }
constexpr float kInvSqrtD = 0.17677669529663687f;   // 1 / sqrt(32): the variant's scale of phi(q)

// phi = ELU + 1 of 8 packed bf16 values, times `scale`, as bf16 hi and lo (hi + lo equals the
// fp32 value to 2^-17 relative)
__device__ __forceinline__ void phi_elu1_hilo(uint4 w, float scale, uint4& hi, uint4& lo) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = phi_elu1(__uint_as_float(u[i] << 16)) * scale;
    const float x1 = phi_elu1(__uint_as_float(u[i] & 0xFFFF0000u)) * scale;
    __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
    h[i] = *reinterpret_cast<uint32_t*>(&hp);
    __nv_bfloat162 lp = __floats2bfloat162_rn(x0 - __uint_as_float(h[i] << 16), x1 - __uint_as_float(h[i] & 0xFFFF0000u));
    l[i] = *reinterpret_cast<uint32_t*>(&lp);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int kMap>
__global__ void __launch_bounds__(RedCfg<kMap>::kThreads, 1)
litela_reduce_tc(const __grid_constant__ CUtensorMap tmap, float* __restrict__ partials,
                 int* __restrict__ err, TcPlan p) {
  using namespace sm100;
  constexpr uint32_t kStageBytes = RedCfg<kMap>::kStageBytes;
  constexpr int kStages = RedCfg<kMap>::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  uint8_t* ones = smem + kStages * kStageBytes;                 // 16 x 16 bf16 ones
  uint64_t* full = reinterpret_cast<uint64_t*>(ones + 512);
  uint64_t* relu_done = full + kStages;
  uint64_t* empty = relu_done + kStages;
  uint64_t* done = empty + kStages;      // a block's products are done (one phase per block)
  uint64_t* tfree = done + 1;            // the epilogue has read a block's accumulator
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfree + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int x = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  // this CTA's blocks [bb0, bb1) (several only with one chunk per block), its chunk ch of each;
  // block k's tokens [n0, n1) and 64-token tiles
  const int bb0 = p.bpc > 1 ? x * p.bpc : x / p.cpb;
  const int bb1 = p.bpc > 1 ? min(bb0 + p.bpc, p.nblk) : bb0 + 1;
  const int ch = p.bpc > 1 ? 0 : x - bb0 * p.cpb;
  auto span = [&](int k, int& n0, int& n1) {
    n0 = k * p.T + ch * p.chunk;
    n1 = min(n0 + p.chunk, min((k + 1) * p.T, p.N));
    return n1 > n0 ? (n1 - n0 + kRedTile - 1) / kRedTile : 0;
  };
  int n0, n1;
  const int ntiles = span(bb0, n0, n1);   // the first block's (the L2 prefetch covers it)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&relu_done[s], 32 * RedCfg<kMap>::kMapWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(tfree, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 128; i += kRedThreads) reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_holder, kRedTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  if (warp == 0 && lane == 0) {
    // while the previous kernel drains: warm L2 with this CTA's first k|v tiles (a prefetch
    // changes no memory contents).  The backward at 4096px: 310.2 -> 306.1 us; the three-kernel
    // forward (B=8, N=4096, H=80): 159.9 -> 158.0 us (12 tiles were slower)
    const int kx0 = p.H * kD + g * (kRedHeads * kD), vx0 = 2 * p.H * kD + g * (kRedHeads * kD);
    for (int i = 0; i < kRedPrefetchTiles && i < ntiles; ++i) {
      const int y = n0 + i * kRedTile;
      tma_prefetch_3d(&tmap, kx0, y, b);
      tma_prefetch_3d(&tmap, kx0 + 64, y, b);
      tma_prefetch_3d(&tmap, vx0, y, b);
      tma_prefetch_3d(&tmap, vx0 + 64, y, b);
    }
  }
  // launched as a programmatic dependent of the previous kernel in the stream: everything
  // above is private set-up; qkv and the workspace are touched only after that kernel is done
  pdl_wait_primary();
  // Only now may the next kernels launch.  This kernel opens a call, and the later kernels of
  // the call read their inputs (q, the incoming gradient) before their own waits: releasing
  // them after this wait means that whatever produced those inputs upstream has finished.
  pdl_launch_dependents();

  const int kx = p.H * kD + g * (kRedHeads * kD);       // first key channel of the group
  const int vx = 2 * p.H * kD + g * (kRedHeads * kD);   // first value channel of the group

  if (warp == 0) {
    if (lane == 0) {
      // k and v are read once: with the ReLU map their L2 lines go first (measured faster for
      // the three-kernel forward; the ELU + 1 map keeps the default policy)
      const uint64_t pol = l2_policy_evict_first();
      auto load = [&](void* dst, uint64_t* bar, int x, int y) {
        if (kMap == 0)
          tma_load_3d(dst, &tmap, bar, x, y, b, pol);
        else
          tma_load_3d(dst, &tmap, bar, x, y, b);
      };
      int issued = 0, i = 0;
      bool stop = false;
      for (int k = bb0; k < bb1 && !stop; ++k) {
        int a0, a1;
        const int nt = span(k, a0, a1);
        for (int j = 0; j < nt; ++j, ++i) {
          const int s = i % kStages;
          if (i >= kStages &&
              !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, abort_flag, err, kErrReduceProducer | s)) {
            stop = true;
            break;
          }
          uint8_t* st = stages + s * kStageBytes;
          const int y = a0 + j * kRedTile;
          mbar_arrive_expect_tx(&full[s], kRedStageBytes);
          load(st, &full[s], kx, y);
          load(st + kRedBoxBytes, &full[s], kx + 64, y);
          load(st + 2 * kRedBoxBytes, &full[s], vx, y);
          load(st + 3 * kRedBoxBytes, &full[s], vx + 64, y);
          issued = i + 1;
        }
      }
      if (*abort_flag) {   // let the copies still in flight land before the CTA exits (bounded)
        for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
          mbar_drain(&full[i % kStages], (i / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_num = idesc_bf16_f32(128, 128, true, true);
      constexpr uint32_t idesc_den = idesc_bf16_f32(128, 16, true, false);
      const uint64_t ones_desc = smem_desc(smem_u32(ones), 128, 256, kSwizzleNone);
      int i = 0;
      bool stop = false;
      for (int k = bb0; k < bb1 && !stop; ++k) {
        int a0, a1;
        const int nt = span(k, a0, a1);
        // the accumulator is overwritten by this block's first product: the epilogue has read
        // the previous block's
        if (k > bb0 && !mbar_wait(tfree, (k - bb0 - 1) & 1, abort_flag, err, kErrReduceMma | 8)) break;
        for (int j = 0; j < nt; ++j, ++i) {
          const int s = i % kStages;
          if (!mbar_wait(&relu_done[s], (i / kStages) & 1, abort_flag, err, kErrReduceMma | s)) {
            stop = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t kbase = smem_u32(stages + s * kStageBytes);
          const uint32_t vbase = kbase + 2 * kRedBoxBytes;
#pragma unroll
          for (int ks = 0; ks < kRedTile / 16; ++ks) {
            // MN-major, 128B swizzle: 8-token row groups 1024 B apart, 64-channel blocks one box apart
            const uint64_t a = smem_desc(kbase + ks * 2048, kRedBoxBytes, 1024, kSwizzle128B);
            const uint64_t bv = smem_desc(vbase + ks * 2048, kRedBoxBytes, 1024, kSwizzle128B);
            const uint32_t acc = (j | ks) != 0;
            umma_bf16(tmem, a, bv, idesc_num, acc);
            umma_bf16(tmem + 128, a, ones_desc, idesc_den, acc);
            if (kMap) {   // the lo halves of phi(k)
              const uint64_t al = smem_desc(kbase + 4 * kRedBoxBytes + ks * 2048, kRedBoxBytes, 1024, kSwizzle128B);
              umma_bf16(tmem, al, bv, idesc_num, 1u);
              umma_bf16(tmem + 128, al, ones_desc, idesc_den, 1u);
            }
          }
          umma_commit(&empty[s]);
        }
        if (!stop) umma_commit(done);
      }
    }
  } else {
    constexpr int kMapThreads = 32 * RedCfg<kMap>::kMapWarps;
    const int t = threadIdx.x - 64;
    const int64_t nparts = (int64_t)p.nblk * p.cpb;
    int i = 0;
    bool ok = true;
    for (int k = bb0; k < bb1; ++k) {
      int a0, a1;
      const int nt = span(k, a0, a1);
      for (int j = 0; ok && j < nt; ++j, ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1, abort_flag, err, kErrReduceRelu | s)) {
          ok = false;
          break;
        }
        uint8_t* st = stages + s * kStageBytes;
        const int valid = min(kRedTile, a1 - (a0 + j * kRedTile));   // tokens of this chunk in the tile
#pragma unroll 4
        for (int w = t; w < 1024; w += kMapThreads) {   // k: 2 boxes x 64 rows x 8 chunks of 16 B
          uint4* c = reinterpret_cast<uint4*>(st + w * 16);
          const int row = (w >> 3) & (kRedTile - 1);
          if (kMap == 0) {
            *c = row < valid ? relu_bf16x8(*c) : make_uint4(0u, 0u, 0u, 0u);
          } else {
            uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
            if (row < valid) phi_elu1_hilo(*c, 1.0f, hi, lo);
            *c = hi;
            *reinterpret_cast<uint4*>(st + 4 * kRedBoxBytes + w * 16) = lo;
          }
        }
        if (valid < kRedTile) {
          for (int w = t; w < 1024; w += kMapThreads) {
            const int row = (w >> 3) & (kRedTile - 1);
            if (row >= valid) *reinterpret_cast<uint4*>(st + 2 * kRedBoxBytes + w * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&relu_done[s]);
      }
      // epilogue (warps 2..5): block k's partial state; warp quarter q reads TMEM lanes
      // 32q..32q+31 = head q's key channels c, then frees the accumulator for the next block
      if (warp < 6) {
        const int q = warp & 3;
        float sv[kRows];
        bool got = ok && nt > 0;
        if (got) got = mbar_wait(done, (k - bb0) & 1, abort_flag, err, kErrReduceEpi);
        got = __all_sync(0xffffffffu, got);
        if (got) {
          tc_fence_after_sync();
          uint32_t r[32], zr;
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16);
          tmem_ld_x32(ta + q * 32, r);
          tmem_ld_x1(ta + 128, zr);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) sv[jj] = __uint_as_float(r[jj]);
          sv[32] = __uint_as_float(zr);
        } else {
#pragma unroll
          for (int jj = 0; jj < kRows; ++jj) sv[jj] = 0.f;
        }
        tc_fence_before_sync();
        mbar_arrive(tfree);
        float* dst = partials + ((((int64_t)b * p.ngroups + g) * nparts + (int64_t)k * p.cpb + ch) * kRedHeads + q) *
                                    kStateFloats;
#pragma unroll
        for (int jj = 0; jj < kRows; ++jj) dst[jj * kD + lane] = sv[jj];   // S[r = jj][c = lane]
      }
      if (!ok) break;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kRedTmemCols);
  }
}

// address of partial `part` (block * cpb + chunk) of head h of batch b
__device__ __forceinline__ const float* partial_ptr(const float* partials, const TcPlan& p, int b, int h,
                                                    int part) {
  const int g = h / kRedHeads, hl = h - g * kRedHeads;
  return partials + ((((int64_t)b * p.ngroups + g) * ((int64_t)p.nblk * p.cpb) + part) * kRedHeads + hl) *
                        kStateFloats;
}

// litela_state_scan: partial states -> per-(batch, head, block) inclusive prefix states, summed in
// fixed order (deterministic).  Writes each one as the apply's B-operand image (bf16 hi rows
// 0..32, lo rows 40..72, zero rows in between and after; S = hi + lo to 2^-17 relative), when
// `images_t` is not null also as the transposed image of its first 32 rows (rows c: hi 0..31,
// lo 32..63, K = r; the B operand of products with S[0:32]^T), and, when `states` is not null,
// as fp32 [B][H][nblk][33][32].  With `reverse` the blocks are visited last to first, giving
// the inclusive SUFFIX sums over blocks (the gradient of a prefix-summed state).  With `rows64`
// the images hold only rows 0..31 (hi rows 0..31, lo rows 32..63: kImageTBytes each, no zero
// rows) and row 32 goes to `zrows` in fp32 ([B][H][nblk][32]).  `state_in` (fp32 [B][H][33][32], may be
// null) is a state carried from earlier chunks of the sequence and starts every prefix;
// `state_out` (may be null, may alias state_in) receives the final prefix.  Grid-stride over the state elements,
// one per thread, with at most kScanCtasPerSm CTAs per SM; each thread keeps 8 partial loads in
// flight per round.  A thread's work is one long chain (a conversion and stores at every block
// end), so the scan needs many warps per SM: with one CTA per SM and 2 elements a thread,
// block-causal calls with many blocks took 3-11 % longer.
constexpr int kScanThreads = 256;
constexpr int kScanCtasPerSm = 4;
constexpr int kScanZeros = 14 * kD;   // zero elements of one image
constexpr int kScanElems = 1;         // state elements per thread and round

__global__ void __launch_bounds__(kScanThreads)
litela_state_scan(const float* __restrict__ partials, uint8_t* __restrict__ images, uint8_t* __restrict__ images_t,
                  float* __restrict__ states, const float* __restrict__ state_in, float* __restrict__ state_out,
                  bool reverse, bool rows64, float* __restrict__ zrows, TcPlan p) {
  using namespace sm100;
  pdl_launch_dependents();
  const int64_t stride = (int64_t)gridDim.x * kScanThreads;
  const int64_t tid = (int64_t)blockIdx.x * kScanThreads + threadIdx.x;
  // the partials come from the reduction grid; the images may be read by the previous call's
  // apply until that grid (which waited for it) is done
  pdl_wait_primary();
  if (images != nullptr && !rows64) {   // zero rows of every image
    const int64_t nz = (int64_t)p.B * p.H * p.nblk * kScanZeros;
    for (int64_t i = tid; i < nz; i += stride) {
      const int64_t im = i / kScanZeros;
      const int k = (int)(i - im * kScanZeros);
      const int zr = k >> 5, c = k & 31;
      const int nrow = zr < 7 ? kRows + zr : kImageLoRow + kRows + (zr - 7);
      *reinterpret_cast<__nv_bfloat16*>(images + im * kImageBytes + image_offset(nrow, c)) = __float2bfloat16_rn(0.f);
    }
  }
  const int nparts = p.nblk * p.cpb;
  const int64_t pstride = (int64_t)kRedHeads * kStateFloats;
  const int64_t total = (int64_t)p.B * p.H * kStateFloats;
  constexpr int kE = kScanElems;
  for (int64_t base = tid; base < total; base += kE * stride) {
    const float* src[kE]; int64_t bh[kE]; int e[kE]; bool ok[kE];
#pragma unroll
    for (int j = 0; j < kE; ++j) {
      const int64_t i = base + j * stride;
      ok[j] = i < total;
      bh[j] = ok[j] ? i / kStateFloats : 0;
      e[j] = ok[j] ? (int)(i - bh[j] * kStateFloats) : 0;
      const int b = (int)(bh[j] / p.H), h = (int)(bh[j] - (int64_t)b * p.H);
      const int g = h / kRedHeads, hl = h - g * kRedHeads;
      src[j] = partials + ((((int64_t)b * p.ngroups + g) * nparts) * kRedHeads + hl) * kStateFloats + e[j];
    }
    float run[kE], sum[kE];
#pragma unroll
    for (int j = 0; j < kE; ++j) {   // the carried state of earlier chunks starts every prefix
      run[j] = (state_in != nullptr && ok[j]) ? state_in[bh[j] * kStateFloats + e[j]] : 0.f;
      sum[j] = 0.f;
    }
    for (int k0 = 0; k0 < nparts; k0 += 8) {
      float v[kE][8];
#pragma unroll
      for (int j = 0; j < kE; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int k = reverse ? nparts - 1 - (k0 + i) : k0 + i;
          v[j][i] = (ok[j] && k0 + i < nparts) ? __ldcg(src[j] + (int64_t)k * pstride) : 0.f;
        }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (k0 + i >= nparts) break;
        const int k = reverse ? nparts - 1 - (k0 + i) : k0 + i;
        // last chunk of block k / cpb in visiting order
        const bool block_end = reverse ? (k % p.cpb == 0) : ((k + 1) % p.cpb == 0);
        const int blk = k / p.cpb;
#pragma unroll
        for (int j = 0; j < kE; ++j) {
          sum[j] += v[j][i];
          if (block_end && ok[j]) {   // extend the prefix and store it
            run[j] += sum[j];
            sum[j] = 0.f;
            const int r = e[j] >> 5, c = e[j] & 31;
            const __nv_bfloat16 hi = __float2bfloat16_rn(run[j]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(run[j] - __bfloat162float(hi));
            const int64_t im = bh[j] * p.nblk + blk;
            if (images != nullptr && !rows64) {
              uint8_t* img = images + im * kImageBytes;
              *reinterpret_cast<__nv_bfloat16*>(img + image_offset(r, c)) = hi;
              *reinterpret_cast<__nv_bfloat16*>(img + image_offset(kImageLoRow + r, c)) = lo;
            }
            if (images != nullptr && rows64 && r < kD) {
              uint8_t* img = images + im * kImageTBytes;
              *reinterpret_cast<__nv_bfloat16*>(img + image_offset(r, c)) = hi;
              *reinterpret_cast<__nv_bfloat16*>(img + image_offset(kD + r, c)) = lo;
            }
            if (zrows != nullptr && r == kD) zrows[im * kD + c] = run[j];
            if (images_t != nullptr && r < kD) {
              uint8_t* imt = images_t + im * kImageTBytes;
              *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(c, r)) = hi;
              *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(kD + c, r)) = lo;
            }
            if (states != nullptr) states[(bh[j] * p.nblk + blk) * kStateFloats + e[j]] = run[j];
          }
        }
      }
    }
    if (state_out != nullptr) {
#pragma unroll
      for (int j = 0; j < kE; ++j)
        if (ok[j]) state_out[bh[j] * kStateFloats + e[j]] = run[j];
    }
  }
}

// litela_state_images: fp32 states [n][33][32] (n = B * H * nblk, already the states the
// queries use) -> the apply's B-operand images (bf16 hi rows 0..32, lo rows 40..72, zero rows)
// and, when images_t is not null, the transposed images of rows 0..31.  Used by the backward
// when the forward's states are supplied instead of recomputed.
__global__ void __launch_bounds__(kScanThreads)
litela_state_images(const float* __restrict__ states, uint8_t* __restrict__ images, uint8_t* __restrict__ images_t,
                    long long n) {
  using namespace sm100;
  pdl_wait_primary();
  // This kernel opens a call; the kernels after it read the call's inputs before their own
  // waits, so they are released only once whatever came before in the stream has finished.
  pdl_launch_dependents();
  const int64_t stride = (int64_t)gridDim.x * kScanThreads;
  const int64_t tid = (int64_t)blockIdx.x * kScanThreads + threadIdx.x;
  for (int64_t i = tid; i < n * kScanZeros; i += stride) {   // zero rows 33..39 and 73..79
    const int64_t im = i / kScanZeros;
    const int k = (int)(i - im * kScanZeros), zr = k >> 5, c = k & 31;
    const int nrow = zr < 7 ? kRows + zr : kImageLoRow + kRows + (zr - 7);
    *reinterpret_cast<__nv_bfloat16*>(images + im * kImageBytes + image_offset(nrow, c)) = __float2bfloat16_rn(0.f);
  }
  for (int64_t i = tid; i < n * kStateFloats; i += stride) {
    const int64_t im = i / kStateFloats;
    const int e = (int)(i - im * kStateFloats), r = e >> 5, c = e & 31;
    const float v = states[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    uint8_t* img = images + im * kImageBytes;
    *reinterpret_cast<__nv_bfloat16*>(img + image_offset(r, c)) = hi;
    *reinterpret_cast<__nv_bfloat16*>(img + image_offset(kImageLoRow + r, c)) = lo;
    if (images_t != nullptr && r < kD) {
      uint8_t* imt = images_t + im * kImageTBytes;
      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(c, r)) = hi;
      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(kD + c, r)) = lo;
    }
  }
}

// ---------------------------------------------------------------------------------------
// apply

constexpr int kApThreads = 256;   // w0 TMA, w1 MMA, w2..3 ReLU, w4..7 epilogue
constexpr uint32_t kQBoxBytes = kApTile * 128;         // 128 tokens x 64 channels x bf16 (one pair)
constexpr int kApAccSlots = 3;
constexpr uint32_t kApAccCols = kApHeads * kImageRows; // 160 fp32 columns per slot (one pair)
constexpr uint32_t kApTmemCols = 512;
constexpr uint32_t kApSbufBytes = kApUnitHeads * kImageBytes;
constexpr uint32_t kOutBoxBytes = kApTile * 128;       // one 128B-swizzled box: 128 rows x 128 B
constexpr int kApReluThreads = 64;

template <typename OutT, int kMap = 0>
struct ApplyCfg {
  // shared memory split (bf16 output: 3 q stages, 2 output slots, 2 state buffers = 202 KB;
  // fp32 output: 2 q stages, 1 output slot, 2 state buffers; ELU + 1: 2 q stages of twice the
  // size (phi(q) hi and lo), 1 state buffer).  Two state buffers let the next segment's image
  // load while the last one's tiles are applied: block-causal calls with short blocks change
  // segment every few tiles (T = 512: 92.0 -> 84.4 us against 4 q stages and 1 buffer).
  static constexpr int kQStages = kMap ? 2 : (sizeof(OutT) == 2 ? 3 : 2);
  static constexpr int kOutSlots = sizeof(OutT) == 2 ? 2 : 1;
  static constexpr int kSBufs = kMap ? 1 : 2;
  // warps: 0 TMA, 1 MMA, 2.. feature map (2 warps for ReLU, 6 for ELU + 1), then 4 epilogue warps
  static constexpr int kMapWarps = kMap ? 8 : 2;
  static constexpr int kThreads = 32 * (2 + kMapWarps + 4);
  static constexpr int kEpiWarp0 = 2 + kMapWarps;
  static constexpr int kBoxChannels = 128 / (int)sizeof(OutT);     // output channels per box
  static constexpr int kOutBoxes = kApUnitHeads * kD / kBoxChannels;
  static constexpr uint32_t kQStageBytes = (kMap ? 4 : 2) * kQBoxBytes;
  static constexpr uint32_t kOutSlotBytes = kOutBoxes * kOutBoxBytes;
  static constexpr uint32_t kSmemBytes =
      kQStages * kQStageBytes + kOutSlots * kOutSlotBytes + kSBufs * kApSbufBytes + 512 + 1024;
};

struct ApUnit {
  int b, quad, blk, tok0, tok1;
  long long seg;
};

// Work assignment.  When the CTAs can be split evenly over the head quads (gridDim.x a multiple
// of nquads), CTA c owns quad c % nquads and a contiguous share (c / nquads) of that quad's
// units in (batch, block, tile) order: all quads then advance through the same token rows at
// the same time, so together the CTAs read and write whole q / output rows (DRAM locality),
// and each CTA changes state only at batch / block boundaries.  Otherwise CTA c takes a
// contiguous range of units in (batch, quad, block, tile) order.
struct ApRange {
  long long u0, u1;   // local unit range
  int quad;           // fixed quad, or -1 for the general order
};

__device__ __forceinline__ ApRange ap_range(const TcPlan& p) {
  ApRange R;
  if (gridDim.x % p.nquads == 0) {
    const int per = gridDim.x / p.nquads, r = blockIdx.x / p.nquads;
    const long long L = (long long)p.B * p.nblk * p.tpb;
    R.quad = blockIdx.x % p.nquads;
    R.u0 = (long long)r * L / per;
    R.u1 = (long long)(r + 1) * L / per;
  } else {
    R.quad = -1;
    R.u0 = (long long)blockIdx.x * p.units / gridDim.x;
    R.u1 = (long long)(blockIdx.x + 1) * p.units / gridDim.x;
  }
  return R;
}

__device__ __forceinline__ ApUnit ap_decode(long long u, const ApRange& R, const TcPlan& p) {
  ApUnit U;
  const int tile = (int)(u % p.tpb);
  long long r = u / p.tpb;
  U.blk = (int)(r % p.nblk);
  r /= p.nblk;
  if (R.quad >= 0) {
    U.quad = R.quad;
    U.b = (int)r;
  } else {
    U.quad = (int)(r % p.nquads);
    U.b = (int)(r / p.nquads);
  }
  U.seg = ((long long)U.b * p.nquads + U.quad) * p.nblk + U.blk;
  U.tok0 = U.blk * p.T + tile * kApTile;
  U.tok1 = min(U.tok0 + kApTile, min((U.blk + 1) * p.T, p.N));
  return U;
}

// heads of pair h (0 or 1) of a unit
__device__ __forceinline__ int pair_heads_h(int H, int quad, int h) {
  return max(0, min(kApHeads, H - quad * kApUnitHeads - h * kApHeads));
}
__device__ __forceinline__ int pair_heads(const TcPlan& p, int quad, int h) { return pair_heads_h(p.H, quad, h); }

// 8 floats -> 8 packed bf16 (round to nearest even)
__device__ __forceinline__ uint4 pack_bf16x8(const float* x) {
  uint32_t u[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 v2 = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    u[i] = *reinterpret_cast<uint32_t*>(&v2);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

__device__ __forceinline__ void pack_out(__nv_bfloat16*, const float* o, uint4* w) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 v2 = __floats2bfloat162_rn(o[i * 8 + 2 * j], o[i * 8 + 2 * j + 1]);
      u[j] = *reinterpret_cast<uint32_t*>(&v2);
    }
    w[i] = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

__device__ __forceinline__ void pack_out(float*, const float* o, uint4* w) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = make_uint4(__float_as_uint(o[4 * i]), __float_as_uint(o[4 * i + 1]), __float_as_uint(o[4 * i + 2]),
                      __float_as_uint(o[4 * i + 3]));
}

template <typename OutT, int kMap = 0>
__global__ void __launch_bounds__(ApplyCfg<OutT, kMap>::kThreads, 1)
litela_apply_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_out,
                const uint8_t* __restrict__ images, OutT* __restrict__ out, int* __restrict__ err, TcPlan p) {
  using namespace sm100;
  using Cfg = ApplyCfg<OutT, kMap>;
  constexpr int kQStages = Cfg::kQStages;
  constexpr int kSBufs = Cfg::kSBufs;
  constexpr int kChunksPerHead = kD * (int)sizeof(OutT) / 16;   // 16-byte chunks of one head's row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* qst = smem;                                              // q tiles (2 boxes per stage)
  uint8_t* obuf = qst + kQStages * Cfg::kQStageBytes;               // output staging slots
  uint8_t* sbuf = obuf + Cfg::kOutSlots * Cfg::kOutSlotBytes;       // state buffers (4 heads each)
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sbuf + kSBufs * kApSbufBytes);
  uint64_t* qrelu = qfull + kQStages;
  uint64_t* qempty = qrelu + kQStages;
  uint64_t* sfull = qempty + kQStages;
  uint64_t* sempty = sfull + kSBufs;
  uint64_t* tfull = sempty + kSBufs;
  uint64_t* tempty = tfull + kApAccSlots;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + kApAccSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ApRange R = ap_range(p);
  const long long u0 = R.u0, u1 = R.u1;

  pdl_launch_dependents();   // the next kernel waits for this grid before touching memory
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qrelu[s], 32 * Cfg::kMapWarps);
      mbar_init(&qempty[s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int s = 0; s < kApAccSlots; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kApTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_out);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---- producer: q tiles, 128 tokens x (2 pairs x 64 channels) per unit, and the state
    // images of each segment (bulk copies of the scan kernel's output)
    if (lane == 0) {
      auto load_q = [&](long long u) {
        const int lu = (int)(u - u0);
        const ApUnit U = ap_decode(u, R, p);
        const int s = lu % kQStages;
        const int np = pair_heads(p, U.quad, 1) > 0 ? 2 : 1;
        mbar_arrive_expect_tx(&qfull[s], np * kQBoxBytes);
        for (int h = 0; h < np; ++h)
          tma_load_3d(qst + s * Cfg::kQStageBytes + h * kQBoxBytes, &tmap_q, &qfull[s],
                      U.quad * kApUnitHeads * kD + h * kApHeads * kD, U.tok0, U.b);
      };
      // q does not depend on the preceding grids: fill the ring before waiting for them
      const long long pre = (u1 - u0) < kQStages ? (u1 - u0) : kQStages;
      for (long long u = u0; u < u0 + pre; ++u) load_q(u);
      int issued = (int)pre, seg_loaded = -1;
      pdl_wait_primary();   // the state images are written by the preceding scan grid
      long long prev = -1;
      int seg_n = -1;
      for (long long u = u0; u < u1; ++u) {
        const int lu = (int)(u - u0);
        const ApUnit U = ap_decode(u, R, p);
        if (lu >= pre) {   // q first: it does not wait for the state buffer to free up
          const int s = lu % kQStages;
          if (!mbar_wait(&qempty[s], ((lu / kQStages) - 1) & 1, abort_flag, err, kErrApplyProducer | s)) break;
          load_q(u);
          issued = lu + 1;
        }
        if (U.seg != prev) {
          prev = U.seg;
          ++seg_n;
          const int sb = seg_n % kSBufs;
          if (seg_n >= kSBufs && !mbar_wait(&sempty[sb], ((seg_n / kSBufs) - 1) & 1, abort_flag, err,
                                            kErrApplyProducer | 8 | sb))
            break;
          const int nh = min(kApUnitHeads, p.H - U.quad * kApUnitHeads);
          mbar_arrive_expect_tx(&sfull[sb], nh * kImageBytes);
          for (int j = 0; j < nh; ++j) {
            const uint8_t* src =
                images + (((int64_t)U.b * p.H + U.quad * kApUnitHeads + j) * p.nblk + U.blk) * kImageBytes;
            bulk_load(sbuf + sb * kApSbufBytes + j * kImageBytes, src, kImageBytes, &sfull[sb]);
          }
          seg_loaded = seg_n;
        }
      }
      if (*abort_flag) {   // let the copies still in flight land before the CTA exits (bounded)
        for (int i = (issued > kQStages ? issued - kQStages : 0); i < issued; ++i)
          mbar_drain(&qfull[i % kQStages], (i / kQStages) & 1);
        for (int k = (seg_loaded >= kSBufs ? seg_loaded - kSBufs + 1 : 0); k <= seg_loaded; ++k)
          mbar_drain(&sfull[k % kSBufs], (k / kSBufs) & 1);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: one head pair at a time into TMEM slot (pair counter) % 3
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kImageRows, false, false);
      long long prev = -1;
      int seg_n = -1, sb = 0, pn = 0;
      bool stop = false;
      for (long long u = u0; u < u1 && !stop; ++u) {
        const int lu = (int)(u - u0);
        const ApUnit U = ap_decode(u, R, p);
        if (U.seg != prev) {
          prev = U.seg;
          ++seg_n;
          sb = seg_n % kSBufs;
          if (!mbar_wait(&sfull[sb], (seg_n / kSBufs) & 1, abort_flag, err, kErrApplyMma | 8 | sb)) break;
        }
        const int s = lu % kQStages;
        if (!mbar_wait(&qrelu[s], (lu / kQStages) & 1, abort_flag, err, kErrApplyMma | s)) break;
        const uint32_t qaddr = smem_u32(qst + s * Cfg::kQStageBytes);
        const uint32_t saddr = smem_u32(sbuf + sb * kApSbufBytes);
        for (int h = 0; h < 2; ++h) {
          const int nh = pair_heads(p, U.quad, h);
          if (nh == 0) break;
          const int a = pn % kApAccSlots;
          if (pn >= kApAccSlots &&
              !mbar_wait(&tempty[a], ((pn / kApAccSlots) - 1) & 1, abort_flag, err, kErrApplyMma | 12 | a)) {
            stop = true;
            break;
          }
          tc_fence_after_sync();
          for (int j = 0; j < nh; ++j) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              // A: K-major 128B swizzle, 8-token groups 1024 B apart; head j's 32 channels at +64j B
              const uint64_t ad = smem_desc(qaddr + h * kQBoxBytes + j * 64 + ks * 32, 16, 1024, kSwizzle128B);
              // B: K-major no swizzle, K-direction core matrices 128 B apart, row groups 512 B apart
              const uint64_t bd =
                  smem_desc(saddr + (h * kApHeads + j) * kImageBytes + ks * 256, 128, 512, kSwizzleNone);
              umma_bf16(tmem + a * kApAccCols + j * kImageRows, ad, bd, idesc, ks);
              if (kMap) {   // the lo halves of phi(q)
                const uint64_t al =
                    smem_desc(qaddr + 2 * kQBoxBytes + h * kQBoxBytes + j * 64 + ks * 32, 16, 1024, kSwizzle128B);
                umma_bf16(tmem + a * kApAccCols + j * kImageRows, al, bd, idesc, 1u);
              }
            }
          }
          umma_commit(&tfull[a]);
          ++pn;
        }
        if (stop) break;
        umma_commit(&qempty[s]);
        const bool seg_ends = (u + 1 >= u1) || (ap_decode(u + 1, R, p).seg != U.seg);
        if (seg_ends) umma_commit(&sempty[sb]);
      }
    }
  } else if (warp < Cfg::kEpiWarp0) {
    // ---- feature map of the q tiles in place (ReLU; or ELU + 1 with its lo halves)
    const int t = threadIdx.x - 64;
    for (long long u = u0; u < u1; ++u) {
      const int lu = (int)(u - u0);
      const int s = lu % kQStages;
      if (!mbar_wait(&qfull[s], (lu / kQStages) & 1, abort_flag, err, kErrApplyRelu | s)) break;
      const ApUnit U = ap_decode(u, R, p);
      const int nchunks = (pair_heads(p, U.quad, 1) > 0 ? 2 : 1) * (int)(kQBoxBytes / 16);
      uint8_t* st = qst + s * Cfg::kQStageBytes;
#pragma unroll 4
      for (int j = t; j < nchunks; j += 32 * Cfg::kMapWarps) {
        uint4* c = reinterpret_cast<uint4*>(st + j * 16);
        if (kMap == 0) {
          *c = relu_bf16x8(*c);
        } else {   // phi(q) / sqrt(d): hi in place, lo two boxes further
          uint4 hi, lo;
          phi_elu1_hilo(*c, kInvSqrtD, hi, lo);
          *c = hi;
          *reinterpret_cast<uint4*>(st + 2 * kQBoxBytes + j * 16) = lo;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&qrelu[s]);
    }
  } else {
    // ---- epilogue: TMEM -> normalise -> staged TMA store (or row stores for partial tiles)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool leader = (warp == Cfg::kEpiWarp0 && lane == 0);
    int nstaged = 0, pn = 0;
    bool stop = false;
    for (long long u = u0; u < u1 && !stop; ++u) {
      const ApUnit U = ap_decode(u, R, p);
      const int n = U.tok0 + row;
      const bool staged = (U.tok1 - U.tok0 == kApTile) || (U.tok1 == p.N);
      uint8_t* slot = obuf + (nstaged % Cfg::kOutSlots) * Cfg::kOutSlotBytes;
      if (staged) {
        if (leader) bulk_wait_group_read<Cfg::kOutSlots - 1>();   // the store that last used this slot has read it
        bar_sync(2, 128);
        ++nstaged;
      }
      for (int h = 0; h < 2; ++h) {
        const int nh = pair_heads(p, U.quad, h);
        if (nh == 0) break;
        const int a = pn % kApAccSlots;
        const bool ok = mbar_wait(&tfull[a], (pn / kApAccSlots) & 1, abort_flag, err, kErrApplyEpi | a);
        if (bar_any(1, 128, !ok)) {
          stop = true;
          break;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + a * kApAccCols;
        for (int j = 0; j < nh; ++j) {
          uint32_t v[kImageRows];
#pragma unroll
          for (int k = 0; k < kImageRows / 16; ++k) tmem_ld_x16(ta + j * kImageRows + k * 16, v + k * 16);
          tmem_wait_ld();
          if (j == nh - 1) {
            tc_fence_before_sync();
            mbar_arrive(&tempty[a]);
          }
          // LiteLA adds eps to the denominator; the ELU + 1 variant clamps it from below (p.eps)
          const float y_d = __uint_as_float(v[kD]) + __uint_as_float(v[kImageLoRow + kD]);
          const float den = kMap ? fmaxf(y_d, p.eps) : y_d + p.eps;
          const float inv = 1.0f / den;
          float o[kD];
#pragma unroll
          for (int r = 0; r < kD; ++r)
            o[r] = (__uint_as_float(v[r]) + __uint_as_float(v[kImageLoRow + r])) * inv;
          uint4 w[kChunksPerHead];
          pack_out(static_cast<OutT*>(nullptr), o, w);
          const int hu = h * kApHeads + j;   // head within the unit
          if (staged) {
            // 16-byte chunk ck of the unit's output row lands in box ck/8 at chunk
            // (ck%8) ^ (row%8): the 128B swizzle the TMA store expects
#pragma unroll
            for (int k = 0; k < kChunksPerHead; ++k) {
              const int ck = hu * kChunksPerHead + k;
              uint8_t* box = slot + (ck >> 3) * kOutBoxBytes;
              *reinterpret_cast<uint4*>(box + row * 128 + (((ck & 7) ^ (row & 7)) << 4)) = w[k];
            }
          } else if (n < U.tok1) {
            uint4* dst = reinterpret_cast<uint4*>(
                out + (((int64_t)U.b * p.N + n) * p.H + U.quad * kApUnitHeads + hu) * kD);
#pragma unroll
            for (int k = 0; k < kChunksPerHead; ++k) dst[k] = w[k];
          }
        }
        ++pn;
      }
      if (stop) break;
      if (staged) {
        fence_proxy_async_smem();
        bar_sync(2, 128);
        if (leader) {
          const int x0 = U.quad * kApUnitHeads * kD;
#pragma unroll
          for (int bx = 0; bx < Cfg::kOutBoxes; ++bx)
            if (x0 + bx * Cfg::kBoxChannels < p.H * kD)
              tma_store_3d(&tmap_out, slot + bx * kOutBoxBytes, x0 + bx * Cfg::kBoxChannels, U.tok0, U.b);
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_group<0>();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kApTmemCols);
  }
}

}  // namespace litela
