// LiteLA backward on the 5th-generation tensor cores: the gradients of L = sum(dout * out)
// with respect to q, k and v, for the non-causal and the block-causal forward.
//
// Method.  The pages give the forward (Sana explainer, "What LiteLA actually computes"; instagit
// page "How Linear Attention Improves Efficiency in DiT for High-Resolution Images", sections
// "Mathematical Foundation" and "Video Generation and Constant-Memory KV Cache"); its gradient
// follows from the chain rule through the state route.  Per (batch, head), with
// k~ = relu(k), q~ = relu(q), S = [V;1] . k~^T ((d+1) x d; block-causal: the prefix state of
// the token's block), y = S q~, den = y[d] + eps, out = y[0:d] / den and g = dout:
//   dy[r] = g[r] / den (r < d),  dy[d] = h = -(g . out) / den
//   dq~   = S^T dy = (S[0:d]^T g) / den + h * S[d]              dq = dq~ * (q > 0)
//   dS    = sum over the tokens that use S of dy q~^T          (block-causal: the gradient of
//           block b's own state is the SUFFIX sum over blocks >= b of these per-block sums)
//   dk~   = dS^T [v;1] = dS[0:d]^T v + dS[d]                   dk = dk~ * (k > 0)
//   dv    = dS[0:d] k~
// relu'(0) = 0, as in PyTorch's ReLU backward.
//
// A call runs five kernels chained with programmatic dependent launch (three with one block per
// sequence: the dq and dk/dv kernels then sum the partial states into their images themselves,
// in the scans' order, and the two scans are not launched):
//   litela_reduce_tc, litela_state_scan   S (as in the forward) as B-operand images: S (rows r)
//                                         and S[0:d]^T (rows c), bf16 hi + lo
//   litela_bwd_q_tc                        per 128-token tile and head: y = q~ . S^T and
//                                          T = g . S[0:d] (tcgen05, TMEM), the epilogue forms dq
//                                          and writes g/den and h (bf16 hi + lo) into shared
//                                          memory; then, per tile, dS^T += q~^T . [g/den ; h]
//                                          accumulates in TMEM (4 heads at once: M = 4 x 32
//                                          query channels, N = 4 x 32 + 16) and each CTA writes
//                                          its partial dS
//   litela_state_scan (reverse)            partial dS -> per-block suffix sums, as images
//   litela_bwd_kv_tc                       per tile and head: dk~ = v . dS[0:d] (+ dS[d]) and
//                                          dv = k~ . dS[0:d]^T; masks and stores dk, dv
// Every product of bf16 inputs is exact in fp32; fp32 operands (S, dS, g/den, h) enter the
// tensor cores as bf16 hi + lo pairs (2^-17 relative), as in the forward's apply.
//
// Every mbarrier wait is bounded (sm100::mbar_wait): on a time-out the kernel records an error
// code, stops its loops, waits (bounded) for its own TMA copies, frees its TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "litela_plan.h"
#include "litela_tc.cuh"
#include "sm100_ptx.cuh"

namespace litela {

struct BwdPlan {
  int B, N, H, T, nblk, nquads, cpb, chunk;   // cpb CTAs of `chunk` tokens per (batch, quad, block)
  float eps;
  // fold_fwd > 0: the dq kernel forms its S images itself from the reduction's fold_fwd partial
  // states per quad (one block only), instead of loading a scan's images; fold_bwd > 0: the
  // dk/dv kernel forms its dS images from the dq kernel's fold_bwd partials per quad
  int fold_fwd, fold_bwd;
};

// The states of one block as a scan over that block's partials forms them (one block: the plain
// sum of its parts, visited first to last, or last to first for the reverse scan), for the
// nh * 33 * 32 elements (head j, element e) of this quad's partials at `base` (part k of element
// (j, e) at base + (k * 4 + j) * 33 * 32 + e).  Threads t = 0..nthreads-1 share the elements, 4
// at a time with 8 parts each in flight; write(j, r, c, sum, hi, lo) stores one element (row r,
// column c) with its bf16 hi + lo rounding.
template <typename Write>
__device__ __forceinline__ void fold_states(const float* __restrict__ base, int nh, int nparts, bool reverse, int t,
                                            int nthreads, Write write) {
  constexpr int kF = 4;
  constexpr int64_t kStride = (int64_t)kRedHeads * kStateFloats;
  const int total = nh * kStateFloats;
  for (int i0 = t; i0 < total; i0 += kF * nthreads) {
    const float* src[kF];
    bool ok[kF];
    float sum[kF];
#pragma unroll
    for (int f = 0; f < kF; ++f) {
      const int i = i0 + f * nthreads;
      ok[f] = i < total;
      src[f] = base + (ok[f] ? i : 0);   // (j, e) at j * 33 * 32 + e = i
      sum[f] = 0.f;
    }
    for (int k0 = 0; k0 < nparts; k0 += 8) {
      float v[kF][8];
#pragma unroll
      for (int f = 0; f < kF; ++f)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int k = reverse ? nparts - 1 - (k0 + q) : k0 + q;
          v[f][q] = (ok[f] && k0 + q < nparts) ? __ldcg(src[f] + k * kStride) : 0.f;
        }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (k0 + q < nparts) {
#pragma unroll
          for (int f = 0; f < kF; ++f) sum[f] += v[f][q];
        }
    }
#pragma unroll
    for (int f = 0; f < kF; ++f) {
      if (!ok[f]) continue;
      const int i = i0 + f * nthreads, j = i / kStateFloats, e = i - j * kStateFloats;
      const __nv_bfloat16 hi = __float2bfloat16_rn(sum[f]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(sum[f] - __bfloat162float(hi));
      write(j, e >> 5, e & 31, sum[f], hi, lo);
    }
  }
}

enum : int {
  kErrBwdQProducer = 0x510, kErrBwdQMma = 0x520, kErrBwdQRelu = 0x530, kErrBwdQEpi = 0x540,
  kErrBwdKvProducer = 0x610, kErrBwdKvMma = 0x620, kErrBwdKvRelu = 0x630, kErrBwdKvEpi = 0x640,
};

// w0 TMA (lane 0; in the dq kernel lane 1 issues the dS products), w1 MMA, w2..3 ReLU,
// w4..11 epilogue in two groups of 4 warps (group g takes the heads j with j % 2 == g; each
// group covers all 128 TMEM lanes)
constexpr int kBwThreads = 384;
constexpr int kBwEpiThreads = 256;
constexpr int kBwStages = 2;
constexpr uint32_t kBwBoxBytes = kApTile * 128;        // 128 tokens x 64 channels (one head pair)
constexpr uint32_t kBwTileBytes = 2 * kBwBoxBytes;     // 4 heads
constexpr uint32_t kBwStageBytes = 2 * kBwTileBytes;   // two tensors: (q, dout) or (k, v)
constexpr uint32_t kBwHBytes = (kApTile / 16) * 512;   // 16 columns x 128 tokens, K-major
constexpr uint32_t kBwImgBytes = kApUnitHeads * (kImageBytes + kImageTBytes);
// TMEM: two accumulator slots (slot g serves epilogue group g) of 144 columns: the products with
// an S (or dS) image (N = 80: hi rows 0..39, lo rows 40..79) and with an S^T image (N = 64: hi
// columns 0..31, lo 32..63); the epilogue adds the hi and lo halves.
constexpr uint32_t kBwSlotCols = kImageRows + kImageTRows;
constexpr uint32_t kBwDsCol = 2 * kBwSlotCols;          // dS^T accumulator (128 columns)
constexpr uint32_t kBwDhCol = kBwDsCol + 128;           // its ones-row part (16 columns)
constexpr uint32_t kBwTmemCols = 512;
// litela_bwd_q_tc shared memory
constexpr uint32_t kBqOffGlo = kBwStages * kBwStageBytes;
constexpr uint32_t kBqOffH = kBqOffGlo + kBwTileBytes;
constexpr uint32_t kBqOffImg = kBqOffH + kBwHBytes;
constexpr uint32_t kBqOffBars = kBqOffImg + kBwImgBytes;
constexpr uint32_t kBqOffZ = kBqOffBars + 256;            // ones rows S[d] in fp32, [4][32]
constexpr uint32_t kDqBoxBytes = kApTile * 64;            // one head's dq: 128 tokens x 32 channels
constexpr uint32_t kBqOffDq = (kBqOffZ + 512 + 1023) / 1024 * 1024;   // a staging box per group
constexpr uint32_t kBqSmemBytes = kBqOffDq + 2 * kDqBoxBytes + 1024;
// litela_bwd_kv_tc: 3 stages; the dS images hold rows 0..31 only (hi rows 0..31, lo rows 32..63)
// and the ones row dS[d] comes in fp32
constexpr int kBkStages = 3;
constexpr uint32_t kBkSlotCols = 2 * kImageTRows;          // dk~ (hi | lo) + dv (hi | lo)
constexpr uint32_t kBkOffImg = kBkStages * kBwStageBytes;
constexpr uint32_t kBkOffZ = kBkOffImg + kApUnitHeads * 2 * kImageTBytes;   // [4][32] fp32
constexpr uint32_t kBkOffBars = kBkOffZ + 512;
constexpr uint32_t kBkSmemBytes = kBkOffBars + 256 + 1024;

static_assert(kBqSmemBytes <= 232448 && kBkSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");
static_assert(2 * kBwSlotCols + 128 + 16 <= kBwTmemCols && 2 * kBkSlotCols <= kBwTmemCols, "TMEM columns");

// byte offset of bf16 element (token t, channel ch of the 4 heads) in a tile of two 128B-swizzled
// TMA boxes (64 channels x 128 tokens each)
__device__ __forceinline__ uint32_t sw_offset(int t, int ch) {
  return (uint32_t)((ch >> 6) * kBwBoxBytes + t * 128 + ((((ch >> 3) & 7) ^ (t & 7)) << 4) + (ch & 7) * 2);
}

// byte offset of bf16 element (token t, channel c < 32) in a 64B-swizzled TMA box of 32 channels
// x 128 tokens (16-byte chunk c/8 of row t sits at chunk (c/8) ^ ((t/2) & 3))
__device__ __forceinline__ uint32_t sw64_offset(int t, int c) {
  return (uint32_t)(t * 64 + ((((c >> 3) & 3) ^ ((t >> 1) & 3)) << 4) + (c & 7) * 2);
}

// byte offset of element (column j, token t) in the 16-column K-major tile of the h values
// (8 x 8 core matrices: K-direction stride 128 B, column-group stride 256 B, 512 B per 16 tokens)
__device__ __forceinline__ uint32_t h_offset(int j, int t) {
  return (uint32_t)((t >> 4) * 512 + (j >> 3) * 256 + ((t >> 3) & 1) * 128 + (j & 7) * 16 + (t & 7) * 2);
}

__device__ __forceinline__ void unpack_bf16x8(uint4 w, float* x) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(u[i] << 16);
    x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float bf16_at(const uint8_t* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(p)) << 16);
}

// true for element e (0..7) of 8 packed bf16 values that are not +0 (for values that went
// through ReLU: the element is > 0)
__device__ __forceinline__ bool bf16_nonzero(uint4 w, int e) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  return ((e & 1) ? (u[e >> 1] >> 16) : (u[e >> 1] & 0xFFFFu)) != 0u;
}

// fp32 copies (hi + lo) of the ones rows (row d) of the nh state images at `img`, into zf[j][c]
// (epilogue threads et = 0..127)
__device__ __forceinline__ void ones_rows_fp32(const uint8_t* img, int nh, float* zf, int et) {
  const int j = et >> 5, c = et & 31;
  if (j < nh)
    zf[et] = bf16_at(img + j * kImageBytes + image_offset(kD, c)) +
             bf16_at(img + j * kImageBytes + image_offset(kImageLoRow + kD, c));
}

// stores 32 values of one head's row to global memory (bf16: 4 x 16 B, fp32: 8 x 16 B)
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float* x) {
#pragma unroll
  for (int k = 0; k < 4; ++k) reinterpret_cast<uint4*>(dst)[k] = pack_bf16x8(x + 8 * k);
}
__device__ __forceinline__ void store_row32(float* dst, const float* x) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    reinterpret_cast<float4*>(dst)[k] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
}

// CTA (x = block * cpb + chunk, quad, b) covers tokens [n0, n1) of one causal block
struct BwSpan {
  int blk, n0, n1, ntiles, nh, np;
};
__device__ __forceinline__ BwSpan bw_span(const BwdPlan& p) {
  BwSpan s;
  const int x = blockIdx.x;
  s.blk = x / p.cpb;
  const int ch = x - s.blk * p.cpb;
  const int blk_end = min((s.blk + 1) * p.T, p.N);
  s.n0 = s.blk * p.T + ch * p.chunk;
  s.n1 = min(s.n0 + p.chunk, blk_end);
  s.ntiles = s.n1 > s.n0 ? (s.n1 - s.n0 + kApTile - 1) / kApTile : 0;
  s.nh = min(kApUnitHeads, p.H - (int)blockIdx.y * kApUnitHeads);
  s.np = s.nh > kApHeads ? 2 : 1;
  return s;
}

// ---------------------------------------------------------------------------------------
// dq and the partial dS

template <typename OutT>
__global__ void __launch_bounds__(kBwThreads, 1)
litela_bwd_q_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_g,
                const __grid_constant__ CUtensorMap tmap_dq, const uint8_t* __restrict__ images,
                const uint8_t* __restrict__ images_t, const float* __restrict__ fold_src,
                float* __restrict__ dpartials, OutT* __restrict__ dqkv, int* __restrict__ err, BwdPlan p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* glo = smem + kBqOffGlo;    // g/den, lo halves (same layout as the g tile)
  uint8_t* hbuf = smem + kBqOffH;     // h hi (column j) and lo (column 4 + j) per token
  uint8_t* simg = smem + kBqOffImg;   // 4 S images, then 4 S^T images
  uint8_t* stimg = simg + kApUnitHeads * kImageBytes;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + kBqOffBars);
  uint64_t* qrelu = qfull + kBwStages;        // [stage][box]: ReLU done for head pair `box`
  uint64_t* qempty = qrelu + 2 * kBwStages;
  uint64_t* sfull = qempty + kBwStages;
  uint64_t* tfull = sfull + 1;                 // one per TMEM slot
  uint64_t* tempty = tfull + 2;
  uint64_t* gready = tempty + 2;
  uint64_t* gfree = gready + 1;
  uint64_t* dsfull = gfree + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dsfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto qtile = [&](int s) { return smem + s * kBwStageBytes; };
  auto gtile = [&](int s) { return smem + s * kBwStageBytes + kBwTileBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = blockIdx.y, b = blockIdx.z;
  const BwSpan sp = bw_span(p);

  pdl_launch_dependents();   // the next kernel waits for this grid before touching memory
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qrelu[2 * s], kApReluThreads);
      mbar_init(&qrelu[2 * s + 1], kApReluThreads);
      mbar_init(&qempty[s], 1);
    }
    mbar_init(sfull, p.fold_fwd > 0 ? kBwEpiThreads : 1);   // the images: the epilogue's fold, or bulk copies
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(gready, kBwEpiThreads);
    mbar_init(gfree, 1);
    mbar_init(dsfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the lo tile and the h tile start at zero: columns of absent heads stay zero
  for (uint32_t i = threadIdx.x; i < (kBwTileBytes + kBwHBytes) / 16; i += kBwThreads)
    reinterpret_cast<uint4*>(glo)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_holder, kBwTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_g);
    prefetch_tensormap(&tmap_dq);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  // The dS product of tile i (issued by warp 0's lane 1, beside the head products of warp 1,
  // so that neither kind of product queues behind the other)
  constexpr uint32_t idesc_ds = idesc_bf16_f32(128, 128, true, true);
  constexpr uint32_t idesc_dh = idesc_bf16_f32(128, 16, true, false);
  const uint32_t la = smem_u32(glo), ha = smem_u32(hbuf);
  // the dS product of tile i, once its epilogue has written g/den (hi over the g tile, lo
  // into glo) and h
  auto ds_product = [&](int i) {
    const int s = i % kBwStages;
    tc_fence_after_sync();
    const uint32_t qa = smem_u32(qtile(s)), ga = smem_u32(gtile(s));
#pragma unroll
    for (int ks = 0; ks < kApTile / 16; ++ks) {
      // dS^T[c][r] += sum over 16 tokens of q~[t][c] (g/den)[t][r]: A = q~ MN-major (M = 4 heads
      // x 32 channels, the two boxes kBwBoxBytes apart), B = g/den MN-major, hi then lo
      const uint64_t ad = smem_desc(qa + ks * 2048, kBwBoxBytes, 1024, kSwizzle128B);
      const uint32_t acc = (i | ks) != 0;
      umma_bf16(tmem + kBwDsCol, ad, smem_desc(ga + ks * 2048, kBwBoxBytes, 1024, kSwizzle128B), idesc_ds, acc);
      umma_bf16(tmem + kBwDsCol, ad, smem_desc(la + ks * 2048, kBwBoxBytes, 1024, kSwizzle128B), idesc_ds, 1u);
      // the ones row: sum of q~[t][c] h[t] (h hi in column j, lo in column 4 + j)
      umma_bf16(tmem + kBwDhCol, ad, smem_desc(ha + ks * 512, 128, 256, kSwizzleNone), idesc_dh, acc);
    }
    umma_commit(&qempty[s]);
    umma_commit(gfree);
  };

  if (warp == 0) {
    if (lane == 0) {
      auto load = [&](int i) {
        const int s = i % kBwStages;
        const int y = sp.n0 + i * kApTile;
        mbar_arrive_expect_tx(&qfull[s], 2 * sp.np * kBwBoxBytes);
        for (int h = 0; h < sp.np; ++h) {
          const int x = quad * kApUnitHeads * kD + h * kApHeads * kD;
          tma_load_3d(qtile(s) + h * kBwBoxBytes, &tmap_q, &qfull[s], x, y, b);
          tma_load_3d(gtile(s) + h * kBwBoxBytes, &tmap_g, &qfull[s], x, y, b);
        }
      };
      // q and dout are inputs of the call: the call's first kernel released this chain only
      // after their producers finished, so they are read before waiting for the scan
      const int pre = sp.ntiles < kBwStages ? sp.ntiles : kBwStages;
      for (int i = 0; i < pre; ++i) load(i);
      int issued = pre;
      bool images_loaded = false;
      pdl_wait_primary();   // the S images come from the preceding scan
      if (sp.ntiles > 0 && p.fold_fwd == 0) {
        mbar_arrive_expect_tx(sfull, sp.nh * (kImageBytes + kImageTBytes));
        for (int j = 0; j < sp.nh; ++j) {
          const int64_t im = ((int64_t)b * p.H + quad * kApUnitHeads + j) * p.nblk + sp.blk;
          bulk_load(simg + j * kImageBytes, images + im * kImageBytes, kImageBytes, sfull);
          bulk_load(stimg + j * kImageTBytes, images_t + im * kImageTBytes, kImageTBytes, sfull);
        }
        images_loaded = true;
      }
      for (int i = pre; i < sp.ntiles; ++i) {
        const int s = i % kBwStages;
        if (!mbar_wait(&qempty[s], ((i / kBwStages) - 1) & 1, abort_flag, err, kErrBwdQProducer | s)) break;
        load(i);
        issued = i + 1;
      }
      if (*abort_flag) {   // let the copies still in flight land before the CTA exits (bounded)
        for (int i = (issued > kBwStages ? issued - kBwStages : 0); i < issued; ++i)
          mbar_drain(&qfull[i % kBwStages], (i / kBwStages) & 1);
        if (images_loaded) mbar_drain(sfull, 0);
      }
    } else if (lane == 1) {
      // the dS product of each tile once both epilogue groups have written its g/den and h
      // (gready); it frees the stage (qempty) and glo / hbuf (gfree).  dsfull follows the last.
      int i = 0;
      for (; i < sp.ntiles; ++i) {
        if (!mbar_wait(gready, i & 1, abort_flag, err, kErrBwdQMma | 13)) break;
        ds_product(i);
      }
      if (sp.ntiles > 0 && i == sp.ntiles) umma_commit(dsfull);
    }
  } else if (warp == 1) {
    if (lane == 0 && sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdQMma | 8)) {
      constexpr uint32_t idesc_y = idesc_bf16_f32(128, kImageRows, false, false);
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, kImageTRows, false, false);
      // The head products of tile i, once tile i's ReLU is done; each waits for its TMEM slot,
      // which the epilogue frees before it waits for any dS product (issued by another thread).
      int use[2] = {0, 0};
      bool stop = false;
      for (int i = 0; i < sp.ntiles && !stop; ++i) {
        const int s = i % kBwStages;
        if (!mbar_wait(&qrelu[2 * s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQMma | 12)) break;
        tc_fence_after_sync();
        const uint32_t qa = smem_u32(qtile(s)), ga = smem_u32(gtile(s));
        for (int j = 0; j < sp.nh; ++j) {
          const int a = j & 1;   // the slot of epilogue group j % 2
          if (j == kApHeads && !mbar_wait(&qrelu[2 * s + 1], (i / kBwStages) & 1, abort_flag, err, kErrBwdQMma | 3)) {
            stop = true;
            break;
          }
          if (use[a] > 0 && !mbar_wait(&tempty[a], (use[a] - 1) & 1, abort_flag, err, kErrBwdQMma | 4 | a)) {
            stop = true;
            break;
          }
          ++use[a];
          tc_fence_after_sync();
          const uint32_t off = (j >> 1) * kBwBoxBytes + (j & 1) * 64;   // head j's 32 channels
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // y = q~ . S^T: A K-major 128B swizzle (8-token groups 1024 B apart), B = S image
            umma_bf16(tmem + a * kBwSlotCols, smem_desc(qa + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(simg + j * kImageBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_y, ks);
            // T = g . S[0:d]: A = the raw dout tile, B = the S^T image
            umma_bf16(tmem + a * kBwSlotCols + kImageRows, smem_desc(ga + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(stimg + j * kImageTBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_t,
                      ks);
          }
          umma_commit(&tfull[a]);
        }
      }
    }
  } else if (warp < 4) {
    // ReLU of the q tiles in place (the raw dout tile is not touched), one head-pair box at a
    // time so that the first pair's products can start early
    const int t = threadIdx.x - 64;
    for (int i = 0; i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      if (!mbar_wait(&qfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQRelu | s)) break;
      for (int h = 0; h < sp.np; ++h) {
        uint8_t* st = qtile(s) + h * kBwBoxBytes;
#pragma unroll 8
        for (int j = t; j < (int)(kBwBoxBytes / 16); j += kApReluThreads) {
          uint4* c = reinterpret_cast<uint4*>(st + j * 16);
          *c = relu_bf16x8(*c);
        }
        fence_proxy_async_smem();
        mbar_arrive(&qrelu[2 * s + h]);
      }
    }
  } else {
    // epilogue: group g takes heads g, g + 2 through TMEM slot g; thread = token row (TMEM lane)
    const int g = (warp - 4) >> 2, wq = warp & 3, row = wq * 32 + lane;
    const int gbar = 1 + 2 * g;   // the group's named barrier (1 or 3)
    float* zf = reinterpret_cast<float*>(smem + kBqOffZ);
    // bf16 dq of a whole tile (or of the tile that ends at N) is staged in the group's box and
    // stored with TMA by the group's first thread; otherwise each thread stores its row
    uint8_t* dqbuf = smem + kBqOffDq + g * kDqBoxBytes;
    const bool storer = lane == 0 && wq == 0;
    if (p.fold_fwd > 0 && sp.ntiles > 0) {
      // the S and S^T images of the quad's heads from the reduction's partial states
      pdl_wait_primary();
      const int et = threadIdx.x - 128;
      fold_states(fold_src + ((int64_t)b * p.nquads + quad) * p.fold_fwd * kRedHeads * kStateFloats, sp.nh,
                  p.fold_fwd, false, et, kBwEpiThreads,
                  [&](int j, int r, int c, float, __nv_bfloat16 hi, __nv_bfloat16 lo) {
                    uint8_t* img = simg + j * kImageBytes;
                    *reinterpret_cast<__nv_bfloat16*>(img + image_offset(r, c)) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(img + image_offset(kImageLoRow + r, c)) = lo;
                    if (r < kD) {
                      uint8_t* imt = stimg + j * kImageTBytes;
                      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(c, r)) = hi;
                      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(kD + c, r)) = lo;
                    }
                  });
      for (int i = et; i < sp.nh * (kImageRows - 2 * kRows) * kD; i += kBwEpiThreads) {   // the zero rows
        const int j = i / ((kImageRows - 2 * kRows) * kD), k = i - j * ((kImageRows - 2 * kRows) * kD);
        const int zr = k >> 5, c = k & 31, half = kImageLoRow - kRows;
        const int nrow = zr < half ? kRows + zr : kImageLoRow + kRows + (zr - half);
        *reinterpret_cast<__nv_bfloat16*>(simg + j * kImageBytes + image_offset(nrow, c)) = __float2bfloat16_rn(0.f);
      }
      fence_proxy_async_smem();
      mbar_arrive(sfull);
    }
    bool ok = sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdQEpi | 8);
    if (ok && threadIdx.x < 256) ones_rows_fp32(simg, sp.nh, zf, threadIdx.x - 128);
    bar_sync(2, kBwEpiThreads);
    int use = 0;
    for (int i = 0; ok && i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      const int tok0 = sp.n0 + i * kApTile, tok = tok0 + row;
      const bool valid = tok < sp.n1;
      const bool staged = sizeof(OutT) == 2 && (tok0 + kApTile <= sp.n1 || sp.n1 == p.N);
      // the tile's TMA data (this thread reads dout and q~ from it; the stage cannot be refilled
      // before this epilogue releases it)
      if (!mbar_wait(&qfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQEpi | 14)) ok = false;
      if (bar_any(gbar, 128, !ok)) {
        ok = false;
        break;
      }
      bool first = true;
      for (int j = g; j < sp.nh; j += 2) {
        const bool okw = mbar_wait(&tfull[g], use & 1, abort_flag, err, kErrBwdQEpi | g);
        ++use;
        if (storer) bulk_wait_group_read<0>();   // the group's previous dq store has read its box
        if (bar_any(gbar, 128, !okw)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + (static_cast<uint32_t>(wq * 32) << 16) + g * kBwSlotCols;
        uint8_t* gt = gtile(s);
        const uint8_t* qt = qtile(s);
        // g (raw dout) of this token and head, from shared memory
        uint4 gw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) gw[k] = *reinterpret_cast<const uint4*>(gt + sw_offset(row, j * kD + k * 8));
        // den and h = -(g . out) / den = -(g . y[0:d]) / den^2
        float inv, h;
        {
          uint32_t v[kImageRows];
#pragma unroll
          for (int k = 0; k < kImageRows / 16; ++k) tmem_ld_x16(ta + k * 16, v + k * 16);
          tmem_wait_ld();
          inv = 1.0f / ((__uint_as_float(v[kD]) + __uint_as_float(v[kImageLoRow + kD])) + p.eps);
          float dot = 0.f;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float g8[8];
            unpack_bf16x8(gw[k], g8);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dot = fmaf(g8[e], __uint_as_float(v[8 * k + e]) + __uint_as_float(v[kImageLoRow + 8 * k + e]), dot);
          }
          h = -dot * inv * inv;
        }
        uint32_t tv[kImageTRows];
#pragma unroll
        for (int k = 0; k < kImageTRows / 16; ++k) tmem_ld_x16(ta + kImageRows + k * 16, tv + k * 16);
        tmem_wait_ld();
        tc_fence_before_sync();
        mbar_arrive(&tempty[g]);
        // dq = relu'(q) * (S[0:d]^T g / den + h S[d]); relu(q) > 0 <=> its bf16 bits are not 0
        const float4* z4 = reinterpret_cast<const float4*>(zf + j * kD);
        float dq[kD];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 qw = *reinterpret_cast<const uint4*>(qt + sw_offset(row, j * kD + k * 8));
          const float4 za = z4[2 * k], zb = z4[2 * k + 1];
          const float z[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = 8 * k + e;
            const float t = (__uint_as_float(tv[c]) + __uint_as_float(tv[kD + c])) * inv;
            dq[c] = bf16_nonzero(qw, e) ? fmaf(z[e], h, t) : 0.f;
          }
        }
        if (staged) {
#pragma unroll
          for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(dqbuf + sw64_offset(row, 8 * k)) = pack_bf16x8(dq + 8 * k);
          fence_proxy_async_smem();
          bar_sync(gbar, 128);
          if (storer) {
            tma_store_3d(&tmap_dq, dqbuf, (quad * kApUnitHeads + j) * kD, tok0, b);
            bulk_commit_group();
          }
        } else if (valid) {
          store_row32(dqkv + ((int64_t)b * p.N + tok) * (3 * p.H * kD) + (quad * kApUnitHeads + j) * kD, dq);
        }
        // the previous tile's dS product has read glo and hbuf (the columns of other heads of
        // the g tile are not touched below)
        if (first && i > 0) {
          const bool okg = mbar_wait(gfree, (i - 1) & 1, abort_flag, err, kErrBwdQEpi | 12);
          if (bar_any(gbar, 128, !okg)) {
            ok = false;
            break;
          }
        }
        first = false;
        // operands of the dS product: g/den over the g tile (hi) and into glo (lo); h hi / lo
        const float sc = valid ? inv : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t gu[4] = {gw[k].x, gw[k].y, gw[k].z, gw[k].w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float x0 = __uint_as_float(gu[e2] << 16) * sc, x1 = __uint_as_float(gu[e2] & 0xFFFF0000u) * sc;
            __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
            const uint32_t hu = *reinterpret_cast<uint32_t*>(&hp);
            __nv_bfloat162 lp = __floats2bfloat162_rn(x0 - __uint_as_float(hu << 16), x1 - __uint_as_float(hu & 0xFFFF0000u));
            hw[e2] = hu;
            lw[e2] = *reinterpret_cast<uint32_t*>(&lp);
          }
          const uint32_t off = sw_offset(row, j * kD + k * 8);
          *reinterpret_cast<uint4*>(gt + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(glo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        const float hv = valid ? h : 0.f;
        const __nv_bfloat16 hh = __float2bfloat16_rn(hv);
        const __nv_bfloat16 hl = __float2bfloat16_rn(hv - __bfloat162float(hh));
        *reinterpret_cast<__nv_bfloat16*>(hbuf + h_offset(j, row)) = hh;
        *reinterpret_cast<__nv_bfloat16*>(hbuf + h_offset(kApUnitHeads + j, row)) = hl;
      }
      if (!ok) break;
      // a group without heads in this quad (nh == 1) skips to here and still takes part; it
      // too waits for the previous tile's dS product first, so that its arrival cannot run a
      // tile ahead and complete this tile's phase before the other group has written g/den
      if (first && i > 0) {
        const bool okg = mbar_wait(gfree, (i - 1) & 1, abort_flag, err, kErrBwdQEpi | 15);
        if (bar_any(gbar, 128, !okg)) {
          ok = false;
          break;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(gready);
    }
    if (storer) bulk_wait_group<0>();
    // the CTA's partial dS (group 0): warp quarter wq holds head wq's query channels (TMEM lanes)
    if (g == 0) {
      float sv[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) sv[r] = 0.f;
      if (ok && sp.ntiles > 0) ok = mbar_wait(dsfull, 0, abort_flag, err, kErrBwdQEpi | 13);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && sp.ntiles > 0 && wq < sp.nh) {
        tc_fence_after_sync();
        uint32_t rr[32], hh[16];
        const uint32_t ta = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        tmem_ld_x32(ta + kBwDsCol + wq * 32, rr);
        tmem_ld_x16(ta + kBwDhCol, hh);
        tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < kD; ++r) sv[r] = __uint_as_float(rr[r]);
        // columns wq and 4 + wq of the ones-row part (selected without dynamic register indexing)
        float zsum = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (c == wq || c == kApUnitHeads + wq) zsum += __uint_as_float(hh[c]);
        sv[kD] = zsum;
      }
      const int64_t nparts = (int64_t)p.nblk * p.cpb;
      float* dst = dpartials + ((((int64_t)b * p.nquads + quad) * nparts + blockIdx.x) * kRedHeads + wq) * kStateFloats;
#pragma unroll
      for (int r = 0; r < kRows; ++r) dst[r * kD + lane] = sv[r];   // dS[r][c = lane]
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// dk and dv

template <typename OutT>
__global__ void __launch_bounds__(kBwThreads, 1)
litela_bwd_kv_tc(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_dqkv,
                 const uint8_t* __restrict__ dimages, const uint8_t* __restrict__ dimages_t,
                 const float* __restrict__ dzrows, const float* __restrict__ fold_src, OutT* __restrict__ dqkv,
                 int* __restrict__ err, BwdPlan p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* dimg = smem + kBkOffImg;   // 4 dS images (rows r), then 4 dS^T images (rows c)
  uint8_t* dtimg = dimg + kApUnitHeads * kImageTBytes;
  float* zf = reinterpret_cast<float*>(smem + kBkOffZ);   // dS[d] of the 4 heads
  uint64_t* kvfull = reinterpret_cast<uint64_t*>(smem + kBkOffBars);
  uint64_t* krelu = kvfull + kBkStages;        // [stage][box]: ReLU done for head pair `box`
  uint64_t* kvempty = krelu + 2 * kBkStages;   // the MMAs' commit + the epilogue's storing thread
  uint64_t* sfull = kvempty + kBkStages;
  uint64_t* tfull = sfull + 1;             // one per TMEM slot
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto ktile = [&](int s) { return smem + s * kBwStageBytes; };
  auto vtile = [&](int s) { return smem + s * kBwStageBytes + kBwTileBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = blockIdx.y, b = blockIdx.z;
  const BwSpan sp = bw_span(p);

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBkStages; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&krelu[2 * s], kApReluThreads);
      mbar_init(&krelu[2 * s + 1], kApReluThreads);
      mbar_init(&kvempty[s], 2);
    }
    mbar_init(sfull, p.fold_bwd > 0 ? kBwEpiThreads : 1);   // the images: the epilogue's fold, or bulk copies
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kBwTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_kv);
    prefetch_tensormap(&tmap_dqkv);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      auto load = [&](int i) {
        const int s = i % kBkStages;
        const int y = sp.n0 + i * kApTile;
        mbar_arrive_expect_tx(&kvfull[s], 2 * sp.np * kBwBoxBytes);
        for (int h = 0; h < sp.np; ++h) {
          const int x = quad * kApUnitHeads * kD + h * kApHeads * kD;
          tma_load_3d(ktile(s) + h * kBwBoxBytes, &tmap_kv, &kvfull[s], p.H * kD + x, y, b);
          tma_load_3d(vtile(s) + h * kBwBoxBytes, &tmap_kv, &kvfull[s], 2 * p.H * kD + x, y, b);
        }
      };
      const int pre = sp.ntiles < kBkStages ? sp.ntiles : kBkStages;
      for (int i = 0; i < pre; ++i) load(i);   // inputs: see litela_bwd_q_tc
      int issued = pre;
      bool images_loaded = false;
      pdl_wait_primary();   // the dS images come from the preceding scan
      if (sp.ntiles > 0 && p.fold_bwd == 0) {
        mbar_arrive_expect_tx(sfull, sp.nh * (2 * kImageTBytes + kD * 4));
        for (int j = 0; j < sp.nh; ++j) {
          const int64_t im = ((int64_t)b * p.H + quad * kApUnitHeads + j) * p.nblk + sp.blk;
          bulk_load(dimg + j * kImageTBytes, dimages + im * kImageTBytes, kImageTBytes, sfull);
          bulk_load(dtimg + j * kImageTBytes, dimages_t + im * kImageTBytes, kImageTBytes, sfull);
          bulk_load(zf + j * kD, dzrows + im * kD, kD * 4, sfull);
        }
        images_loaded = true;
      }
      for (int i = pre; i < sp.ntiles; ++i) {
        const int s = i % kBkStages;
        if (!mbar_wait(&kvempty[s], ((i / kBkStages) - 1) & 1, abort_flag, err, kErrBwdKvProducer | s)) break;
        load(i);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > kBkStages ? issued - kBkStages : 0); i < issued; ++i)
          mbar_drain(&kvfull[i % kBkStages], (i / kBkStages) & 1);
        if (images_loaded) mbar_drain(sfull, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdKvMma | 8)) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kImageTRows, false, false);
      int use[2] = {0, 0};
      bool stop = false;
      for (int i = 0; i < sp.ntiles && !stop; ++i) {
        const int s = i % kBkStages;
        if (!mbar_wait(&krelu[2 * s], (i / kBkStages) & 1, abort_flag, err, kErrBwdKvMma | s)) break;
        tc_fence_after_sync();
        const uint32_t ka = smem_u32(ktile(s)), va = smem_u32(vtile(s));
        for (int j = 0; j < sp.nh; ++j) {
          const int a = j & 1;
          if (j == kApHeads && !mbar_wait(&krelu[2 * s + 1], (i / kBkStages) & 1, abort_flag, err, kErrBwdKvMma | 3)) {
            stop = true;
            break;
          }
          if (use[a] > 0 && !mbar_wait(&tempty[a], (use[a] - 1) & 1, abort_flag, err, kErrBwdKvMma | 4 | a)) {
            stop = true;
            break;
          }
          ++use[a];
          tc_fence_after_sync();
          const uint32_t off = (j >> 1) * kBwBoxBytes + (j & 1) * 64;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // dk~ (before the ones row) = v . dS[0:d]: A = v (K-major), B = the dS^T image
            umma_bf16(tmem + a * kBkSlotCols, smem_desc(va + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(dtimg + j * kImageTBytes) + ks * 256, 128, 512, kSwizzleNone), idesc, ks);
            // dv = k~ . dS[0:d]^T: A = k~ (K-major), B = the dS image (rows r)
            umma_bf16(tmem + a * kBkSlotCols + kImageTRows, smem_desc(ka + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(dimg + j * kImageTBytes) + ks * 256, 128, 512, kSwizzleNone), idesc, ks);
          }
          umma_commit(&tfull[a]);
        }
        if (stop) break;
        umma_commit(&kvempty[s]);
      }
    }
  } else if (warp < 4) {
    // ReLU of the k tiles in place, one head-pair box at a time
    const int t = threadIdx.x - 64;
    for (int i = 0; i < sp.ntiles; ++i) {
      const int s = i % kBkStages;
      if (!mbar_wait(&kvfull[s], (i / kBkStages) & 1, abort_flag, err, kErrBwdKvRelu | s)) break;
      for (int h = 0; h < sp.np; ++h) {
        uint8_t* st = ktile(s) + h * kBwBoxBytes;
#pragma unroll 8
        for (int j = t; j < (int)(kBwBoxBytes / 16); j += kApReluThreads) {
          uint4* c = reinterpret_cast<uint4*>(st + j * 16);
          *c = relu_bf16x8(*c);
        }
        fence_proxy_async_smem();
        mbar_arrive(&krelu[2 * s + h]);
      }
    }
  } else {
    // epilogue: group g takes heads g, g + 2 through TMEM slot g; thread = token row (TMEM lane)
    const int g = (warp - 4) >> 2, wq = warp & 3, row = wq * 32 + lane;
    const int gbar = 1 + 2 * g;
    if (p.fold_bwd > 0 && sp.ntiles > 0) {
      // the dS images (rows 0..d-1 and their transposes) and dS[d] of the quad's heads from the
      // dq kernel's partials, summed last to first as the reverse scan does
      pdl_wait_primary();
      fold_states(fold_src + ((int64_t)b * p.nquads + quad) * p.fold_bwd * kRedHeads * kStateFloats, sp.nh,
                  p.fold_bwd, true, threadIdx.x - 128, kBwEpiThreads,
                  [&](int j, int r, int c, float sum, __nv_bfloat16 hi, __nv_bfloat16 lo) {
                    if (r < kD) {
                      uint8_t* img = dimg + j * kImageTBytes;
                      *reinterpret_cast<__nv_bfloat16*>(img + image_offset(r, c)) = hi;
                      *reinterpret_cast<__nv_bfloat16*>(img + image_offset(kD + r, c)) = lo;
                      uint8_t* imt = dtimg + j * kImageTBytes;
                      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(c, r)) = hi;
                      *reinterpret_cast<__nv_bfloat16*>(imt + image_offset(kD + c, r)) = lo;
                    } else {
                      zf[j * kD + c] = sum;
                    }
                  });
      fence_proxy_async_smem();
      mbar_arrive(sfull);
    }
    bool ok = sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdKvEpi | 8);
    // bf16 results of a whole tile are written over the k and v tiles they came from (each
    // head's columns once its products are done and its mask is read) and stored with TMA:
    // when the quad's heads fill whole boxes and the tile is whole or ends at N (a TMA store is
    // clipped only at N).  Otherwise each thread stores its row.
    const bool stage_ok = sizeof(OutT) == 2 && (sp.nh % 2) == 0;
    const bool storer = threadIdx.x == 128;
    int pending = -1;   // (storer) stage whose TMA stores may still be reading it
    int use = 0;
    for (int i = 0; ok && i < sp.ntiles; ++i) {
      const int s = i % kBkStages;
      const int tok0 = sp.n0 + i * kApTile, tok = tok0 + row;
      const bool valid = tok < sp.n1;
      const bool staged = stage_ok && (tok0 + kApTile <= sp.n1 || sp.n1 == p.N);
      uint8_t* kt = ktile(s);
      uint8_t* vt = vtile(s);
      // the tile's TMA data (k~ is read here; the stage is refilled only after its release)
      if (!mbar_wait(&kvfull[s], (i / kBkStages) & 1, abort_flag, err, kErrBwdKvEpi | 14)) ok = false;
      if (bar_any(2, kBwEpiThreads, !ok)) {
        ok = false;
        break;
      }
      for (int j = g; j < sp.nh; j += 2) {
        const bool okw = mbar_wait(&tfull[g], use & 1, abort_flag, err, kErrBwdKvEpi | g);
        ++use;
        if (bar_any(gbar, 128, !okw)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + (static_cast<uint32_t>(wq * 32) << 16) + g * kBkSlotCols;
        const float4* z4 = reinterpret_cast<const float4*>(zf + j * kD);
        const int64_t rowbase = ((int64_t)b * p.N + tok) * (3 * p.H * kD) + (quad * kApUnitHeads + j) * kD;
        float x[kD];
        {
          uint32_t v[kImageTRows];
#pragma unroll
          for (int k = 0; k < kImageTRows / 16; ++k) tmem_ld_x16(ta + k * 16, v + k * 16);
          tmem_wait_ld();
          // dk = relu'(k) * (v . dS[0:d] + dS[d]); relu(k) > 0 <=> its bf16 bits are not 0
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 kw = *reinterpret_cast<const uint4*>(kt + sw_offset(row, j * kD + k * 8));
            const float4 za = z4[2 * k], zb = z4[2 * k + 1];
            const float z[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = 8 * k + e;
              const float t = (__uint_as_float(v[c]) + __uint_as_float(v[kD + c])) + z[e];
              x[c] = bf16_nonzero(kw, e) ? t : 0.f;
            }
          }
        }
        if (staged) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(kt + sw_offset(row, j * kD + k * 8)) = pack_bf16x8(x + 8 * k);
        } else if (valid) {
          store_row32(dqkv + rowbase + p.H * kD, x);
        }
        {
          uint32_t v[kImageTRows];
#pragma unroll
          for (int k = 0; k < kImageTRows / 16; ++k) tmem_ld_x16(ta + kImageTRows + k * 16, v + k * 16);
          tmem_wait_ld();
          tc_fence_before_sync();
          mbar_arrive(&tempty[g]);
#pragma unroll
          for (int r = 0; r < kD; ++r) x[r] = __uint_as_float(v[r]) + __uint_as_float(v[kD + r]);
        }
        if (staged) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(vt + sw_offset(row, j * kD + k * 8)) = pack_bf16x8(x + 8 * k);
        } else if (valid) {
          store_row32(dqkv + rowbase + 2 * p.H * kD, x);
        }
      }
      fence_proxy_async_smem();
      if (bar_any(2, kBwEpiThreads, !ok)) {   // every epilogue thread has written its rows
        ok = false;
        break;
      }
      if (storer) {
        // a stage is released (kvempty) once the stores out of it have read it; that wait is
        // deferred by one tile so that the epilogue goes on with the next tile meanwhile
        if (staged) {
          for (int h = 0; h < sp.np; ++h) {
            const int x0 = quad * kApUnitHeads * kD + h * kApHeads * kD;
            tma_store_3d(&tmap_dqkv, kt + h * kBwBoxBytes, p.H * kD + x0, tok0, b);
            tma_store_3d(&tmap_dqkv, vt + h * kBwBoxBytes, 2 * p.H * kD + x0, tok0, b);
          }
          bulk_commit_group();
          if (pending >= 0) {
            bulk_wait_group_read<1>();
            mbar_arrive(&kvempty[pending]);
          }
          pending = s;
        } else {
          if (pending >= 0) {
            bulk_wait_group_read<0>();
            mbar_arrive(&kvempty[pending]);
            pending = -1;
          }
          mbar_arrive(&kvempty[s]);
        }
      }
    }
    if (storer) {
      bulk_wait_group<0>();
      if (pending >= 0) mbar_arrive(&kvempty[pending]);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

}  // namespace litela
