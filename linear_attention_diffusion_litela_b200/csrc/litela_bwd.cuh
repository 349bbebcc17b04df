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
// A call runs five kernels chained with programmatic dependent launch:
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
};

enum : int {
  kErrBwdQProducer = 0x510, kErrBwdQMma = 0x520, kErrBwdQRelu = 0x530, kErrBwdQEpi = 0x540,
  kErrBwdKvProducer = 0x610, kErrBwdKvMma = 0x620, kErrBwdKvRelu = 0x630, kErrBwdKvEpi = 0x640,
};

constexpr int kBwThreads = 256;   // w0 TMA, w1 MMA, w2..3 ReLU, w4..7 epilogue
constexpr int kBwStages = 2;
constexpr uint32_t kBwBoxBytes = kApTile * 128;        // 128 tokens x 64 channels (one head pair)
constexpr uint32_t kBwTileBytes = 2 * kBwBoxBytes;     // 4 heads
constexpr uint32_t kBwStageBytes = 2 * kBwTileBytes;   // two tensors: (q, dout) or (k, v)
constexpr uint32_t kBwHBytes = (kApTile / 16) * 512;   // 16 columns x 128 tokens, K-major
constexpr uint32_t kBwImgBytes = kApUnitHeads * (kImageBytes + kImageTBytes);
constexpr uint32_t kBwSlotCols = 144;                   // TMEM columns per head: 80 + 64
constexpr uint32_t kBwDsCol = 2 * kBwSlotCols;          // dS^T accumulator (128 columns)
constexpr uint32_t kBwDhCol = kBwDsCol + 128;           // its ones-row part (16 columns)
constexpr uint32_t kBwTmemCols = 512;
// litela_bwd_q_tc shared memory
constexpr uint32_t kBqOffGlo = kBwStages * kBwStageBytes;
constexpr uint32_t kBqOffH = kBqOffGlo + kBwTileBytes;
constexpr uint32_t kBqOffImg = kBqOffH + kBwHBytes;
constexpr uint32_t kBqOffBars = kBqOffImg + kBwImgBytes;
constexpr uint32_t kBqSmemBytes = kBqOffBars + 256 + 1024;
// litela_bwd_kv_tc shared memory
constexpr uint32_t kBkOffImg = kBwStages * kBwStageBytes;
constexpr uint32_t kBkOffBars = kBkOffImg + kBwImgBytes;
constexpr uint32_t kBkSmemBytes = kBkOffBars + 256 + 1024;

// byte offset of bf16 element (token t, channel ch of the 4 heads) in a tile of two 128B-swizzled
// TMA boxes (64 channels x 128 tokens each)
__device__ __forceinline__ uint32_t sw_offset(int t, int ch) {
  return (uint32_t)((ch >> 6) * kBwBoxBytes + t * 128 + ((((ch >> 3) & 7) ^ (t & 7)) << 4) + (ch & 7) * 2);
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
                const uint8_t* __restrict__ images, const uint8_t* __restrict__ images_t,
                float* __restrict__ dpartials, OutT* __restrict__ dqkv, int* __restrict__ err, BwdPlan p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* glo = smem + kBqOffGlo;    // g/den, lo halves (same layout as the g tile)
  uint8_t* hbuf = smem + kBqOffH;     // h hi (column j) and lo (column 4 + j) per token
  uint8_t* simg = smem + kBqOffImg;   // 4 S images, then 4 S^T images
  uint8_t* stimg = simg + kApUnitHeads * kImageBytes;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + kBqOffBars);
  uint64_t* qrelu = qfull + kBwStages;
  uint64_t* qempty = qrelu + kBwStages;
  uint64_t* sfull = qempty + kBwStages;
  uint64_t* tfull = sfull + 1;
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
      mbar_init(&qrelu[s], kApReluThreads);
      mbar_init(&qempty[s], 1);
    }
    mbar_init(sfull, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(gready, 128);
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
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

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
      if (sp.ntiles > 0) {
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
    }
  } else if (warp == 1) {
    if (lane == 0 && sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdQMma | 8)) {
      constexpr uint32_t idesc_y = idesc_bf16_f32(128, kImageRows, false, false);
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, kImageTRows, false, false);
      constexpr uint32_t idesc_ds = idesc_bf16_f32(128, 128, true, true);
      constexpr uint32_t idesc_dh = idesc_bf16_f32(128, 16, true, false);
      int hc = 0;
      bool stop = false;
      for (int i = 0; i < sp.ntiles && !stop; ++i) {
        const int s = i % kBwStages;
        if (!mbar_wait(&qrelu[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQMma | s)) break;
        tc_fence_after_sync();
        const uint32_t qa = smem_u32(qtile(s)), ga = smem_u32(gtile(s));
        for (int j = 0; j < sp.nh; ++j, ++hc) {
          const int a = hc & 1;
          if (hc >= 2 && !mbar_wait(&tempty[a], ((hc >> 1) - 1) & 1, abort_flag, err, kErrBwdQMma | 4 | a)) {
            stop = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t off = (j >> 1) * kBwBoxBytes + (j & 1) * 64;   // head j's 32 channels
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // y = q~ . S^T: A K-major 128B swizzle (8-token groups 1024 B apart), B = S image
            umma_bf16(tmem + a * kBwSlotCols, smem_desc(qa + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(simg + j * kImageBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_y, ks);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // T = g . S[0:d]: A = the raw dout tile, B = the S^T image
            umma_bf16(tmem + a * kBwSlotCols + kImageRows, smem_desc(ga + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(stimg + j * kImageTBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_t,
                      ks);
          }
          umma_commit(&tfull[a]);
        }
        if (stop) break;
        // the epilogue has written g/den (hi over the g tile, lo into glo) and h for this tile
        if (!mbar_wait(gready, i & 1, abort_flag, err, kErrBwdQMma | 12)) break;
        tc_fence_after_sync();
        const uint32_t la = smem_u32(glo), ha = smem_u32(hbuf);
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
      }
      umma_commit(dsfull);
    }
  } else if (warp < 4) {
    // ReLU of the q tiles in place (the raw dout tile is not touched)
    const int t = threadIdx.x - 64;
    const int nchunks = sp.np * (int)(kBwBoxBytes / 16);
    for (int i = 0; i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      if (!mbar_wait(&qfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQRelu | s)) break;
      uint8_t* st = qtile(s);
#pragma unroll 4
      for (int j = t; j < nchunks; j += kApReluThreads) {
        uint4* c = reinterpret_cast<uint4*>(st + j * 16);
        *c = relu_bf16x8(*c);
      }
      fence_proxy_async_smem();
      mbar_arrive(&qrelu[s]);
    }
  } else {
    // epilogue: thread = token row of the tile (TMEM lane)
    const int wq = warp & 3, row = wq * 32 + lane;
    bool ok = sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdQEpi | 8);
    int hc = 0;
    for (int i = 0; ok && i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      const int tok = sp.n0 + i * kApTile + row;
      const bool valid = tok < sp.n1;
      // the tile's TMA data (this thread reads dout and q~ from it; the stage cannot be refilled
      // before this epilogue releases it), and the previous tile's dS product has read glo, hbuf
      if (!mbar_wait(&qfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdQEpi | 14)) ok = false;
      if (ok && i > 0 && !mbar_wait(gfree, (i - 1) & 1, abort_flag, err, kErrBwdQEpi | 12)) ok = false;
      if (bar_any(1, 128, !ok)) {
        ok = false;
        break;
      }
      for (int j = 0; j < sp.nh; ++j, ++hc) {
        const int a = hc & 1;
        const bool okw = mbar_wait(&tfull[a], (hc >> 1) & 1, abort_flag, err, kErrBwdQEpi | a);
        if (bar_any(1, 128, !okw)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + (static_cast<uint32_t>(wq * 32) << 16) + a * kBwSlotCols;
        float o[kD], den;
        {
          uint32_t v[kImageRows];
#pragma unroll
          for (int k = 0; k < kImageRows / 16; ++k) tmem_ld_x16(ta + k * 16, v + k * 16);
          tmem_wait_ld();
          den = (__uint_as_float(v[kD]) + __uint_as_float(v[kImageLoRow + kD])) + p.eps;
          const float inv = 1.0f / den;
#pragma unroll
          for (int r = 0; r < kD; ++r) o[r] = (__uint_as_float(v[r]) + __uint_as_float(v[kImageLoRow + r])) * inv;
        }
        const float inv = 1.0f / den;
        // g (raw dout) of this token and head, from shared memory; h = -(g . out) / den
        float g[kD];
        uint8_t* gt = gtile(s);
        const uint8_t* qt = qtile(s);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          unpack_bf16x8(*reinterpret_cast<const uint4*>(gt + sw_offset(row, j * kD + k * 8)), g + 8 * k);
        float dot = 0.f;
#pragma unroll
        for (int r = 0; r < kD; ++r) dot = fmaf(g[r], o[r], dot);
        const float h = -dot * inv;
        uint32_t tv[kImageTRows];
#pragma unroll
        for (int k = 0; k < kImageTRows / 16; ++k) tmem_ld_x16(ta + kImageRows + k * 16, tv + k * 16);
        tmem_wait_ld();
        tc_fence_before_sync();
        mbar_arrive(&tempty[a]);
        // dq = relu'(q) * (S[0:d]^T g / den + h S[d]); S[d] (the ones row) from the S image
        const uint8_t* im = simg + j * kImageBytes;
        float dq[kD];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float qr[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(qt + sw_offset(row, j * kD + k * 8)), qr);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = 8 * k + e;
            const float z = bf16_at(im + image_offset(kD, c)) + bf16_at(im + image_offset(kImageLoRow + kD, c));
            const float t = (__uint_as_float(tv[c]) + __uint_as_float(tv[kD + c])) * inv;
            dq[c] = qr[e] > 0.f ? fmaf(z, h, t) : 0.f;
          }
        }
        if (valid) store_row32(dqkv + ((int64_t)b * p.N + tok) * (3 * p.H * kD) + (quad * kApUnitHeads + j) * kD, dq);
        // operands of the dS product: g/den over the g tile (hi) and into glo (lo); h hi / lo
        float ghi[8], glo8[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = valid ? g[8 * k + e] * inv : 0.f;
            ghi[e] = __bfloat162float(__float2bfloat16_rn(x));
            glo8[e] = x - ghi[e];
          }
          const uint32_t off = sw_offset(row, j * kD + k * 8);
          *reinterpret_cast<uint4*>(gt + off) = pack_bf16x8(ghi);
          *reinterpret_cast<uint4*>(glo + off) = pack_bf16x8(glo8);
        }
        const float hv = valid ? h : 0.f;
        const __nv_bfloat16 hh = __float2bfloat16_rn(hv);
        const __nv_bfloat16 hl = __float2bfloat16_rn(hv - __bfloat162float(hh));
        *reinterpret_cast<__nv_bfloat16*>(hbuf + h_offset(j, row)) = hh;
        *reinterpret_cast<__nv_bfloat16*>(hbuf + h_offset(kApUnitHeads + j, row)) = hl;
      }
      if (!ok) break;
      fence_proxy_async_smem();
      mbar_arrive(gready);
    }
    // the CTA's partial dS: warp quarter wq holds head wq's query channels (TMEM lanes)
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
      sv[kD] = __uint_as_float(hh[wq]) + __uint_as_float(hh[kApUnitHeads + wq]);
    }
    const int64_t nparts = (int64_t)p.nblk * p.cpb;
    float* dst = dpartials + ((((int64_t)b * p.nquads + quad) * nparts + blockIdx.x) * kRedHeads + wq) * kStateFloats;
#pragma unroll
    for (int r = 0; r < kRows; ++r) dst[r * kD + lane] = sv[r];   // dS[r][c = lane]
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
litela_bwd_kv_tc(const __grid_constant__ CUtensorMap tmap_kv, const uint8_t* __restrict__ dimages,
                 const uint8_t* __restrict__ dimages_t, OutT* __restrict__ dqkv, int* __restrict__ err, BwdPlan p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* dimg = smem + kBkOffImg;   // 4 dS images, then 4 dS^T images
  uint8_t* dtimg = dimg + kApUnitHeads * kImageBytes;
  uint64_t* kvfull = reinterpret_cast<uint64_t*>(smem + kBkOffBars);
  uint64_t* krelu = kvfull + kBwStages;
  uint64_t* kvempty = krelu + kBwStages;   // the MMAs' commit + the 128 epilogue threads
  uint64_t* sfull = kvempty + kBwStages;
  uint64_t* tfull = sfull + 1;
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
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&krelu[s], kApReluThreads);
      mbar_init(&kvempty[s], 1 + 128);
    }
    mbar_init(sfull, 1);
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
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_kv);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      auto load = [&](int i) {
        const int s = i % kBwStages;
        const int y = sp.n0 + i * kApTile;
        mbar_arrive_expect_tx(&kvfull[s], 2 * sp.np * kBwBoxBytes);
        for (int h = 0; h < sp.np; ++h) {
          const int x = quad * kApUnitHeads * kD + h * kApHeads * kD;
          tma_load_3d(ktile(s) + h * kBwBoxBytes, &tmap_kv, &kvfull[s], p.H * kD + x, y, b);
          tma_load_3d(vtile(s) + h * kBwBoxBytes, &tmap_kv, &kvfull[s], 2 * p.H * kD + x, y, b);
        }
      };
      const int pre = sp.ntiles < kBwStages ? sp.ntiles : kBwStages;
      for (int i = 0; i < pre; ++i) load(i);   // inputs: see litela_bwd_q_tc
      int issued = pre;
      bool images_loaded = false;
      pdl_wait_primary();   // the dS images come from the preceding scan
      if (sp.ntiles > 0) {
        mbar_arrive_expect_tx(sfull, sp.nh * (kImageBytes + kImageTBytes));
        for (int j = 0; j < sp.nh; ++j) {
          const int64_t im = ((int64_t)b * p.H + quad * kApUnitHeads + j) * p.nblk + sp.blk;
          bulk_load(dimg + j * kImageBytes, dimages + im * kImageBytes, kImageBytes, sfull);
          bulk_load(dtimg + j * kImageTBytes, dimages_t + im * kImageTBytes, kImageTBytes, sfull);
        }
        images_loaded = true;
      }
      for (int i = pre; i < sp.ntiles; ++i) {
        const int s = i % kBwStages;
        if (!mbar_wait(&kvempty[s], ((i / kBwStages) - 1) & 1, abort_flag, err, kErrBwdKvProducer | s)) break;
        load(i);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > kBwStages ? issued - kBwStages : 0); i < issued; ++i)
          mbar_drain(&kvfull[i % kBwStages], (i / kBwStages) & 1);
        if (images_loaded) mbar_drain(sfull, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdKvMma | 8)) {
      constexpr uint32_t idesc_k = idesc_bf16_f32(128, kImageTRows, false, false);
      constexpr uint32_t idesc_v = idesc_bf16_f32(128, kImageRows, false, false);
      int hc = 0;
      bool stop = false;
      for (int i = 0; i < sp.ntiles && !stop; ++i) {
        const int s = i % kBwStages;
        if (!mbar_wait(&krelu[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdKvMma | s)) break;
        tc_fence_after_sync();
        const uint32_t ka = smem_u32(ktile(s)), va = smem_u32(vtile(s));
        for (int j = 0; j < sp.nh; ++j, ++hc) {
          const int a = hc & 1;
          if (hc >= 2 && !mbar_wait(&tempty[a], ((hc >> 1) - 1) & 1, abort_flag, err, kErrBwdKvMma | 4 | a)) {
            stop = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t off = (j >> 1) * kBwBoxBytes + (j & 1) * 64;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // dk~ (before the ones row) = v . dS[0:d]: A = v (K-major), B = the dS^T image
            umma_bf16(tmem + a * kBwSlotCols, smem_desc(va + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(dtimg + j * kImageTBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_k, ks);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            // dv = k~ . dS^T: A = k~ (K-major), B = the dS image (rows r)
            umma_bf16(tmem + a * kBwSlotCols + kImageTRows, smem_desc(ka + off + ks * 32, 16, 1024, kSwizzle128B),
                      smem_desc(smem_u32(dimg + j * kImageBytes) + ks * 256, 128, 512, kSwizzleNone), idesc_v, ks);
          }
          umma_commit(&tfull[a]);
        }
        if (stop) break;
        umma_commit(&kvempty[s]);
      }
    }
  } else if (warp < 4) {
    const int t = threadIdx.x - 64;
    const int nchunks = sp.np * (int)(kBwBoxBytes / 16);
    for (int i = 0; i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      if (!mbar_wait(&kvfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdKvRelu | s)) break;
      uint8_t* st = ktile(s);
#pragma unroll 4
      for (int j = t; j < nchunks; j += kApReluThreads) {
        uint4* c = reinterpret_cast<uint4*>(st + j * 16);
        *c = relu_bf16x8(*c);
      }
      fence_proxy_async_smem();
      mbar_arrive(&krelu[s]);
    }
  } else {
    const int wq = warp & 3, row = wq * 32 + lane;
    bool ok = sp.ntiles > 0 && mbar_wait(sfull, 0, abort_flag, err, kErrBwdKvEpi | 8);
    int hc = 0;
    for (int i = 0; ok && i < sp.ntiles; ++i) {
      const int s = i % kBwStages;
      const int tok = sp.n0 + i * kApTile + row;
      const bool valid = tok < sp.n1;
      const uint8_t* kt = ktile(s);
      // the tile's TMA data (k~ is read here; the stage is refilled only after this thread's
      // arrival on kvempty)
      if (!mbar_wait(&kvfull[s], (i / kBwStages) & 1, abort_flag, err, kErrBwdKvEpi | 14)) ok = false;
      if (bar_any(1, 128, !ok)) {
        ok = false;
        break;
      }
      for (int j = 0; j < sp.nh; ++j, ++hc) {
        const int a = hc & 1;
        const bool okw = mbar_wait(&tfull[a], (hc >> 1) & 1, abort_flag, err, kErrBwdKvEpi | a);
        if (bar_any(1, 128, !okw)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t ta = tmem + (static_cast<uint32_t>(wq * 32) << 16) + a * kBwSlotCols;
        const uint8_t* im = dimg + j * kImageBytes;
        float x[kD];
        {
          uint32_t v[kImageTRows];
#pragma unroll
          for (int k = 0; k < kImageTRows / 16; ++k) tmem_ld_x16(ta + k * 16, v + k * 16);
          tmem_wait_ld();
          float kr[kD];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            unpack_bf16x8(*reinterpret_cast<const uint4*>(kt + sw_offset(row, j * kD + k * 8)), kr + 8 * k);
#pragma unroll
          for (int c = 0; c < kD; ++c) {
            const float z = bf16_at(im + image_offset(kD, c)) + bf16_at(im + image_offset(kImageLoRow + kD, c));
            const float t = (__uint_as_float(v[c]) + __uint_as_float(v[kD + c])) + z;
            x[c] = kr[c] > 0.f ? t : 0.f;
          }
        }
        const int64_t rowbase = ((int64_t)b * p.N + tok) * (3 * p.H * kD) + (quad * kApUnitHeads + j) * kD;
        if (valid) store_row32(dqkv + rowbase + p.H * kD, x);
        {
          uint32_t v[kImageRows];
#pragma unroll
          for (int k = 0; k < kImageRows / 16; ++k) tmem_ld_x16(ta + kImageTRows + k * 16, v + k * 16);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < kD; ++r) x[r] = __uint_as_float(v[r]) + __uint_as_float(v[kImageLoRow + r]);
        }
        tc_fence_before_sync();
        mbar_arrive(&tempty[a]);
        if (valid) store_row32(dqkv + rowbase + 2 * p.H * kD, x);
      }
      if (!ok) break;
      mbar_arrive(&kvempty[s]);   // this thread no longer reads the k tile
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
