// SIMT (CUDA-core fp32 FMA) kernels of the LiteLA forward.
//
//   litela_reduce_simt : phi(K) = ReLU(K) fused with the state reduction
//                        S = [V;1] . phi(K)^T over one chunk of tokens, written as a partial
//                        state; the last chunk of a (batch, head) to finish merges the
//                        partials in fixed order into the per-block (prefix) states.
//   litela_apply_simt  : y = S . ReLU(q), out = y[:d] / (y[d] + eps).
//
// Method: Sana explainer "Sana: the autoencoder does more of the work than the linear
// attention", section "What LiteLA actually computes" (ReLU kernel, ones-padded V, two
// contractions, division by the last row plus eps); block-causal prefix: instagit page "How
// Linear Attention Improves Efficiency in DiT for High-Resolution Images", section "Video
// Generation and Constant-Memory KV Cache".
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "litela_plan.h"

namespace litela {

struct DevPlan {
  int B, N, H, T, nblk, chunks_per_block, chunk, tiles_per_block;
  float eps;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Reduce: grid (nblk * chunks_per_block, H, B), 256 threads.
// Work split inside the CTA: 4 token lanes x (8 row groups x 8 column groups) of 4x4.
constexpr int kReduceThreads = 256;

__global__ void __launch_bounds__(kReduceThreads)
litela_reduce_simt(const __nv_bfloat16* __restrict__ qkv, float* __restrict__ partials,
                   float* __restrict__ states, unsigned* __restrict__ counters, DevPlan p) {
  __shared__ __align__(16) float ks[kReduceTile][kD];      // relu(k), fp32
  __shared__ __align__(16) float vs[kReduceTile][kD];      // v, fp32
  __shared__ __align__(16) float red[4][kStateFloats];     // per token-lane partial states
  __shared__ bool is_last;

  const int x = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int blk = x / p.chunks_per_block, ch = x - blk * p.chunks_per_block;
  const int blk_end = min((blk + 1) * p.T, p.N);
  const int n0 = blk * p.T + ch * p.chunk;
  const int n1 = min(n0 + p.chunk, blk_end);

  const int t = threadIdx.x;
  const int tl = t >> 6, u = t & 63, rg = u >> 3, cg = u & 7;
  float acc[4][4] = {};
  float z[4] = {};

  const int64_t row = 3LL * p.H * kD;                      // elements per token row
  const __nv_bfloat16* base = qkv + (int64_t)b * p.N * row;
  // loader role: threads 0..127 load k, 128..255 load v; 4 x 16 B per token
  const int lt = (t & 127) >> 2, part = t & 3;
  const int which = (t < 128) ? 1 : 2;                      // 1 = k, 2 = v
  const int64_t col = ((int64_t)which * p.H + h) * kD + part * 8;

  for (int tile0 = n0; tile0 < n1; tile0 += kReduceTile) {
    const int n = tile0 + lt;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (n < n1) w = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)n * row + col));
    float f[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                  bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
    float* dst = (which == 1) ? &ks[lt][part * 8] : &vs[lt][part * 8];
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = (which == 1) ? fmaxf(f[i], 0.f) : f[i];
    __syncthreads();
#pragma unroll 4
    for (int tk = tl; tk < kReduceTile; tk += 4) {
      const float4 k4 = *reinterpret_cast<const float4*>(&ks[tk][cg * 4]);
      const float4 v4 = *reinterpret_cast<const float4*>(&vs[tk][rg * 4]);
      const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
      const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(vv[i], kk[j], acc[i][j]);
      if (rg == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) z[j] += kk[j];
      }
    }
    __syncthreads();
  }

  // combine the 4 token lanes in fixed order
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[tl][(rg * 4 + i) * kD + cg * 4 + j] = acc[i][j];
  if (rg == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) red[tl][kD * kD + cg * 4 + j] = z[j];
  }
  __syncthreads();
  const int64_t head = (int64_t)b * p.H + h;
  const int64_t nparts = (int64_t)p.nblk * p.chunks_per_block;
  float* part_out = partials + (head * nparts + x) * kStateFloats;
  for (int e = t; e < kStateFloats; e += kReduceThreads)
    part_out[e] = ((red[0][e] + red[1][e]) + red[2][e]) + red[3][e];

  // last-arriving CTA of this (batch, head) merges: no waiting, only an arrival count
  __threadfence();
  __syncthreads();
  if (t == 0) is_last = (atomicAdd(&counters[head], 1u) == (unsigned)(nparts - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const float* hp = partials + head * nparts * kStateFloats;
  float* hs = states + head * p.nblk * kStateFloats;
  for (int e = t; e < kStateFloats; e += kReduceThreads) {
    float run = 0.f;
    for (int bb = 0; bb < p.nblk; ++bb) {
      float s = 0.f;
      for (int c = 0; c < p.chunks_per_block; ++c)
        s += __ldcg(hp + ((int64_t)bb * p.chunks_per_block + c) * kStateFloats + e);
      run += s;
      hs[(int64_t)bb * kStateFloats + e] = run;
    }
  }
  if (t == 0) counters[head] = 0u;
}

// Apply: grid (nblk * tiles_per_block, H, B), kApplyTile threads, one query token each.
template <typename OutT>
__device__ __forceinline__ void store_out(OutT* dst, const float* o);

template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, const float* o) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 v2 = __floats2bfloat162_rn(o[i * 8 + 2 * j], o[i * 8 + 2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&v2);
    }
    d4[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <>
__device__ __forceinline__ void store_out<float>(float* dst, const float* o) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d4[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

template <typename OutT>
__global__ void __launch_bounds__(kApplyTile)
litela_apply_simt(const __nv_bfloat16* __restrict__ qkv, const float* __restrict__ states,
                  OutT* __restrict__ out, DevPlan p) {
  constexpr int kRowsPad = 36;                               // 33 rows padded to 9 float4
  __shared__ __align__(16) float St[kD][kRowsPad];           // St[c][r] = S[r][c]
  const int x = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int blk = x / p.tiles_per_block, tile = x - blk * p.tiles_per_block;
  const int64_t head = (int64_t)b * p.H + h;
  const float* S = states + (head * p.nblk + blk) * kStateFloats;
  for (int e = threadIdx.x; e < kD * kRowsPad; e += kApplyTile) {
    const int c = e / kRowsPad, r = e - c * kRowsPad;
    St[c][r] = (r < kRows) ? S[r * kD + c] : 0.f;
  }
  __syncthreads();

  const int n = blk * p.T + tile * kApplyTile + threadIdx.x;
  const int blk_end = min((blk + 1) * p.T, p.N);
  if (n >= blk_end) return;
  const int64_t row = 3LL * p.H * kD;
  const uint4* qp = reinterpret_cast<const uint4*>(qkv + ((int64_t)b * p.N + n) * row + (int64_t)h * kD);
  float q[kD];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldg(qp + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      q[i * 8 + 2 * j] = fmaxf(bf16_lo(ws[j]), 0.f);
      q[i * 8 + 2 * j + 1] = fmaxf(bf16_hi(ws[j]), 0.f);
    }
  }
  float y[kRowsPad] = {};
#pragma unroll
  for (int c = 0; c < kD; ++c) {
#pragma unroll
    for (int r4 = 0; r4 < kRowsPad / 4; ++r4) {
      const float4 s = *reinterpret_cast<const float4*>(&St[c][r4 * 4]);
      y[r4 * 4 + 0] = fmaf(s.x, q[c], y[r4 * 4 + 0]);
      y[r4 * 4 + 1] = fmaf(s.y, q[c], y[r4 * 4 + 1]);
      y[r4 * 4 + 2] = fmaf(s.z, q[c], y[r4 * 4 + 2]);
      y[r4 * 4 + 3] = fmaf(s.w, q[c], y[r4 * 4 + 3]);
    }
  }
  const float inv = 1.0f / (y[kD] + p.eps);                  // IEEE reciprocal (no fast-math)
  float o[kD];
#pragma unroll
  for (int r = 0; r < kD; ++r) o[r] = y[r] * inv;
  store_out<OutT>(out + ((int64_t)b * p.N + n) * p.H * kD + (int64_t)h * kD, o);
}

}  // namespace litela
