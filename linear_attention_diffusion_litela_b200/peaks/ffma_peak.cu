// fp32 FMA throughput microbenchmark.  The LiteLA roofline is the slower of two bounds: the
// minimal HBM traffic at the copy bandwidth, and the method's 4*B*H*N*d*(d+1) FLOPs (the state
// reduction and the apply, counted as fp32 multiply-adds) at the fp32 FMA peak.  This kernel
// measures that peak on the running GPU at the clock it actually holds under load.
//
// Every thread runs kChains independent multiply-add chains (enough to hide the FMA latency at
// full occupancy) for iters x kUnroll rounds.  The chains converge to a fixed point and their
// sum is stored only under a condition that never holds, which keeps the work alive without
// any memory traffic.
#include <cuda_runtime.h>

#include "litela_ffma_peak.h"

namespace {

constexpr int kChains = 8;
constexpr int kUnroll = 16;

__global__ void __launch_bounds__(512) ffma_loop(float* __restrict__ sink, long long iters, float a, float b) {
  float x[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) x[k] = 1.0f + 1e-6f * (float)(threadIdx.x + k);
  for (long long i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
      for (int k = 0; k < kChains; ++k) x[k] = fmaf(x[k], a, b);
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChains; ++k) s += x[k];
  if (s == -1.0f) sink[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

extern "C" {

long long litela_ffma_flops(int blocks, int threads, long long iters) {
  if (blocks <= 0 || threads <= 0 || iters <= 0) return 0;
  return 2LL * blocks * threads * iters * kUnroll * kChains;
}

int litela_ffma_launch(float* sink, int blocks, int threads, long long iters, cudaStream_t stream) {
  if (sink == nullptr || blocks <= 0 || threads <= 0 || threads > 512 || (threads & 31) || iters <= 0) return 1;
  ffma_loop<<<blocks, threads, 0, stream>>>(sink, iters, 0.999f, 0.001f);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

}  // extern "C"
