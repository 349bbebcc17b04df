/* fp32 FMA peak microbenchmark (liblitela_ffma_peak.so).
 *
 * Not part of the LiteLA method: the benchmark uses it for the fp32-FMA side of the roofline
 * (4*B*H*N*d*(d+1) FLOPs of the forward at the measured FMA rate), measured in the same run as
 * the kernels, at the clock the GPU holds under load.
 */
#ifndef LITELA_FFMA_PEAK_H
#define LITELA_FFMA_PEAK_H

#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

/* FLOPs (2 per fused multiply-add) that one litela_ffma_launch with these arguments performs;
 * 0 for non-positive arguments. */
long long litela_ffma_flops(int blocks, int threads, long long iters);

/* Launches the FMA loop on `stream`: `blocks` CTAs of `threads` threads (a multiple of 32, at
 * most 512), each thread doing iters x 128 multiply-adds.  `sink` is a caller-owned device
 * buffer of blocks * threads floats that the kernel may write (in practice never does).
 * Returns 0, 1 for an invalid argument (nothing launched) or 4 for a launch error.  The caller
 * times the launch with events on `stream`. */
int litela_ffma_launch(float* sink, int blocks, int threads, long long iters, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif
