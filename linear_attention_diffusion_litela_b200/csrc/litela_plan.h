// Host-side partition of one LiteLA call into reduce chunks, blocks and apply tiles.
// Plain C++ (no CUDA), so the same arithmetic is compiled into the library and can be
// queried on a machine without a GPU.
#pragma once

#include <cstddef>
#include <cstdint>

namespace litela {

constexpr int kD = 32;             // head dim (Sana's linear_head_dim)
constexpr int kRows = kD + 1;      // state rows: d value channels + the ones (denominator) row
constexpr int kStateFloats = kRows * kD;

struct Plan {
  int B = 0, N = 0, H = 0;
  int T = 0;                 // tokens per causal block (N when non-causal)
  int nblk = 0;              // number of blocks, ceil(N / T)
  int chunks_per_block = 0;  // reduce CTAs per (batch, head, block)
  int chunk = 0;             // tokens per reduce CTA (a multiple of kReduceTile)
  int tiles_per_block = 0;   // apply CTAs per (batch, head, block)
  int apply_tile = 0;        // tokens per apply CTA
  // state workspace layout, in bytes from its base (each region 256-byte aligned)
  size_t off_partials = 0, off_states = 0, bytes = 0;
  // arrival counters, one per (batch, head); they live in a separate zero-initialised
  // buffer that the kernels leave at zero when they finish
  size_t counters = 0;
};

constexpr int kReduceTile = 32;     // tokens staged per reduce iteration
constexpr int kApplyTile = 256;     // tokens per apply CTA (one per thread)
constexpr int kTargetReduceCtas = 148 * 8;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// tokens_per_block <= 0 or >= N selects the non-causal form.  Returns false for an empty
// problem (B, N or H == 0); sizes must already be validated as non-negative.
inline bool make_plan(int B, int N, int H, int tokens_per_block, Plan* p) {
  *p = Plan{};
  if (B <= 0 || N <= 0 || H <= 0) return false;
  p->B = B; p->N = N; p->H = H;
  p->T = (tokens_per_block <= 0 || tokens_per_block >= N) ? N : tokens_per_block;
  p->nblk = (N + p->T - 1) / p->T;
  const int64_t heads = (int64_t)B * H * p->nblk;
  int64_t want = (kTargetReduceCtas + heads - 1) / heads;           // chunks per block
  int64_t max_chunks = (p->T + kReduceTile - 1) / kReduceTile;
  if (want > max_chunks) want = max_chunks;
  if (want < 1) want = 1;
  int64_t chunk = (p->T + want - 1) / want;
  chunk = (chunk + kReduceTile - 1) / kReduceTile * kReduceTile;
  p->chunk = (int)chunk;
  p->chunks_per_block = (int)((p->T + chunk - 1) / chunk);
  p->apply_tile = kApplyTile;
  p->tiles_per_block = (p->T + kApplyTile - 1) / kApplyTile;
  const size_t partials = (size_t)heads * p->chunks_per_block * kStateFloats * sizeof(float);
  const size_t states = (size_t)heads * kStateFloats * sizeof(float);
  p->off_partials = 0;
  p->off_states = align_up(partials, 256);
  p->bytes = p->off_states + align_up(states, 256);
  p->counters = (size_t)B * H;
  return true;
}

}  // namespace litela
