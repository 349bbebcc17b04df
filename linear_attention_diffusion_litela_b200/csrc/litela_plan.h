// Host-side partition of one LiteLA call into causal blocks, state-reduction CTAs and apply
// work items, and the layout of the workspace.  Plain C++ (no CUDA), so the same arithmetic is
// compiled into the library and can be queried on a machine without a GPU.
#pragma once

#include <cstddef>
#include <cstdint>

namespace litela {

constexpr int kD = 32;             // head dim (Sana's linear_head_dim)
constexpr int kRows = kD + 1;      // state rows: d value channels + the ones (denominator) row
constexpr int kStateFloats = kRows * kD;

// state reduction: a CTA owns 4 heads (the MMA's M = 4 x 32 key channels) and one chunk of
// tokens inside one causal block, streamed in stages of 64 tokens
constexpr int kRedHeads = 4;
constexpr int kRedTile = 64;
constexpr int kRedCtasPerSm = 2;
// apply: a work unit is 4 heads (256-byte q and output rows) x one 128-token tile inside one
// causal block; the MMA and the accumulators work on one head pair at a time
constexpr int kApUnitHeads = 4;
constexpr int kApHeads = 2;
constexpr int kApTile = 128;
// one head's state in the apply MMA's B-operand layout (in shared memory): 80 rows (33 hi rows
// + 7 zero rows, 33 lo rows + 7 zero rows) x 32 bf16
constexpr int kImageRows = 80;
constexpr int kImageLoRow = 40;
constexpr int kImageBytes = kImageRows * kD * 2;
// the transposed image of a state's first d rows (rows c: hi 0..31, lo 32..63; K = r, 32 wide),
// the B operand of the backward's products with S[0:d]^T
constexpr int kImageTRows = 2 * kD;
constexpr int kImageTBytes = kImageTRows * kD * 2;
// small zero-initialised control buffer: word 0 is the kernels' error word (a bounded wait that
// timed out); the fused kernel's sibling counters start at word kCounterBase
constexpr int kErrWords = 64;
// the paired form of the fused path is taken when a sibling's chunk has at least this many
// tokens: with shorter chunks one quad's reduction is too short to hide the other's merge
constexpr int kPairedMinChunk = 1024;
constexpr int kCounterBase = kErrWords;

struct Plan {
  int B = 0, N = 0, H = 0;
  int T = 0;                 // tokens per causal block (N when non-causal)
  int nblk = 0;              // number of blocks, ceil(N / T)
  int ngroups = 0;           // reduce head groups, ceil(H / 4)
  int chunks_per_block = 0;  // reduce CTAs per (batch, group, block)
  int chunk = 0;             // tokens per reduce CTA (a multiple of kRedTile)
  int red_bpc = 1;           // consecutive blocks per reduce CTA (> 1 only with one chunk per block)
  int nquads = 0;            // apply head quads, ceil(H / 4)
  int tiles_per_block = 0;   // apply tiles per (batch, quad, block)
  int64_t units = 0;         // apply work units
  // workspace, in bytes from its base (each region 256-byte aligned):
  //   partial states fp32 [B][ngroups][nblk * chunks_per_block][4][33][32]
  //   state images (the apply's B operand) bf16 [B][H][nblk][kImageBytes]
  size_t off_images = 0, bytes = 0;
  // fused single-kernel path (non-causal, B * nquads <= SMs): CTA (b, quad, r), r < fused_cpb;
  // workspace = fused partials [B][nquads][fused_cpb][4][33][32]; control words: B * nquads
  // arrival counters, a finish counter and a ticket counter
  bool fused = false;
  int fused_cpb = 0, fused_chunk = 0, fused_ntiles = 0;
  size_t fused_bytes = 0, counters = 0;
  // its paired form (fused_paired, ReLU only): CTA r of sibling group g works on quads g and
  // g + ceil(B * nquads / 2) (index b * nquads + q), paired_cpb siblings per quad of
  // paired_chunk tokens each;
  // workspace = partials [B * nquads][paired_cpb][4][33][32]; the same control words
  bool fused_paired = false;
  int paired_cpb = 0, paired_chunk = 0;
  size_t paired_bytes = 0;
  // block-causal fused path (fused_causal): CTA (b, quad, r) owns blocks [r * fused_bpc, ...),
  // at most 2; workspace = block states [B][nquads][nblk][4][33][32], then the CTA totals
  // [B][nquads][fused_cpb][4][33][32] at fused_off_totals; control words: an arrival flag per
  // CTA, the finish and ticket counters
  bool fused_causal = false;
  int fused_bpc = 0;
  size_t fused_off_totals = 0;
  // backward (make_bwd_plan): the forward's reduction and scan (partials, images above), then
  //   S^T images bf16 [B][H][nblk][kImageTBytes]                       at off_images_t
  //   dS partials fp32 [B][nquads][nblk * bwd_cpb][4][33][32]           at off_dpartials
  //   dS images, rows 0..d-1 [B][H][nblk][kImageTBytes], dS^T images (the same size) and the
  //   ones rows dS[d] fp32 [B][H][nblk][d]                  at off_dimages, off_dimages_t, off_dzrows
  int bwd_cpb = 0, bwd_chunk = 0;   // CTAs per (batch, quad, block); tokens per CTA (multiple of 128)
  size_t off_images_t = 0, off_dpartials = 0, off_dimages = 0, off_dimages_t = 0, off_dzrows = 0, bwd_bytes = 0;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// tokens_per_block <= 0 or >= N selects the non-causal form.  Returns false for an empty
// problem (B, N or H == 0); sizes must already be validated as non-negative.  num_sms is the
// device's SM count (148 on B200); paired_min_chunk the chunk length (tokens) from which the
// non-causal fused path takes its paired form.
inline bool make_plan(int B, int N, int H, int tokens_per_block, int num_sms, Plan* p,
                      int paired_min_chunk = kPairedMinChunk) {
  *p = Plan{};
  if (B <= 0 || N <= 0 || H <= 0) return false;
  p->B = B; p->N = N; p->H = H;
  p->T = (tokens_per_block <= 0 || tokens_per_block >= N) ? N : tokens_per_block;
  p->nblk = (N + p->T - 1) / p->T;
  p->ngroups = (H + kRedHeads - 1) / kRedHeads;
  const int64_t units = (int64_t)B * p->ngroups * p->nblk;
  const int64_t target = (int64_t)(num_sms > 0 ? num_sms : 148) * kRedCtasPerSm;
  int64_t want = target / units;                                  // chunks per block
  const int64_t max_chunks = (p->T + kRedTile - 1) / kRedTile;
  if (want > max_chunks) want = max_chunks;
  if (want < 1) want = 1;
  int64_t chunk = (p->T + want - 1) / want;
  chunk = (chunk + kRedTile - 1) / kRedTile * kRedTile;
  p->chunk = (int)chunk;
  p->chunks_per_block = (int)((p->T + chunk - 1) / chunk);
  // one chunk per block and more blocks than the target number of CTAs: a reduction CTA walks
  // several consecutive blocks (one partial state each) instead of launching a CTA per block
  const int64_t ctas_per_group = target / ((int64_t)B * p->ngroups) > 0 ? target / ((int64_t)B * p->ngroups) : 1;
  if (p->chunks_per_block == 1 && p->nblk > ctas_per_group)
    p->red_bpc = (int)((p->nblk + ctas_per_group - 1) / ctas_per_group);
  p->nquads = (H + kApUnitHeads - 1) / kApUnitHeads;
  p->tiles_per_block = (p->T + kApTile - 1) / kApTile;
  p->units = (int64_t)B * p->nquads * p->nblk * p->tiles_per_block;
  const size_t partials = (size_t)units * p->chunks_per_block * kRedHeads * kStateFloats * sizeof(float);
  const size_t images = (size_t)B * H * p->nblk * kImageBytes;
  p->off_images = align_up(partials, 256);
  p->bytes = p->off_images + align_up(images, 256);
  const int sms = num_sms > 0 ? num_sms : 148;
  if (p->nblk == 1 && (int64_t)B * p->nquads <= sms) {
    p->fused = true;
    p->fused_ntiles = (N + kApTile - 1) / kApTile;
    int cpb = sms / (B * p->nquads);
    if (cpb > p->fused_ntiles) cpb = p->fused_ntiles;
    if (cpb < 1) cpb = 1;
    int64_t chunk = ((int64_t)N + cpb - 1) / cpb;
    chunk = (chunk + kRedTile - 1) / kRedTile * kRedTile;
    p->fused_cpb = cpb;
    p->fused_chunk = (int)chunk;
    p->fused_bytes = align_up((size_t)B * p->nquads * cpb * kRedHeads * kStateFloats * sizeof(float), 256);
    p->counters = (size_t)B * p->nquads + 2;   // an arrival counter per quad; finish, ticket
    const int64_t nq = (int64_t)B * p->nquads;
    const int64_t groups = (nq + 1) / 2;
    int64_t S = sms / groups;
    if (S > p->fused_ntiles) S = p->fused_ntiles;
    if (S < 1) S = 1;
    int64_t ch = ((int64_t)N + S - 1) / S;
    ch = (ch + kRedTile - 1) / kRedTile * kRedTile;
    if (nq >= 2 && ch >= paired_min_chunk) {
      p->fused_paired = true;
      p->paired_chunk = (int)ch;
      p->paired_cpb = (int)(((int64_t)N + ch - 1) / ch);
      p->paired_bytes = align_up((size_t)nq * p->paired_cpb * kRedHeads * kStateFloats * sizeof(float), 256);
    }
  } else if (p->nblk > 1 && p->T % kApTile == 0 && (int64_t)B * p->nquads <= sms) {
    int cpb = sms / (B * p->nquads);
    if (cpb > p->nblk) cpb = p->nblk;
    const int bpc = (p->nblk + cpb - 1) / cpb;
    if (bpc <= 2) {   // each CTA keeps the images of its blocks in shared memory
      cpb = (p->nblk + bpc - 1) / bpc;
      p->fused = p->fused_causal = true;
      p->fused_cpb = cpb;
      p->fused_bpc = bpc;
      p->fused_ntiles = (N + kApTile - 1) / kApTile;
      const size_t part = (size_t)kRedHeads * kStateFloats * sizeof(float);
      p->fused_off_totals = align_up((size_t)B * p->nquads * p->nblk * part, 256);
      p->fused_bytes = p->fused_off_totals + align_up((size_t)B * p->nquads * cpb * part, 256);
      p->counters = (size_t)B * p->nquads * cpb + 2;   // an arrival flag per CTA; finish, ticket
    }
    // paired block-causal form, where the plain form gives each CTA two consecutive blocks: the
    // same CTAs, but sibling r of quad c owns its blocks r and r + S (S = ceil(nblk / 2)), so that
    // block r's prefix is merged while the CTA reduces block r + S; workspace = block states
    // [B * nquads][nblk][4][33][32]; control words: a flag per (quad, block), the finish and
    // ticket counters
    const int64_t nq = (int64_t)B * p->nquads, S = (p->nblk + 1) / 2;
    if (bpc == 2 && p->T >= paired_min_chunk) {
      const size_t part = (size_t)kRedHeads * kStateFloats * sizeof(float);
      p->fused = p->fused_causal = p->fused_paired = true;
      p->fused_ntiles = (N + kApTile - 1) / kApTile;
      p->paired_cpb = (int)S;
      p->paired_chunk = p->T;
      p->paired_bytes = align_up((size_t)nq * p->nblk * part, 256);
      p->counters = (size_t)nq * p->nblk + 2;
    }
  }
  return true;
}

// Adds the backward's partition and workspace layout to a plan made by make_plan: one CTA per
// (batch, head quad, block, chunk of the block), about one CTA per SM in total.
inline void make_bwd_plan(int num_sms, Plan* p) {
  const int sms = num_sms > 0 ? num_sms : 148;
  const int64_t segs = (int64_t)p->B * p->nquads * p->nblk;
  int64_t want = sms / segs;
  if (want > p->tiles_per_block) want = p->tiles_per_block;
  if (want < 1) want = 1;
  int64_t chunk = (p->T + want - 1) / want;
  chunk = (chunk + kApTile - 1) / kApTile * kApTile;
  p->bwd_chunk = (int)chunk;
  p->bwd_cpb = (int)((p->T + chunk - 1) / chunk);
  const size_t img_t = (size_t)p->B * p->H * p->nblk * kImageTBytes;
  const size_t zrows = (size_t)p->B * p->H * p->nblk * kD * sizeof(float);
  const size_t dpart = (size_t)segs * p->bwd_cpb * kRedHeads * kStateFloats * sizeof(float);
  p->off_images_t = align_up(p->bytes, 256);
  p->off_dpartials = p->off_images_t + align_up(img_t, 256);
  p->off_dimages = p->off_dpartials + align_up(dpart, 256);
  p->off_dimages_t = p->off_dimages + align_up(img_t, 256);
  p->off_dzrows = p->off_dimages_t + align_up(img_t, 256);
  p->bwd_bytes = p->off_dzrows + align_up(zrows, 256);
}

}  // namespace litela
