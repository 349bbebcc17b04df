/*
 * liblitela — LiteLA forward (Sana's ReLU linear self-attention) for NVIDIA B200 (sm_100a).
 *
 * The operation (Sana explainer "Sana: the autoencoder does more of the work than the linear
 * attention", section "What LiteLA actually computes"; instagit page "How Linear Attention
 * Improves Efficiency in DiT for High-Resolution Images", sections "Mathematical Foundation"
 * and "Implementation Details"): for every (batch b, head h), with phi = ReLU applied to q and
 * k only and V padded with a row of ones,
 *
 *     S    = [V ; 1] . phi(K)^T                  a (d+1) x d state, accumulated in fp32
 *     y_n  = S . phi(q_n)                         d+1 values per query token n
 *     out_n[r] = y_n[r] / (y_n[d] + eps)          r = 0 .. d-1
 *
 * which equals sum_j w_nj v_j / (sum_j w_nj + eps) with w_nj = phi(q_n).phi(k_j).
 *
 * Layouts (all row-major, densely packed, no padding between rows):
 *   qkv : bf16 [B, N, 3*H*d]; one token row is [q | k | v], each head-major, i.e. element
 *         (b, n, h, c) of q, k, v is at ((b*N + n)*3*H + {0, 1, 2}*H + h)*d + c.
 *   out : [B, N, H*d]; element (b, n, h, c) at ((b*N + n)*H + h)*d + c; bf16 (round to
 *         nearest even) for the plain entry points, fp32 for the *_f32out ones.
 *
 * Ownership: the caller owns qkv and out (device memory, at least 16-byte aligned, not
 * overlapping).  The library owns a per-(device, stream) workspace of partial states (a few
 * MB, see lite_la_workspace_bytes) that it allocates on first use, grows on demand (both after
 * synchronising that stream, so the first call with a new size must not happen during graph
 * capture) and keeps until lite_la_release_workspace().  Calls are asynchronous with respect to
 * the host; calls on one stream are ordered by that stream, calls on different streams use
 * different workspaces.  Once a stream's workspace has the size a call needs, the call may be
 * captured into a CUDA graph on that stream: every call leaves the workspace's control words
 * as it found them, so the graph may be replayed any number of times, between eager calls.
 *
 * Errors: every entry point returns a litela_status and never throws.  Argument errors are
 * detected on the host before anything is launched.  A kernel launch failure returns
 * LITELA_ERR_CUDA; a fault that happens later in an asynchronous kernel surfaces at the next
 * synchronisation, as usual in CUDA.  lite_la_last_error() gives a message for the calling
 * thread's last failure.
 *
 * Only d = 32 (Sana's linear_head_dim) is built; other d give LITELA_ERR_UNSUPPORTED.
 * B, N or H equal to 0 is an empty problem: the call returns LITELA_OK and touches nothing.
 */
#ifndef LITELA_H_
#define LITELA_H_

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LITELA_OK = 0,
  LITELA_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, misaligned or overlapping
                                      buffers, eps < 0 or not finite, tokens_per_block < 1,
                                      sizes whose element count overflows int64 */
  LITELA_ERR_UNSUPPORTED = 2,      /* d != 32 */
  LITELA_ERR_OUT_OF_MEMORY = 3,    /* workspace allocation failed */
  LITELA_ERR_CUDA = 4,             /* a CUDA runtime call or kernel launch failed */
  LITELA_ERR_DEVICE_TIMEOUT = 5    /* a kernel gave up on a bounded wait (lite_la_device_status) */
} litela_status;

/* Non-causal LiteLA forward, bf16 output.
 * qkv: device pointer, bf16 [B, N, 3*H*d] (layout above); out: device pointer, bf16
 * [B, N, H*d].  eps is added to the denominator (Sana uses a tiny eps such as 1e-15).
 * stream: the CUDA stream to run on (0 = legacy default stream). */
litela_status lite_la_fwd(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                          cudaStream_t stream);

/* Block-causal LiteLA forward, bf16 output ("Block-Linear Attention" for video: same instagit
 * page, section "Video Generation and Constant-Memory KV Cache").  Tokens are cut into
 * consecutive blocks of tokens_per_block tokens (the last block may be shorter); a query in
 * block b uses the state summed over the keys/values of blocks 0..b (inclusive prefix).
 * tokens_per_block >= N gives the non-causal result.  Other arguments as lite_la_fwd. */
litela_status lite_la_block_causal_fwd(const void* qkv, void* out, int B, int N, int H, int d,
                                       float eps, int tokens_per_block, cudaStream_t stream);

/* Block-causal LiteLA over one chunk of a longer sequence, carrying the state across chunks
 * (the "constant-memory KV cache" of Block-Linear Attention: same instagit page, section "Video
 * Generation and Constant-Memory KV Cache").  state_in: device fp32 [B, H, d+1, d], the prefix
 * state of every token of the earlier chunks (rows r < d: sum of v_r * relu(k); row d: sum of
 * relu(k)), or NULL for none; it is added to the state of every block of this chunk.
 * state_out: device fp32 [B, H, d+1, d], receives state_in plus the state of all of this chunk's
 * tokens (the state_in of the next chunk), or NULL.  state_out may be state_in (updated in
 * place); neither may overlap qkv or out; both 16-byte aligned.  With chunk lengths that are
 * multiples of tokens_per_block, chaining chunks gives exactly the block-causal result of the
 * whole sequence.  Other arguments as lite_la_block_causal_fwd. */
litela_status lite_la_block_causal_fwd_carry(const void* qkv, void* out, int B, int N, int H, int d,
                                             float eps, int tokens_per_block, const float* state_in,
                                             float* state_out, cudaStream_t stream);
litela_status lite_la_block_causal_fwd_carry_f32out(const void* qkv, float* out, int B, int N, int H,
                                                    int d, float eps, int tokens_per_block,
                                                    const float* state_in, float* state_out,
                                                    cudaStream_t stream);

/* The same two operations with an fp32 output buffer [B, N, H*d] (debug / accuracy mode). */
litela_status lite_la_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d,
                                 float eps, cudaStream_t stream);
litela_status lite_la_block_causal_fwd_f32out(const void* qkv, float* out, int B, int N, int H,
                                              int d, float eps, int tokens_per_block,
                                              cudaStream_t stream);

/* The LiteLA state alone (the first contraction, and the video "KV cache" of Block-Linear
 * Attention): for every batch b, head h and causal block k (one block when tokens_per_block <= 0
 * or >= N) the inclusive prefix state over the tokens of blocks 0..k,
 *     states[b][h][k][r][c] = sum_n v[n][h][r] * relu(k[n][h][c])   for r < d,
 *     states[b][h][k][d][c] = sum_n relu(k[n][h][c])                  (the ones-pad row),
 * fp32, layout [B, H, nblk, d+1, d] row-major, nblk = ceil(N / tokens_per_block).  states is a
 * caller-owned device buffer (16-byte aligned, not overlapping qkv). */
litela_status lite_la_state_fwd(const void* qkv, float* states, int B, int N, int H, int d,
                                int tokens_per_block, cudaStream_t stream);

/* lite_la_fwd with phase timing: the same kernels (without programmatic overlap between them),
 * plus cudaEventRecord of events[0] before the first kernel, events[1] after the state phase
 * (reduction + scan) and events[2] after the apply, all on `stream`; on the fused single-kernel
 * path events[1] and events[2] are both recorded after the kernel.  events: host array of 3
 * caller-created CUDA events.  Used by the benchmark to time the kernels on their stream. */
litela_status lite_la_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                 cudaStream_t stream, cudaEvent_t* events);

/* lite_la_block_causal_fwd with the phase timing of lite_la_fwd_events: events[0] before the
 * reduction, events[1] after the prefix scan, events[2] after the apply (tokens_per_block >= N
 * is the non-causal call and takes its path).  Arguments are validated as for
 * lite_la_block_causal_fwd. */
litela_status lite_la_block_causal_fwd_events(const void* qkv, void* out, int B, int N, int H, int d,
                                              float eps, int tokens_per_block, cudaStream_t stream,
                                              cudaEvent_t* events);

/* Synchronises `stream`, then reads and clears the error word that this library's kernels on
 * the current device set when one of their bounded waits timed out (each wait inside the
 * kernels gives up after about 1.5 s, records a code, frees its tensor memory and returns, so
 * the GPU context stays usable).  Returns LITELA_ERR_DEVICE_TIMEOUT (message with the code) if
 * a kernel of this stream's workspace or of lite_la_fwd_noalloc reported one, else LITELA_OK.
 * This stream's workspace has an error word of its own; lite_la_fwd_noalloc's word is one per
 * device, shared by every stream.  That word is therefore read reliably only once every stream
 * that issued lite_la_fwd_noalloc calls has been synchronised (a call still running on another
 * stream can set it after the read), and a time-out it holds may come from another stream's
 * call; it is reported, and cleared, by whichever stream asks first. */
litela_status lite_la_device_status(cudaStream_t stream);

/* Self-test of that error path: launches on `stream` one thread that waits on a barrier nothing
 * ever completes; after the wait limit (about 1.5 s) it records its code and returns.  The next
 * lite_la_device_status(stream) then returns LITELA_ERR_DEVICE_TIMEOUT, and the stream and the
 * context remain usable.  Nothing faults and nothing hangs. */
litela_status lite_la_selftest_timeout(cudaStream_t stream);

/* ---- ELU + 1 variant ------------------------------------------------------------------
 *
 * Kernelised linear attention as the Sana tutorial page (aifetchly) writes its linear-attention
 * block: phi(x) = ELU(x) + 1 (exp(x) for x <= 0, x + 1 above; alpha = 1) on q and k, phi(q)
 * scaled by 1/sqrt(d), the same state S = [V;1] . phi(K)^T, and the denominator clamped from
 * below instead of adding eps:
 *     out_n[r] = y_n[r] / max(y_n[d], clamp_min),   y_n = S . (phi(q_n) / sqrt(d)).
 * Sana's LiteLA is the ReLU form above; this variant is provided beside it.  tokens_per_block
 * > 0 gives the block-causal form, <= 0 the non-causal one.  clamp_min (the page uses 1e-6)
 * must be finite and >= 0.  Layouts, buffers, streams and status codes as for lite_la_fwd
 * (bf16 output; fp32 for the _f32out form). */
litela_status lite_la_elu1_fwd(const void* qkv, void* out, int B, int N, int H, int d, float clamp_min,
                               int tokens_per_block, cudaStream_t stream);
litela_status lite_la_elu1_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d, float clamp_min,
                                      int tokens_per_block, cudaStream_t stream);
/* lite_la_elu1_fwd with the phase timing of lite_la_fwd_events (three kernels: events[0]
 * before the reduction, events[1] after the scan, events[2] after the apply). */
litela_status lite_la_elu1_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float clamp_min,
                                      int tokens_per_block, cudaStream_t stream, cudaEvent_t* events);

/* ---- backward -------------------------------------------------------------------------
 *
 * Gradients of L = sum over all outputs of dout * out with respect to q, k and v, for the
 * forward of lite_la_fwd (non-causal) or lite_la_block_causal_fwd.  The pages print only the
 * forward (Sana explainer, "What LiteLA actually computes"); Sana trains through it, and these
 * are its derivatives by the chain rule, per (batch, head), with S the state a query uses
 * (block-causal: the prefix state of its block), den = (S relu(q))[d] + eps, g = dout:
 *     dq = relu'(q) * (S[0:d]^T g / den + h * S[d]),   h = -(g . out) / den
 *     dS = sum over the queries that use S of [g / den ; h] relu(q)^T
 *          (block-causal: block b's own state gets the sum of dS over blocks b .. last)
 *     dk = relu'(k) * (dS[0:d]^T v + dS[d]),   dv = dS[0:d] relu(k)
 * relu'(x) = 1 for x > 0, else 0.  eps is a constant; the ones row that pads v has no gradient.
 *
 * qkv  : the forward's input, bf16 [B, N, 3*H*d] (layout as above).
 * dout : the incoming gradient, bf16 [B, N, H*d] (the layout of out).
 * dqkv : the result, [B, N, 3*H*d] in qkv's layout (dq | dk | dv per token row); bf16 (round to
 *        nearest even) for the plain entry points, fp32 for the *_f32out ones.  Every element is
 *        written.
 * All three are caller-owned device buffers, 16-byte aligned; dqkv must not overlap qkv or dout
 * (LITELA_ERR_INVALID_ARGUMENT).  Other arguments, the workspace, streams, status codes and
 * asynchrony as for the forward entry points.  The forward's output is not needed: the
 * backward recomputes the state (minimal HBM traffic 18 bytes per (token, head, channel):
 * k, v read for the state, q and dout read, k and v read again, dq, dk, dv written). */
litela_status lite_la_bwd(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d, float eps,
                          cudaStream_t stream);
litela_status lite_la_block_causal_bwd(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d,
                                       float eps, int tokens_per_block, cudaStream_t stream);
litela_status lite_la_bwd_f32out(const void* qkv, const void* dout, float* dqkv, int B, int N, int H, int d,
                                 float eps, cudaStream_t stream);
litela_status lite_la_block_causal_bwd_f32out(const void* qkv, const void* dout, float* dqkv, int B, int N, int H,
                                              int d, float eps, int tokens_per_block, cudaStream_t stream);

/* The forward and the backward with the state carried between them.  lite_la_fwd_save_state
 * is lite_la_fwd (tokens_per_block <= 0) or lite_la_block_causal_fwd (> 0), bitwise the same
 * output, that also writes the states its queries use, fp32 [B, H, nblk, d+1, d] (the layout of
 * lite_la_state_fwd: the per-block inclusive prefix states; nblk = 1 when non-causal) into the
 * caller's buffer `states` (16-byte aligned, not overlapping qkv or out).
 * lite_la_bwd_from_state is lite_la_bwd / lite_la_block_causal_bwd (bf16 dqkv) given those
 * states: it skips recomputing them (a reduction over k and v and a scan), which saves 4 of the
 * 18 bytes of HBM traffic per (token, head, channel).  `states` must hold the states of the same
 * qkv and tokens_per_block (not checked); other arguments as for lite_la_bwd. */
litela_status lite_la_fwd_save_state(const void* qkv, void* out, float* states, int B, int N, int H, int d,
                                     float eps, int tokens_per_block, cudaStream_t stream);
litela_status lite_la_bwd_from_state(const void* qkv, const void* dout, const float* states, void* dqkv, int B, int N,
                                     int H, int d, float eps, int tokens_per_block, cudaStream_t stream);

/* The backward (bf16 dqkv) with phase timing: events[0] before its first kernel, events[1]
 * after the state (reduction + scan), events[2] after the dq kernel, events[3] after the
 * dk/dv kernels; tokens_per_block <= 0 is the non-causal call.  events: host array of 4
 * caller-created CUDA events.  The kernels run without programmatic overlap. */
litela_status lite_la_bwd_events(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d,
                                 float eps, int tokens_per_block, cudaStream_t stream, cudaEvent_t* events);

/* Size in bytes of the workspace a backward call with these arguments needs (tokens_per_block
 * <= 0 means non-causal; a 148-SM device).  0 for invalid arguments or an empty problem. */
size_t lite_la_bwd_workspace_bytes(int B, int N, int H, int d, int tokens_per_block);

/* Static description of a status code (never NULL). */
const char* lite_la_status_string(litela_status status);

/* Message describing the calling thread's most recent failure ("" if none). */
const char* lite_la_last_error(void);

/* Frees every cached workspace on every device.  Synchronises each device that holds one
 * first, so it must not be called while another thread is capturing a CUDA graph. */
litela_status lite_la_release_workspace(void);

/* Size in bytes of the workspace a call with these arguments needs (tokens_per_block <= 0
 * means non-causal).  Returns 0 for invalid arguments or an empty problem. */
size_t lite_la_workspace_bytes(int B, int N, int H, int d, int tokens_per_block);

/* Number of kernels one forward call with these arguments launches on the current device: 1
 * when it takes a fused single kernel, plain or paired (B * ceil(H/4) <= SM count; block-causal
 * calls also need a block size that is a multiple of 128 tokens and at most two blocks per CTA;
 * lite_la_forward_form says which), 3 otherwise
 * (state reduction, prefix scan, apply); 0 for an empty or invalid problem.  The streaming-carry
 * form always takes the three-kernel path, and so does the ELU+1 variant's block-causal form (its
 * non-causal form takes the fused kernel under the same condition as LiteLA's). */
int lite_la_kernels_per_call(int B, int N, int H, int d, int tokens_per_block);

/* Number of kernels one backward call launches (lite_la_bwd, lite_la_block_causal_bwd when
 * from_state is 0; lite_la_bwd_from_state when it is 1): 3 when the call has one block per
 * sequence (non-causal, or tokens_per_block >= N): the state (the reduction, or the images of
 * the saved states), dq, and dk/dv, the last two summing the partial states into their own
 * images; otherwise 5 (reduction, prefix scan, dq, reverse scan, dk/dv), 4 from saved states.
 * 0 for an empty or invalid problem. */
int lite_la_bwd_kernels_per_call(int B, int N, int H, int d, int tokens_per_block, int from_state);

/* Which form a LiteLA forward call (lite_la_fwd, lite_la_block_causal_fwd and their _f32out
 * forms) with these arguments takes on the current device: LITELA_FORM_THREE_KERNEL (state
 * reduction, prefix scan, apply), LITELA_FORM_FUSED (one kernel: a CTA reduces a chunk of one
 * head quad's tokens, the quad's sibling CTAs merge their partial states, then apply the state to
 * a share of the quad's queries), LITELA_FORM_FUSED_PAIRED (the same work, but every CTA owns a
 * chunk of two head quads, so that one quad's merge runs while the CTA streams the other quad's
 * tokens; taken when a chunk has at least the paired minimum of tokens, see
 * lite_la_set_paired_min_chunk), LITELA_FORM_FUSED_CAUSAL (the fused kernel's block-causal form:
 * a CTA owns one or two consecutive causal blocks of one quad) or LITELA_FORM_FUSED_PAIRED_CAUSAL
 * (the paired kernel's block-causal form: a CTA owns blocks r and r + ceil(nblk/2) of one quad,
 * so that the prefix of its first block is merged while it reduces the second; taken where
 * the plain form would give each CTA two blocks and blocks have at least the paired minimum of
 * tokens); -1 for an empty or invalid problem.  The ELU+1 variant never takes a paired form. */
#define LITELA_FORM_THREE_KERNEL 0
#define LITELA_FORM_FUSED 1
#define LITELA_FORM_FUSED_PAIRED 2
#define LITELA_FORM_FUSED_CAUSAL 3
#define LITELA_FORM_FUSED_PAIRED_CAUSAL 4
int lite_la_forward_form(int B, int N, int H, int d, int tokens_per_block);

/* Sets the chunk length (tokens per sibling CTA and head quad; the block size for block-causal
 * calls) from which LiteLA calls take a paired fused form, for every device and thread of the
 * process; tokens <= 0 restores the default, 1024 (measured on B200: with shorter chunks one
 * quad's state reduction is too short to hide the other's merge, and the plain fused form is
 * faster).  Returns the previous value.  Calls already enqueued are not affected; the result of
 * a call does not depend on the form up to the order of its fp32 partial-state sums. */
int lite_la_set_paired_min_chunk(int tokens);

/* ---- LiteLA with the output projection fused ---------------------------------------------
 *
 * In Sana's block, LiteLA's output feeds the attention's output projection (Sana explainer,
 * "What LiteLA actually computes"; the FLOP ledger of "Two levers" counts qkv + out proj as
 * 4 N d^2 multiply-adds per layer).  The projection is read as a linear layer in PyTorch's
 * convention, y = x W^T (+ b).
 *
 * lite_la_fwd_oproj computes y = LiteLA(qkv) W^T + bias without writing LiteLA's output x to
 * memory: the apply (S . relu(q), normalised) runs in the projection GEMM's operand prologue
 * and x is rounded to bf16 there, as lite_la_fwd's output would be.
 *   qkv  : device, bf16 [B, N, 3*H*d] (layout above); d must be 32.
 *   w_o  : device, bf16 [C_out, H*d], row-major (nn.Linear's weight), 16-byte aligned.
 *   bias : device, fp32 [C_out], or NULL for none.
 *   y    : device, bf16 [B, N, C_out], 16-byte aligned, not overlapping any input.
 *   C_out: a multiple of 8 (16-byte rows), >= 0.  tokens_per_block <= 0 (or >= N): non-causal;
 *          otherwise block-causal, and then it must be a multiple of 128 (LITELA_ERR_UNSUPPORTED
 *          otherwise).
 * Three kernels: the state reduction, the prefix scan (the state images, in this stream's
 * workspace) and the fused apply + projection GEMM (tcgen05, tiles of 128 tokens x 224 output
 * columns).  Errors, workspace and asynchrony as for lite_la_fwd.
 * lite_la_fwd_oproj_events brackets the phases: events[0] before the reduction, events[1]
 * after the scan, events[2] after the projection kernel (no programmatic overlap then).
 *
 * lite_la_out_proj is the projection alone, y = x W^T (+ bias), on a bf16 [B, N, C_in] input x
 * (e.g. lite_la_fwd's output: the unfused chain), with the same GEMM kernel and tiles.  C_in and
 * C_out must be multiples of 8; x, w_o and y 16-byte aligned; y must not overlap the inputs. */
litela_status lite_la_fwd_oproj(const void* qkv, const void* w_o, const float* bias, void* y, int B, int N, int H,
                                int d, int C_out, float eps, int tokens_per_block, cudaStream_t stream);
litela_status lite_la_fwd_oproj_events(const void* qkv, const void* w_o, const float* bias, void* y, int B, int N,
                                       int H, int d, int C_out, float eps, int tokens_per_block, cudaStream_t stream,
                                       cudaEvent_t* events);
litela_status lite_la_out_proj(const void* x, const void* w_o, const float* bias, void* y, int B, int N, int C_in,
                               int C_out, cudaStream_t stream);

/* lite_la_fwd without any allocation.  The pages describe no such call; it exists for callers
 * that cannot let a library allocate device memory: a host that owns all of the device memory
 * through its own pool and hands each op only its input and output buffers, or a latency-bound
 * loop in which a first-use cudaMalloc (and the device synchronisation it may bring) is not
 * acceptable.  Same arguments, layouts and result as lite_la_fwd (bf16 output, non-causal).
 *
 * Its scratch (partial states, merged states, arrival counters) is one fixed array of
 * LITELA_NOALLOC_SCRATCH_BYTES in device memory that the library defines statically; every
 * GPU that loads the library holds it until the process exits.  A problem whose scratch does
 * not fit (lite_la_workspace_bytes() plus a few hundred bytes of control words above the limit)
 * is rejected with LITELA_ERR_INVALID_ARGUMENT and a message before anything is launched.  The
 * 4096px Sana call (B=2, N=16384, H=70) takes the paired fused kernel and needs about 4.9 MB
 * (the partial states of 8 siblings per head quad; 2.4 MB in the plain fused form of the 1024px
 * and 2048px calls); calls with more than 148 head quads (B * ceil(H/4)) take the three-kernel
 * path, whose partial states and state images need more (B=8, N=512, H=80: about 6 MB).  The
 * first call on a device looks up that device's address of the array (once per device); make that first call before any
 * stream capture.  The call never calls cudaMalloc or cudaFree; it clears the counters it needs
 * with cudaMemsetAsync on `stream`.  All calls on a device share the one array and it keeps the
 * last call's contents, so calls that can overlap on the GPU (different streams without an
 * ordering between them) race and give wrong results: order them, e.g. on one stream. */
#define LITELA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
litela_status lite_la_fwd_noalloc(const void* qkv, void* out, int B, int N, int H, int d,
                                  float eps, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LITELA_H_ */
