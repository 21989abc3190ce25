/*
 * gdr.h -- C ABI of libgdr: the chunkwise-parallel forward pass of the gated
 * delta rule on one NVIDIA B200 (sm_100a).
 *
 * The operation (per sequence and head; tokens t in order; state S is dk x dv):
 *
 *     S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with D_t = I (DeltaNet), alpha_t I (Gated DeltaNet, one scalar per token and
 * head) or diag(alpha_t) (KDA, one factor per key channel).
 *
 * Sources:
 *  - "DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
 *    §2 Background: the delta rule is serial gradient descent on a linear
 *    memory; the update is affine in the preceding memory, which is what allows
 *    chunkwise-parallel evaluation while keeping token-level corrections.
 *    §4.1: a gradient step on a linear-regression objective in the memory
 *    matrix is a delta-rule update.  App. B: keys are normalised.
 *  - "Delta-Rule Linear Attention" topic page, FG^2-GDN card: KDA refines the
 *    head-wise decay of Gated DeltaNet into a channel-wise decay; FG^2-GDN
 *    makes the learning rate channel-wise too (gdr_chunk_fwd_fg2).
 *  - Gated DeltaNet-2 abstract, comparative-study page (2607.07953): a
 *    chunkwise WY algorithm with channel-wise decay absorbed into the erase
 *    factors; GDN-2 reduces to KDA and then to Gated DeltaNet.
 *
 * Readings taken where the pages are silent (the pages print no equation):
 *  - decay is applied before the erase: (I - beta k k^T) D S, the order that
 *    type-checks for dk != dv; it only matters for the channel-wise gate;
 *  - o_t reads the state after token t's write (the intra-chunk causal mask
 *    includes the diagonal);
 *  - no query scaling; keys and queries are used as given (callers normalise);
 *  - log_alpha is the natural log of the decay and is expected to be <= 0.
 *
 * Conventions shared by every entry point:
 *  - Every call returns a gdr_status; nothing throws, aborts or traps.
 *  - Argument checks happen on the host before any CUDA call, so a rejected
 *    call has no side effect.
 *  - Compute calls are asynchronous on `stream`; results are valid once the
 *    stream has been synchronised.  Inputs are never modified.
 *  - Scratch memory is allocated and released stream-ordered on `stream`
 *    (cudaMallocAsync / cudaFreeAsync), so calls on different streams do not
 *    share scratch.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDR_OK = 0,
  GDR_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, ...   */
  GDR_ERR_UNSUPPORTED = 2,      /* valid but not implemented (shape, dtype) */
  GDR_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed      */
  GDR_ERR_OUT_OF_MEMORY = 4,    /* scratch allocation failed                 */
  GDR_ERR_TIMEOUT = 5,          /* a bounded device-side wait expired        */
  GDR_ERR_RANGE = 6             /* a value fell outside the fused path's fp16
                                   operand range (non-finite output/state);
                                   the STAGED path has no such limit         */
} gdr_status;

/* Element type of q, k, v and out.  beta, log_alpha and the states are always
 * fp32; arithmetic is fp32 (bf16 only as tensor-core operands). */
typedef enum { GDR_BF16 = 0, GDR_FP32 = 1 } gdr_dtype;

typedef enum {
  GDR_GATE_NONE = 0,    /* alpha = 1 (DeltaNet); log_alpha must be NULL      */
  GDR_GATE_SCALAR = 1,  /* Gated DeltaNet: log_alpha [ntok][H]               */
  GDR_GATE_CHANNEL = 2  /* KDA: log_alpha [ntok][H][dk]                      */
} gdr_gate;

/* Which kernels run.  AUTO takes FUSED_TC where it applies and STAGED
 * otherwise; naming one explicitly returns GDR_ERR_UNSUPPORTED where it does
 * not apply. */
typedef enum {
  GDR_ALGO_AUTO = 0,
  /* four kernels -- (a) segmented log-decay cumsum, (b) intra-chunk WY/UT
   * transform, (c) sequential inter-chunk state passing, (d) chunk output --
   * fp32 CUDA-core arithmetic, intermediates in scratch.  Any supported
   * shape, fp32 or bf16. */
  GDR_ALGO_STAGED = 1,
  /* one persistent kernel per (sequence, head) that runs the same four steps
   * chunk after chunk with every intermediate on chip; chunk products on
   * tcgen05 tensor cores: fp16 operands (inputs converted on chip), fp32
   * accumulation in tensor memory, fp32 state.  bf16 I/O, dk = dv = 128,
   * chunk = 64.  Inputs and on-chip intermediates must lie within fp16
   * range (|x| <= 65504); a violation shows as a non-finite output or
   * state and is reported by gdr_device_error as GDR_ERR_RANGE.  Accuracy:
   * the scalar and no gate stay within about 5e-3 of the output RMS at any
   * decay.  For the channel gate the decay sits inside the contraction, on
   * operands rescaled by e^{+-(g - g_m)} (g_m: the log-decay at a chunk's
   * row 31), which are fp16 while every key channel's log-decay moves by at
   * most 9 between row 31 and the chunk's first or last row (about 3e-3 of
   * the output RMS; the KDA workload's decays stay well inside).  A chunk
   * beyond that window is computed on bf16 operands instead, which are less
   * accurate (up to about 3e-2 at mean log-decays of -1 to -2 per token and
   * channel), and the call reports GDR_ERR_RANGE through gdr_device_error:
   * run such inputs with GDR_ALGO_STAGED, fp32 throughout. */
  GDR_ALGO_FUSED_TC = 2,
  /* gdr_backward only: the reverse token recurrence (see there); every
   * forward entry returns GDR_ERR_UNSUPPORTED for it. */
  GDR_ALGO_RECURRENT = 3
} gdr_algo;

typedef struct {
  gdr_dtype dtype;
  gdr_gate gate;
  /* Packed variable-length batch: device pointer to num_seqs+1 int32 token
   * offsets (0 = first, non-decreasing, last = T), or NULL for fixed-length
   * sequences.  With cu_seqlens, B must be 1 and T is the packed total. */
  const int32_t *cu_seqlens;
  int num_seqs;
  gdr_algo algo;
} gdr_opts;

/*
 * gdr_chunk_fwd -- forward pass over a batch, chunk by chunk.
 *
 * Device pointers, row-major and contiguous, 16-byte aligned:
 *   q, k          [B][T][H][dk]   dtype
 *   v             [B][T][H][dv]   dtype
 *   log_alpha     NULL (GDR_GATE_NONE), [B][T][H] (SCALAR) or
 *                 [B][T][H][dk] (CHANNEL), fp32
 *   beta          [B][T][H] fp32
 *   initial_state [N][H][dk][dv] fp32, or NULL for a zero state
 *   out           [B][T][H][dv]   dtype (written)
 *   final_state   [N][H][dk][dv] fp32 (written), or NULL to skip
 * where N = B for fixed length, or num_seqs with cu_seqlens.
 * The caller owns every buffer; out and final_state must not overlap inputs.
 *
 * Sizes: B, T, H >= 0 (an empty batch is a no-op returning GDR_OK);
 * dk, dv in {16, 32, 64, 128}; chunk in {16, 32, 64} (chunk <= 64 and a
 * multiple of 16).  A sequence length need not be a multiple of chunk: its
 * last chunk is simply shorter.
 *
 * opts may be NULL: bf16, scalar gate, fixed length, AUTO.
 * Returns GDR_ERR_INVALID_ARGUMENT for null or misaligned pointers and
 * inconsistent sizes, GDR_ERR_UNSUPPORTED for shapes outside the list above,
 * GDR_ERR_OUT_OF_MEMORY if scratch cannot be allocated, GDR_ERR_CUDA if a
 * launch fails.  Device-side waits are bounded; an expired one is reported by
 * gdr_device_error().
 */
GDR_API gdr_status gdr_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         const float *initial_state, void *out,
                         float *final_state, int B, int T, int H, int dk,
                         int dv, int chunk, cudaStream_t stream,
                         const gdr_opts *opts);

/*
 * gdr_chunk_fwd_host -- the same computation on HOST buffers.
 *
 * Every tensor pointer (and opts->cu_seqlens) is a host pointer with the
 * layouts above; with cu_seqlens the offsets are checked on the host (first
 * 0, non-decreasing, last T), else GDR_ERR_INVALID_ARGUMENT.
 *
 * The work is cut into up to 8 pieces: fixed-length batches by time, at
 * chunk boundaries (each piece holds the same token range of every sequence
 * and starts from the state the previous piece ended with, kept on the
 * device in fp32, so the results are those of gdr_chunk_fwd bit for bit);
 * packed batches into pieces of whole sequences, each an independent
 * sub-problem.  The call enqueues, and returns without
 * waiting: per piece, the host-to-device copies of its inputs on an upload
 * stream, its computation on `stream`, and the device-to-host copies of its
 * results on a download stream, so that the copies of neighbouring pieces
 * overlap each other and the computation; then `stream` waits for both copy
 * streams and the device buffers are released.  Work enqueued on `stream`
 * after the call sees every result.  The upload and download streams are
 * created per device on first use and kept, as is a device memory pool that
 * holds the largest call's buffers between calls.
 *
 * Host buffers must stay valid until `stream` is synchronised.  With
 * page-locked (pinned) host memory the copies are asynchronous; with pageable
 * memory the CUDA runtime makes them synchronous to the host.
 */
GDR_API gdr_status gdr_chunk_fwd_host(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              const float *initial_state, void *out,
                              float *final_state, int B, int T, int H, int dk,
                              int dv, int chunk, cudaStream_t stream,
                              const gdr_opts *opts);

/*
 * gdr_chunk_fwd_gdn2 -- the forward pass with Gated DeltaNet-2's separate
 * erase and write gates.
 *
 * Gated DeltaNet-2 (abstract on the comparative-study page 2607.07953)
 * replaces the delta rule's one scalar gate beta, which controls both how
 * much old content is erased on the key side and how much new content is
 * written on the value side, by a channel-wise erase gate b_t (per key
 * channel) and a channel-wise write gate w_t (per value channel), and
 * reduces to KDA when both collapse to the same scalar.  The pages print no
 * formula; the update taken here keeps the delta rule's form with the erase
 * gate on the read key and the write gate on the target:
 *   S~_t = D_t S_{t-1},   u_t = w_t . v_t - S~_t^T (b_t . k_t),
 *   S_t  = S~_t + k_t u_t^T,   o_t = S_t^T q_t,
 * which is gdr_chunk_fwd's recurrence when b_t = beta_t 1 and w_t = beta_t 1.
 *
 * Arguments as for gdr_chunk_fwd, with beta replaced by
 *   erase_gate  [B][T][H][dk] fp32 (device, 16-byte aligned), required;
 *   write_gate  [B][T][H][dv] fp32 (device, 16-byte aligned), required;
 * (packed layouts with cu_seqlens as for gdr_chunk_fwd).  The decay form is
 * opts->gate (NONE, SCALAR or CHANNEL) as before.  Paths as for
 * gdr_chunk_fwd (fused tensor-core kernel for bf16, dk = dv = 128,
 * chunk = 64; the staged path otherwise).  The fused kernel runs these gates
 * on its channel-wise decay: a scalar or absent decay is expanded into
 * scratch as the channel-wise decay with every channel equal (ntok * H * 128
 * floats, from `stream`, GDR_ERR_OUT_OF_MEMORY on failure).  On the fused
 * path b . k and w . v are formed in fp32 and rounded once to the fp16
 * operands.  Status codes as for gdr_chunk_fwd (GDR_ERR_RANGE from the fused
 * path as for its channel gate).
 */
GDR_API gdr_status gdr_chunk_fwd_gdn2(const void *q, const void *k,
                                      const void *v, const float *log_alpha,
                                      const float *erase_gate,
                                      const float *write_gate,
                                      const float *initial_state, void *out,
                                      float *final_state, int B, int T, int H,
                                      int dk, int dv, int chunk,
                                      cudaStream_t stream,
                                      const gdr_opts *opts);

/*
 * gdr_chunk_fwd_fg2 -- the forward pass with FG^2-GDN's channel-wise
 * learning rate (and FG^2-GDN+'s value-side scaling).
 *
 * FG^2-GDN ("Delta-Rule Linear Attention" topic page, FG^2-GDN card) turns
 * the delta rule's scalar learning rate beta_t into a vector over channels,
 * as per-coordinate optimisers refine SGD; FG^2-GDN+ scales keys and values
 * separately.  The pages print no formula; the update taken here reads the
 * delta rule as one gradient step on 1/2 ||S^T k_t - v_t||^2 ("DeltaTTT"
 * page, sec. 4.1) with a rate per key channel (row of S), and FG^2-GDN+ as
 * a per-value-channel scaling c_t of the target:
 *   S~_t = D_t S_{t-1},   u_t = c_t . v_t - S~_t^T k_t,
 *   S_t  = S~_t + (beta_t . k_t) u_t^T,   o_t = S_t^T q_t,
 * i.e. write key beta_t . k_t, read key k_t.  beta_t = beta_t 1 with c = 1
 * is gdr_chunk_fwd's recurrence.
 *
 * Arguments as for gdr_chunk_fwd, with beta replaced by
 *   beta_k  [B][T][H][dk] fp32 (device, 16-byte aligned), required: the
 *           per-key-channel rate;
 *   beta_v  [B][T][H][dv] fp32 (device, 16-byte aligned), or NULL for
 *           FG^2-GDN (c = 1): FG^2-GDN+'s per-value-channel scaling;
 * (packed layouts with cu_seqlens as for gdr_chunk_fwd).  The decay form is
 * opts->gate (NONE, SCALAR or CHANNEL).  Paths as for gdr_chunk_fwd_gdn2:
 * the fused tensor-core kernel for bf16, dk = dv = 128, chunk = 64 (any
 * decay form, expanded as there), where it forms beta_k . k and c . v in
 * fp32 and rounds them once to its fp16 operands; the staged path
 * otherwise.  Status codes as for gdr_chunk_fwd.
 */
GDR_API gdr_status gdr_chunk_fwd_fg2(const void *q, const void *k,
                                     const void *v, const float *log_alpha,
                                     const float *beta_k, const float *beta_v,
                                     const float *initial_state, void *out,
                                     float *final_state, int B, int T, int H,
                                     int dk, int dv, int chunk,
                                     cudaStream_t stream,
                                     const gdr_opts *opts);

/*
 * gdr_chunk_fwd_segmented -- gdr_chunk_fwd with context-parallel state
 * passing along each sequence.
 *
 * The update is affine in the preceding state ("DeltaTTT" page, §2
 * Background), so a segment of a sequence maps its incoming state S to
 * M S + N.  Every sequence is cut into up to `segments` pieces of equally
 * many whole chunks; the pieces' M (the recurrence run from the identity
 * with v = 0) and N (run from a zero state) are computed in parallel by the
 * forward kernels, a combine kernel walks each sequence's pieces in order to
 * give every piece its true initial state, and a last forward pass computes
 * the outputs and final states.  The work is about three forward passes, in
 * exchange for `segments` times more independent chains: it pays when the
 * batch has fewer (sequence, head) pairs than the GPU has SMs (one long
 * sequence, few heads).  segments = 1 gives gdr_chunk_fwd's result (with
 * three passes).
 *
 * Arguments and layouts as for gdr_chunk_fwd, plus segments >= 1
 * (GDR_ERR_INVALID_ARGUMENT otherwise).  With cu_seqlens, the offsets are
 * read to the host once (the call synchronises `stream` for that) and
 * checked: first 0, non-decreasing, last T (else GDR_ERR_INVALID_ARGUMENT).
 * Scratch (about one bf16 / fp32 copy of v and out, and five dk x max(dk, dv)
 * fp32 states per piece and head) comes from the library's per-device pool,
 * stream-ordered on `stream`.
 */
GDR_API gdr_status gdr_chunk_fwd_segmented(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta, const float *initial_state, void *out,
    float *final_state, int B, int T, int H, int dk, int dv, int chunk,
    int segments, cudaStream_t stream, const gdr_opts *opts);

/*
 * gdr_chunk_fwd_noalloc -- gdr_chunk_fwd without any device allocation.
 *
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory at call time.  Examples are processes
 * whose device memory is reserved up front by another allocator (a serving
 * runtime whose caching pool already holds all free memory, so a new
 * cudaMalloc / cudaMallocAsync fails), and code that must not allocate during
 * steady-state operation (fixed memory budget, no allocator latency).
 *
 * It runs the STAGED kernels with their scratch in one statically sized
 * device array that lives in this library (GDR_NOALLOC_SCRATCH_BYTES, 64 MiB;
 * every GPU that loads the library holds it until the process exits).  The
 * caller still passes all inputs and outputs, as for gdr_chunk_fwd; the same
 * layouts, sizes and status codes apply, plus:
 *  - opts->algo must be GDR_ALGO_AUTO or GDR_ALGO_STAGED (FUSED_TC returns
 *    GDR_ERR_UNSUPPORTED: it does not use this scratch);
 *  - a problem whose staged scratch would exceed GDR_NOALLOC_SCRATCH_BYTES is
 *    rejected with GDR_ERR_UNSUPPORTED before any CUDA call;
 *  - the current device must be the device of `stream`.  The first call on
 *    each device looks up that device's address of the array
 *    (cudaGetSymbolAddress, once per device, cached); make that first call
 *    before any stream capture.  The cached address is not looked up again:
 *    after a cudaDeviceReset in the calling process this entry point must
 *    not be used on that device again;
 *  - every call on a device shares the one array, which keeps the last call's
 *    contents (nothing in it needs to start at zero: every scratch word is
 *    written before it is read).  Calls whose execution overlaps on the GPU
 *    (different streams, or different host threads, without ordering between
 *    them) race on the array and give undefined results: serialise them.
 * No cudaMalloc, cudaFree or other allocating routine is called.
 */
#define GDR_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

GDR_API gdr_status gdr_chunk_fwd_noalloc(const void *q, const void *k,
                                         const void *v, const float *log_alpha,
                                         const float *beta,
                                         const float *initial_state, void *out,
                                         float *final_state, int B, int T,
                                         int H, int dk, int dv, int chunk,
                                         cudaStream_t stream,
                                         const gdr_opts *opts);

/*
 * gdr_decode_step -- one token per (sequence, head): the recurrent update of
 * a resident state, as used when generating one token at a time after a
 * forward pass over the prompt.
 *
 * The operation is the recurrence above for a single token t (DeltaTTT page,
 * §2 Background and §4.1: the delta rule's one-token gradient step; "Delta-
 * Rule Linear Attention" topic page, GDN decode-accelerator card: decoding
 * reads and writes the whole recurrent state once per token, at under one
 * flop per byte):
 *     S' = (I - beta k k^T) D S + beta k v^T,    o = S'^T q
 *
 * Device pointers, row-major and contiguous, 16-byte aligned:
 *   q, k        [N][H][dk]   dtype
 *   v           [N][H][dv]   dtype
 *   log_alpha   NULL (GDR_GATE_NONE), [N][H] (SCALAR) or [N][H][dk]
 *               (CHANNEL), fp32
 *   beta        [N][H] fp32
 *   state_in    [N][H][dk][dv] fp32, or NULL for a zero state
 *   state_out   [N][H][dk][dv] fp32 (written).  It may be the same buffer as
 *               state_in (the state is then updated in place); otherwise the
 *               two must not overlap (GDR_ERR_INVALID_ARGUMENT).
 *   out         [N][H][dv]   dtype (written)
 *
 * Sizes: N, H >= 0 (N * H == 0 is a no-op returning GDR_OK), N * H < 2^31;
 * dk, dv in {16, 32, 64, 128}.  opts may be NULL (bf16, scalar gate);
 * opts->cu_seqlens must be NULL and opts->num_seqs 0 (one token per
 * sequence: nothing to pack), opts->algo must be GDR_ALGO_AUTO.
 * Arithmetic is fp32.  One kernel launch, no scratch memory; each CTA's wait
 * for its state tile is bounded (an expired wait is reported by
 * gdr_device_error as GDR_ERR_TIMEOUT; the environment variable
 * GDR_FAULT_INJECT_DECODE_TIMEOUT=1 makes every wait expire, for tests of that
 * path: the step is then skipped and state_out is not written).  After a
 * wait that expires on its own (not injected) the CTA skips its work but
 * stays, under a second bounded wait, until the copy it issued has landed,
 * so that no late copy writes into shared memory another CTA has since been
 * given; such a GDR_ERR_TIMEOUT means the device is not answering as it
 * should, and the caller should treat the CUDA context as suspect (finish
 * and restart rather than continue).  Returns GDR_ERR_INVALID_ARGUMENT /
 * GDR_ERR_UNSUPPORTED as described, GDR_ERR_CUDA if the launch fails.
 */
GDR_API gdr_status gdr_decode_step(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   const float *state_in, float *state_out,
                                   void *out, int N, int H, int dk, int dv,
                                   cudaStream_t stream, const gdr_opts *opts);

/*
 * gdr_decode_step_gdn2 -- gdr_decode_step with Gated DeltaNet-2's separate
 * erase and write gates (the update gdr_chunk_fwd_gdn2 documents) for one
 * token per (sequence, head):
 *     S~ = D S,   u = w . v - S~^T (b . k),   S' = S~ + k u^T,   o = S'^T q
 * so that a prompt run through gdr_chunk_fwd_gdn2 can be continued one token
 * at a time.
 *
 * Arguments as for gdr_decode_step, with beta replaced by
 *   erase_gate  [N][H][dk] fp32 (device, 16-byte aligned), required;
 *   write_gate  [N][H][dv] fp32 (device, 16-byte aligned), required.
 * Same kernel, limits, bounded wait and status codes as gdr_decode_step;
 * a NULL gate returns GDR_ERR_INVALID_ARGUMENT.
 */
GDR_API gdr_status gdr_decode_step_gdn2(const void *q, const void *k,
                                        const void *v, const float *log_alpha,
                                        const float *erase_gate,
                                        const float *write_gate,
                                        const float *state_in,
                                        float *state_out, void *out, int N,
                                        int H, int dk, int dv,
                                        cudaStream_t stream,
                                        const gdr_opts *opts);

/*
 * gdr_decode_step_fg2 -- gdr_decode_step with FG^2-GDN's per-key-channel
 * rate (and FG^2-GDN+'s value-side scaling; the update gdr_chunk_fwd_fg2
 * documents) for one token per (sequence, head):
 *     S~ = D S,   u = c . v - S~^T k,   S' = S~ + (beta_k . k) u^T,
 *     o = S'^T q
 * so that a prompt run through gdr_chunk_fwd_fg2 can be continued one token
 * at a time.
 *
 * Arguments as for gdr_decode_step, with beta replaced by
 *   beta_k  [N][H][dk] fp32 (device, 16-byte aligned), required;
 *   beta_v  [N][H][dv] fp32 (device, 16-byte aligned), or NULL (c = 1).
 * Same kernel, limits, bounded wait and status codes as gdr_decode_step;
 * a NULL beta_k returns GDR_ERR_INVALID_ARGUMENT.
 */
GDR_API gdr_status gdr_decode_step_fg2(const void *q, const void *k,
                                       const void *v, const float *log_alpha,
                                       const float *beta_k,
                                       const float *beta_v,
                                       const float *state_in,
                                       float *state_out, void *out, int N,
                                       int H, int dk, int dv,
                                       cudaStream_t stream,
                                       const gdr_opts *opts);

/*
 * gdr_backward -- gradients of gdr_chunk_fwd's outputs with respect to its
 * inputs (the backward pass for training).
 *
 * Given the forward inputs and the upstream gradients dL/d out and
 * dL/d final_state, it writes dL/dq, dL/dk, dL/dv, dL/d log_alpha,
 * dL/d beta and dL/d initial_state of the recurrence above (the same
 * definition gdr_chunk_fwd evaluates, whichever algorithm ran it), all in
 * fp32.  Two algorithms:
 *  - AUTO or STAGED: the chunked backward (the faster of the two on every
 *    shape measured).  The gradients of the chunkwise
 *    (WY) forward, taken product by product over chunks of 64 tokens: the
 *    staged path's per-chunk W, U and T, a forward scan over the chunk
 *    boundaries for the chunk-start states, a reverse scan for dL/dS at
 *    every chunk end, then every chunk's input gradients in parallel
 *    (mma.sync tensor-core products on fp32 operands split into a tf32
 *    part and its remainder, accurate to about 2^-21).  The update being
 *    affine in the preceding memory ("DeltaTTT" page, §2 Background) is
 *    what makes the two scans exact.  Deterministic except for the order in
 *    which a chunk's per-channel shares of the decay gradient are added.
 *  - RECURRENT: the reverse token recurrence.  It runs the recurrence
 *    forward, checkpointing the state every 8 tokens in scratch (16 when dk
 *    or dv is 16), then the reverse token recurrence window by window.  For
 *    dk, dv >= 32 each (sequence, head) runs on dv/32 blocks of 32 value
 *    columns; their per-token shares of the row sums (dq, dk, d_log_alpha,
 *    d_beta) are added in a fixed order, so the result does not depend on
 *    scheduling.
 * FUSED_TC returns GDR_ERR_UNSUPPORTED.
 *
 * Inputs: q, k, v, log_alpha, beta, initial_state, B, T, H, dk, dv and opts
 * exactly as for gdr_chunk_fwd (opts->algo AUTO, STAGED or RECURRENT);
 *   d_out          layout and dtype of out (device), required;
 *   d_final_state  [N][H][dk][dv] fp32, or NULL for a zero gradient.
 * Outputs (device, fp32, 16-byte aligned, written):
 *   dq, dk         [B][T][H][dk];   dv [B][T][H][dv];   d_beta [B][T][H];
 *   d_log_alpha    the layout of log_alpha; NULL iff gate is NONE;
 *   d_initial_state [N][H][dk][dv], or NULL to skip.
 * Scratch, chunked, in floats: (1 + dk + 3 dv) ntok H (g, W, U, V_new,
 * dV_new) plus, per chunk of 64 tokens and head, 2 * 64 * 64 (T, P),
 * 4 dk dv (the chunk-start state, dL/dS at the chunk end, Dm, Bm) and
 * dk * dk (the chunk's state map): about 4 GB at B8 H16 T4096 d128.  Recurrent (dk, dv >= 32): (ntok/8 + N) * H + 8 * N
 * * H states of dk*dv floats, plus the row-sum shares, 2 * (dv/32) * ntok *
 * H * dk floats (3 * for the channel gate); for dk or dv = 16: (ntok/16 +
 * N) * H + 16 * N * H states.  Allocated stream-ordered on `stream` from the library's per-device memory
 * pool, which keeps its memory between calls (the pool gdr_chunk_fwd_host
 * uses); GDR_ERR_OUT_OF_MEMORY on failure.
 * Status codes as for gdr_chunk_fwd.
 */
GDR_API gdr_status gdr_backward(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *initial_state, const void *d_out,
                                const float *d_final_state, float *dq,
                                float *dk, float *dv, float *d_log_alpha,
                                float *d_beta, float *d_initial_state, int B,
                                int T, int H, int dk_dim, int dv_dim,
                                cudaStream_t stream, const gdr_opts *opts);

/*
 * gdr_backward_gdn2 -- gdr_backward for gdr_chunk_fwd_gdn2: the gradients of
 * the forward pass with Gated DeltaNet-2's erase and write gates, the gates'
 * own included (the gate-aware backward the Gated DeltaNet-2 abstract,
 * comparative-study page 2607.07953, pairs with its chunkwise algorithm).
 *
 * The chunked backward of gdr_backward with the read key b . k (erase gate b)
 * on the row side of A and in W, the write key k in the state update and in
 * P, and the target w . v (write gate w) in U; beta is 1.  Gradients, fp32,
 * 16-byte aligned, written:
 *   dq, dk [B][T][H][dk];  dv [B][T][H][dv];  d_log_alpha (layout of
 *   log_alpha; NULL iff gate is NONE);  d_erase (layout of k) and d_write
 *   (layout of v), required;  d_initial_state [N][H][dk][dv] or NULL.
 * Inputs as for gdr_chunk_fwd_gdn2 (erase_gate, write_gate required) plus
 * d_out and d_final_state as for gdr_backward.  opts->algo AUTO or STAGED;
 * RECURRENT and FUSED_TC return GDR_ERR_UNSUPPORTED.  Scratch and status
 * codes as for gdr_backward's chunked algorithm.
 */
GDR_API gdr_status gdr_backward_gdn2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *erase_gate, const float *write_gate,
    const float *initial_state, const void *d_out,
    const float *d_final_state, float *dq, float *dk, float *dv,
    float *d_log_alpha, float *d_erase, float *d_write,
    float *d_initial_state, int B, int T, int H, int dk_, int dv_,
    cudaStream_t stream, const gdr_opts *opts);

/*
 * gdr_backward_fg2 -- gdr_backward for gdr_chunk_fwd_fg2: the gradients of
 * the forward pass with FG^2-GDN's per-key-channel rate (and FG^2-GDN+'s
 * value scaling), the rate's and the scaling's own included.
 *
 * The chunked backward with the write key beta_k . k (rate beta_k) in the
 * state update, in P and on the column side of A, the read key k on A's row
 * side and in W, and the target c . v (c = beta_v, or 1) in U; beta is 1.
 * Gradients, fp32, 16-byte aligned, written: dq, dk, dv, d_log_alpha (NULL
 * iff gate is NONE), d_beta_k (layout of k, required), d_beta_v (layout of
 * v; required iff beta_v is given, else NULL), d_initial_state (or NULL).
 * Inputs as for gdr_chunk_fwd_fg2 plus d_out and d_final_state as for
 * gdr_backward.  opts->algo AUTO or STAGED; RECURRENT and FUSED_TC return
 * GDR_ERR_UNSUPPORTED.  Scratch and status codes as for gdr_backward's
 * chunked algorithm.
 */
GDR_API gdr_status gdr_backward_fg2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta_k, const float *beta_v, const float *initial_state,
    const void *d_out, const float *d_final_state, float *dq, float *dk,
    float *dv, float *d_log_alpha, float *d_beta_k, float *d_beta_v,
    float *d_initial_state, int B, int T, int H, int dk_, int dv_,
    cudaStream_t stream, const gdr_opts *opts);

/*
 * gdr_efla_beta -- exact-flow step size (EFLA) for the delta rule.
 *
 * The delta rule's update is one explicit Euler step of length beta of the
 * flow dS/dtau = -k k^T S + k v^T; EFLA takes the exact flow instead, which
 * for these rank-1 dynamics has the same form ("Delta-Rule Linear Attention"
 * topic page, EFLA card).  Reading taken (the card prints no formula): the
 * exact step is the delta rule with step size
 *     beta'[t][h] = (1 - exp(-beta[t][h] * |k[t][h]|^2)) / |k[t][h]|^2
 * (beta' = beta where |k| = 0), applied after the decay as usual.  Running
 * gdr_chunk_fwd or gdr_decode_step with beta' in place of beta gives the
 * EFLA recurrence with every gate kind.
 *
 * Device pointers, 16-byte aligned: k [ntok][H][dk] in `dtype`, beta and
 * beta_out [ntok][H] fp32.  beta_out may be beta itself (in place);
 * otherwise the two must not overlap.  dk in {16, 32, 64, 128};
 * ntok * H == 0 is a no-op.  One launch on `stream`, no scratch.
 */
GDR_API gdr_status gdr_efla_beta(const void *k, const float *beta,
                                 float *beta_out, int ntok, int H, int dk,
                                 gdr_dtype dtype, cudaStream_t stream);

/*
 * gdr_efla_beta_backward -- the chain rule through gdr_efla_beta, for the
 * EFLA backward pass: run gdr_backward with beta' (its d_beta is then
 * d beta'), then this, which writes
 *   d_beta[row] = d_beta_prime[row] e^{-beta s}        (s = |k_row|^2)
 * and ADDS  d_beta_prime[row] (d beta' / d s) 2 k_row  to dk (fp32, the
 * layout of k, typically gdr_backward's dk), with
 * d beta' / d s = (beta s e^{-beta s} + e^{-beta s} - 1) / s^2 (its Taylor
 * series for small beta s, limit -beta^2 / 2).
 *
 * k [ntok][H][dk] in `dtype`; beta, d_beta_prime, d_beta [ntok][H] fp32; all
 * device, 16-byte aligned.  dk in {16, 32, 64, 128}.  Status codes as for
 * gdr_efla_beta.
 */
GDR_API gdr_status gdr_efla_beta_backward(const void *k, const float *beta,
                                          const float *d_beta_prime,
                                          float *d_beta, float *dk, int ntok,
                                          int H, int dk_, gdr_dtype dtype,
                                          cudaStream_t stream);

/*
 * gdr_device_error -- synchronise `stream`, then read (and clear if `clear`)
 * the library's sticky device-side error word for the current device.
 * Returns GDR_OK if no kernel has reported an error, GDR_ERR_TIMEOUT if a
 * bounded wait expired (the fused kernel's, or the decode step's wait for its
 * state tile), GDR_ERR_RANGE if the fused kernel produced a
 * non-finite output or final state (an input or intermediate beyond the
 * fp16 operand range, |x| > 65504, or a NaN input) or, for the channel gate,
 * met such an input,
 * GDR_ERR_CUDA if synchronisation itself failed.
 */
GDR_API gdr_status gdr_device_error(cudaStream_t stream, int clear);

/*
 * gdr_algo_applies -- 1 if `algo` can run a problem of this dtype, gate and
 * shape (AUTO and STAGED: any supported shape; FUSED_TC: bf16, dk = dv = 128,
 * chunk = 64, any gate), else 0.  Host-only; makes no CUDA call.
 */
GDR_API int gdr_algo_applies(gdr_algo algo, gdr_dtype dtype, gdr_gate gate,
                             int dk, int dv, int chunk);

/* Human-readable name of a status code (static storage; never NULL). */
GDR_API const char *gdr_status_string(gdr_status status);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
