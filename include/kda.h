/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library (libkda.so).
 *
 * The operation ("Kimi Delta Attention: la atencion lineal detras de Kimi K2 y
 * Qwen3", section "Como funciona Kimi Delta Attention paso a paso", the
 * per-token step and the flowchart after it): for every sequence and head, with
 * a state S of shape dk x dv, and for every token t in order,
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = scale * S_t^T q_t,          alpha_t = exp(log_alpha_t)  (per key channel)
 *
 * i.e. decay the state per key channel, predict vhat = S~^T k_t, write the
 * beta-scaled error along k_t, then read with the query.  The page keeps the
 * state as (d_v, d_k) and reads S q; this library keeps S as [dk][dv] (dv
 * innermost) and reads S^T q -- the same arithmetic.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers, contiguous, last dimension
 *    innermost, 16-byte aligned (beta and cu_seqlens: 4-byte aligned).  The
 *    caller owns all of them.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).  Argument
 *    errors are detected on the host and returned before anything is launched;
 *    a failed launch returns KDA_ERR_CUDA.  What only the device can see (a
 *    malformed cu_seqlens array, a state slot out of range, a bounded wait
 *    that gave up) is ORed into the library's device error word, one per GPU
 *    and shared by all calls on it, and stays there until kda_get_error takes
 *    it; see kda_get_error for the bits.  No entry point synchronises the
 *    device unless KDA_DEBUG=1 is set in the environment, in which case every
 *    call takes the error word itself after its own work (so it synchronises
 *    `stream`) and returns KDA_ERR_TIMEOUT or KDA_ERR_INVALID_ARG for the bits
 *    it finds.
 *  - The prefill's kernels other than the fused tensor-core kernel are
 *    launched with programmatic stream serialization and let the next grid on
 *    `stream` be scheduled early; each of them waits for the previous grid to
 *    complete before it touches memory.
 *    Ordinary launches, copies and events after a call are ordered as usual.
 *    A kernel the caller launches after a call WITH programmatic stream
 *    serialization must wait for its dependency (cudaGridDependencySynchronize
 *    or griddepcontrol.wait) before it reads the call's outputs, as that
 *    launch mode requires of every consumer.
 *  - q and k are expected to be L2-normalised per (token, head) by the caller
 *    (the delta rule is only stable for normalised keys, as the same page notes
 *    in its warning on key normalisation); the kernels do not renormalise.
 *  - `scale` multiplies q once, at the read (configurations use 1/sqrt(dk)).
 *  - log_alpha is the natural log of the per-channel decay, finite and <= 0.
 *    The default tensor-core prefill (AUTO / TENSORCORE) and the SIMT paths
 *    hold at any decay rate.  The two-kernel tensor-core forms, when forced
 *    through KDA_PREFILL_TENSORCORE_CHAIN or _SEGMENTED, assume that within
 *    each 64-token chunk no key channel decays by more than e^-80 over 16
 *    consecutive tokens (their exponential factors are referenced to 16-token
 *    sub-chunk starts and would leave the fp32 range beyond that).
 *  - Supported head sizes: dk, dv in {64, 128}.  Anything else returns
 *    KDA_ERR_UNSUPPORTED.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad shape, bad cu_seqlens (debug) */
    KDA_ERR_UNSUPPORTED = 2,   /* head size or dtype not implemented */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_NO_MEMORY = 4,     /* workspace could not be allocated */
    KDA_ERR_TIMEOUT = 5        /* a bounded device-side wait gave up (debug) */
} kda_status_t;

typedef enum {
    KDA_IO_F32 = 0,            /* q, k, v, out are fp32 */
    KDA_IO_BF16 = 1            /* q, k, v, out are bf16 (gates, beta and states stay fp32) */
} kda_io_dtype_t;

/*
 * Tensor-core state walk.  Each (sequence, head) pair is a sequential chain of
 * chunks.  When there are too few chains to fill the GPU (few sequences and
 * heads), the library cuts every chain into segments that are walked in
 * parallel: a segment maps its entry state affinely (S -> M S + B, the
 * recurrence being linear in S), so each segment's M and B are computed
 * independently, the entry states follow from a short composition, and a last
 * parallel walk writes the outputs.  AUTO and TENSORCORE run the fused kernel:
 * one CTA per SM walks chains and builds each chunk's operands on chip while
 * the previous chunk's state update runs, so only the inputs, the outputs and
 * the states cross device memory (no workspace per chunk), and it is exact at
 * any decay rate.  With packed sequences its CTAs take chains from a shared
 * counter as they free up, longest sequences first.  When there are few chains
 * (at most half the SMs), AUTO and TENSORCORE first run the two-kernel form
 * (operand images in the workspace, prepared on every SM; segmented when there
 * are at most a quarter of the SMs' chains); its prep checks every 16-token
 * block against the two-kernel decay range, and if any block is past it the
 * walks do nothing and the fused kernel, launched after them, computes the
 * whole call -- so AUTO stays exact at any decay rate.  The last three values
 * force one form; the forced two-kernel forms (CHAIN, SEGMENTED) keep the
 * decay-range limit stated above.
 */
typedef enum {
    KDA_PREFILL_AUTO = 0,      /* tensor cores for bf16 with dk = dv = 128, SIMT otherwise */
    KDA_PREFILL_SIMT = 1,      /* fp32 SIMT chunk kernels (any supported shape / dtype) */
    KDA_PREFILL_TENSORCORE = 2, /* tcgen05 chunk kernels; bf16, dk = dv = 128, < 2^31 token rows */
    KDA_PREFILL_TENSORCORE_CHAIN = 3,     /* tcgen05, two kernels (operand image in
                                             workspace), one chain per (sequence, head) */
    KDA_PREFILL_TENSORCORE_SEGMENTED = 4, /* tcgen05, segment-parallel walk */
    KDA_PREFILL_TENSORCORE_FUSED = 5      /* tcgen05, one kernel: every chunk's operands
                                             built on chip next to the state walk */
} kda_prefill_impl_t;

/*
 * kda_chunk_fwd -- chunkwise-parallel prefill (64-token chunks).
 *
 * The chunkwise form is the exact reformulation of the token recurrence that
 * "Kimi Linear acaba de superar a la atencion completa en sus propios
 * terminos" (sections on the chunk training algorithm and the
 * diagonal-plus-low-rank transition) says the method uses; it returns the
 * token recurrence's result up to rounding.  Per chunk: cumulative log-decay,
 * intra-chunk WY/UT transform (T = (I + A)^{-1}), state propagation across
 * chunks with the state kept in fp32, and the output.
 *
 *  q, k        [B, T, H, dk]  io_dtype
 *  v           [B, T, H, dv]  io_dtype
 *  log_alpha   [B, T, H, dk]  fp32
 *  beta        [B, T, H]      fp32
 *  h0          [N, H, dk, dv] fp32 initial states, or NULL for zeros
 *  out         [B, T, H, dv]  io_dtype, written; must not alias any input
 *  hT          [N, H, dk, dv] fp32 final states, or NULL (not written); may alias h0
 *  cu_seqlens  NULL, or a DEVICE array of B+1 int32 offsets.  Then the B
 *              sequences are packed along T (q, k, v, log_alpha, beta, out have
 *              a leading axis of 1), cu_seqlens[0] = 0, non-decreasing,
 *              cu_seqlens[B] = T, and N = B.  Empty sequences are allowed
 *              (their hT equals h0).  Offsets are clamped into [0, T] on the
 *              device, so a malformed array never causes an out-of-bounds
 *              access (its results are then unspecified; bit 0 of the error
 *              word reports it).
 *              With NULL, every one of the N = B sequences has length T.
 * Memory: the call allocates stream-ordered workspace from a library-owned
 * CUDA memory pool (bounded, reused across calls); KDA_ERR_NO_MEMORY if that
 * fails.  T = 0 is a no-op apart from hT = h0.
 */
KDA_API kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* beta,
                           const float* h0, void* out, float* hT,
                           const int32_t* cu_seqlens,
                           int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                           float scale, kda_io_dtype_t io_dtype, cudaStream_t stream);

/* Same as kda_chunk_fwd with an explicit choice of implementation. */
KDA_API kda_status_t kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              const float* h0, void* out, float* hT,
                              const int32_t* cu_seqlens,
                              int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                              float scale, kda_io_dtype_t io_dtype,
                              kda_prefill_impl_t impl, cudaStream_t stream);

/*
 * kda_chunk_fwd_noalloc -- the chunkwise prefill for callers that cannot
 * allocate device memory.  The pages have no counterpart to this entry point.
 *
 * Some hosts reserve all GPU memory at start-up and forbid allocation
 * afterwards (serving engines that carve the device into their own pools,
 * plugin interfaces that pass a plugin its tensors but no allocator); for
 * them a library that calls cudaMalloc or a pool allocator mid-request can
 * fail or stall.  This call takes the same arguments as kda_chunk_fwd and runs
 * the fp32 SIMT chunk kernels (any supported dtype and head size), but keeps
 * its intermediate data in a fixed scratch array compiled into the library
 * (KDA_NOALLOC_SCRATCH_BYTES per GPU, held from the first load of the
 * library's kernels on that GPU until the process exits), so it allocates
 * nothing.  The caller still owns and passes every input and output.
 *
 * Limits and rules:
 *  - the problem must fit: with blk = 4*(64*(3*dk + dv + 64) + dk) bytes per
 *    (chunk, head) and C = number of chunk slots (B*ceil(T/64), or
 *    floor(T/64) + B with cu_seqlens), it needs 256 + (cu_seqlens ?
 *    round_up(8*(B+1), 256) : 0) + blk*C bytes for one head at a time (heads
 *    then run in groups that fit).  Otherwise KDA_ERR_UNSUPPORTED is returned
 *    before anything is launched (for dk = dv = 128 that is about 29,000
 *    chunk-tokens per call);
 *  - every call on a GPU shares the one scratch array, which keeps the last
 *    call's contents: calls whose GPU work overlaps (unordered streams) race on
 *    it, so the caller must order them;
 *  - the first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u << 20)
KDA_API kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                           const float* log_alpha, const float* beta,
                                           const float* h0, void* out, float* hT,
                                           const int32_t* cu_seqlens,
                                           int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                                           float scale, kda_io_dtype_t io_dtype,
                                           cudaStream_t stream);

/*
 * kda_recurrent_step -- one decode token per sequence, the per-token step
 * itself, with the state updated in place (HBM-bound: each (sequence, head)
 * state is read once and written once).
 *
 *  q, k        [N, H, dk]  io_dtype
 *  v           [N, H, dv]  io_dtype
 *  log_alpha   [N, H, dk]  fp32
 *  beta        [N, H]      fp32
 *  state       [N, H, dk, dv] fp32, read and overwritten
 *  out         [N, H, dv]  io_dtype
 * No workspace is used.  N = 0 is a no-op.
 */
KDA_API kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta,
                                float* state, void* out,
                                int64_t N, int64_t H, int64_t dk, int64_t dv,
                                float scale, kda_io_dtype_t io_dtype, cudaStream_t stream);

/*
 * Launch accounting of the library's own kernels (no counterpart on the
 * pages; it exists so throughput can be attributed per kernel).  Every
 * launch is counted.  While enabled, each launch is also bracketed by CUDA
 * events recorded on its own stream.  kda_profiler_read() waits for the
 * recorded events, fills up to max_entries stats (one per kernel, in a fixed
 * order), optionally resets the counters, and returns the number of entries,
 * or -1 if an event could not be read.
 */
typedef struct {
    const char* name;          /* static string */
    int64_t launches;          /* launches since the last reset */
    int64_t timed_launches;    /* launches recorded while the profiler was on */
    double total_ms;           /* summed event time of the timed launches */
} kda_kernel_stat_t;

KDA_API void kda_profiler_enable(int on);
KDA_API int kda_profiler_read(kda_kernel_stat_t* out, int max_entries, int reset);

/*
 * Gated DeltaNet, the direct predecessor the pages compare KDA with ("Kimi
 * Delta Attention: la atencion lineal detras de Kimi K2 y Qwen3", comparison
 * table and FAQ; "Cos'e Kimi Delta Attention (KDA)?", section on per-channel
 * gating): the same recurrence with ONE decay per (token, head),
 * Diag(alpha_t) = a_t I.  Same arguments as kda_chunk_fwd_ex /
 * kda_recurrent_step except the gate:
 *  log_a   [B, T, H] (prefill) or [N, H] (decode) fp32, natural log, <= 0,
 *          4-byte aligned.
 * The same kernels run, with the gate broadcast over the key channels.
 */
KDA_API kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v,
                                       const float* log_a, const float* beta,
                                       const float* h0, void* out, float* hT,
                                       const int32_t* cu_seqlens,
                                       int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                                       float scale, kda_io_dtype_t io_dtype,
                                       kda_prefill_impl_t impl, cudaStream_t stream);

KDA_API kda_status_t kda_gdn_recurrent_step(const void* q, const void* k, const void* v,
                                            const float* log_a, const float* beta,
                                            float* state, void* out,
                                            int64_t N, int64_t H, int64_t dk, int64_t dv,
                                            float scale, kda_io_dtype_t io_dtype,
                                            cudaStream_t stream);

/*
 * Pooled recurrent states for serving (continuous batching, prefix reuse,
 * chunked prefill).  The pages single out the recurrent-state layout across
 * chunked prefill, batched decode and prefix caching as what breaks in
 * practice ("Kimi Linear acaba de superar a la atencion completa en sus
 * propios terminos", section on serving reliability); these entry points keep
 * every sequence's state in one caller-owned pool and address it by slot.
 *
 *  state_pool  [P, H, dk, dv] fp32, read and written in place
 *  slots       DEVICE int32 [N]: sequence n uses pool slot slots[n].  A negative
 *              slot means "no cached state": zero initial state, final state
 *              not stored (decode: output row set to 0, nothing else touched).
 *              Slots >= P are not accessed (bit 0 of the error word reports
 *              them).  Two sequences of one call must not share a
 *              slot (their updates would race).
 *
 * kda_chunk_fwd_slots -- kda_chunk_fwd_ex with h0 = hT = state_pool[slots[n]];
 *   a prefill that continues from, and returns to, the pool.  Splitting a
 *   prompt into several calls (chunked prefill) gives the single-call result.
 * kda_recurrent_step_slots -- kda_recurrent_step on pool slots; N is the number
 *   of sequences in this step, P the pool size.
 */
KDA_API kda_status_t kda_chunk_fwd_slots(const void* q, const void* k, const void* v,
                                         const float* log_alpha, const float* beta,
                                         float* state_pool, const int32_t* slots, void* out,
                                         const int32_t* cu_seqlens,
                                         int64_t B, int64_t T, int64_t P, int64_t H,
                                         int64_t dk, int64_t dv, float scale,
                                         kda_io_dtype_t io_dtype, kda_prefill_impl_t impl,
                                         cudaStream_t stream);

KDA_API kda_status_t kda_recurrent_step_slots(const void* q, const void* k, const void* v,
                                              const float* log_alpha, const float* beta,
                                              float* state_pool, const int32_t* slots, void* out,
                                              int64_t N, int64_t P, int64_t H, int64_t dk,
                                              int64_t dv, float scale, kda_io_dtype_t io_dtype,
                                              cudaStream_t stream);

/*
 * kda_chunk_bwd -- gradients of the chunkwise prefill (training).
 *
 * "Kimi Linear acaba de superar a la atencion completa en sus propios
 * terminos" (section on the chunk training algorithm) says the method trains
 * with the chunk form; the pages give no gradient.  This returns the exact
 * gradients (up to rounding) of L = sum(dout * out) + sum(dhT * hT) for the
 * forward kda_chunk_fwd computes on the same arguments, obtained by
 * differentiating the chunk equations in reverse: a forward walk recomputes
 * every chunk's entry state, a reverse walk carries dL/dS back across chunks,
 * and per-chunk kernels form the parameter gradients.  All arithmetic is fp32
 * on the SIMT cores (no tensor cores yet).
 *
 *  q, k, v, log_alpha, beta, h0, cu_seqlens, B, T, H, dk, dv, scale, io_dtype:
 *              exactly as passed to kda_chunk_fwd
 *  dout        [B, T, H, dv]  io_dtype: gradient of out
 *  dhT         [N, H, dk, dv] fp32 gradient of hT, or NULL (zero)
 *  dq, dk      [B, T, H, dk]  io_dtype, written
 *  dv          [B, T, H, dv]  io_dtype, written
 *  dlog_alpha  [B, T, H, dk]  fp32, written
 *  dbeta       [B, T, H]      fp32, written
 *  dh0         [N, H, dk, dv] fp32, written, or NULL (not computed)
 * Outputs must not alias the inputs or one another.  Alignment, varlen rules
 * and supported shapes as for kda_chunk_fwd.  Workspace: about 600 KB per
 * (64-token chunk, head) at dk = dv = 128 from the library pool; heads run in
 * groups that fit the workspace budget.
 */
KDA_API kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, const float* h0,
                                   const void* dout, const float* dhT,
                                   void* dq, void* dk, void* dv, float* dlog_alpha,
                                   float* dbeta, float* dh0, const int32_t* cu_seqlens,
                                   int64_t B, int64_t T, int64_t H, int64_t dk_, int64_t dv_,
                                   float scale, kda_io_dtype_t io_dtype, cudaStream_t stream);

/*
 * kda_gdn_chunk_bwd -- kda_chunk_bwd for the Gated DeltaNet form: log_a
 * [B, T, H] fp32 (one gate per token and head, as kda_gdn_chunk_fwd takes it);
 * dlog_a [B, T, H] fp32 receives its gradient, the sum over the key channels of
 * the per-channel one (the gate multiplies every channel).  Other arguments
 * as for kda_chunk_bwd; log_a and dlog_a need 4-byte alignment.
 */
KDA_API kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v,
                                       const float* log_a, const float* beta, const float* h0,
                                       const void* dout, const float* dhT,
                                       void* dq, void* dk, void* dv, float* dlog_a,
                                       float* dbeta, float* dh0, const int32_t* cu_seqlens,
                                       int64_t B, int64_t T, int64_t H, int64_t dk_, int64_t dv_,
                                       float scale, kda_io_dtype_t io_dtype, cudaStream_t stream);

/*
 * Context parallelism: one long sequence split across GPUs (or across calls).
 *
 * The recurrence is linear in the state, so a run of tokens maps any entry
 * state S to M S + B (M: dk x dk, B: dk x dv).  Splitting a sequence into
 * consecutive pieces, each holder computes its piece's (M, B); the entry state
 * of piece r is then the composition of pieces 0 .. r-1 applied to h0, and a
 * plain kda_chunk_fwd of piece r from that state gives exactly the outputs and
 * final state of the unsplit sequence (up to rounding).  The pages run the
 * method at contexts of about a million tokens ("Kimi Linear acaba de superar
 * a la atencion completa en sus propios terminos", sections on decode timing
 * at 1M tokens and on the open release); the split itself is not on the pages
 * and follows from the linearity of the step.  The exchange between GPUs is
 * left to the caller (an all-gather of (M, B), 2 * 64 KiB per head at d = 128).
 *
 * kda_chunk_fwd_segmap -- (M, B) of every (sequence, head) of a prefill input.
 *  q, k, v, log_alpha, beta, cu_seqlens, B, T, H, dk, dv, io_dtype: as for
 *              kda_chunk_fwd (no output, no scale)
 *  maps        [N, H, dk, dk] fp32, written: M of each (sequence, head)
 *  offs        [N, H, dk, dv] fp32, written: B (the final state from a zero
 *              entry state)
 *  Both 16-byte aligned, not aliasing the inputs.  An empty sequence gives
 *  M = I, B = 0.  bf16 with dk = dv = 128 runs on the tensor cores (M and B
 *  carry the bf16-operand rounding of that path), anything else on the fp32
 *  SIMT kernels.  Allocates workspace like kda_chunk_fwd.
 *
 * kda_affine_prefix -- apply nseg consecutive maps to initial states.
 *  maps        [nseg, NH, dk, dk] fp32 (segment-major: segment s of chain i
 *              at s * NH + i)
 *  offs        [nseg, NH, dk, dv] fp32
 *  h0          [NH, dk, dv] fp32, or NULL for zeros
 *  out         [NH, dk, dv] fp32, written: M_{nseg-1}(...(M_0 h0 + B_0)...) +
 *              B_{nseg-1}; may alias h0, must not alias maps or offs.
 *  nseg = 0 copies h0 (or zeros).  fp32 FMA arithmetic on the device; all
 *  pointers 16-byte aligned; dk, dv in {64, 128}.  Allocates nothing.
 */
KDA_API kda_status_t kda_chunk_fwd_segmap(const void* q, const void* k, const void* v,
                                          const float* log_alpha, const float* beta,
                                          float* maps, float* offs,
                                          const int32_t* cu_seqlens,
                                          int64_t B, int64_t T, int64_t H, int64_t dk,
                                          int64_t dv, kda_io_dtype_t io_dtype,
                                          cudaStream_t stream);

KDA_API kda_status_t kda_affine_prefix(const float* maps, const float* offs, const float* h0,
                                       float* out, int64_t nseg, int64_t NH, int64_t dk,
                                       int64_t dv, cudaStream_t stream);

/*
 * kda_debug_prep_image -- test hook, not part of the method: runs only the
 * tensor-core prep kernel (cumulative decay and intra-chunk transform) of a
 * fixed-length bf16 batch with dk = dv = 128 and leaves its per-(chunk, head)
 * operand images in `image` (device, caller-owned, B * ceil(T / 64) * H blocks of
 * 66560 bytes, block (chunk c of sequence n, head h) at index (n * ceil(T/64) + c)
 * * H + h), in the 128-byte-swizzled bf16 layout the state kernel reads:
 * -W^T ([channel][token]) | Q e^G | [Aqk^T | K e^{G_last - G}] | T diag(beta) |
 * e^{G_last} (fp32).  Q e^G and Aqk carry no `scale`: the state kernel applies it
 * to the output.  log_alpha is [B, T, H, dk], or [B, T, H] with gate_scalar != 0
 * (Gated DeltaNet prep).  Lets the tests check the intra-chunk kernels against the
 * fp64 chunk equations one quantity at a time.
 */
KDA_API kda_status_t kda_debug_prep_image(const void* q, const void* k, const float* log_alpha,
                                          const float* beta, void* image, int64_t B, int64_t T,
                                          int64_t H, int gate_scalar, cudaStream_t stream);

/*
 * kda_debug_bounded_wait -- self-test, not part of the method: one CTA waits on
 * an mbarrier that nothing completes, with the two bounded waits the library's
 * kernels use on their copies, MMAs and warp hand-offs: `polls` suspended polls
 * (each at most ~0.1 ms; bit 1 of `err_word` when it gives up), then a spinning
 * poll bounded at `polls` x 200000 clock cycles (bit 2).  `err_word` is device
 * memory, caller-owned, 4-byte aligned, zeroed first; or NULL, and then the
 * bits go to the library's error word (taken with kda_get_error) and the call
 * returns KDA_OK.  The CTA returns with nothing in flight.  Synchronises
 * `stream`.  Returns KDA_ERR_TIMEOUT when the wait gave up on `err_word` (the
 * expected outcome), KDA_OK otherwise, KDA_ERR_INVALID_ARG for polls outside
 * [1, 20000] or a misaligned pointer.  Lets the tests check that a wait that
 * runs out is reported and leaves the context usable.
 */
KDA_API kda_status_t kda_debug_bounded_wait(int32_t polls, int32_t* err_word, cudaStream_t stream);

/*
 * kda_get_error -- takes the current device's error word: reads it and clears
 * it in one atomic exchange queued on `stream`, then waits for `stream` and
 * stores the bits in *word (host memory).  The word collects the bits of every
 * call made on this device since the last take, from any stream; bits of work
 * still running on another stream may land after the exchange (and are then
 * returned by the next take).  No kernel reads the word, so bits left in it
 * never change what a later call computes.
 *   bit 0      a malformed cu_seqlens array, or a state slot >= P
 *   bits 1-6   a bounded device-side wait gave up (1: input copies, 2-3: the
 *              operand MMAs, 4: state copies, 5: state-walk MMAs, 6: hand-offs
 *              between warps); the kernel stopped that work without faulting
 *              and its outputs are unspecified
 * Returns KDA_ERR_INVALID_ARG for word == NULL, KDA_ERR_CUDA if a CUDA call
 * failed, KDA_OK otherwise.
 */
KDA_API kda_status_t kda_get_error(cudaStream_t stream, int32_t* word);

/*
 * kda_workspace_high_water -- the most bytes of workspace that calls on the
 * current device had allocated at once from the library's pool since the last
 * reset (the pool's used-memory high-water mark; allocations are counted as
 * the pool rounds them), stored in *bytes; reset != 0 then restarts the mark
 * at the bytes in use now.  The fused tensor-core prefill (the default when the
 * chains outnumber half the SMs) needs a fixed 1 KiB (plus at most 20 bytes per
 * sequence with cu_seqlens) whatever T is; the two-kernel and SIMT forms grow
 * with the number of chunks up to the workspace budget, beyond which heads run
 * in groups; the decode step allocates nothing.
 * KDA_ERR_INVALID_ARG for bytes == NULL, KDA_ERR_CUDA if a CUDA call failed.
 */
KDA_API kda_status_t kda_workspace_high_water(int64_t* bytes, int reset);

/* Static, NUL-terminated description of a status code. */
KDA_API const char* kda_status_string(kda_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
KDA_API int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
