/*
 * wkv7.h - C ABI of the WKV7 recurrence library (libwkv7.so, CUDA sm_100a).
 *
 * The operation (per batch b, head h; the state S is an N x N fp32 matrix,
 * row i = value index, column j = key index):
 *
 *     S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T
 *     y_t = S_t r_t                     (read after the write of token t)
 *
 * This is the RWKV-7 "generalized delta rule with vector-valued gating and
 * in-context learning rates" (RWKV-7 "Goose" with Expressive Dynamic State
 * Evolution, abstract): a "diagonal plus rank one" state transition with a
 * vector-valued, data-dependent decay and separate removal / replacement
 * keys (Paper Review: RWKV-7 "Goose", section "Architecture"), updated per
 * head and read out by the receptance vector (same review, section "The
 * approach").  w is the decay itself (0 < w <= 1 in the intended use), not its
 * logarithm; a is the removal key, b the learning-rate-scaled replacement
 * key; k, v the write key and value; r the receptance.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers owned by the caller (wkv7_forward_host
 *    takes host tensors).  The library allocates no memory; scratch comes
 *    from the caller through the *_workspace_size queries.  Every pointer
 *    must be 16-byte aligned.
 *  - Tensors are contiguous, row-major.  Per-token tensors (r, w, k, v, a, b,
 *    y, dy and their gradients) are [B, T, H, N]; a decode step's tensors are
 *    [B, H, N]; states (s0, sT, dsT, ds0, state) are [B, H, N, N] fp32 with
 *    element S[b][h][i][j] (i = value row, j = key column).
 *  - Calls are asynchronous on `stream`; they never synchronize (except
 *    wkv7_get_last_status).  Launch errors are reported as WKV7_ERR_CUDA.
 *  - Arguments are validated on the host before any launch; an invalid
 *    argument returns WKV7_ERR_INVALID_ARG (N other than 64 returns
 *    WKV7_ERR_UNSUPPORTED) and launches nothing.
 *  - B, T, H may be 0 (nothing to do; with T = 0 the forward copies s0, or
 *    zeros, to sT and the backward copies dsT, or zeros, to ds0).
 *  - No exception crosses the ABI.  The library is safe to call from several
 *    host threads as long as each call's buffers are its own.
 */
#ifndef WKV7_H
#define WKV7_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define WKV7_API __attribute__((visibility("default")))
#else
#define WKV7_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WKV7_OK = 0,
    WKV7_ERR_INVALID_ARG = 1,  /* bad pointer / size / dtype / alignment      */
    WKV7_ERR_UNSUPPORTED = 2,  /* valid request that this library does not implement */
    WKV7_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed        */
    WKV7_ERR_TIMEOUT = 4,      /* a device-side bounded wait gave up          */
    WKV7_ERR_RANGE = 5,        /* device-side: input outside the chunked
                                  form's numeric domain (see wkv7_forward)   */
    WKV7_ERR_TOO_LARGE = 6     /* problem needs more scratch than the fixed
                                  array of wkv7_backward_noalloc holds       */
} wkv7_status;

typedef enum { WKV7_F32 = 0, WKV7_BF16 = 1 } wkv7_dtype;

typedef enum {
    WKV7_ALGO_AUTO = 0,   /* library picks: CHUNK for bf16 inputs when T >= 64, else SEQ */
    WKV7_ALGO_SEQ = 1,    /* token-by-token scan, state kept on chip            */
    WKV7_ALGO_CHUNK = 2   /* chunked (parallel-in-time) form on tensor cores    */
} wkv7_algo;

/* ABI version of this header (bumped on any incompatible change). */
#define WKV7_ABI_VERSION 1
WKV7_API int wkv7_abi_version(void);

/* Static, human-readable name of a status code (never NULL). */
WKV7_API const char *wkv7_status_string(wkv7_status status);

/*
 * Bytes of scratch wkv7_forward can use for these arguments on the current
 * device (0 when the chosen algorithm needs none).  The split it pays for
 * rests on the state update being affine in S: the transition is a diagonal
 * plus a rank-one term built from the token's own inputs (Paper Review:
 * RWKV-7 "Goose", section "Architecture"), so a stretch of tokens maps its
 * entry state S to S M + E.  The chunked form uses it to
 * split long sequences into segments that run in parallel when B*H heads are
 * too few to fill the GPU (a per-segment summary S -> S M + E, a scan of the
 * entry states, then every segment from its entry state).  Without it (NULL
 * or too small) the chunked form runs in one pass; the results are the same.
 */
WKV7_API size_t wkv7_forward_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                   wkv7_algo algo, int chunk_len);

/*
 * Forward over a whole sequence (when the chunked form splits the sequence into
 * segments, the state crosses segment boundaries through the summary scan).
 *   r, w, k, v, a, b : [B, T, H, N] of in_dtype (fp32 or bf16), read only
 *   s0               : [B, H, N, N] fp32 initial state, or NULL for zeros
 *   y                : [B, T, H, N] of y_dtype, written
 *   sT               : [B, H, N, N] fp32 final state, or NULL to skip.
 *                      sT may alias s0 (in-place continuation); no other
 *                      output may alias an input.
 *   algo, chunk_len  : algorithm choice; chunk_len 0 means 32, the only
 *                      length the chunked form implements (any other value
 *                      returns WKV7_ERR_UNSUPPORTED; the result of the
 *                      recurrence does not depend on the chunk length).
 *   workspace        : wkv7_forward_workspace_size() bytes, or NULL if 0.
 * The chunked form needs the per-chunk decay product of every channel to stay
 * in fp32's normal range (prod of 32 consecutive w >= 1e-30); a chunk outside
 * it raises WKV7_ERR_RANGE in the device status word (read it with
 * wkv7_get_last_status) and its outputs are unspecified.  The SEQ form has no
 * such limit: callers whose decays can be that strong poll the status word
 * or choose WKV7_ALGO_SEQ.
 */
WKV7_API wkv7_status wkv7_forward(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype y_dtype,
                         const void *r, const void *w, const void *k, const void *v,
                         const void *a, const void *b, const float *s0, void *y, float *sT,
                         wkv7_algo algo, int chunk_len, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * Sequence (context) parallel forward, in three calls around an exchange.
 * The recurrence is affine in the state (the transition diag(w_t) + a_t b_t^T
 * does not depend on S: RWKV-7 "Goose" paper review, section "Architecture"),
 * so a stretch of T tokens maps its entry state to its final state as
 *     S_out = S_in M + E,
 *     M = prod_t (diag(w_t) + a_t b_t^T)      (t in order, right-multiplied)
 *     E = the final state of the stretch started from S = 0.
 * A sequence split over P devices in order runs, on device i with stretch i:
 *   wkv7_forward_summary   -> [E_i; M_i]
 *   (exchange the P summaries: an all-gather)
 *   wkv7_compose_states    -> the entry state of every stretch
 *   wkv7_forward_continue  -> y of stretch i from its entry state
 * which gives the same y and final state as one wkv7_forward over the whole
 * sequence.  All three take bf16 inputs (the chunked form); fp32 inputs return
 * WKV7_ERR_UNSUPPORTED.
 */

/* Bytes of scratch that lets wkv7_forward_summary / wkv7_forward_continue
 * split a stretch into segments that run in parallel (0 when one pass fills
 * the GPU).  Both calls of a pair must get the same workspace. */
WKV7_API size_t wkv7_forward_summary_workspace_size(int B, int T, int H, int N);

/*
 * Summary of one stretch.
 *   r, w, k, v, a, b : [B, T, H, N] bf16
 *   summary          : [2, B, H, N, N] fp32, written: summary[0] = E,
 *                      summary[1] = M.  T = 0 gives E = 0, M = I.
 *   workspace        : wkv7_forward_summary_workspace_size() bytes, or NULL.
 *                      With it the stretch runs as segments whose summaries
 *                      are chained into E and M and stay in the workspace for
 *                      wkv7_forward_continue, with every token's two partial
 *                      outputs (fp32, 512 B per head-token); without it, one launch that
 *                      carries both states through the stretch (from S = 0,
 *                      and from S = I with v read as 0).
 * Shares the chunked form's numeric domain (see wkv7_forward).
 */
WKV7_API wkv7_status wkv7_forward_summary(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                          const void *r, const void *w, const void *k, const void *v,
                                          const void *a, const void *b, float *summary, void *workspace,
                                          size_t workspace_bytes, cudaStream_t stream);

/*
 * Forward of one stretch from its entry state s_in (NULL = zeros), after
 * wkv7_forward_summary ran on the SAME inputs with the SAME workspace pointer
 * and size, and nothing wrote the workspace in between (the segment summaries
 * and per-token partial outputs it left there are reused; the results are
 * unspecified otherwise).  With that workspace it does no chunk work: a
 * segment's state at token t is S_in M_{<=t} + E_{<=t}, so its output is
 * y0_t + S_in q_t, where y0 (the output from S = 0) and q_t = M_{<=t} r_t
 * come from the summary pass; the call chains the segments' entry states
 * and adds S_in q.  With a NULL workspace it is a plain one-pass chunked
 * forward from s_in.
 *   y  : [B, T, H, N] of y_dtype, written
 *   sT : [B, H, N, N] fp32 final state of the stretch, or NULL
 */
WKV7_API wkv7_status wkv7_forward_continue(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                           wkv7_dtype y_dtype, const void *r, const void *w, const void *k,
                                           const void *v, const void *a, const void *b, const float *s_in,
                                           void *y, float *sT, void *workspace, size_t workspace_bytes,
                                           cudaStream_t stream);

/*
 * Entry states of nseg consecutive stretches from their summaries:
 *     states[0] = s0 (or zeros when s0 is NULL)
 *     states[k + 1] = states[k] M_k + E_k,  k = 0 .. nseg - 1
 *   summaries : [nseg, 2, B, H, N, N] fp32, summaries[k] as written by
 *               wkv7_forward_summary for stretch k (may be NULL if nseg = 0)
 *   states    : [nseg + 1, B, H, N, N] fp32, written; states[k] is the state
 *               before stretch k and states[nseg] the final state.  states
 *               must not overlap s0 or summaries.
 * fp32 on CUDA cores, one launch; nseg >= 0.
 */
WKV7_API wkv7_status wkv7_compose_states(int nseg, int B, int H, int N, const float *s0,
                                         const float *summaries, float *states, cudaStream_t stream);

/*
 * Sequence-parallel backward, the forward's steps in reverse.  The state
 * gradient is affine too: for a stretch with summary M (see above),
 *     dL/dS_in = dL/dS_out M^T + F,
 * F being the stretch's own contribution (dL/dS_in with dL/dS_out = 0).  On
 * device i with stretch i, after the sequence-parallel forward:
 *   wkv7_state_gradient (dsT = NULL) -> F_i
 *   (exchange the P F's: an all-gather)
 *   wkv7_compose_adjoints            -> dL/dS before and after every stretch
 *   wkv7_backward (s0 = the stretch's entry state, dsT = dL/dS after it)
 * which gives the gradients of one wkv7_backward over the whole sequence.
 */

/*
 * dL/dS_0 of L = sum(dy * y) + sum(dsT * S_T) over a stretch: the reverse
 * sweep of the state gradient alone (G += dy_t r_t^T, then G <- G A_t^T).
 * Needs neither k, v nor the states.  With a workspace of at least
 * wkv7_state_gradient_workspace_size bytes, a sweep over few heads runs as
 * segments side by side (each carrying G from 0 and a second G from I, the
 * two chained afterwards), else as one pass per head.
 *   r, w, a, b, dy : [B, T, H, N] of in_dtype
 *   dsT            : [B, H, N, N] fp32, or NULL for zeros
 *   ds0            : [B, H, N, N] fp32, written
 *   workspace      : device scratch, 16-byte aligned, or NULL
 */
WKV7_API size_t wkv7_state_gradient_workspace_size(int B, int T, int H, int N);
WKV7_API wkv7_status wkv7_state_gradient(int B, int T, int H, int N, wkv7_dtype in_dtype, const void *r,
                                         const void *w, const void *a, const void *b, const void *dy,
                                         const float *dsT, float *ds0, void *workspace, size_t workspace_bytes,
                                         cudaStream_t stream);

/*
 * dL/dS before every one of nseg consecutive stretches, last stretch first:
 *     adj[nseg] = dsT (or zeros when dsT is NULL)
 *     adj[k] = adj[k + 1] M_k^T + F_k,  k = nseg - 1 .. 0
 *   summaries : [nseg, 2, B, H, N, N] fp32 as for wkv7_compose_states (M_k in
 *               summaries[k][1]; may be NULL if nseg = 0)
 *   F         : [nseg, B, H, N, N] fp32, the stretches' own state gradients
 *   adj       : [nseg + 1, B, H, N, N] fp32, written; stretch k's backward
 *               takes dsT = adj[k + 1], and adj[0] is the whole sequence's ds0.
 *               adj must not overlap the inputs.
 */
WKV7_API wkv7_status wkv7_compose_adjoints(int nseg, int B, int H, int N, const float *dsT, const float *summaries,
                                           const float *F, float *adj, cudaStream_t stream);

/*
 * wkv7_forward with r..b, s0, y and sT in HOST memory (page-locked memory
 * lets the copies overlap the computation; pageable memory works, slower).
 * The sequence is cut into up to 8 time slices of whole 32-token chunks; the
 * upload of slice k+1 and the download of slice k-1's y run on two internal
 * streams while slice k computes on `stream`, and the state is carried from
 * slice to slice on the device.  The algorithm is resolved once for the whole
 * T.  Results equal wkv7_forward's up to the chunked form's segment choice,
 * which is made per slice.
 *   host tensors : same shapes and dtypes as wkv7_forward; s0 / sT may be NULL
 *   workspace    : DEVICE scratch of wkv7_forward_host_workspace_size() bytes
 *                  (two slots of slice inputs and y, the state, the forward's
 *                  own workspace); required, also for T = 0.
 * Asynchronous on `stream` like every call: the host buffers must stay valid
 * and unmodified (y, sT unread) until `stream` reaches this point.  Each call
 * creates two streams and a few events and releases them before returning
 * (the driver frees them when their work completes), so it is not meant for
 * stream capture.
 */
WKV7_API size_t wkv7_forward_host_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                                 wkv7_dtype y_dtype, wkv7_algo algo, int chunk_len);
WKV7_API wkv7_status wkv7_forward_host(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype y_dtype,
                                       const void *r, const void *w, const void *k, const void *v, const void *a,
                                       const void *b, const float *s0, void *y, float *sT, wkv7_algo algo,
                                       int chunk_len, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The algorithm wkv7_forward runs for these arguments (WKV7_ALGO_SEQ or
 * WKV7_ALGO_CHUNK; AUTO picks CHUNK for bf16 inputs with T >= 64), or -1 for
 * an invalid dtype / algorithm.  The chunked form takes bf16 inputs only.
 */
WKV7_API int wkv7_forward_resolve_algo(int T, wkv7_dtype in_dtype, wkv7_algo algo);

/*
 * Forward with the time-mix block's output epilogue.  The pages describe it in
 * words (Paper Review: RWKV-7 "Goose" with Expressive Dynamic State Evolution,
 * section "The approach"): after the state update the receptance reads the
 * state; the block also attends to the current token directly, without that
 * token being stored in the state; the result is normalised per head, the
 * heads are combined, and a gate is applied (the linear layer that follows
 * needs trained weights and is not part of this call).  Our reading of those
 * words, per (b, t, h):
 *     o_t = S_t r_t + (sum_j r_t[j] rho[h][j] k_t[j]) v_t
 *     z_t[i] = g_t[i] * (gamma[h][i] (o_t[i] - mean(o_t)) / sqrt(var(o_t) + eps) + beta[h][i])
 * with the mean and the population variance over the head's N channels.
 *   r..b, s0, sT, algo, chunk_len : as wkv7_forward (sT is the plain
 *                      recurrence's final state: the current-token term never
 *                      enters the state)
 *   rho              : [H, N] fp32 current-token weight (required; zeros give
 *                      the normalised readout)
 *   gamma, beta      : [H, N] fp32, or NULL for 1 and 0
 *   g                : [B, T, H, N] of in_dtype gate values, or NULL for 1
 *   eps              : >= 0, added to the variance
 *   z                : [B, T, H, N] of out_dtype, written
 *   workspace        : wkv7_forward_timemix_workspace_size() bytes.  The
 *                      chunked form applies the epilogue inside its kernel
 *                      (same scratch as wkv7_forward); the sequential scan
 *                      writes an fp32 y there and maps it to z in a second pass.
 */
WKV7_API size_t wkv7_forward_timemix_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                                    wkv7_algo algo, int chunk_len);
WKV7_API wkv7_status wkv7_forward_timemix(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype out_dtype,
                                          const void *r, const void *w, const void *k, const void *v,
                                          const void *a, const void *b, const float *s0, const float *rho,
                                          const float *gamma, const float *beta, const void *g, float eps,
                                          void *z, float *sT, wkv7_algo algo, int chunk_len, void *workspace,
                                          size_t workspace_bytes, cudaStream_t stream);

/*
 * One decode token (T = 1) for every (b, h), updating the state IN PLACE
 * (constant memory and time per token: RWKV-7 "Goose" abstract).
 *   r, w, k, v, a, b : [B, H, N] of in_dtype
 *   state            : [B, H, N, N] fp32, read and overwritten with S_t
 *   y                : [B, H, N] of y_dtype
 */
WKV7_API wkv7_status wkv7_step(int B, int H, int N, wkv7_dtype in_dtype, wkv7_dtype y_dtype,
                      const void *r, const void *w, const void *k, const void *v,
                      const void *a, const void *b, float *state, void *y, cudaStream_t stream);

/* Bytes of scratch wkv7_backward takes: per (b, h), the state before every
 * 32-token chunk, dL/dS at the end of every chunk, and the final state
 * (fp32, 16 KiB each); for few heads over many tokens also 3 states per
 * segment of the state-gradient sweep (see below); and every chunk's
 * transition image (24 KiB per chunk, used for bf16 inputs).  The call also
 * runs with less, down to this size minus the transition images (dL/dS then
 * comes from the per-token sweep).  Depends on the current device's SM
 * count.  The checkpoints are what lets the backward run its chunks in
 * parallel instead of token by token: the method is presented as keeping
 * training parallelisable (RWKV-7 "Goose" with Expressive Dynamic State
 * Evolution, abstract). */
WKV7_API size_t wkv7_backward_workspace_size(int B, int T, int H, int N);

/*
 * Backward: gradients of L = sum(dy * y) + sum(dsT * sT) with respect to every
 * input and the initial state, i.e. the training pass of the recurrence above.
 * The pages give no gradient formula; they say the formulation keeps training
 * parallelisable (RWKV-7 "Goose" with Expressive Dynamic State Evolution,
 * abstract), and this call is the reverse-mode derivative of the recurrence
 * taken chunk by chunk.  Three steps: state checkpoints every 32
 * tokens, dL/dS at every chunk end (and ds0), then the input gradients of
 * every chunk independently (the adjoint of the chunked form of the
 * recurrence): on the tensor cores for bf16 inputs (bf16 hi/lo operands, fp32
 * accumulation), in fp32 on the CUDA cores for fp32 inputs.
 * dL/dS comes, for bf16 inputs with the full workspace, from the chunks'
 * transitions: the chunk's state map is affine, S_out = S_in M + E with
 * y_t = S_in q_t + (terms without S_in), so dS_in = dS_out M^T + dY^T Q, one
 * tensor-core product per chunk ([M^T; Q] exported by the checkpoint pass).
 * Otherwise it comes from a reverse sweep of the state gradient, token by
 * token.  When the heads leave most SMs idle that sweep runs as segments
 * side by side: a dual pass per segment (dL/dS from 0 with dy, and the
 * segment's transposed transition product from I), a chain of those for
 * every segment's exit adjoint, and a second pass that records dS.  A cost
 * model picks the chain or the sweep; the results agree within the bf16
 * bound.
 *   r..b, s0         : the forward's inputs (s0 NULL = zeros)
 *   dy               : [B, T, H, N] of in_dtype
 *   dsT              : [B, H, N, N] fp32, or NULL for zeros
 *   dr, dw, dk, dv, da, db : [B, T, H, N] of grad_dtype, overwritten
 *   ds0              : [B, H, N, N] fp32, overwritten (required)
 *   workspace        : wkv7_backward_workspace_size() bytes (at least that
 *                      size minus the transition images; less is
 *                      WKV7_ERR_INVALID_ARG)
 * dw is dL/dw for the decay value w itself.
 */
WKV7_API wkv7_status wkv7_backward(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype grad_dtype,
                          const void *r, const void *w, const void *k, const void *v,
                          const void *a, const void *b, const float *s0, const void *dy,
                          const float *dsT, void *dr, void *dw, void *dk, void *dv, void *da,
                          void *db, float *ds0, void *workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/*
 * Training pair: a forward that also keeps what the backward needs, and a
 * backward that starts from it instead of recomputing the states (saves the
 * checkpoint pass, about a quarter of wkv7_backward on the training workload).
 *
 * Bytes of the saved states: the state before every 32-token chunk,
 * [B, H, ceil(T / 32), N, N] fp32 (512 B per head-token at N = 64), then,
 * from the next multiple of 256 bytes on, every chunk's transition image
 * (24 KiB per chunk: 768 B per head-token; written for bf16 inputs, opaque).
 */
WKV7_API size_t wkv7_saved_states_size(int B, int T, int H, int N);

/*
 * wkv7_forward that also writes `states` (wkv7_saved_states_size() bytes,
 * device, overwritten; states[b][h][c] = the state before token 32 c, then
 * the chunks' transitions).  sT is required here (the backward reads it as
 * the state after the last chunk).  Same arguments, algorithms, results and
 * errors as wkv7_forward otherwise.  For bf16 inputs the states and the
 * transitions always come from the chunked form (the backward's dS chain
 * needs the transitions): when the call runs the scan (WKV7_ALGO_SEQ, or
 * AUTO below 64 tokens) y and sT come from the scan and one chunked pass
 * without y writes the states and transitions.
 */
WKV7_API wkv7_status wkv7_forward_train(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype y_dtype,
                                        const void *r, const void *w, const void *k, const void *v,
                                        const void *a, const void *b, const float *s0, void *y, float *sT,
                                        float *states, wkv7_algo algo, int chunk_len, void *workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

/* Bytes of scratch wkv7_backward_from_states needs: dL/dS at the end of every
 * 32-token chunk, fp32, and the segmented sweep's scratch. */
WKV7_API size_t wkv7_backward_from_states_workspace_size(int B, int T, int H, int N);

/*
 * wkv7_backward given the states and sT that wkv7_forward_train wrote for the
 * same inputs (s0 is not needed: states[.][.][0] is it).  Two launches:
 * dL/dS at every chunk end (bf16 inputs: the transition chain over the saved
 * transitions; fp32: the per-token sweep) and the chunk gradients.  Same
 * gradients, dtypes and errors as wkv7_backward (for bf16 inputs bit for bit
 * with wkv7_backward given its full workspace when the forward ran the
 * chunked form).
 */
WKV7_API wkv7_status wkv7_backward_from_states(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                               wkv7_dtype grad_dtype, const void *r, const void *w,
                                               const void *k, const void *v, const void *a, const void *b,
                                               const float *states, const float *sT, const void *dy,
                                               const float *dsT, void *dr, void *dw, void *dk, void *dv,
                                               void *da, void *db, float *ds0, void *workspace,
                                               size_t workspace_bytes, cudaStream_t stream);

/*
 * wkv7_backward without workspace: the same computation, arguments and
 * outputs, with its scratch taken from a fixed 32 MiB array in device memory
 * that belongs to the library.  The pages have no counterpart of this call; it
 * exists for callers that cannot allocate device memory where they run the
 * backward (an engine plugin whose enqueue path must not call the allocator,
 * or a framework whose memory pool already holds the device's memory).
 *   - Every GPU that loads the library keeps the 32 MiB array until exit.
 *   - Problems whose wkv7_backward_workspace_size() without the transition
 *     images exceeds 32 MiB return WKV7_ERR_TOO_LARGE and launch nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it: make that first call before any
 *     stream capture.
 *   - All calls share the array, which keeps the previous call's contents
 *     (the backward overwrites every scratch byte before reading it).  Calls
 *     that overlap on the GPU race on the array: do not run two at once.
 *   - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 */
WKV7_API wkv7_status wkv7_backward_noalloc(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                           wkv7_dtype grad_dtype, const void *r, const void *w, const void *k,
                                           const void *v, const void *a, const void *b, const float *s0,
                                           const void *dy, const float *dsT, void *dr, void *dw, void *dk,
                                           void *dv, void *da, void *db, float *ds0, cudaStream_t stream);

/*
 * Bound, in SM clock cycles, on every device-side wait of kernels launched
 * afterwards from this process (the tensor-core round handshakes of the
 * chunked forward and of the backward's chunk gradients).  A wait that runs out sets WKV7_ERR_TIMEOUT in the device status
 * word, lets already-committed tensor-core work finish, frees its tensor
 * memory and returns; the context stays usable.  0 restores the default
 * (about one second).  Meant for testing that path.
 */
WKV7_API void wkv7_set_wait_limit(long long cycles);

/*
 * Synchronizes `stream`, then returns and clears the sticky device-side status
 * word of the current device (WKV7_OK, WKV7_ERR_TIMEOUT or WKV7_ERR_RANGE), or
 * WKV7_ERR_CUDA if the synchronization itself failed.  Kernels cannot return
 * a status to the host, so conditions found on the device (a bounded wait
 * that ran out; a chunk whose decay product leaves the chunked form's range,
 * which matters because the recurrence is sensitive to numerical precision:
 * Elamur Research summary of RWKV-7 "Goose", section "Limitations") are
 * recorded in this word until read.  A caller of the chunked form that wants
 * to know its outputs are valid calls this after the work it cares about.
 */
WKV7_API wkv7_status wkv7_get_last_status(cudaStream_t stream);

/* The same call as wkv7_get_last_status, under its earlier name. */
WKV7_API wkv7_status wkv7_get_device_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV7_H */
