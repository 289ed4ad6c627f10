/*
 * flare.h - C ABI of the B200 (sm_100a) FLARE / FLARE++ mixer, forward and
 * backward (gradients).
 *
 * What the calls compute (FLARE++ paper, arXiv 2608.11519, section "Method"):
 *
 *   flare_mixer_fwd      FLARE, section "FLARE: fixed-query latent routing"
 *                        (eq. 5-6): per head h, with learned queries Q_h (M x D)
 *                          Z_h = softmax_n(Q_h K_h^T * scale) V_h        (encode)
 *                          Y_h = softmax_m(K_h Q_h^T * scale) Z_h        (decode)
 *
 *   flarepp_mixer_fwd    FLARE++, section "FLARE++: dynamic token routing"
 *                        (eq. 7-11): per head h
 *                          K~_h = X W~_K,h,  V~_h = X W~_V,h             (eq. 7)
 *                          Q_h(X) = softmax_n(Q~_h K~_h^T * scale) V~_h  (eq. 8)
 *                          K_h = X W_K,h,  V_h = X W_V,h                 (eq. 9)
 *                          Z_h = softmax_n(Q_h(X) K_h^T * scale) V_h     (eq. 10)
 *                          Y_h = softmax_m(K_h Q_h(X)^T * scale) Z_h     (eq. 11)
 *                        W_{.,h} is column block [h*D, (h+1)*D) of the C x C
 *                        matrix W (section "Full self-attention": H heads of
 *                        width D = C/H).
 *
 * flarepp_mixer_out_fwd adds the head concatenation and the output projection
 * of section "Full self-attention" (the heads' outputs side by side, times
 * the C x C matrix W_O); the other calls return Y per head.
 *
 * Conventions shared by every call
 * --------------------------------
 *   - bf16 tensors are passed as pointers to 16-bit bit patterns (flare_bf16),
 *     float tensors as float*.  All tensors are dense, row-major, in DEVICE
 *     memory, and every pointer must be 16-byte aligned.
 *   - Layouts: X [B][N][C]; W [C][C] with K = X @ W (row-vector convention);
 *     K, V, Y [B][H][N][D]; Q, Q0 [H][M][D] (shared by the whole batch);
 *     debug outputs Q(X) and Z are float [B][H][M][D].
 *   - Supported sizes: B, H, N >= 1; D in {16, 32}; M a multiple of 16 in
 *     [16, 512]; FLARE++ also needs C = H*D, C a multiple of 64, C <= 256.
 *   - lengths: optional DEVICE int32[B] (NULL = every token valid).  Tokens
 *     n >= lengths[b] are padding: they are not keys of the synthesis and
 *     encode softmaxes and their rows of Y are written as zeros.  A length
 *     outside [1, N] is clamped to [0, N] and reported by
 *     flare_last_device_status() as FLARE_ERR_SHAPE.
 *   - scale <= 0 selects the default 1/sqrt(D).
 *   - workspace: caller-owned DEVICE scratch of at least
 *     flare_workspace_bytes(...) bytes, 256-byte aligned.  The library never
 *     allocates or frees memory and keeps no state between calls; two calls
 *     that may run concurrently need two workspaces.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work on that stream and returns; inputs must
 *     stay valid until the stream has executed the work.  No call
 *     synchronises except flare_last_device_status().
 *   - Results are deterministic: the same inputs give bitwise-identical
 *     outputs on every run (fixed split count and fixed merge order, no
 *     floating-point atomics).
 *   - Errors: argument errors are detected on the host before anything is
 *     enqueued and returned as a flare_status.  A CUDA error while
 *     enqueueing returns FLARE_ERR_LAUNCH.  Errors found while the kernels
 *     run (a bounded wait that expired, an invalid length) are recorded in
 *     the workspace and returned by flare_last_device_status().  No call
 *     traps the device.
 */
#ifndef FLARE_H_
#define FLARE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLARE_API __attribute__((visibility("default")))
#else
#define FLARE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t flare_bf16; /* bfloat16 bit pattern */

typedef enum {
  FLARE_OK = 0,
  FLARE_ERR_NULL = 1,        /* a required pointer is NULL                        */
  FLARE_ERR_SHAPE = 2,       /* a size is out of range or inconsistent            */
  FLARE_ERR_UNSUPPORTED = 3, /* valid math, but a size this build does not cover  */
  FLARE_ERR_ALIGN = 4,       /* a pointer is not 16-byte (workspace: 256) aligned */
  FLARE_ERR_WORKSPACE = 5,   /* workspace smaller than flare_workspace_bytes()    */
  FLARE_ERR_LAUNCH = 6,      /* CUDA error while enqueueing (no sm_100 device...) */
  FLARE_ERR_TIMEOUT = 7,     /* a device-side bounded wait expired                */
  FLARE_ERR_UNDERFLOW = 8,   /* context parallelism without the exact step: a merged
                                row's sums underflowed and were not recomputed  */
  FLARE_ERR_NO_FORWARD = 9   /* a *_bwd_train call found no *_fwd_train state in
                                its workspace (none run, or already used)       */
} flare_status;

/* Variant selector for flare_workspace_bytes(). */
#define FLARE_VARIANT_FLARE 0
#define FLARE_VARIANT_FLAREPP 1
#define FLARE_VARIANT_FLAREPP_OUT 2 /* flarepp_mixer_out_fwd */
#define FLARE_VARIANT_FLARE_BWD 3   /* flare_mixer_bwd */
#define FLARE_VARIANT_FLAREPP_BWD 4 /* flarepp_mixer_bwd */

/*
 * Workspace size in bytes for one call with these sizes (C is ignored for
 * FLARE).  Returns 0 when the sizes are not supported.  Pure host function.
 */
FLARE_API size_t flare_workspace_bytes(int variant, int B, int H, int N, int M, int D, int C);

/*
 * FLARE mixer forward (eq. 5-6).
 *   K, V    [B][H][N][D] bf16, read only
 *   Q       [H][M][D]    bf16, read only (learned latent queries)
 *   Y       [B][H][N][D] bf16, written
 *   Z_out   [B][H][M][D] float, written if not NULL (latent values, debug)
 */
FLARE_API flare_status flare_mixer_fwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                             int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                             void* workspace, size_t workspace_bytes, void* stream, float* Z_out);

/*
 * FLARE++ mixer forward (eq. 7-11).
 *   X                       [B][N][C] bf16, read only
 *   Wk, Wv, Wk_syn, Wv_syn  [C][C]    bf16, read only (W_K, W_V, W~_K, W~_V)
 *   Q0                      [H][M][D] bf16, read only (learned seeds Q~)
 *   Y                       [B][H][N][D] bf16, written
 *   Qx_out, Z_out           [B][H][M][D] float, written if not NULL (the
 *                           synthesised routing queries Q(X) and the latent
 *                           values Z, for inspection)
 * Passing the same pointers as Wk_syn/Wv_syn and Wk/Wv selects the shared
 * projection variant (W~ = W, so K~ = K and V~ = V): the result is the same
 * as with two copies of the weights, and only two projections are computed.
 */
FLARE_API flare_status flarepp_mixer_fwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                               flare_bf16* Y, int B, int N, int C, int H, int M, int D,
                               const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                               void* stream, float* Qx_out, float* Z_out);

/*
 * FLARE++ mixer forward with the head concatenation and the output
 * projection (section "Full self-attention"):
 *   Out[b][n][:] = (Y_1[b][n][:], ..., Y_H[b][n][:]) @ W_O
 * with Y_h as in flarepp_mixer_fwd.
 *   X, Wk, Wv, Wk_syn, Wv_syn, Q0   as in flarepp_mixer_fwd
 *   Wo    [C][C] bf16, read only (W_O, row-vector convention: Out = Ycat @ Wo)
 *   Out   [B][N][C] bf16, written; rows of padding tokens are zero
 * Needs flare_workspace_bytes(FLARE_VARIANT_FLAREPP_OUT, ...) bytes of
 * workspace (the FLARE++ workspace plus Y with the heads side by side).
 */
FLARE_API flare_status flarepp_mixer_out_fwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                             const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                             const flare_bf16* Q0, const flare_bf16* Wo, flare_bf16* Out, int B,
                                             int N, int C, int H, int M, int D, const int32_t* lengths, float scale,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Profiling variants: identical work, plus cudaEventRecord() of caller-created
 * events (cudaEvent_t passed as void*) on `stream` between the stages, so a
 * caller can time each kernel on the stream it runs on.  A NULL array (or a
 * NULL entry) records nothing.
 *   flare_mixer_fwd_profiled:   5 events around key norms | encode | merge |
 *                               decode   (events[i] precedes stage i,
 *                               events[4] follows the decode)
 *   flarepp_mixer_fwd_profiled: 7 events around projections | synthesis
 *                               encode | synthesis merge | encode | merge |
 *                               decode   (events[6] follows the decode)
 */
FLARE_API flare_status flare_mixer_fwd_profiled(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                                flare_bf16* Y, int B, int H, int N, int M, int D,
                                                const int32_t* lengths, float scale, void* workspace,
                                                size_t workspace_bytes, void* stream, float* Z_out,
                                                void* const* stage_events);
FLARE_API flare_status flarepp_mixer_fwd_profiled(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                                  const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                                  const flare_bf16* Q0, flare_bf16* Y, int B, int N, int C, int H,
                                                  int M, int D, const int32_t* lengths, float scale,
                                                  void* workspace, size_t workspace_bytes, void* stream,
                                                  float* Qx_out, float* Z_out, void* const* stage_events);

/*
 * Inspection variants: identical work and outputs, plus Y_f32_out
 * [B][H][N][D] float (written, required): the fp32 values that the decoder
 * rounds to the bf16 Y (zeros for padding tokens).  They let a caller check
 * the token-dependent part of Y (the routing of eq. 6 / eq. 11) more finely
 * than bf16 resolves it.  Other arguments as in flare_mixer_fwd /
 * flarepp_mixer_fwd.
 */
FLARE_API flare_status flare_mixer_fwd_inspect(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                               flare_bf16* Y, int B, int H, int N, int M, int D,
                                               const int32_t* lengths, float scale, void* workspace,
                                               size_t workspace_bytes, void* stream, float* Z_out,
                                               float* Y_f32_out);
FLARE_API flare_status flarepp_mixer_fwd_inspect(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                                 const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                                 const flare_bf16* Q0, flare_bf16* Y, int B, int N, int C, int H,
                                                 int M, int D, const int32_t* lengths, float scale,
                                                 void* workspace, size_t workspace_bytes, void* stream,
                                                 float* Qx_out, float* Z_out, float* Y_f32_out);

/*
 * Backward (gradients of a scalar loss, given dY = dLoss/dY).
 *
 * The pages name the paper's backward equations (eq. 13-40) without
 * printing them; every step of the mixer is one SDPA call, so these calls
 * compute the SDPA backward of each step (for O = softmax_rows(s Qa Ka^T) Va:
 * dVa = P^T dO, dS = P (dO Va^T - rowsum(P (dO Va^T))), dQa = s dS Ka,
 * dKa = s dS^T Qa), chained through the mixer.  Each call is
 * self-contained: it takes the forward's inputs and dY, not the forward's
 * outputs, and first runs the training forward's kernels (below) into its
 * workspace without storing Y, so that what the forward produced (the
 * projections, Q(X), Z and the softmax normalisers) comes from the forward's
 * own launches; then the training backward's launches.  The gradients equal
 * those of the training pair on the same inputs bit for bit.  Outputs are
 * written (not accumulated).  Rows of dY for padding tokens are ignored;
 * padding tokens get zero gradients.  Same size limits as the forward, and
 * B*H <= 65535.  Arithmetic: the score and gradient products of the four
 * softmax passes and the projection gradients dX and dW on the tcgen05
 * tensor cores, each fp32 operand as the sum of two bf16 parts (high and
 * low), fp32 accumulation; softmax weights, normalisers and every reduction
 * in fp32.  (The context-parallel phases below recompute the forward's state
 * and run their softmax passes with tf32 tensor-core products; bf16 inputs
 * are exact in tf32.)  Deterministic like the forward.
 *
 * flare_mixer_bwd (FLARE, eq. 5-6), workspace variant FLARE_VARIANT_FLARE_BWD:
 *   K, V, Q, lengths, scale   as in flare_mixer_fwd
 *   dY    [B][H][N][D] bf16, read only
 *   dK, dV [B][H][N][D] bf16, written (dK sums the encoder's and the
 *          decoder's parts)
 *   dQ    [H][M][D] float, written (summed over the batch)
 */
FLARE_API flare_status flare_mixer_bwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                       const flare_bf16* dY, flare_bf16* dK, flare_bf16* dV, float* dQ, int B, int H,
                                       int N, int M, int D, const int32_t* lengths, float scale, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * flarepp_mixer_bwd (FLARE++, eq. 7-11), workspace variant
 * FLARE_VARIANT_FLAREPP_BWD:
 *   X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths, scale   as in flarepp_mixer_fwd
 *   dY    [B][H][N][D] bf16, read only (gradient of the per-head output Y)
 *   dX    [B][N][C] bf16, written
 *   dWk, dWv, dWk_syn, dWv_syn   [C][C] float, written
 *   dQ0   [H][M][D] float, written (summed over the batch)
 * With the shared-projection variant (Wk_syn == Wk and Wv_syn == Wv as
 * pointers) dWk and dWv receive the whole gradient of the shared weights;
 * dWk_syn and dWv_syn may then be NULL and, if given, receive the same
 * values.
 */
FLARE_API flare_status flarepp_mixer_bwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                         const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                         const flare_bf16* dY, flare_bf16* dX, float* dWk, float* dWv,
                                         float* dWk_syn, float* dWv_syn, float* dQ0, int B, int N, int C, int H,
                                         int M, int D, const int32_t* lengths, float scale, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * Training pair: a forward that keeps its state for the backward.
 *
 * The forward of a training step computes most of what the backward would
 * otherwise recompute: the projections K, V, K~, V~ (FLARE++), Q(X) and Z,
 * and the log-normaliser of every row of the synthesis and encode softmaxes
 * (eq. 8 and 10 of the FLARE++ paper; eq. 5 of the FLARE paper).  The
 * *_fwd_train calls run the forward and keep that state in the BACKWARD's
 * workspace (flare_workspace_bytes(FLARE_VARIANT_FLAREPP_BWD or
 * FLARE_VARIANT_FLARE_BWD, ...)); the *_bwd_train calls read it instead of
 * recomputing the projections and the synthesis and encode passes.  At
 * D = 16 the training forward's decoder runs its value product on fp16
 * operands (Z and the softmax weights in fp16 instead of bf16) so that Y sees
 * Z to 2^-12, and keeps the fp32 Y and the decoder's per-token
 * log-normalisers (eq. 11; eq. 6), which the backward then takes instead of
 * recomputing them; at D = 32 the backward recomputes those.
 *
 *   flarepp_mixer_fwd_train   arguments as flarepp_mixer_fwd; writes Y
 *   flarepp_mixer_bwd_train   arguments as flarepp_mixer_bwd
 *   flare_mixer_fwd_train     arguments as flare_mixer_fwd; writes Y
 *   flare_mixer_bwd_train     arguments as flare_mixer_bwd
 *
 * A *_bwd_train call must get the same workspace, inputs, sizes, lengths
 * and scale as the *_fwd_train call before it, with nothing else run in that
 * workspace in between.  The forward marks the workspace; every other entry
 * point clears the mark when it starts, and the backward checks it on the
 * device (no host synchronisation) and clears it when done, so one forward
 * serves one backward.  A backward without the mark still runs to its end on
 * whatever the workspace holds and reports FLARE_ERR_NO_FORWARD through
 * flare_last_device_status; its outputs are then meaningless.  Inputs changed
 * between the two calls are not detected.
 *
 * The backward's scores take the bf16 Q(X) that the forward's tensor-core
 * products took, unscaled, with the scale applied to the fp32 product as in
 * the forward, so that the forward's normalisers fit them; Z and the
 * synthesis' gamma use the forward's fp32 Z and Q(X).  The gradients equal
 * flarepp_mixer_bwd's (flare_mixer_bwd's) bit for bit.  At
 * D = 32 Y is written by the forward exactly as flarepp_mixer_fwd
 * (flare_mixer_fwd) writes it; at D = 16 it is the bf16 rounding of a Y
 * computed with fp16 Z and weights, within the forward's tolerance and no
 * further from the exact Y.
 */
FLARE_API flare_status flarepp_mixer_fwd_train(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                               const flare_bf16* Q0, flare_bf16* Y, int B, int N, int C, int H,
                                               int M, int D, const int32_t* lengths, float scale, void* workspace,
                                               size_t workspace_bytes, void* stream);
FLARE_API flare_status flarepp_mixer_bwd_train(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                               const flare_bf16* Q0, const flare_bf16* dY, flare_bf16* dX,
                                               float* dWk, float* dWv, float* dWk_syn, float* dWv_syn, float* dQ0,
                                               int B, int N, int C, int H, int M, int D, const int32_t* lengths,
                                               float scale, void* workspace, size_t workspace_bytes, void* stream);
FLARE_API flare_status flare_mixer_fwd_train(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                             flare_bf16* Y, int B, int H, int N, int M, int D,
                                             const int32_t* lengths, float scale, void* workspace,
                                             size_t workspace_bytes, void* stream);
FLARE_API flare_status flare_mixer_bwd_train(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                             const flare_bf16* dY, flare_bf16* dK, flare_bf16* dV, float* dQ, int B,
                                             int H, int N, int M, int D, const int32_t* lengths, float scale,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Context-parallel FLARE++ backward (the token-sharded encoder of section
 * "Multi-GPU context parallelism", eq. 13-14, with its backward).
 *
 * Token sharding as for the forward phases (rank r holds tokens
 * [r*N, (r+1)*N) of sequences of world*N tokens; X, dY and dX are the shard's
 * rows; `lengths` counts tokens of the whole sequences).  The backward runs in
 * FLARE_CP_BWD_PHASES phases, all with the same arguments except `phase`,
 * `gathered` and `exchange`:
 *
 *   for phase = 0 .. FLARE_CP_BWD_PHASES - 1:
 *     flarepp_cp_bwd_phase(phase, ..., gathered, exchange, ...)
 *     gathered = all-gather of every rank's `exchange`, in rank order
 *
 * Phase p (< FLARE_CP_BWD_PHASES - 1) writes flarepp_cp_bwd_exchange_bytes(p,
 * ...) bytes (fp32) to `exchange`; phase p > 0 reads `gathered` = world of
 * those buffers of phase p - 1, rank-major (NULL for phase 0; `exchange` is
 * NULL for the last phase).  Every rank merges the gathered buffers in the
 * same ascending (rank, split) order, so every rank ends with bitwise the
 * same dW_K, dW_V, dW~_K, dW~_V and dQ0 (written by the last two phases);
 * dX holds the shard's rows.  The phases recompute the forward's state
 * themselves (the projections, then Q(X), Z and the normalisers with the
 * backward's own tensor-core passes), so with world == 1 the result matches
 * flarepp_mixer_bwd to rounding, not bit for bit; both are within the same
 * tolerance of the exact gradients.  The phases of one rank share its workspace
 * (flare_workspace_bytes(FLARE_VARIANT_FLAREPP_BWD, ...) with the shard's N)
 * and carry the shard's state in it; the other arguments are as for
 * flarepp_mixer_bwd.  An out-of-range phase returns FLARE_ERR_SHAPE.
 */
#define FLARE_CP_BWD_PHASES 7
FLARE_API size_t flarepp_cp_bwd_exchange_bytes(int phase, int B, int N, int C, int H, int M, int D);
FLARE_API flare_status flarepp_cp_bwd_phase(int phase, const flare_bf16* X, const flare_bf16* Wk,
                                            const flare_bf16* Wv, const flare_bf16* Wk_syn,
                                            const flare_bf16* Wv_syn, const flare_bf16* Q0, const flare_bf16* dY,
                                            const float* gathered, float* exchange, flare_bf16* dX, float* dWk,
                                            float* dWv, float* dWk_syn, float* dWv_syn, float* dQ0, int B, int N,
                                            int C, int H, int M, int D, const int32_t* lengths, int rank,
                                            int world, float scale, void* workspace, size_t workspace_bytes,
                                            void* stream);

/*
 * Context-parallel FLARE backward (token sharding as for flare_cp_begin /
 * flare_cp_end; K, V, dY, dK and dV are the shard's rows, `lengths` counts
 * tokens of the whole sequences).  The backward of flare_mixer_bwd runs in
 * FLARE_CP_BWD_PHASES_FLARE phases with the same protocol as
 * flarepp_cp_bwd_phase: phase p (< last) writes
 * flare_cp_bwd_exchange_bytes(p, ...) bytes to `exchange`, the caller
 * all-gathers them in rank order and passes the result as `gathered` to phase
 * p + 1.  Every rank merges in ascending (rank, split) order, so every rank
 * ends with bitwise the same dQ (written by the last phase); dK and dV hold
 * the shard's rows (written by phase 2).  As for FLARE++, the phases
 * recompute the encoder's state, so with world == 1 the result matches
 * flare_mixer_bwd to rounding.  The phases of one rank share its workspace (FLARE_VARIANT_FLARE_BWD with the
 * shard's N).  An out-of-range phase returns FLARE_ERR_SHAPE.
 */
#define FLARE_CP_BWD_PHASES_FLARE 4
FLARE_API size_t flare_cp_bwd_exchange_bytes(int phase, int B, int H, int N, int M, int D);
FLARE_API flare_status flare_cp_bwd_phase(int phase, const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                          const flare_bf16* dY, const float* gathered, float* exchange,
                                          flare_bf16* dK, flare_bf16* dV, float* dQ, int B, int H, int N, int M,
                                          int D, const int32_t* lengths, int rank, int world, float scale,
                                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, reads the device error word of `workspace` and
 * returns FLARE_OK, FLARE_ERR_TIMEOUT, FLARE_ERR_SHAPE (invalid lengths) or
 * FLARE_ERR_UNDERFLOW (context-parallel merges only).
 * The word is cleared at the start of every mixer call.
 */
FLARE_API flare_status flare_last_device_status(void* workspace, void* stream);

/* Static, human-readable name of a status. */
FLARE_API const char* flare_status_string(flare_status status);

/*
 * Context parallelism (section "Multi-GPU context parallelism", eq. 13-14).
 *
 * The tokens of every sequence are split into `world` shards of N tokens, one
 * per rank: rank r holds tokens [r*N, (r+1)*N) of sequences of world*N tokens
 * (X, K, V and Y are the shard's rows; `lengths`, if given, counts tokens of
 * the whole sequence).  Each encoder pass produces per-split partial sums
 * ("partials", flare_cp_partials_bytes() bytes per rank, fp32); the caller
 * concatenates the partials of all ranks in rank order (an all-gather,
 * [world][...]) and passes them to the next phase, which merges them with
 * the log-sum-exp rule in a fixed order, so every rank holds bitwise the
 * same Q(X) and Z.  The projections and the decoder only touch local rows.
 *
 *   FLARE++ : flarepp_cp_begin -> all-gather (P1) -> flarepp_cp_exact(0, P1)
 *             -> all-gather (E1) -> flarepp_cp_middle(P1, E1)
 *             -> all-gather (P2) -> flarepp_cp_exact(1, P2)
 *             -> all-gather (E2) -> flarepp_cp_end(P2, E2)
 *   FLARE   : flare_cp_begin -> all-gather (P) -> flare_cp_exact(P)
 *             -> all-gather (E) -> flare_cp_end(P, E)
 *
 * The exact step: a row of an encoder whose fast-path sums may have lost
 * mass to underflow (the encoder shifts each split by a norm bound, which
 * can be far above the row's largest score) is recomputed exactly on one
 * GPU from all keys.  Across shards no rank holds all keys, so every rank
 * finds the same such rows in the gathered partials (the merge's own test)
 * and writes, for them, the exact partial sums of its own tokens (max,
 * sum, weighted values; two passes in fp32) to `exact_out`
 * (flare_cp_exact_bytes() bytes, fp32; other rows are marked empty).  The
 * all-gathered exact partials (E, [world][...] rank-major) let every rank's
 * merge combine those rows exactly with the same log-sum-exp rule, so the
 * result is exact for any split of the tokens.  The exact step does real
 * work only for rows that need it.  Passing NULL as exact_all skips it: a
 * row that needs it is then reported as FLARE_ERR_UNDERFLOW by
 * flare_last_device_status.
 *
 * The phases of one rank share its workspace (flare_workspace_bytes of the
 * same variant with the shard's N) and stream; the workspace carries the
 * projections, Q(X) and Z from one phase to the next.  All ranks must call
 * with the same sizes.  With world == 1 the result equals flare_mixer_fwd /
 * flarepp_mixer_fwd.
 */
FLARE_API size_t flare_cp_partials_bytes(int B, int H, int N, int M, int D);
FLARE_API size_t flare_cp_exact_bytes(int B, int H, int M, int D);

FLARE_API flare_status flarepp_cp_begin(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                        const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                        int B, int N, int C, int H, int M, int D, const int32_t* lengths, int rank,
                                        int world, float scale, void* workspace, size_t workspace_bytes,
                                        void* stream, float* partials);
/* pass 0: the query synthesis (after flarepp_cp_begin); pass 1: the encode
 * (after flarepp_cp_middle).  The weight pointers only tell the shared-
 * projection variant apart, as in flarepp_cp_begin; Q0 is read in pass 0. */
FLARE_API flare_status flarepp_cp_exact(int pass, const float* partials_all, const flare_bf16* Wk,
                                        const flare_bf16* Wv, const flare_bf16* Wk_syn, const flare_bf16* Wv_syn,
                                        const flare_bf16* Q0, int B, int N, int C, int H, int M, int D,
                                        const int32_t* lengths, int rank, int world, float scale, void* workspace,
                                        size_t workspace_bytes, void* stream, float* exact_out);
FLARE_API flare_status flarepp_cp_middle(const float* partials_all, const float* exact_all, int B, int N, int C,
                                         int H, int M, int D, const int32_t* lengths, int rank, int world,
                                         float scale, void* workspace, size_t workspace_bytes, void* stream,
                                         float* partials, float* Qx_out);
FLARE_API flare_status flarepp_cp_end(const float* partials_all, const float* exact_all, flare_bf16* Y, int B,
                                      int N, int C, int H, int M, int D, const int32_t* lengths, int rank, int world,
                                      float scale, void* workspace, size_t workspace_bytes, void* stream,
                                      float* Z_out);
FLARE_API flare_status flare_cp_begin(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, int B, int H,
                                      int N, int M, int D, const int32_t* lengths, int rank, int world, float scale,
                                      void* workspace, size_t workspace_bytes, void* stream, float* partials);
FLARE_API flare_status flare_cp_exact(const float* partials_all, const flare_bf16* K, const flare_bf16* V,
                                      const flare_bf16* Q, int B, int H, int N, int M, int D,
                                      const int32_t* lengths, int rank, int world, float scale, void* workspace,
                                      size_t workspace_bytes, void* stream, float* exact_out);
FLARE_API flare_status flare_cp_end(const float* partials_all, const float* exact_all, const flare_bf16* K,
                                    const flare_bf16* Q, flare_bf16* Y, int B, int H, int N, int M, int D,
                                    const int32_t* lengths, int rank, int world, float scale, void* workspace,
                                    size_t workspace_bytes, void* stream, float* Z_out);

/*
 * FLARE mixer forward for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call; it exists for callers that
 * must not call cudaMalloc (or any allocating routine) themselves, for
 * example code running where device allocation is forbidden or has to stay
 * under a fixed budget.  It computes exactly what flare_mixer_fwd computes,
 * with the same arguments minus the workspace: its scratch lives in a
 * fixed array of FLARE_STATIC_SCRATCH_BYTES bytes inside the library's
 * device image, which every GPU that loads the library keeps until the
 * process exits.  The call allocates nothing.
 *
 *   - Sizes whose workspace (flare_workspace_bytes(FLARE_VARIANT_FLARE, ...))
 *     exceeds FLARE_STATIC_SCRATCH_BYTES are rejected with
 *     FLARE_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on each device looks up the array's device address
 *     with that device current (cudaGetSymbolAddress); make that first call
 *     before any stream capture.
 *   - Every call, on every stream, shares the one array, and the array keeps
 *     the last call's contents (the words that must start at zero are
 *     cleared by each call).  Calls whose execution overlaps on the GPU race
 *     on the scratch and give wrong results: serialise them.
 *   - The device error word (an expired bounded wait, a length outside
 *     [1, N]) lives at the start of the shared array and is cleared by each
 *     call; read it with flare_static_last_device_status().
 */
#define FLARE_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
FLARE_API flare_status flare_mixer_fwd_static(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                              flare_bf16* Y, int B, int H, int N, int M, int D,
                                              const int32_t* lengths, float scale, void* stream, float* Z_out);

/*
 * flare_last_device_status() for flare_mixer_fwd_static: synchronises
 * `stream` and reads the device error word of the static scratch (the last
 * static call's, whichever stream it ran on).  Same return values.
 */
FLARE_API flare_status flare_static_last_device_status(void* stream);

/*
 * Pipe-throughput probes (no counterpart in the pages: they measure the
 * denominators of the exp-unit roofline on the device at hand).  Runs two
 * short kernels on `stream` -- independent chains of ex2.approx.f32 on the
 * special-function unit and of fp32 fma on the FMA pipe, one wave of CTAs
 * on every SM -- synchronises the stream and writes the results per SM
 * clock (from each SM's own clock64 counter, so independent of the clock
 * frequency) to *ex2_per_clk_sm and *ffma_per_clk_sm.  `scratch`: caller-
 * owned DEVICE memory of flare_probe_scratch_bytes() bytes, 256-byte
 * aligned.  Not for use during stream capture.
 */
FLARE_API size_t flare_probe_scratch_bytes(void);
FLARE_API flare_status flare_probe_pipe_rates(void* scratch, size_t scratch_bytes, void* stream,
                                              double* ex2_per_clk_sm, double* ffma_per_clk_sm);

/*
 * Self-test of the bounded-wait error path: enqueues one small kernel that
 * waits on an mbarrier nothing ever completes, with a limit of `timeout_ns`
 * nanoseconds (clamped to [1e3, 1e9]).  The wait expires, the kernel records
 * FLARE_ERR_TIMEOUT in the workspace error word and returns normally; read
 * it with flare_last_device_status().  workspace needs 256 bytes.
 */
FLARE_API flare_status flare_selftest_wait_timeout(void* workspace, void* stream, unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* FLARE_H_ */
