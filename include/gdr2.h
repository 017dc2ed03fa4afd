/*
 * gdr2.h -- C ABI of the B200 (sm_100a) Gated Delta Rule-2 sequence-mixer library (libgdr2.so).
 *
 * The operation is the Gated Delta Rule-2 recurrence of "Gated DeltaNet-2: Decoupling Erase and
 * Write in Linear Attention" (Hatamizadeh, Choi, Kautz), Eq. 10, restated step by step in the
 * review page's section "The Gated Delta Rule-2 State Update" (Steps 1-5). Per (batch b, head h),
 * with an fp32 state S in R^{dk x dv} (row = key channel, column = value channel):
 *
 *     alpha_t = exp(log_alpha_t)                           (section "Gate Parameterization", Eq. 12)
 *     S_t = (I - k_t (b_t (.) k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t (.) v_t)^T        (Eq. 10)
 *     o_t = S_t^T q_t                                      (Step 5: read of the updated state)
 *
 * log_alpha is the channel-wise log-decay (<= 0 in normal use), b the channel-wise erase gate on the
 * key axis (in [0,1], or [0,2] for the negative-eigenvalue variant of Eq. 11), w the channel-wise
 * write gate on the value axis. There is no query scale and no normalisation inside the mixer.
 *
 * Conventions shared by every entry point
 *   Pointers    : device pointers (memory of the current CUDA device) unless stated otherwise.
 *                 Every pointer must be 16-byte aligned.
 *   Layouts     : contiguous, row-major. Token tensors q, k, log_alpha, b, dq, dk, dlog_alpha, db
 *                 are [B, T, H, dk]; v, w, o, dv, dw, d_o are [B, T, H, dv]; states and their
 *                 gradients are [B, H, dk, dv]. Decode drops the T axis.
 *   dtype       : q, k, v, b, w, o and dq, dk, dv, db, dw, d_o are fp32 (GDR2_F32) or bf16
 *                 (GDR2_BF16). log_alpha, dlog_alpha, all states and state gradients are fp32
 *                 whatever the dtype (the pages keep the log-decay and the state in fp32).
 *   Sizes       : B, T, H >= 1; dk, dv in {64, 128} for the chunk entry points; decode takes dk in
 *                 {64, 128} and dv a multiple of 64 up to 256.
 *   Ownership   : the caller owns every buffer, workspaces included. The library never allocates,
 *                 frees or synchronises; all work is enqueued on `stream` (a cudaStream_t; NULL is
 *                 the legacy default stream) and results are valid once that stream reaches them.
 *                 Inputs are read only. Outputs must not overlap inputs or each other (except the
 *                 decode state, updated in place).
 *   Errors      : every function returns a status (GDR2_OK = 0) and never aborts or prints. Invalid
 *                 arguments are rejected before anything is launched. A failed launch returns
 *                 GDR2_ERR_CUDA. gdr2_status_string() names a status.
 *   Threads     : entry points are re-entrant; concurrent calls on different streams are safe if
 *                 their buffers (workspaces included) are distinct. The exception is
 *                 gdr2_chunk_fwd_noalloc, whose calls share one scratch array per device (see there).
 */
#ifndef GDR2_H
#define GDR2_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDR2_API __attribute__((visibility("default")))
#else
#define GDR2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { GDR2_F32 = 0, GDR2_BF16 = 1 } gdr2_dtype;

enum {
    GDR2_OK = 0,
    GDR2_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, non-positive size, bad dtype */
    GDR2_ERR_UNSUPPORTED = 2,  /* head dimensions the library has no kernel for */
    GDR2_ERR_WORKSPACE = 3,    /* workspace missing or smaller than gdr2_workspace_bytes() */
    GDR2_ERR_CUDA = 4,         /* a CUDA launch or device query failed */
    GDR2_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired (reported by gdr2_check) */
    GDR2_ERR_RANGE = 6,        /* a chunk's cumulative log-decay left the supported range (gdr2_check) */
    GDR2_ERR_BOUNDS = 7        /* debug build only: an index check in a kernel failed (gdr2_check) */
};

/* Library version as 10000*major + 100*minor + patch. */
GDR2_API int gdr2_version(void);

/* Static text for a status code (never NULL). */
GDR2_API const char *gdr2_status_string(int status);

/*
 * Device-side status of the calls made so far. The kernels never trap: a bounded wait that gives up
 * (about 2^26 polls of an mbarrier) or an input the chunk form cannot represent sets a bit in a device
 * status word and the kernel finishes. gdr2_check synchronises `stream` (a cudaStream_t; NULL = the
 * legacy default stream), reads and clears those words, and returns
 *   GDR2_ERR_TIMEOUT  a bounded wait expired: the outputs of the calls since the last check are not valid;
 *   GDR2_ERR_RANGE    in some chunk a channel's cumulative log-decay G_C (the sum of log_alpha over the
 *                     chunk's 64 rows) left [-160, 160] on the tensor-core path (dtype GDR2_BF16 with
 *                     dk = dv = 128) or [-80, 80] on the fp32 path, or was NaN: the chunk form scales keys
 *                     and erase keys by exponentials of the in-chunk log-decay in fp32 (relative to the
 *                     mid-chunk value on the tensor-core path), which leave its normal range there, so the
 *                     outputs of those calls are not valid (a mean log_alpha of -2.5, resp. -1.25, per
 *                     token over a full chunk reaches the bound; decode steps have no such limit), or,
 *                     on the per-chain path (gdr2_set_chunk_path), an fp16 operand of the chunk form
 *                     (w (.) v, the WY factors, the state) exceeded 65504 in magnitude;
 *   GDR2_ERR_BOUNDS   (only in the debug build, libgdr2_debug.so, compiled with -DGDR2_DEBUG) an index check in
 *                     a kernel failed: a chunk, chain, tile row or column, TMEM column or output index outside
 *                     its range; this is a library bug, reported first;
 *   GDR2_ERR_CUDA     the synchronisation or the read failed;
 *   GDR2_OK           otherwise.
 * It blocks the host until `stream` is idle; call it where a synchronisation is acceptable.
 */
GDR2_API int gdr2_check(void *stream);

/*
 * Kernel path of the chunk entry points for bf16 operands with dk = dv = 128 (unpacked batches, one value
 * head per key head). Both paths compute the chunkwise algorithm of the review's section "Chunkwise
 * Parallel Training via WY Representation"; they differ in how the work is laid out on the GPU:
 *   1  per-chain: one CTA walks each (batch, head) chain's chunks in order, reading every input once and
 *      keeping every derived operand on chip; fastest when the B*H chains fill most of a wave of SMs;
 *   2  chunk-parallel: the chunk-local work runs over all chunks at once and the serial state passes
 *      read its intermediates from the workspace, with the chunk-level scan when B*H is small;
 *   0  automatic (default): path 1 when a cost model with the step times measured on B200 favours it (B*H from
 *      91 to 148 chains, from 181 to 296, ...), path 2 otherwise.
 * The setting is process-wide and read at each call: gdr2_workspace_bytes() reports the size for the
 * path in force, so query it after changing the path, and keep the same path for a gdr2_chunk_fwd_train /
 * gdr2_chunk_bwd_saved pair. Results agree within the library's tolerances, not bit for bit. Returns
 * GDR2_ERR_INVALID_ARG for a value outside {0, 1, 2}.
 */
GDR2_API int gdr2_set_chunk_path(int path);
GDR2_API int gdr2_get_chunk_path(void);

/*
 * Bytes of device workspace that gdr2_chunk_fwd (for_bwd = 0) or gdr2_chunk_bwd (for_bwd = 1)
 * needs for these sizes. Returns 0 for invalid sizes. The workspace holds per-chunk intermediates of
 * the chunkwise algorithm (section "Chunkwise Parallel Training via WY Representation"): the WY
 * factors of Eq. 20, the chunk-boundary states of Eq. 23 and, for the backward, their gradients. It
 * needs no initialisation and its contents are meaningless after the call.
 */
GDR2_API size_t gdr2_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype, int for_bwd);

/*
 * Chunkwise-parallel forward, C = 64 (review sections "Chunkwise Parallel Training via WY
 * Representation", Steps 1-3, Eqs. 20-24, and Appendix C.2). Computes o_t for every token and the
 * state after the last token, exactly the Eq. 10 recurrence up to floating-point rounding.
 *   q, k, b        [B,T,H,dk] dtype     v, w  [B,T,H,dv] dtype     log_alpha [B,T,H,dk] fp32
 *   initial_state  [B,H,dk,dv] fp32, or NULL for a zero state
 *   o              [B,T,H,dv] dtype (written)
 *   final_state    [B,H,dk,dv] fp32 (written), or NULL when not wanted
 *   T may be any value >= 1; a partial last chunk behaves as identity transitions.
 */
GDR2_API int gdr2_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                   const void *b, const void *w, const float *initial_state,
                   void *o, float *final_state,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gate-aware chunkwise backward (review section "Gate-Aware Backward Pass", Eqs. 64-65, the
 * triangular-inverse VJP, the gate gradients dB = dEbar*gamma*K, dW = dZ*V, dV = dZ*W, and the
 * in-chunk reverse cumulative sum for the log-decay). The forward inputs are passed again and the
 * forward is recomputed inside; nothing from a previous gdr2_chunk_fwd call is needed.
 *   d_o            [B,T,H,dv] dtype, or NULL for zero      d_final_state [B,H,dk,dv] fp32 or NULL
 *   dq, dk, db     [B,T,H,dk] dtype (written)              dv, dw [B,T,H,dv] dtype (written)
 *   dlog_alpha     [B,T,H,dk] fp32 (written)
 *   d_initial_state[B,H,dk,dv] fp32 (written), or NULL when not wanted
 * These are the gradients of L = <o, d_o> + <S_T, d_final_state> with respect to q, k, v,
 * log_alpha, b, w and the initial state.
 */
GDR2_API int gdr2_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                   const void *b, const void *w, const float *initial_state,
                   const void *d_o, const float *d_final_state,
                   void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                   float *d_initial_state,
                   int B, int T, int H, int dk_, int dv_, int dtype,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Training pair: forward that keeps what the backward needs, and the backward that uses it.
 * gdr2_chunk_fwd_train computes exactly what gdr2_chunk_fwd computes (o, final_state) and, in the
 * same pass, fills `workspace` with the per-chunk intermediates of the chunkwise algorithm (WY
 * factors, decay-scaled operands and chunk-boundary states of Eqs. 20-24). The workspace must hold
 * gdr2_workspace_bytes(..., for_bwd = 1) bytes.
 * gdr2_chunk_bwd_saved then computes exactly what gdr2_chunk_bwd computes, reading those
 * intermediates instead of recomputing the forward. Its arguments are those of gdr2_chunk_bwd; the
 * inputs, sizes, dtype and workspace must be the ones of the gdr2_chunk_fwd_train call that filled
 * the workspace, with nothing else written to the workspace in between (the library cannot check
 * this; a mismatch gives wrong gradients, not an error).
 */
GDR2_API int gdr2_chunk_fwd_train(const void *q, const void *k, const void *v, const float *log_alpha,
                                  const void *b, const void *w, const float *initial_state,
                                  void *o, float *final_state,
                                  int B, int T, int H, int dk, int dv, int dtype,
                                  void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_saved(const void *q, const void *k, const void *v, const float *log_alpha,
                                  const void *b, const void *w, const float *initial_state,
                                  const void *d_o, const float *d_final_state,
                                  void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                  float *d_initial_state,
                                  int B, int T, int H, int dk_, int dv_, int dtype,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Grouped value heads (review, "Headed architecture and grouped-value attention" and Appendix C.3):
 * Hv = G H value heads share each key head. The key-side tensors stay on the key-head axis and value
 * head j reads key head floor(j / G); v, w, o and the states live on the value-head axis:
 *   q, k, log_alpha, b and dq, dk, dlog_alpha, db   [B, T, H, dk]
 *   v, w, o, d_o and dv, dw                          [B, T, Hv, dv]
 *   initial_state, final_state, d_final_state, d_initial_state   [B, Hv, dk, dv] fp32
 * Value head j computes exactly the recurrence of Eq. 10 with q, k, log_alpha, b of key head j / G
 * (the key side "repeated across the value-head group"); the key-side gradients are the sums of the
 * group's value heads' gradients. The four calls mirror gdr2_chunk_fwd, gdr2_chunk_fwd_train,
 * gdr2_chunk_bwd and gdr2_chunk_bwd_saved; the key-side work of a chunk is done once per group.
 * Hv must be a positive multiple of H (Hv = H is the plain layout); GDR2_BF16 with dk = dv = 128
 * only (others return GDR2_ERR_UNSUPPORTED). gdr2_workspace_bytes_gva returns 0 for invalid or
 * unsupported sizes.
 */
GDR2_API size_t gdr2_workspace_bytes_gva(int B, int T, int H, int Hv, int dk, int dv, int dtype, int for_bwd);

GDR2_API int gdr2_chunk_fwd_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                const void *b, const void *w, const float *initial_state,
                                void *o, float *final_state,
                                int B, int T, int H, int Hv, int dk, int dv, int dtype,
                                void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_fwd_train_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                      const void *b, const void *w, const float *initial_state,
                                      void *o, float *final_state,
                                      int B, int T, int H, int Hv, int dk, int dv, int dtype,
                                      void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                const void *b, const void *w, const float *initial_state,
                                const void *d_o, const float *d_final_state,
                                void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                float *d_initial_state,
                                int B, int T, int H, int Hv, int dk_, int dv_, int dtype,
                                void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_saved_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                      const void *b, const void *w, const float *initial_state,
                                      const void *d_o, const float *d_final_state,
                                      void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                      float *d_initial_state,
                                      int B, int T, int H, int Hv, int dk_, int dv_, int dtype,
                                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * Packed variable-length batches (review, Appendix C.6: sequences of different lengths packed along
 * one token axis, the state reset at every sequence start). The token tensors are [T, H, d] (B = 1):
 * the N sequences lie back to back, sequence n on tokens [cu_seqlens[n], cu_seqlens[n+1]).
 *   cu_seqlens     int32 [N + 1] DEVICE array, 0 = c_0 <= c_1 <= ... <= c_N = T (read on the stream;
 *                  the host never looks at it). Empty sequences are allowed. Other contents are not
 *                  an error the host can see: sequence n then covers [max_{m<=n} c_m, max_{m<=n+1} c_m)
 *                  clamped to [0, T], and tokens outside every sequence keep unspecified outputs.
 *   initial_state, final_state, d_final_state, d_initial_state
 *                  [N, H, dk, dv] fp32: one state per sequence (initial_state NULL = zeros).
 * Each sequence is computed exactly as a batch of one by gdr2_chunk_fwd / gdr2_chunk_bwd: a sequence
 * whose length is not a multiple of 64 ends in a partial chunk, and no chunk spans two sequences.
 * The four calls mirror gdr2_chunk_fwd, gdr2_chunk_fwd_train, gdr2_chunk_bwd and
 * gdr2_chunk_bwd_saved (the training pair shares one workspace of
 * gdr2_workspace_bytes_varlen(..., for_bwd = 1) bytes; the saved backward must get the same
 * cu_seqlens contents). Supported: dtype GDR2_BF16 with dk = dv = 128 (others return
 * GDR2_ERR_UNSUPPORTED); N <= 65535.
 * gdr2_workspace_bytes_varlen depends on N, T and H only (room for T/64 + N chunks per head, the
 * chunk and sequence tables, and one staging tile per sequence and head for the outputs of its
 * partial last chunk); it returns 0 for invalid or unsupported sizes.
 */
GDR2_API size_t gdr2_workspace_bytes_varlen(int N, int T, int H, int dk, int dv, int dtype, int for_bwd);

GDR2_API int gdr2_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                                   const void *b, const void *w, const float *initial_state,
                                   void *o, float *final_state, const int *cu_seqlens,
                                   int N, int T, int H, int dk, int dv, int dtype,
                                   void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_fwd_train_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                                         const void *b, const void *w, const float *initial_state,
                                         void *o, float *final_state, const int *cu_seqlens,
                                         int N, int T, int H, int dk, int dv, int dtype,
                                         void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                                   const void *b, const void *w, const float *initial_state,
                                   const void *d_o, const float *d_final_state,
                                   void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                   float *d_initial_state, const int *cu_seqlens,
                                   int N, int T, int H, int dk_, int dv_, int dtype,
                                   void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_saved_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                                         const void *b, const void *w, const float *initial_state,
                                         const void *d_o, const float *d_final_state,
                                         void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                         float *d_initial_state, const int *cu_seqlens,
                                         int N, int T, int H, int dk_, int dv_, int dtype,
                                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Packed variable-length batches with grouped value heads: the two layouts above together. The token
 * tensors q, k, b, log_alpha are [T, H, dk] and v, w, o (and dv, dw, d_o) are [T, Hv, dv] with
 * Hv = G H, value head j reading key head j / G; the states are [N, Hv, dk, dv], one per (sequence,
 * value head). cu_seqlens, the sequence semantics and the workspace rules are those of the packed
 * calls, with gdr2_workspace_bytes_varlen_gva(..., for_bwd) bytes. Each sequence is computed exactly as
 * a batch of one by the grouped-head calls. Supported: dtype GDR2_BF16 with dk = dv = 128, Hv a
 * multiple of H, N and Hv <= 65535 (others return GDR2_ERR_INVALID_ARG or GDR2_ERR_UNSUPPORTED).
 */
GDR2_API size_t gdr2_workspace_bytes_varlen_gva(int N, int T, int H, int Hv, int dk, int dv, int dtype,
                                                int for_bwd);

GDR2_API int gdr2_chunk_fwd_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                       const void *b, const void *w, const float *initial_state,
                                       void *o, float *final_state, const int *cu_seqlens,
                                       int N, int T, int H, int Hv, int dk, int dv, int dtype,
                                       void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_fwd_train_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                             const void *b, const void *w, const float *initial_state,
                                             void *o, float *final_state, const int *cu_seqlens,
                                             int N, int T, int H, int Hv, int dk, int dv, int dtype,
                                             void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                       const void *b, const void *w, const float *initial_state,
                                       const void *d_o, const float *d_final_state,
                                       void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                                       float *d_initial_state, const int *cu_seqlens,
                                       int N, int T, int H, int Hv, int dk_, int dv_, int dtype,
                                       void *workspace, size_t workspace_bytes, void *stream);

GDR2_API int gdr2_chunk_bwd_saved_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                             const void *b, const void *w, const float *initial_state,
                                             const void *d_o, const float *d_final_state,
                                             void *dq, void *dk, void *dv, float *dlog_alpha, void *db,
                                             void *dw, float *d_initial_state, const int *cu_seqlens,
                                             int N, int T, int H, int Hv, int dk_, int dv_, int dtype,
                                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gate and normalisation prologue: the steps immediately upstream of the mixer ("Gated DeltaNet-2",
 * review page, section "Gate Parameterization", Eqs. 11-12, and "Block Design", steps 2-3). Per
 * (token, head), from the branch pre-activations:
 *     q = x_q / ||x_q||,  k = x_k / ||x_k||      (L2 norm over the head's dk channels; a zero
 *                                                 vector gives zero, with zero gradient)
 *     log_alpha = -exp(a) (.) softplus(x_f + delta)          computed and stored in fp32 (Eq. 12)
 *     b = sigmoid(x_b), or 2 sigmoid(x_b) when neg_eig != 0  (Eq. 11, negative-eigenvalue variant)
 *     w = sigmoid(x_w)                                       (Eq. 11)
 * The outputs are exactly the inputs gdr2_chunk_fwd / gdr2_decode_step take.
 *   xq, xk, xf, xb [B,T,H,dk] dtype     xw [B,T,H,dv] dtype     a, delta [H,dk] fp32
 *   q, k, b [B,T,H,dk] dtype (written)  w [B,T,H,dv] dtype      log_alpha [B,T,H,dk] fp32
 * gdr2_gate_prologue_bwd takes the same inputs and the gradients of those outputs (dq, dk, db
 * [B,T,H,dk] dtype, dlog_alpha [B,T,H,dk] fp32, dw [B,T,H,dv] dtype) and writes dxq, dxk, dxf, dxb
 * [B,T,H,dk], dxw [B,T,H,dv] (dtype) and da, ddelta [H,dk] fp32 (sums over every token; computed
 * in a fixed order, so repeated calls give identical bits). Its workspace holds per-block partial
 * sums: gdr2_gate_prologue_workspace_bytes(...) bytes. Sizes, dtypes and errors as for the chunk
 * entry points (dk, dv in {64, 128}).
 */
GDR2_API size_t gdr2_gate_prologue_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);

GDR2_API int gdr2_gate_prologue_fwd(const void *xq, const void *xk, const void *xf, const void *xb,
                                    const void *xw, const float *a, const float *delta, int neg_eig,
                                    void *q, void *k, float *log_alpha, void *b, void *w,
                                    int B, int T, int H, int dk, int dv, int dtype, void *stream);

GDR2_API int gdr2_gate_prologue_bwd(const void *xq, const void *xk, const void *xf, const void *xb,
                                    const void *xw, const float *a, const float *delta, int neg_eig,
                                    const void *dq, const void *dk, const float *dlog_alpha,
                                    const void *db, const void *dw,
                                    void *dxq, void *dxk, void *dxf, void *dxb, void *dxw,
                                    float *da, float *ddelta,
                                    int B, int T, int H, int dk_, int dv, int dtype,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * One-token recurrent decode step (review, Appendix C.5 "Recurrent decoding kernel"): for every
 * (b, h) the fp32 state is decayed by exp(log_alpha), read along b (.) k, written with w (.) v along
 * k, and o = S^T q is returned from the updated state.
 *   q, k, b    [B,H,dk] dtype      v, w  [B,H,dv] dtype      log_alpha [B,H,dk] fp32
 *   state      [B,H,dk,dv] fp32, read and overwritten in place with the new state
 *   o          [B,H,dv] dtype (written)
 * Needs no workspace.
 */
GDR2_API int gdr2_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                     const void *b, const void *w, float *state, void *o,
                     int B, int H, int dk, int dv, int dtype, void *stream);

/*
 * gdr2_chunk_fwd for callers that cannot allocate device memory. The paper has no counterpart to
 * this entry point: it exists for callers that only receive input and output buffers -- plugins in a
 * host framework that owns all device memory through its own pool, or latency-critical loops where a
 * cudaMalloc (which may synchronise the device) is not allowed -- and so cannot pass the workspace
 * that gdr2_chunk_fwd needs.
 * Arguments and results are those of gdr2_chunk_fwd without the workspace pair; the computation is
 * the plain fp32-FMA chunkwise forward. Its scratch is one fixed 32 MiB array compiled into the
 * library, which every GPU that loads the library holds until the process exits.
 *   Limit   : B*H*ceil(T/64) * (6*64*dk + 2*64*dv + 2*64*64) * 4 bytes must not exceed 32 MiB, i.e.
 *             B*H*ceil(T/64) <= 113 (dk = dv = 128), 204 (dk = dv = 64), 170 (dk = 64, dv = 128) or
 *             128 (dk = 128, dv = 64). Larger problems (including sizes whose products would not fit
 *             in 64 bits) return GDR2_ERR_WORKSPACE before anything is launched.
 *   Set-up  : every call looks up the array's device address (cudaGetSymbolAddress, with the caller's
 *             device current), so the address stays right after a device reset or a rebuilt primary
 *             context. The first call on a device (and the first after such a reset) may load the
 *             library's device code; make it before any stream capture.
 *   Sharing : all calls in the process share the one array per device, which keeps the last call's
 *             contents (every scratch element is written before it is read, so nothing needs
 *             clearing). Calls whose kernels overlap on the GPU race on it: issue them on one stream
 *             or otherwise order them.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine is called.
 */
GDR2_API int gdr2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                    const void *b, const void *w, const float *initial_state,
                                    void *o, float *final_state,
                                    int B, int T, int H, int dk, int dv, int dtype, void *stream);

/*
 * Benchmark support (not part of the method): per-kernel device time. gdr2_profile_enable(1) makes
 * every later kernel launch of this library record a CUDA event pair on its own stream (events come
 * from a pool created on first use; at most 8192 launches are held, later ones are counted in
 * *dropped). gdr2_profile_collect waits for the recorded events, writes up to max_entries distinct
 * kernel names (NUL-terminated, name_stride bytes apart in `names`) with their launch counts and summed
 * milliseconds, clears the records, and returns the number of entries (or minus a status code).
 * `names`, `launches`, `ms` and `dropped` are host pointers.
 */
GDR2_API int gdr2_profile_enable(int on);
GDR2_API int gdr2_profile_collect(char *names, int name_stride, int *launches, double *ms, int max_entries,
                                  int *dropped);

#ifdef __cplusplus
}
#endif

#endif /* GDR2_H */
