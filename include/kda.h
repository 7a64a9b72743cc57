/*
 * kda.h -- C ABI of libkda: the chunked forward of KDA incremental linear attention
 * (a gated delta rule with per-channel decay) with the lower-bounded decay gate, its
 * backward (the gradients of every input), and its single-token decode step, for NVIDIA
 * B200 (sm_100a).
 *
 * The operation.  The pages ("Trillion-Scale MoE Multimodal Models: Practical
 * Techniques for Ultra-Long Context ...", section 3; "Breaking Through
 * Trillion-Parameter Multimodal MoE ...", section 2.1; "Trillion-Parameter MoE
 * Multimodal Models: Engineering Long-Context ...", section 3.2) describe a linear
 * attention whose state is updated incrementally token by token and computed in
 * chunks with a cumulative decay Gamma, with the log-decay bounded below:
 *
 *     g_t = g_min * sigmoid(a_t)                                   (per key channel)
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * S is a dk x dv matrix per (batch, head).  No 1/sqrt(dk) scale is applied; q and k
 * are expected L2-normalised by the caller (the library does not normalise), beta is
 * passed post-activation in (0, 1), and a is the gate pre-activation (the projection
 * that produces it lives upstream).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major (innermost index last) and 16-byte aligned, except beta, which needs only
 *     its element size (so [T, H] slices at any token offset are accepted).  The library allocates
 *     no device memory; scratch space is passed in by the caller.
 *   - Token tensors are [B, T, H, d]; beta is [B, T, H]; states are [B, H, dk, dv]
 *     float32.  dtype KDA_BF16 means q, k, v, a, beta and o are bfloat16 (state and
 *     accumulation stay float32); KDA_F32 means they are float32 (a CUDA-core path
 *     kept for debugging at tight tolerance).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream).  Arguments are validated synchronously before any launch; an invalid
 *     call launches nothing and returns an error status.  Calls keep no state between
 *     invocations and may be made from several host threads.
 *   - Errors detected inside a kernel (a bounded wait that ran out) are recorded in a
 *     per-device status word and reported by kda_device_status().
 *   - libkda_debug.so is the same library built with KDA_DEBUG_CHECKS: its prep, scan,
 *     state-gradient scan and gradient-kernel CTAs check the record and token ranges they
 *     derive from their grid coordinates against the buffers they were given and, on a
 *     mismatch, record KDA_ERR_DEVICE_BOUNDS and return without touching memory.
 *   - Gradients (kda_chunk_bwd*) are float32 in the layouts of their inputs.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (identical to cudaStream_t / CUstream). */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_BF16 = 0, /* bfloat16 token tensors, float32 state and accumulation */
    KDA_F32 = 1   /* float32 everywhere (CUDA-core debug path)              */
} kda_dtype;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,    /* null pointer, negative size, bad dtype, bad g_min  */
    KDA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (head dim, g_min range)  */
    KDA_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned                   */
    KDA_ERR_ALIAS = 4,          /* an output overlaps an input it must not overlap    */
    KDA_ERR_CUDA = 5,           /* a CUDA runtime call or kernel launch failed        */
    KDA_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out (kda_device_status) */
    KDA_ERR_WORKSPACE = 7,      /* workspace pointer missing or smaller than required */
    KDA_ERR_DEVICE_BOUNDS = 8   /* debug build: a kernel's index check failed (kda_device_status) */
} kda_status;

/* The decay gate of the chunked forward. */
typedef enum {
    KDA_GATE_BOUNDED = 0,   /* g = g_min * sigmoid(a), g_min in [KDA_G_MIN_LOWEST, 0)          */
    KDA_GATE_LOGSIGMOID = 1 /* g = log(sigmoid(a)), unbounded: the ablation path (see below)  */
} kda_gate;

/* Supported range of g_min: finite, KDA_G_MIN_LOWEST <= g_min < 0.  The pages fix
 * g_min = -5 so that 1/Gamma inside any 16-token tile stays in range; with the tile's
 * middle token as reference the largest exponent is 8*|g_min| <= 43.2, far inside
 * float32/bfloat16's range (e^88.7).                                                 */
#define KDA_G_MIN_LOWEST (-5.4f)

/* Token chunk of the bfloat16 path (state carried every KDA_CHUNK tokens) and the
 * decay tile inside it (the pages' 16-token tile). */
#define KDA_CHUNK 64
#define KDA_TILE 16

/*
 * kda_gate_fwd -- the bounded gate on its own: g[i] = g_min * sigmoid(a[i]).
 * Passage: "Trillion-Scale ..." section 3.2 (g = g_min * Sigmoid(...), g_min = -5) and
 * "Breaking Through ..." section 2.1 (g_t = g_min * sigma(w x_t + b), range [g_min, 0)).
 *   a      device, n elements of a_dtype (bf16 or f32), any shape flattened.
 *   g      device, n float32 outputs.  Evaluated in float64 and rounded once to
 *          float32 (round-to-nearest-even), so the result is bit-exact against an
 *          fp64 reference.  NaN propagates; a = +inf gives g_min; a = -inf gives -0.
 *   n      number of elements (0 is a no-op).
 * Errors: INVALID_ARG (null pointer with n > 0, bad dtype, g_min not finite or >= 0),
 * UNSUPPORTED (g_min < KDA_G_MIN_LOWEST), ALIGNMENT, ALIAS (g overlaps a), CUDA.
 */
kda_status kda_gate_fwd(const void *a, kda_dtype a_dtype, float g_min, float *g, int64_t n,
                        kda_stream_t stream);

/*
 * kda_gate_fwd_heads -- the gate with a per-head scale on its argument:
 *     g[t, h, c] = g_min * sigmoid(e^{A_log[h]} * a[t, h, c])
 * Passage: "Trillion-Scale ..." section 3.2 (g = g_min * Sigmoid(e^A * h * z), with `a`
 * the projection h * z and one A per head).
 *   a        device, [n_tok, H, dk] of a_dtype (bf16 or f32); dk a multiple of 8.
 *   A_log    device, H float32 values (4-byte aligned).
 *   g        device, [n_tok, H, dk] float32.  The scaled argument and the gate are
 *            evaluated in float64 and rounded once, as in kda_gate_fwd.
 * Errors: INVALID_ARG, UNSUPPORTED (dk not a multiple of 8, g_min range), ALIGNMENT,
 * ALIAS (g overlaps a or A_log), CUDA.
 */
kda_status kda_gate_fwd_heads(const void *a, kda_dtype a_dtype, float g_min, const float *A_log, int64_t n_tok,
                              int H, int dk, float *g, kda_stream_t stream);

/*
 * kda_chunk_fwd_workspace -- bytes of device scratch kda_chunk_fwd needs for this
 * shape (0 when none).  Pure host computation; never fails (returns 0 for invalid
 * shapes, which kda_chunk_fwd then rejects).
 */
size_t kda_chunk_fwd_workspace(int B, int T, int H, int dk, int dv, kda_dtype dtype);

/*
 * kda_chunk_fwd -- chunked forward over a whole sequence batch (prefill / training
 * forward), state carried in and out.
 * Passages: chunked computation with cumulative decay Gamma and its inverse
 * ("Trillion-Scale ..." section 3.1), all 16-token tiles as dense tensor-core GEMMs
 * thanks to the bound ("Trillion-Scale ..." section 3.3; "Breaking Through ..."
 * section 2.1), Delta-Net-style state update ("Breaking Through ..." section 2.1),
 * chunk recursion with a constant-size state ("Trillion-Parameter MoE ... Engineering"
 * section 3.2).
 *   B, T, H    batch, tokens, heads (B, H >= 1; T >= 0; T need not be a multiple of
 *              anything).  T == 0 copies S0 (or zeros) to S_T and writes no o.
 *   dk, dv     head dims; supported: dk == dv, 64 or 128.
 *   dtype      KDA_BF16 or KDA_F32 (applies to q, k, v, a, beta, o).
 *   q, k, a    [B, T, H, dk];  v: [B, T, H, dv];  beta: [B, T, H].
 *   g_min      gate lower bound, KDA_G_MIN_LOWEST <= g_min < 0 (the pages use -5).
 *   S0         [B, H, dk, dv] float32 initial state, or NULL for zeros.
 *   o          [B, T, H, dv] output (dtype).  Must not overlap any input or S_T.
 *   S_T        [B, H, dk, dv] float32 final state, or NULL to skip.  May be the same
 *              pointer as S0 (in-place carry across segment calls); partial overlap
 *              is rejected.
 *   workspace  device scratch of at least kda_chunk_fwd_workspace(...) bytes, 16-byte
 *              aligned, overlapping no tensor argument (may be NULL when that size is
 *              0).  Its contents on entry are ignored and on exit unspecified: the
 *              bf16 path writes its per-chunk records there, then a table of the gate at
 *              every bfloat16 input (the values kda_gate_fwd returns, one float each),
 *              from which the kernels read g.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS, WORKSPACE, CUDA.
 */
kda_status kda_chunk_fwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q,
                         const void *k, const void *v, const void *a, const void *beta,
                         float g_min, const float *S0, void *o, float *S_T, void *workspace,
                         size_t ws_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_logsigmoid -- the ablation of the bounded gate: the same chunked forward
 * with the unbounded gate g = log(sigmoid(a)) and no g_min.
 * Passages: the unbounded log-sigmoid gate ("Breaking Through ..." section 2.1), and the
 * path the bound replaced ("Trillion-Scale ..." sections 3.1 and 3.3; "Breaking Through
 * ..." section 2.1).  Without a lower bound on g, the inverse decay inside a 16-token
 * tile cannot be factored into tensor-core operands, so the pairs (r, j) of the diagonal
 * tiles are computed element by element on CUDA cores, one exponential per pair and key
 * channel (the slow position-pair path).  The off-diagonal tiles stay dense products,
 * with references chosen so that every factor is at most 1.  Everything after the tiles
 * (solve, record, scan) is the kda_chunk_fwd path unchanged.
 *   Arguments, layouts, workspace (kda_chunk_fwd_workspace), aliasing rules and errors
 *   are those of kda_chunk_fwd without g_min; only dtype KDA_BF16 is implemented
 *   (KDA_F32 returns UNSUPPORTED).  Every finite a is accepted; the result is
 *   unspecified for infinite or NaN a.
 */
kda_status kda_chunk_fwd_logsigmoid(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q,
                                    const void *k, const void *v, const void *a, const void *beta,
                                    const float *S0, void *o, float *S_T, void *workspace, size_t ws_bytes,
                                    kda_stream_t stream);

/*
 * kda_chunk_fwd_varlen -- the chunked forward over a packed batch of variable-length
 * sequences: N sequences stored back to back on one token axis of T tokens, sequence s
 * being tokens [cu_seqlens[s], cu_seqlens[s+1]).  Each sequence starts from its own state
 * S0[s] (or zeros) and ends in S_T[s]; nothing flows across a boundary, and no chunk
 * spans two sequences.  Equal-length sequences give exactly kda_chunk_fwd's result.
 * Passage: many documents packed into one long training sequence ("Breaking Through ..."
 * section 3, the packing used for the long-context stages); the per-sequence recurrence
 * is kda_chunk_fwd's.
 *   N            sequences (>= 1; N * H <= 65535).
 *   cu_seqlens   DEVICE pointer to N + 1 int32 offsets, 4-byte aligned: cu[0] = 0,
 *                non-decreasing, cu[N] = T (empty sequences allowed).  Checked on the
 *                device: an invalid array records KDA_ERR_INVALID_ARG in the device status
 *                word (kda_device_status), writes no o, and S_T gets S0 (or zeros).
 *   T            tokens on the packed axis (0 .. 2^31 - 65).
 *   dk, dv       dk == dv in {64, 128}; dtype must be KDA_BF16.
 *   gate, g_min, A_log  as in kda_chunk_fwd_prep.
 *   q, k, a      [T, H, dk];  v, o: [T, H, dv];  beta: [T, H]   (bfloat16)
 *   S0, S_T      [N, H, dk, dv] float32, or NULL (zeros / not stored); S_T may be S0.
 *   workspace    >= kda_chunk_fwd_varlen_workspace(N, T, H, dk, dv, dtype) bytes (records
 *                for ceil(T/64) + N chunks per head, plus the chunk table), 16-byte aligned.
 *   Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS, WORKSPACE, CUDA.
 */
size_t kda_chunk_fwd_varlen_workspace(int N, int T, int H, int dk, int dv, kda_dtype dtype);
kda_status kda_chunk_fwd_varlen(int N, const int32_t *cu_seqlens, int T, int H, int dk, int dv, kda_dtype dtype,
                                kda_gate gate, float g_min, const float *A_log, const void *q, const void *k,
                                const void *v, const void *a, const void *beta, const float *S0, void *o,
                                float *S_T, void *workspace, size_t ws_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_prep, kda_chunk_fwd_scan -- the two stages of the bfloat16 kda_chunk_fwd
 * as separate calls, for callers that schedule them apart (timing each stage, or running
 * the fully parallel prep of one batch while other work waits for the serial scan).
 * kda_chunk_fwd(bf16) is exactly kda_chunk_fwd_prep followed by kda_chunk_fwd_scan on the
 * same stream with the same workspace.
 *
 * kda_chunk_fwd_prep: everything inside each 64-token chunk (gate, cumulative decay,
 * tile products, the delta-rule solve and the chunk's contributions), written as one
 * record per (batch*head, chunk) into `workspace`.  All chunks are independent.
 *   gate, g_min  KDA_GATE_BOUNDED with g_min as in kda_chunk_fwd, or KDA_GATE_LOGSIGMOID
 *                (g_min unused) as in kda_chunk_fwd_logsigmoid.
 *   A_log        NULL, or a DEVICE array of H float32 values (4-byte aligned): the gate's
 *                argument becomes e^{A_log[h]} * a, the per-head scale of g = g_min *
 *                Sigmoid(e^A * h * z) ("Trillion-Scale ..." section 3.2; `a` is the
 *                projection h * z), fused here instead of a separate pass over a.
 *   q, k, v, a, beta, workspace, ws_bytes: as in kda_chunk_fwd, bfloat16 only.
 *   Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS (workspace overlaps an input),
 *   WORKSPACE, CUDA.  T == 0 does nothing.
 *
 * kda_chunk_fwd_scan: the chunk recursion over the records, serial over chunks per
 * (batch, head, 32-column block of the state): writes o and, if S_T is not NULL, the
 * final state.
 *   workspace    the records of a kda_chunk_fwd_prep call with the same B, T, H, dk, dv,
 *                ordered before this call (same stream, or an event).  Other contents give
 *                unspecified o and S_T but no access outside the buffers.
 *   S0, o, S_T   as in kda_chunk_fwd (S_T may be S0; o overlaps nothing else).
 *   Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS, WORKSPACE, CUDA.  T == 0 copies S0
 *   (or zeros) to S_T.
 */
kda_status kda_chunk_fwd_prep(int B, int T, int H, int dk, int dv, kda_gate gate, float g_min, const float *A_log,
                              const void *q, const void *k, const void *v, const void *a, const void *beta,
                              void *workspace, size_t ws_bytes, kda_stream_t stream);
kda_status kda_chunk_fwd_scan(int B, int T, int H, int dk, int dv, const void *workspace, size_t ws_bytes,
                              const float *S0, void *o, float *S_T, kda_stream_t stream);

/*
 * kda_chunk_fwd_segmented -- the bf16 chunked forward of long sequences, taken seg_T tokens
 * at a time with the state carried, the prep of each stretch overlapping the scan of the one
 * before it.  The result equals kda_chunk_fwd on the whole problem bit for bit (stretches are
 * whole 64-token chunks and the state is carried in float32 either way).
 * Passages: the context stages of long-context training, up to 1M tokens ("Trillion-Scale
 * ..." section 2.3; "Trillion-Parameter MoE ... Engineering" section 5.1), over the chunk
 * recursion with a constant-size state ("... Engineering" section 3.2).
 * Why: a stretch's scan is serial over its chunks and occupies one SM per (head, 32 value
 * columns), so with few heads (the 1M stage's 16: 64 of 148 SMs) most SMs idle while it
 * runs; the next stretch's prep, which does not depend on the state, fills them.
 *   B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, S0, o:  as in kda_chunk_fwd; dtype must
 *              be KDA_BF16 (the bounded gate, as kda_chunk_fwd).
 *   seg_T      tokens per stretch: a positive multiple of 64.  Each batch element's
 *              sequence is cut into ceil(T / seg_T) stretches (the last may be shorter), and
 *              the stretches of all elements run in order, element by element.
 *   S_T        [B, H, dk, dv] float32, required (it carries the state from stretch to
 *              stretch); may be the same pointer as S0.
 *   workspace  at least kda_chunk_fwd_segmented_workspace(...) bytes (two stretches'
 *              records), 16-byte aligned, overlapping no tensor argument.
 *   stream     the call's work starts after the work already on it and the work queued on
 *              it later follows the call's.  Inside, the preps run on a stream of the call
 *              at the lowest priority and the scans on one at the highest (so that a scan's
 *              CTAs are placed ahead of the next prep's), ordered by events.  The call
 *              creates two streams and four events and releases them (CUDA frees them once
 *              their work is done); it is not meant for stream capture.
 * Errors: INVALID_ARG (seg_T not a positive multiple of 64, S_T NULL), UNSUPPORTED (dtype
 * not KDA_BF16, shapes kda_chunk_fwd rejects), ALIGNMENT, ALIAS, WORKSPACE, CUDA.  Every
 * check is done before the first launch.  T == 0 copies S0 (or zeros) to S_T.
 */
size_t kda_chunk_fwd_segmented_workspace(int B, int T, int H, int dk, int dv, int seg_T);
kda_status kda_chunk_fwd_segmented(int B, int T, int H, int dk, int dv, kda_dtype dtype, int seg_T, const void *q,
                                   const void *k, const void *v, const void *a, const void *beta, float g_min,
                                   const float *S0, void *o, float *S_T, void *workspace, size_t ws_bytes,
                                   kda_stream_t stream);

/*
 * Sequence parallelism: one long sequence split into R consecutive segments, one per GPU
 * ("Breaking Through ..." section 3: sequence parallelism for the million-token stage).
 * Over a segment the state map is affine, S_out = M S_in + S_zero, with M the product of
 * the segments' per-chunk maps Diag(Gamma) - N and S_zero the state the segment reaches
 * from S_in = 0.  Each GPU preps its segment (kda_chunk_fwd_prep), computes (S_zero, M)
 * (kda_chunk_fwd_scan_affine), all-gathers them, forms every segment's incoming state
 * (kda_state_combine), and scans its segment again from its own incoming state
 * (kda_chunk_fwd_scan) to write o.  The result equals one kda_chunk_fwd over the whole
 * sequence up to rounding.
 *
 * kda_chunk_fwd_scan_affine -- (S_zero, M) of the segment whose records `workspace` holds.
 *   workspace    the records of kda_chunk_fwd_prep(B, T, H, dk, dv, ...), ordered before.
 *   S_zero       [B, H, dk, dv] float32 out: the final state from a zero initial state.
 *   M            [B, H, dk, dk] float32 out: the segment's transfer map (T == 0: identity).
 *   Writes no o.  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS, WORKSPACE, CUDA.
 *
 * kda_state_combine -- incoming states of R consecutive segments:
 *     S_in[0] = S0 (or zeros),  S_in[r + 1] = M[r] S_in[r] + S_zero[r],  r < R
 *   M, S_zero    [R, B, H, dk, dv] float32 (dk == dv), as gathered from the segments.
 *   S0           [B, H, dk, dv] float32 or NULL.
 *   S_in         [R + 1, B, H, dk, dv] float32 out; S_in[R] is the whole sequence's final
 *                state.  Float32 arithmetic.
 *   Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS (S_in overlaps an input), CUDA.
 */
kda_status kda_chunk_fwd_scan_affine(int B, int T, int H, int dk, int dv, const void *workspace, size_t ws_bytes,
                                     float *S_zero, float *M, kda_stream_t stream);
kda_status kda_state_combine(int R, int B, int H, int dk, int dv, const float *M, const float *S_zero,
                             const float *S0, float *S_in, kda_stream_t stream);

/*
 * kda_chunk_bwd -- gradients of the bfloat16 chunked forward (bounded gate, optionally with
 * the per-head scale e^{A_log[h]} on the gate's argument) with respect to every input,
 * given the gradient of the loss with respect to o and to the final state.  Passage: long
 * sequences are trained by recursing in chunks ("Trillion-Parameter MoE ... Engineering"
 * section 3.2); the pages print no backward, so this is the derivative of kda_chunk_fwd's
 * recurrence, computed in the same chunked form:
 *     dS = (Diag(Gamma) - N)^T dS' + Q'^T dO        (state gradient, chunks in reverse)
 * and, inside each chunk, the reverse of the chunk's products (see chunk_bf16.cu).  It
 * recomputes the forward (prep and scan) inside the call; nothing of a forward call is
 * needed.  All gradients are float32.
 *   B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, S0: exactly as in kda_chunk_fwd
 *                (dtype must be KDA_BF16; S0 may be NULL for zeros).
 *   A_log        NULL, or a DEVICE array of H float32 values (4-byte aligned): the gate is
 *                g = g_min * sigmoid(e^{A_log[h]} a), as in kda_chunk_fwd_prep.
 *   dO           [B, T, H, dv] bfloat16: dL/do.
 *   dS_T         [B, H, dk, dv] float32 or NULL (zero): dL/dS_T.
 *   dq, dk_, da  [B, T, H, dk] float32 out;  dv_: [B, T, H, dv] float32 out;
 *   dbeta        [B, T, H] float32 out;  dS0: [B, H, dk, dv] float32 out or NULL.
 *                da is the gradient with respect to the gate's input a.
 *   dA_log       [H] float32 out, or NULL (needs A_log): dL/dA_log, the sum over the head's
 *                tokens and channels of da * a, reduced in a fixed order.
 *   workspace    >= kda_chunk_bwd_workspace(B, T, H, dk, dv, dtype) bytes, 16-byte
 *                aligned: the forward's records, the state entering every chunk and the
 *                gradient of the state after it (float32, dk x dv per (b, h, chunk), in
 *                that order, from the byte offsets kda_chunk_bwd_offsets gives), then the
 *                gradient kernel's scratch.
 * The outputs must not overlap each other, an input or the workspace.
 * Errors: INVALID_ARG, UNSUPPORTED (also when B * H * ceil(T / 64) * dk >= 2^31: the saved
 * state arrays are written as that many rows of dv floats, by row index), ALIGNMENT, ALIAS,
 * WORKSPACE, CUDA.  T == 0 writes dS0 = dS_T (or zeros), dA_log = 0, and nothing else.
 *
 * kda_chunk_bwd_varlen -- the same over a packed batch of N sequences on one token axis, as
 * kda_chunk_fwd_varlen lays it out (cu_seqlens on the device and checked there; each
 * sequence starts from S0[s] and ends with the gradient dS_T[s]).  Token tensors and their
 * gradients are [T, H, .], states [N, H, dk, dv].  Workspace: kda_chunk_bwd_varlen_workspace.
 * An invalid cu_seqlens records KDA_ERR_INVALID_ARG in the device status word; the
 * gradients are then unspecified but nothing outside the buffers is touched.
 */
size_t kda_chunk_bwd_workspace(int B, int T, int H, int dk, int dv, kda_dtype dtype);
kda_status kda_chunk_bwd_offsets(int B, int T, int H, int dk, int dv, size_t *states_offset,
                                 size_t *dstates_offset);
kda_status kda_chunk_bwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                         const void *v, const void *a, const void *beta, float g_min, const float *A_log,
                         const float *S0, const void *dO, const float *dS_T, float *dq, float *dk_, float *dv_,
                         float *da, float *dbeta, float *dS0, float *dA_log, void *workspace, size_t ws_bytes,
                         kda_stream_t stream);
/*
 * kda_chunk_bwd_recorded -- kda_chunk_bwd for a training step that keeps the forward's
 * records: the backward's workspace starts with the same layout as kda_chunk_fwd's (the
 * records, then the gate table), so a bf16 kda_chunk_fwd (or kda_chunk_fwd_prep with the
 * same gate and A_log) given this workspace writes exactly what kda_chunk_bwd's first launch
 * would; this call skips that launch and runs the other three.  Same arguments, checks and
 * errors as kda_chunk_bwd; the gradients equal kda_chunk_bwd's bit for bit when the records
 * come from the same q, k, v, a, beta, g_min and A_log, ordered before this call.  Other
 * contents give unspecified gradients but no access outside the buffers.
 */
kda_status kda_chunk_bwd_recorded(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                                  const void *v, const void *a, const void *beta, float g_min, const float *A_log,
                                  const float *S0, const void *dO, const float *dS_T, float *dq, float *dk_,
                                  float *dv_, float *da, float *dbeta, float *dS0, float *dA_log, void *workspace,
                                  size_t ws_bytes, kda_stream_t stream);
size_t kda_chunk_bwd_varlen_workspace(int N, int T, int H, int dk, int dv, kda_dtype dtype);
kda_status kda_chunk_bwd_varlen(int N, const int32_t *cu_seqlens, int T, int H, int dk, int dv, kda_dtype dtype,
                                float g_min, const float *A_log, const void *q, const void *k, const void *v,
                                const void *a, const void *beta, const float *S0, const void *dO, const float *dS_T,
                                float *dq, float *dk_, float *dv_, float *da, float *dbeta, float *dS0,
                                float *dA_log, void *workspace, size_t ws_bytes, kda_stream_t stream);

/*
 * kda_decode_step -- one token for N independent sequences, state updated in place.
 * Passage: the incremental state of constant size used at inference ("Trillion-
 * Parameter MoE ... Engineering" section 3.2).  Per (n, h):
 *     S_dec = Diag(exp g) S;  u = beta (v - S_dec^T k);  S' = S_dec + k u^T;
 *     o = S'^T q                     (the recurrence above for a single token)
 *   N, H       sequences and heads (>= 1); dk == dv in {64, 128}.
 *   q, k, a    [N, H, dk];  v: [N, H, dv];  beta: [N, H]   (dtype)
 *   S          [N, H, dk, dv] float32, read and overwritten with S'.
 *   o          [N, H, dv] (dtype); must not overlap S or any input.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, ALIAS, CUDA.
 */
kda_status kda_decode_step(int N, int H, int dk, int dv, kda_dtype dtype, const void *q,
                           const void *k, const void *v, const void *a, const void *beta,
                           float g_min, float *S, void *o, kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for the library's users.
 * Code that runs during CUDA graph capture (allocation is not allowed there), serving
 * loops that must never call cudaMalloc (it can synchronise the device), and hosts whose
 * device memory is owned by another allocator cannot provide the workspace that
 * kda_chunk_fwd takes.  This entry point takes the same arguments minus the workspace and
 * uses a fixed scratch array built into the library instead: kda_chunk_fwd_noalloc_max_
 * scratch() bytes (64 MiB) of device memory on every GPU that loads the library, held
 * until the process exits.  It allocates nothing and computes exactly what kda_chunk_fwd
 * computes: inputs longer than the scratch holds are processed in stretches of whole
 * 64-token chunks with the float32 state carried between them.
 *   - Every call looks up the scratch array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing); the first such lookup on a device
 *     may load the library's module there, so make the first call before any stream
 *     capture.
 *   - All checks (shapes, alignment, overlaps between any two tensors, across batch
 *     elements too) run on the whole problem before the first launch, as in kda_chunk_fwd.
 *   - All calls share the one array, and it keeps whatever the last call left there;
 *     nothing in it needs to start at zero.  Calls whose GPU work overlaps (other
 *     streams, other host threads) race on the array: serialise them.
 *   - Errors: as kda_chunk_fwd, plus WORKSPACE when even one 64-token chunk of all heads
 *     (with the state carry slot) does not fit the scratch (roughly H > 600 at
 *     dk = dv = 128), and CUDA if the scratch address cannot be looked up.
 */
kda_status kda_chunk_fwd_noalloc(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q,
                                 const void *k, const void *v, const void *a, const void *beta,
                                 float g_min, const float *S0, void *o, float *S_T, kda_stream_t stream);

/* Size in bytes of the built-in scratch array kda_chunk_fwd_noalloc uses. */
size_t kda_chunk_fwd_noalloc_max_scratch(void);

/*
 * kda_device_status -- synchronise `stream`, then return and clear the current
 * device's kernel status word: KDA_OK; KDA_ERR_DEVICE_TIMEOUT if a kernel gave up on a
 * bounded wait since the last call; KDA_ERR_INVALID_ARG if kda_chunk_fwd_varlen found
 * its cu_seqlens invalid; KDA_ERR_DEVICE_BOUNDS if a debug-build index check failed;
 * KDA_ERR_CUDA if the synchronisation failed.  The first error
 * recorded since the last call is the one reported.
 */
kda_status kda_device_status(kda_stream_t stream);

/*
 * kda_selftest_device_timeout -- exercise the kernels' failure path.  Launches one small
 * kernel whose bounded wait, on an mbarrier that nothing completes, runs out after
 * `limit_us` microseconds (1 .. 2 000 000); it then records KDA_ERR_DEVICE_TIMEOUT in the
 * device status word exactly as a real timeout would, and returns.  The GPU and the CUDA
 * context stay usable: the next kda_device_status() returns KDA_ERR_DEVICE_TIMEOUT and
 * clears the word.  The pages have no counterpart; it exists to test error handling.
 * Errors: INVALID_ARG (limit out of range), CUDA.
 */
kda_status kda_selftest_device_timeout(uint32_t limit_us, kda_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status status);

/* Library version, major*10000 + minor*100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
