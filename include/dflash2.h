/*
 * dflash2.h -- C ABI of the DFlash 2 draft -> select -> verify step on B200.
 *
 * The library (libdflash2.so) runs the step that follows the drafter and
 * target forwards of one-pass block-parallel speculative decoding:
 *
 *   dflash2_topk_softmax   softmax over the vocabulary and the 16 best
 *                          candidates of every drafted position
 *   dflash2_pair_select    bilinear adjacent-pair scores and the exact best
 *                          path through the 16 candidates per position
 *   dflash2_verify_greedy  greedy lossless verify (longest prefix match)
 *   dflash2_verify_sample  sampling lossless verify (rejection sampling with
 *                          residual resample and bonus draw)
 *   dflash2_verify_sample_trunc  the same on top-k / top-p truncated
 *                          distributions
 *   dflash2_dynconv2       two-tap dynamic depthwise conv fused with its tap
 *                          projection and the residual add
 *
 * Source pages (cited by title and section):
 *   [tamsi]    "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie",
 *              sections "L’idée, sans le papier" and "Les chiffres qui
 *              comptent sur Qwen3.8-27B".
 *   [myaiexp]  "DFlash 2" (myaiexp.com), section "主な機能" (features).
 *   [latenode] "DFlash 2: un drafter de 3.43× que cae a 1.45× bajo carga",
 *              sections "Un drafter que adivina el bloque entero de una vez",
 *              "El desacuerdo empieza en las propias tablas del proveedor",
 *              "Preguntas frecuentes".
 *   [psi]      "Qwen 3.8 27B + DFlash2: 140 Token/Sec?", section "Résumé".
 *   [philox]   Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
 *              SC'11, section 5.
 *
 * Conventions for every call:
 *   - Tensor arguments are DEVICE pointers owned by the caller; the library
 *     never frees or keeps them.  Layouts are dense row-major unless a stride
 *     is given.  bf16 data is passed as its 16-bit storage.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream) and never synchronises the host.
 *   - The return value is a dflash2_status.  Host-side validation happens
 *     before anything is enqueued: on any status other than DFLASH2_OK no
 *     work was enqueued, except DFLASH2_ECUDA, which reports a failed launch
 *     or memset (read with cudaGetLastError, which also clears it).
 *   - Preconditions the library does not check on the device: logits,
 *     embeddings and weights are finite; output buffers do not overlap
 *     inputs.  Token ids (drafted tokens, candidate ids, the anchor) belong
 *     in [0, V); one outside it is never used as an address: the verifies
 *     treat it as not accepted (greedy: a mismatch; sampling: r = 0, so it
 *     is rejected), the selector gives it a zero embedding, and the call
 *     sets device error flag 32 (dflash2_device_errors).
 *   - Calls that take a workspace (`ws`, `ws_bytes`): a device buffer of at
 *     least dflash2_workspace_bytes(B, G, V) bytes, 256-byte aligned, used
 *     for arrival counters and per-chunk partial results.  Its first 64 KB
 *     hold the counters of every call and must be ZERO when the workspace is
 *     first used (e.g. cudaMemset once after allocating it); every call that
 *     completes leaves them zero again (its kernels reset what they used), so
 *     one workspace serves any sequence of calls on a stream without further
 *     clearing.  After dflash2_device_errors reports a failure, zero those
 *     64 KB again before reusing the workspace.  The rest of the workspace
 *     needs no initialisation.  Two calls that may run concurrently need
 *     separate workspaces.
 *   - Results are deterministic: a sequence's outputs depend only on its own
 *     inputs (and seq_id), not on the batch it runs in or on B -- except that
 *     dflash2_pair_select picks its implementation by B (see
 *     dflash2_pair_select_ex, which fixes it).
 */
#ifndef DFLASH2_H
#define DFLASH2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point is exported from the shared library; nothing else is. */
#if defined(__GNUC__)
#define DFLASH2_API __attribute__((visibility("default")))
#else
#define DFLASH2_API
#endif

/* The driver stream handle; identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* dflash2_stream_t;

typedef enum {
    DFLASH2_OK = 0,
    DFLASH2_EINVAL = 1,     /* null pointer, non-finite or non-positive scalar */
    DFLASH2_EDTYPE = 2,     /* dtype not DFLASH2_F32 / DFLASH2_BF16 */
    DFLASH2_ESHAPE = 3,     /* size out of the supported range */
    DFLASH2_EWORKSPACE = 4, /* ws NULL, misaligned or smaller than required */
    DFLASH2_ECUDA = 5,      /* a CUDA launch or memset failed */
    DFLASH2_EALIGN = 6      /* a pointer or stride violates the stated alignment */
} dflash2_status;

typedef enum { DFLASH2_F32 = 0, DFLASH2_BF16 = 1 } dflash2_dtype;
typedef enum { DFLASH2_Q_SOFTMAX = 0, DFLASH2_Q_ONEHOT = 1 } dflash2_qmode;

/* Candidates kept per drafted position ([tamsi] "L’idée, sans le papier":
 * the right token is in the drafter's top 16 far more often than at top 1). */
#define DFLASH2_K 16
/* Largest block size (drafted positions + 1) the verify and select calls take. */
#define DFLASH2_MAX_BLOCK 32

/* Human-readable name of a status code (static storage, never NULL). */
DFLASH2_API const char* dflash2_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
DFLASH2_API int dflash2_version(void);

/* Workspace bytes that any call with at most B sequences, G drafted positions
 * per sequence (B*G rows for dflash2_topk_softmax) and vocabulary V needs.
 * Returns 0 for B < 0, G < 1, G >= DFLASH2_MAX_BLOCK or V < 1. */
DFLASH2_API size_t dflash2_workspace_bytes(int B, int G, int64_t V);

/*
 * Softmax and top-16 per drafted position.  [tamsi] "L’idée, sans le papier";
 * [myaiexp] "主な機能" (the selector keeps the 16 best candidates per position).
 *
 * For each of `rows` rows (row r starts at logits + r * row_stride elements):
 *   z_v = x_v * inv_temperature,  logz = log(sum_v exp(z_v)),
 *   idx[r][k]  = the k-th best v by (x_v descending, v ascending), -0 == +0,
 *   prob[r][k] = exp(z_idx - logz),  logp[r][k] = z_idx - logz.
 *
 * logits      [rows, row_stride] of `dtype`; rows V..row_stride-1 unused.
 * rows        >= 0 (0 is a no-op); V in [16, 2^31 - 1]; row_stride >= V.
 * inv_temperature  finite, > 0.
 * idx         [rows, 16] int32;  prob, logp [rows, 16] float;  logz [rows] float.
 * ws          workspace for B*G >= rows sequences-positions at this V.
 * Rows whose start is 16-byte aligned are read with 128-bit loads; others are
 * read element by element (correct, slower).
 */
DFLASH2_API int dflash2_topk_softmax(const void* logits, int dtype, int64_t rows, int64_t V,
                         int64_t row_stride, float inv_temperature, int32_t* idx, float* prob,
                         float* logp, float* logz, void* ws, size_t ws_bytes,
                         dflash2_stream_t stream);

/*
 * dflash2_topk_softmax plus each row's normaliser in a form the sampling
 * verify can reuse (the fused cycle: [tamsi] "L’idée, sans le papier" runs the
 * drafter softmax once; dflash2_verify_sample_ex then needs no second pass
 * over the draft rows).  Same arguments and results as
 * dflash2_topk_softmax, and:
 * row_max     [rows] float or NULL: max_v x_v (an element's value, exact);
 * row_lse     [rows] float or NULL: ln sum_v exp((x_v - row_max) * inv_temperature),
 *             so that logz = row_max * inv_temperature + row_lse.
 */
DFLASH2_API int dflash2_topk_softmax_ex(const void* logits, int dtype, int64_t rows, int64_t V,
                                        int64_t row_stride, float inv_temperature, int32_t* idx,
                                        float* prob, float* logp, float* logz, float* row_max,
                                        float* row_lse, void* ws, size_t ws_bytes,
                                        dflash2_stream_t stream);

/*
 * Allocation-free dflash2_topk_softmax.  The paper has no counterpart: this
 * entry exists for callers that cannot give the library device memory -- an
 * inference engine that reserved nearly all of the GPU for its own pools at
 * start-up and does not let plugins call cudaMalloc, or a latency-critical
 * path where cudaMalloc could synchronise the device.
 *
 * Same arguments, results and errors as dflash2_topk_softmax, minus the
 * workspace: the scratch is a fixed array of DFLASH2_NOALLOC_SCRATCH_BYTES in
 * the library's own device memory, present on every GPU that loads the
 * library until the process exits.  The call allocates nothing (no
 * cudaMalloc, no cudaFree, no allocating library routine); it clears the
 * array's counters with cudaMemsetAsync on `stream` before every call.
 *   - Limit: 64 KB + rows * ceil(V / L) * 144 bytes (L = 4096 for bf16, 2048
 *     for fp32: the rows are reduced in chunks of 8 KB; rounded up to 256)
 *     must fit in the array; larger shapes return DFLASH2_EWORKSPACE
 *     and enqueue nothing.  At V = 151,936 in bf16 that is up to 754 rows.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind: two calls that can overlap on the GPU (different streams without
 *     an ordering between them) race and give wrong results.
 *   - The first call in each CUDA context looks up the array's device
 *     address (cudaGetSymbolAddress, with that context current) and keeps it
 *     under the context's unique id (cuCtxGetId), so a context created later
 *     (after cudaDeviceReset, say) looks it up anew; make the first call in a
 *     context before any stream capture.
 *   - Every argument is checked before anything is enqueued; on DFLASH2_OK
 *     the call enqueues one cudaMemsetAsync of the array's counters, then the
 *     kernel.
 */
#define DFLASH2_NOALLOC_SCRATCH_BYTES (4u << 20)
DFLASH2_API int dflash2_topk_softmax_noalloc(const void* logits, int dtype, int64_t rows, int64_t V,
                                             int64_t row_stride, float inv_temperature,
                                             int32_t* idx, float* prob, float* logp, float* logz,
                                             dflash2_stream_t stream);

/*
 * Bilinear adjacent-pair selector and the exact best path.  [tamsi] "L’idée,
 * sans le papier" (choose a coherent path through the top-16 lists);
 * [myaiexp] "主な機能" (adjacent candidate pairs are scored); [psi] "Résumé"
 * (candidates chosen by a bilinear attention).  The pages give the selector
 * in outline only; this call fixes it as
 *   score(path) = sum_i logp[i][k_i] + pair(anchor, c[0][k_0])
 *               + sum_{i>0} pair(c[i-1][k_{i-1}], c[i][k_i]),
 *   pair(a, b)  = e(a)^T W e(b),
 * maximised exactly over all 16^G paths (max-sum recursion over positions);
 * on equal scores the smaller rank wins at every back-pointer and at the end.
 *
 * idx, logp   [B, G, 16] as written by dflash2_topk_softmax (c = idx).
 * anchor      [B] int32 last accepted token per sequence, or NULL (no term).
 * emb         [V, d] of `emb_dtype`, 16-byte aligned; d in {64, 128}.
 * W           [d, d] float, row-major (W[j][l] at j * d + l), 16-byte aligned.
 * B >= 0, 1 <= G < DFLASH2_MAX_BLOCK.
 * path_tok    [B, G] int32 chosen tokens; path_rank [B, G] int32 their ranks;
 * path_score  [B] float score of the chosen path.
 */
DFLASH2_API int dflash2_pair_select(const int32_t* idx, const float* logp, const int32_t* anchor,
                        const void* emb, int emb_dtype, int64_t V, int d, const float* W, int B,
                        int G, int32_t* path_tok, int32_t* path_rank, float* path_score,
                        void* ws, size_t ws_bytes, dflash2_stream_t stream);

/*
 * dflash2_pair_select with the implementation named.  Results of the two
 * differ only in fp32 rounding (both accumulate in fp32; the path can differ
 * only where two paths' scores are within that rounding).
 * impl  DFLASH2_SELECT_AUTO: the tensor cores for bf16 tables when
 *       B >= DFLASH2_SELECT_TC_MIN_B, else the CUDA cores (what
 *       dflash2_pair_select does).  The threshold is where the tensor path
 *       became the faster one in measurements on B200 (block 8, d = 128, L2
 *       cold): 18.4 us at every B up to 128 against the CUDA cores' 16.4 us
 *       up to B = 16, 20.5 us at 32 and 45 us at 128.  A sequence's path_score
 *       can therefore differ in its last bits between batches on either side
 *       of the threshold; a caller that needs the same bits at every B names
 *       the implementation;
 *       DFLASH2_SELECT_SIMT: the CUDA cores, fp32 FMAs, one CTA per
 *       (sequence, position) and a last-CTA recursion (any table);
 *       DFLASH2_SELECT_TENSOR: one CTA per sequence, F = E W on tcgen05 with
 *       W split into three bf16 planes (fp32 accuracy), the 16 x 16 blocks
 *       F E^T on tcgen05 as well (F split the same way), the recursion in
 *       shared memory (bf16 tables only: DFLASH2_EDTYPE otherwise); needs no
 *       workspace, though ws is checked as for the other implementations.
 * Other values: DFLASH2_EINVAL.
 */
#define DFLASH2_SELECT_AUTO 0
#define DFLASH2_SELECT_SIMT 1
#define DFLASH2_SELECT_TENSOR 2
#define DFLASH2_SELECT_TC_MIN_B 32
DFLASH2_API int dflash2_pair_select_ex(const int32_t* idx, const float* logp, const int32_t* anchor,
                                       const void* emb, int emb_dtype, int64_t V, int d,
                                       const float* W, int B, int G, int32_t* path_tok,
                                       int32_t* path_rank, float* path_score, int impl, void* ws,
                                       size_t ws_bytes, dflash2_stream_t stream);

/*
 * Greedy lossless verify.  [tamsi] "Les chiffres qui comptent sur
 * Qwen3.8-27B" (greedy output is exactly the target's); [latenode] "El
 * desacuerdo..." (acceptance length = tokens completed per verify step).
 *
 * target      [B, G+1, V] of `dtype`: row j scores drafted position j, row G
 *             the position after the block.
 * draft_tok   [B, G] int32 drafted tokens (the selected path).
 * t_j = argmax_v target[j][v] (lowest v on ties, -0 == +0);
 * n = first j with draft_tok[j] != t_j, else G.
 * n_accept    [B] int32 = n;  out_tok [B, G+1] int32 = draft_tok[0..n-1],
 *             then t_n (correction, or bonus when n = G), then -1.
 */
DFLASH2_API int dflash2_verify_greedy(const void* target, int dtype, int B, int G, int64_t V,
                          const int32_t* draft_tok, int32_t* n_accept, int32_t* out_tok,
                          void* ws, size_t ws_bytes, dflash2_stream_t stream);

/*
 * dflash2_verify_greedy with early exit: the same arguments and bit-identical
 * results, but target rows after a sequence's first mismatch are not read.
 * Row j mismatches exactly when one of its elements has a larger (value,
 * -index) key than draft_tok[j]'s; the rows are streamed in step (all
 * sequences' row 0 first, then row 1, ...), and a chunk of a row after a
 * mismatch already found is skipped rather than read, so only rows 0..n are
 * guaranteed to be read and the bytes saved depend on the acceptance.
 * Workspace: dflash2_workspace_bytes(B, G, V).  Rows that are not 16-byte
 * aligned, or V * element size not a multiple of 16, run dflash2_verify_greedy.
 */
DFLASH2_API int dflash2_verify_greedy_early_exit(const void* target, int dtype, int B, int G,
                                                 int64_t V, const int32_t* draft_tok,
                                                 int32_t* n_accept, int32_t* out_tok, void* ws,
                                                 size_t ws_bytes, dflash2_stream_t stream);

/*
 * Sampling lossless verify by rejection sampling.  [tamsi] "Les chiffres qui
 * comptent sur Qwen3.8-27B" (rejection sampling keeps the target
 * distribution); uniforms from Philox4x32-10 ([philox]).
 *
 * p_j = softmax(target[j] * inv_temperature), q_j = softmax(draft[j] * inv_temperature).
 * For j = 0, 1, ...: r_j = p_j(d_j) / q_j(d_j); accept iff u_j < r_j; stop at
 * the first rejection; n = accepted count.  If n < G the last token is drawn
 * from max(0, p_n - q_n) (normalised; p_n if that is empty by rounding),
 * else the bonus token is drawn from p_G.  A draw takes t = u' * R (R the
 * total mass) and returns the smallest v whose inclusive prefix sum exceeds t
 * (the last v with mass if rounding leaves none).
 * q_mode DFLASH2_Q_ONEHOT: q_j is a point mass on d_j (the reading for a
 * deterministic selector): r_j = p_j(d_j), residual = p_n without d_n, and
 * `draft` is not read (may be NULL).
 * Uniforms: Philox4x32-10 with key (seed low 32, seed high 32) and counter
 * (step, seq_id[b], position, purpose); u = (word0 >> 8) * 2^-24; purpose 0
 * for u_j, 1 for u' (position = n).
 *
 * target [B, G+1, V], draft [B, G, V] of `dtype`, rows 16-byte aligned for
 * the fast path; B <= 65535 and B * (2G+1) * ceil(V / L) < 2^31 (L = 4096
 * for bf16, 2048 for fp32; DFLASH2_ESHAPE otherwise); draft_tok [B, G]
 * int32; seq_id [B] uint32 or NULL (= b).  One cooperative launch (every
 * CTA resident; DFLASH2_ECUDA if the device cannot hold the grid).
 * n_accept [B], out_tok [B, G+1] as in dflash2_verify_greedy.
 * ratio_dbg [B, G] float r_j for every j, u_dbg [B, G] float u_j; both
 * optional (NULL).
 */
DFLASH2_API int dflash2_verify_sample(const void* target, const void* draft, int dtype, int B, int G,
                          int64_t V, const int32_t* draft_tok, float inv_temperature,
                          uint64_t seed, uint32_t step, const uint32_t* seq_id, int q_mode,
                          int32_t* n_accept, int32_t* out_tok, float* ratio_dbg, float* u_dbg,
                          void* ws, size_t ws_bytes, dflash2_stream_t stream);

/*
 * dflash2_verify_sample with the drafter's normalisers given (the fused
 * cycle): draft_max, draft_lse [B, G] float as written by
 * dflash2_topk_softmax_ex (row_max, row_lse) for the draft rows of the same
 * inv_temperature.  Then q_j(d_j) = exp((x - draft_max) * inv_temperature
 * - draft_lse) and the draft rows are not streamed: `draft` is read only at
 * the drafted tokens and in the one row a residual draw uses.  Results as
 * dflash2_verify_sample up to the float rounding of draft_lse (its ulp, at
 * most 1e-6 for rows up to e^16 effective tokens, enters the ratios).
 * draft_max and draft_lse are both given or both NULL (DFLASH2_EINVAL
 * otherwise); both NULL, or q_mode DFLASH2_Q_ONEHOT, is
 * dflash2_verify_sample exactly.
 */
DFLASH2_API int dflash2_verify_sample_ex(const void* target, const void* draft, int dtype, int B,
                                         int G, int64_t V, const int32_t* draft_tok,
                                         const float* draft_max, const float* draft_lse,
                                         float inv_temperature, uint64_t seed, uint32_t step,
                                         const uint32_t* seq_id, int q_mode, int32_t* n_accept,
                                         int32_t* out_tok, float* ratio_dbg, float* u_dbg, void* ws,
                                         size_t ws_bytes, dflash2_stream_t stream);

/*
 * Sampling verify of distributions truncated by top-k and top-p.
 * [latenode] "Preguntas frecuentes" (the Qwen targets are sampled at
 * temperature 1.0, top-p 0.95, top-k 20); rejection sampling as in
 * dflash2_verify_sample.  The pages do not say how truncation meets the
 * verification; this call reads it as: the truncated distribution is the one
 * a token is drawn from, so the verify keeps the truncated target p~ exactly
 * against the drafter's truncated q~.
 *
 * Truncation of a row (z = x * inv_temperature): order the tokens by
 * (z descending, index ascending); keep the first min(top_k, V); renormalise
 * over them; keep the shortest prefix whose cumulative sum reaches top_p
 * (at least one token; top_p = 1 keeps all); renormalise again (fp64).
 * r_j = p~_j(d_j) / q~_j(d_j) (q~(d) = 0 < p~(d): r = +inf; both 0: r = 0),
 * or r_j = p~_j(d_j) for DFLASH2_Q_ONEHOT; accept iff u_j < r_j, stop at the
 * first rejection; n < G: the last token is drawn from max(0, p~_n - q~_n)
 * (one-hot: p~_n without d_n; p~_n if that is empty by rounding), n = G: the
 * bonus from p~_G; the draw takes t = u' R and returns the smallest kept
 * index whose inclusive prefix in index order exceeds t (the last index with
 * mass if none).  Uniforms as in dflash2_verify_sample.
 *
 * Arguments as dflash2_verify_sample, and:
 * top_k       1 <= top_k <= 32 (DFLASH2_ESHAPE otherwise); top_k > V keeps V.
 * top_p       0 < top_p <= 1, finite (DFLASH2_EINVAL otherwise), compared in
 *             fp64 after widening.
 * Every row is streamed once for its exact 32 best (value, index) keys; the
 * full-row normaliser cancels in the truncated distributions, so no
 * exponential of the row is taken.  ratio_dbg holds every r_j as float (+inf
 * where q~(d) = 0 < p~(d)).  Workspace: dflash2_workspace_bytes(B, G, V).
 * The cut, sums and draw are fp64 in an order of their own: outputs can
 * differ from an fp64 reference taking another order only where a top-p cut,
 * an accept test or a draw sits within rounding of its boundary.
 */
DFLASH2_API int dflash2_verify_sample_trunc(const void* target, const void* draft, int dtype, int B,
                                            int G, int64_t V, const int32_t* draft_tok,
                                            float inv_temperature, int top_k, float top_p,
                                            uint64_t seed, uint32_t step, const uint32_t* seq_id,
                                            int q_mode, int32_t* n_accept, int32_t* out_tok,
                                            float* ratio_dbg, float* u_dbg, void* ws,
                                            size_t ws_bytes, dflash2_stream_t stream);

/*
 * Two-tap dynamic depthwise conv fused with its tap projection and the
 * residual add.  [tamsi] "L’idée, sans le papier" (two-tap conv before and
 * after each attention and MLP); [myaiexp] "主な機能" (2-tap dynamic conv).
 *
 *   [a_t; b_t] = W_tap x_t  (W_tap [2H, H]: rows 0..H-1 give a, H..2H-1 give b)
 *   out_t = x_t + a_t * x_t + b_t * x_{t-1},   x_{-1} = x_prev
 * x [B, T, H], x_prev [B, H], w_tap [2H, H], out [B, T, H], all of `dtype`,
 * 16-byte aligned; H a multiple of 64; B, T >= 0, B * T <= 2^30 - 1.  fp32
 * accumulation, one rounding at the output.
 * bf16 runs on the tensor cores with the K dimension of a 64-channel tile
 * possibly split between SMs; the split depends on B * T, H and the SM
 * count only, and the parts are added in K order, so a given shape on a
 * given device always rounds the same way.  It needs a workspace of
 * dflash2_dynconv2_workspace_bytes bytes (256-byte aligned; the same
 * contract as the other calls' workspaces: the first 64 KB zero on first use,
 * left zero by every completed call; one call at a time per workspace); fp32 needs none
 * (ws may be NULL).
 */
DFLASH2_API int dflash2_dynconv2(const void* x, const void* x_prev, const void* w_tap, int dtype, int B,
                     int T, int H, void* out, void* ws, size_t ws_bytes, dflash2_stream_t stream);

/* Workspace bytes dflash2_dynconv2 needs for these arguments (0 when it
 * needs none or the arguments are invalid). */
DFLASH2_API size_t dflash2_dynconv2_workspace_bytes(int dtype, int B, int T, int H);

/*
 * The tap weights in the tensor-core path's own layout, for a caller that
 * keeps the weights across calls (they are model parameters).  The pages
 * have no counterpart: this is a storage format.  In nn.Linear layout every
 * 16 KB stage the kernel streams is 128 row pieces of 128 bytes, H * 2 bytes
 * apart; packed, each stage is one contiguous 16 KB block, read with one bulk
 * copy.  The arithmetic, and so every output bit, is that of dflash2_dynconv2.
 *
 * dflash2_dynconv2_packed_bytes  bytes of the packed form (4 H^2 for bf16;
 *   0 for fp32, which has no tensor-core path, or an invalid H).
 * dflash2_dynconv2_pack  w_tap [2H, H] bf16 (16-byte aligned) -> w_packed
 *   (256-byte aligned, dflash2_dynconv2_packed_bytes bytes), one launch on
 *   `stream`; bf16 only (DFLASH2_EDTYPE otherwise).  The layout is internal:
 *   block (hb, kb) at (hb * H/64 + kb) * 16 KB holds channels 64 hb ..
 *   64 hb + 63 of W_a and W_b (interleaved by 16) over K elements 64 kb ..
 *   64 kb + 63, 128-byte swizzled.
 * dflash2_dynconv2_packed  dflash2_dynconv2 with the packed weights; the
 *   same arguments otherwise, the same workspace, the same results.
 */
DFLASH2_API size_t dflash2_dynconv2_packed_bytes(int dtype, int H);
DFLASH2_API int dflash2_dynconv2_pack(const void* w_tap, int dtype, int H, void* w_packed,
                                      dflash2_stream_t stream);
DFLASH2_API int dflash2_dynconv2_packed(const void* x, const void* x_prev, const void* w_packed,
                                        int dtype, int B, int T, int H, void* out, void* ws,
                                        size_t ws_bytes, dflash2_stream_t stream);

/*
 * Device-side error flags of the kernels on the current device (0 = none).
 * Every wait inside the kernels (on a TMA copy, a tensor-core MMA, or
 * another CTA's result in the same launch) is bounded to one second; a wait
 * that runs out sets a flag bit (1 producer, 2 MMA issuer, 4 epilogue,
 * 8 drain, 16 streamed copy or cross-CTA wait), the kernel waits (bounded)
 * for its own copies in flight, releases its tensor memory and returns, and
 * the call's outputs are not valid; zero the workspace's first 64 KB before
 * reusing it.  Bit 32: a token id was outside [0, V) (see the conventions
 * above; the outputs follow the stated rule).  Synchronous (reads device
 * memory); clear != 0 resets the flags.  Returns 0xFFFFFFFF if the flags
 * cannot be read.
 */
DFLASH2_API unsigned dflash2_device_errors(int clear);

#ifdef __cplusplus
}
#endif

#endif /* DFLASH2_H */
