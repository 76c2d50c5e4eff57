/*
 * qsa.h -- C ABI of libqsa, a B200 (sm_100a) implementation of the Qwen
 * Sparse Attention (QSA) layer: micro-block pooling, a lightweight MQA
 * indexer with top-k block selection, and exact softmax attention over the
 * tokens of the selected blocks, for prefill and decode; plus dense causal
 * GQA attention on the same tensors (the speed-up baseline).  For training,
 * the first stage's indexer distillation loss and gradients and the second
 * stage's sparse attention backward; and the gated delta rule of the
 * hybrid's Gated DeltaNet layers (prefill and decode).
 *
 * Sources (web pages about the Qwen3.8-Flash-Next architecture):
 *   [ART]  "用125亿分之6的参数，打平3970亿的旗舰模型", section
 *          "稀疏注意力：给检索建索引，也得先学会省纸".
 *   [SUM]  "On the Design of Qwen3.8-Next Architecture: Evaluation,
 *          Efficiency, and Training Stability", token-mixing paragraph.
 *   [NEWS] "Qwen3.8-Flash发布并开源：6B激活参数背后，是Qwen4架构的第一次公开
 *          亮相", section "二、架构 / 1. 注意力机制".
 *
 * Conventions, for every entry point:
 *   - Tensor arguments are DEVICE pointers to contiguous row-major arrays
 *     (last dimension innermost), 16-byte aligned, allocated and owned by the
 *     caller.  bf16 tensors are passed as raw 16-bit patterns (qsa_bf16_t).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  All work is enqueued asynchronously on it; the library never
 *     allocates, frees or synchronises, except qsa_check_device_status.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned synchronously (QSA_ERR_INVALID_ARG / _UNSUPPORTED_SHAPE /
 *     _WORKSPACE).  A device that is not sm_100 gives QSA_ERR_ARCH.  A failed
 *     launch gives QSA_ERR_CUDA.
 *   - Errors detected by a kernel (an out-of-range value read from a device
 *     array) are recorded in the status word at the start of the workspace
 *     and read back with qsa_check_device_status.  Kernels never trap.
 *   - Workspace sizes from the *_workspace_size functions are byte counts;
 *     0 is never returned for a valid shape (the status header is included).
 *     SIZE_MAX means the arguments are invalid.
 *   - Calls that share a workspace must be ordered on one stream.
 *   - Supported shapes on the GPU: r = 4; D in {64, 128}; Di in {32, 64};
 *     Hi in {1, 2, 4}; Hkv in {1, 2, 4}; G = Hq / Hkv in {1, 2, 4, 8};
 *     budget a multiple of r with budget / r <= 1024.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QSA_OK = 0,
    QSA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad ratio */
    QSA_ERR_UNSUPPORTED_SHAPE = 2, /* valid but outside the GPU kernels' set */
    QSA_ERR_WORKSPACE = 3,         /* workspace missing or too small */
    QSA_ERR_ARCH = 4,              /* current device is not sm_100 */
    QSA_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    QSA_ERR_TIMEOUT = 6,           /* a bounded device-side wait ran out */
    QSA_ERR_DEVICE = 7             /* a kernel met an out-of-range input value */
} qsa_status_t;

typedef uint16_t qsa_bf16_t; /* raw bf16 bit pattern */

/*
 * Micro-block mean pooling [ART: consecutive tokens packed into a micro-block
 * and mean-pooled into one representative key; SUM: compression ratio 4].
 *
 *   k_pooled[b, j, :] = bf16_rne( ((k[4j] + k[4j+1]) + (k[4j+2] + k[4j+3])) * 0.25 )
 *
 * with the sums in fp32, for every batch row b and every block j in
 * [blk_begin, blk_end).  Other blocks of k_pooled are left untouched, so a
 * decode loop pools exactly the block a new token completes.
 *   k_idx    [B, T, Di] bf16   indexer keys (one shared key head)
 *   k_pooled [B, T / r, Di] bf16
 * Requires r == 4, Di % 8 == 0, 0 <= blk_begin <= blk_end <= T / r.
 */
QSA_API qsa_status_t qsa_pool(const qsa_bf16_t *k_idx, int B, int64_t T, int Di, int r,
                      int64_t blk_begin, int64_t blk_end, qsa_bf16_t *k_pooled,
                      void *stream);

/*
 * Indexer scores and top-k block selection for a run of query tokens
 * [ART: a lightweight MQA indexer gives every micro-block a score and the
 * highest-scoring blocks are kept; SUM: indexing cost O(n^2 / r), token
 * budget 2048].
 *
 * Query t of batch row b sits at absolute position p = q_pos0[b] + t
 * (q_pos0 == NULL: p = t).  Its candidates are the complete blocks
 * j < c = floor(p / r), scored in fp32 as
 *     s(t, j) = sum_h w[b, t, h] * max(0, q_idx[b, t, h, :] . k_pooled[b, j, :]).
 * It keeps the kb - 1 best candidates (score descending, lower block index
 * first on equal scores), adds its own block c, and writes them ascending,
 * padded with -1, kb = budget / r entries per query.
 *   q_idx     [B, Tq, Hi, Di] bf16
 *   w         [B, Tq, Hi] fp32 per-token head weights
 *   k_pooled  [B, n_blocks, Di] bf16 (may be NULL when n_blocks == 0: every
 *             query then keeps its own block only)
 *   q_pos0    [B] int64 device array, or NULL
 *   sel       [B, Tq, kb] int32 (output)
 *   sel_score [B, Tq, kb] fp32 (output, may be NULL): the score of each kept
 *             block; +inf for the own block, -inf for padding
 *   ws        device workspace of at least qsa_index_topk_workspace_size(...)
 *             bytes; its first 256 bytes hold the device status word
 * A position whose floor(p / r) exceeds n_blocks is clamped to n_blocks and
 * recorded as QSA_ERR_DEVICE in the status word.  Tq == 0 is a no-op.
 */
QSA_API size_t qsa_index_topk_workspace_size(int B, int64_t Tq, int64_t n_blocks, int Hi,
                                     int Di, int r, int budget);
QSA_API qsa_status_t qsa_index_topk(const qsa_bf16_t *q_idx, const float *w,
                            const qsa_bf16_t *k_pooled, const int64_t *q_pos0,
                            int B, int64_t Tq, int64_t n_blocks, int Hi, int Di,
                            int r, int budget, int32_t *sel, float *sel_score,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Decode-step selection: one new query per sequence at p = seqlens[b] - 1,
 * same scores, ranking and output as qsa_index_topk with Tq = 1, but the
 * candidates of each sequence are split across many CTAs and merged, so a
 * batch of 64 sequences fills the GPU.
 *   q_idx [B, Hi, Di] bf16, w [B, Hi] fp32, k_pooled [B, n_blocks, Di] bf16
 *   (may be NULL when n_blocks == 0),
 *   seqlens [B] int32 device array (1 <= seqlens[b] and
 *   floor((seqlens[b] - 1) / r) <= n_blocks, else clamped and recorded as
 *   QSA_ERR_DEVICE), sel [B, kb] int32, sel_score [B, kb] fp32 (nullable).
 */
QSA_API size_t qsa_index_topk_decode_workspace_size(int B, int64_t n_blocks, int r,
                                            int budget);
QSA_API qsa_status_t qsa_index_topk_decode(const qsa_bf16_t *q_idx, const float *w,
                                   const qsa_bf16_t *k_pooled,
                                   const int32_t *seqlens, int B,
                                   int64_t n_blocks, int Hi, int Di, int r,
                                   int budget, int32_t *sel, float *sel_score,
                                   void *ws, size_t ws_bytes, void *stream);

/*
 * Sparse prefill attention [ART: the selected blocks are expanded back into
 * their original tokens, which take part in the real attention; NEWS:
 * full-precision attention over the selected blocks only].
 *
 * Query t of batch row b at position p = q_pos0[b] + t (q_pos0 NULL: p = t)
 * attends to the tokens S = { r*j + i : j in sel[b, t, :], j >= 0,
 * 0 <= i < r, r*j + i <= p }.  For head h, with g = h / (Hq / Hkv):
 *     o[b, t, h] = sum_{u in S} softmax_u(scale * q[b, t, h] . k[b, u, g]) v[b, u, g]
 *     lse[b, t, h] = ln sum_{u in S} exp(scale * q[b, t, h] . k[b, u, g])
 * Logits, softmax statistics and accumulation in fp32; the probabilities are
 * rounded to bf16 for the P.V product; o rounded to bf16.
 *   q [B, Tq, Hq, D] bf16; k, v [B, Tk, Hkv, D] bf16 (p < Tk required);
 *   sel [B, Tq, kb] int32 (any order; entries < 0 or with r*j > p ignored);
 *   q_pos0 [B] int64 or NULL; o [B, Tq, Hq, D] bf16; lse [B, Tq, Hq] fp32
 *   or NULL.  An empty token set gives o = 0 and lse = -inf.
 */
QSA_API qsa_status_t qsa_sparse_attn_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                     const qsa_bf16_t *v, const int32_t *sel,
                                     const int64_t *q_pos0, int B, int64_t Tq,
                                     int64_t Tk, int Hq, int Hkv, int D, int r,
                                     int budget, float scale, qsa_bf16_t *o,
                                     float *lse, void *stream);

/*
 * Sparse decode attention: the same definition for one query per sequence at
 * p = seqlens[b] - 1, over the KV caches.  The selected tokens are split
 * across CTAs and the partial results merged with their log-sum-exp.
 *   q [B, Hq, D] bf16; k_cache, v_cache [B, L_max, Hkv, D] bf16;
 *   seqlens [B] int32 (1..L_max, else the row is treated as empty and
 *   QSA_ERR_DEVICE recorded); sel [B, kb] int32; o [B, Hq, D] bf16;
 *   lse [B, Hq] fp32 or NULL.
 */
QSA_API size_t qsa_sparse_attn_decode_workspace_size(int B, int Hq, int D, int r,
                                             int budget);
QSA_API qsa_status_t qsa_sparse_attn_decode(const qsa_bf16_t *q, const qsa_bf16_t *k_cache,
                                    const qsa_bf16_t *v_cache,
                                    const int32_t *seqlens, int64_t L_max,
                                    const int32_t *sel, int B, int Hq, int Hkv,
                                    int D, int r, int budget, float scale,
                                    qsa_bf16_t *o, float *lse, void *ws,
                                    size_t ws_bytes, void *stream);

/*
 * Sparse decode attention without a caller workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory where they run a decode step (for example an engine plugin
 * whose enqueue must not allocate, or a server whose device memory budget is
 * fixed at start-up) and so cannot provide the workspace that
 * qsa_sparse_attn_decode takes.
 *
 * Same arguments, definition and outputs as qsa_sparse_attn_decode, minus the
 * workspace.  The split partials live in one library-owned device array of
 * QSA_NOALLOC_SCRATCH_BYTES (8 MiB) per GPU, held from library load until
 * process exit; the call allocates nothing.  Requirements and behaviour:
 *   - B * nsplit * Hq * (D + 2) * 4 bytes must fit in the array, with
 *     nsplit = min(ceil(512 / B), max(1, kb / 16)); larger problems return
 *     QSA_ERR_WORKSPACE before anything is enqueued (the 64 x 16-head x 128
 *     decode batch needs 4.3 MB).
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the array: calls that may run at the same
 *     time on the GPU (other streams, other threads) race and must be
 *     serialised by the caller.  Nothing in the array needs to start at zero:
 *     every partial a call reads is written by that call first.
 *   - Out-of-range seqlens are handled as in qsa_sparse_attn_decode but not
 *     recorded (there is no workspace status word).
 */
#define QSA_NOALLOC_SCRATCH_BYTES (8u << 20)
QSA_API qsa_status_t qsa_sparse_attn_decode_noalloc(
    const qsa_bf16_t *q, const qsa_bf16_t *k_cache, const qsa_bf16_t *v_cache,
    const int32_t *seqlens, int64_t L_max, const int32_t *sel, int B, int Hq, int Hkv, int D,
    int r, int budget, float scale, qsa_bf16_t *o, float *lse, void *stream);

/*
 * Dense causal GQA attention, prefill: every query t attends to all tokens
 * u <= t (the full-attention layer QSA replaces; speed-up baseline).
 *   q [B, T, Hq, D], k, v [B, T, Hkv, D], o [B, T, Hq, D] bf16;
 *   lse [B, T, Hq] fp32 or NULL.
 */
QSA_API qsa_status_t qsa_dense_gqa_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                   const qsa_bf16_t *v, int B, int64_t T, int Hq,
                                   int Hkv, int D, float scale, qsa_bf16_t *o,
                                   float *lse, void *stream);

/*
 * Dense GQA attention, decode: one query per sequence over all seqlens[b]
 * cached tokens, split across CTAs and merged by log-sum-exp.
 */
QSA_API size_t qsa_dense_gqa_decode_workspace_size(int B, int64_t L_max, int Hq, int D);
QSA_API qsa_status_t qsa_dense_gqa_decode(const qsa_bf16_t *q, const qsa_bf16_t *k_cache,
                                  const qsa_bf16_t *v_cache,
                                  const int32_t *seqlens, int64_t L_max, int B,
                                  int Hq, int Hkv, int D, float scale,
                                  qsa_bf16_t *o, float *lse, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Backward of the sparse prefill attention, for the second training stage
 * [ART: after the dense distillation, the indexer and the backbone are trained
 * together on the sparse pattern].  The selection is held fixed.  With the
 * forward of qsa_sparse_attn_prefill (q_pos0 NULL: query t at p = t, token set
 * S(t) = { r*j + i <= p : j in sel[b, t, :], j >= 0 }, P the softmax of
 * scale * q . k over S(t)) and an output gradient d_o:
 *   D_h      = sum_{u in S} P(u) (d_o_h . v_g(u))
 *   dS(u)    = P(u) (d_o_h . v_g(u) - D_h)
 *   dq_h     = scale * sum_{u in S} dS(u) k_g(u)
 *   dk_g(u) += scale * dS(u) q_h;   dv_g(u) += P(u) d_o_h
 * summed over every query and head that reads token u (g = h / (Hq / Hkv)).
 *   q, d_o [B, T, Hq, D] bf16; k, v [B, T, Hkv, D] bf16; sel [B, T, budget/r]
 *   int32 (distinct entries; negative or future blocks ignored);
 *   dq [B, T, Hq, D], dk, dv [B, T, Hkv, D] fp32 outputs (overwritten).
 * Softmax statistics are recomputed (no forward lse needed); dk and dv are
 * accumulated with atomics, so their low-order bits vary from run to run.
 * T == 0 is a no-op.  Shapes as for qsa_sparse_attn_prefill.
 */
QSA_API qsa_status_t qsa_sparse_attn_backward(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                              const qsa_bf16_t *v, const int32_t *sel,
                                              const qsa_bf16_t *d_o, int B, int64_t T, int Hq,
                                              int Hkv, int D, int r, int budget, float scale,
                                              float *dq, float *dk, float *dv, void *stream);

/*
 * Stage-1 indexer distillation: loss and indexer gradients [ART: QSA is trained
 * in two stages; the first, dense distillation, trains only the indexer, to
 * imitate the full-attention model's attention distribution, with a
 * KL-divergence loss; SUM: QSA first distils the dense attention distribution].
 *
 * For query t of batch row b at position p = t, with candidates the complete
 * blocks j < c = floor(p / r) (the blocks qsa_index_topk ranks):
 *   a(t, j)  = sum over all Hq heads h and the r tokens u of block j of
 *              exp(scale * q[b,t,h] . k[b,u,h/(Hq/Hkv)] - lse[b,t,h])
 *   pi(t, j) = a(t, j) / sum_{j' < c} a(t, j')          (the teacher)
 *   s(t, j)  = sum_h w[b,t,h] * max(0, q_idx[b,t,h,:] . k_pooled[b,j,:])
 *   kl[b,t]  = KL(pi(t, .) || softmax_j s(t, .)), 0 when c < 2
 * and the gradients of L = sum_{b,t} kl[b,t] (the teacher is a constant), with
 * g(t, j) = softmax_j s(t, j) - pi(t, j) and the ReLU's derivative 1[x > 0]:
 *   dq_idx[b,t,h,:] = sum_j g w_h 1[q_idx_h . Kp_j > 0] k_pooled[b,j,:]
 *   dw[b,t,h]       = sum_j g max(0, q_idx_h . Kp_j)
 *   dk_pooled[b,j,:] = sum_t sum_h g w_h 1[q_idx_h . Kp_j > 0] q_idx[b,t,h,:]
 *   dk_idx[b,u,:]   = dk_pooled[b, u / r, :] / r for u < r * floor(T / r), else 0
 *                     (the bf16 rounding of the pooled key taken as identity)
 *   q, k     [B, T, Hq, D] / [B, T, Hkv, D] bf16: the main attention's inputs
 *   lse      [B, T, Hq] fp32: natural-log softmax normalisers of the dense
 *            causal attention at `scale` (qsa_dense_gqa_prefill writes them)
 *   q_idx [B, T, Hi, Di] bf16, w [B, T, Hi] fp32, k_pooled [B, floor(T/r), Di]
 *            bf16 (qsa_pool of the indexer keys; NULL allowed when T < r)
 *   kl [B, T], dq_idx [B, T, Hi, Di], dw [B, T, Hi], dk_pooled [B, floor(T/r), Di]
 *            fp32 outputs; dk_idx [B, T, Di] fp32 or NULL
 *   ws       at least qsa_index_distill_workspace_size(B, T, Hkv, r) bytes,
 *            first 256 bytes zeroed once (status word); it holds the teacher's
 *            block mass, 4 * Hkv * B * T * floor(T / r) bytes (about Hkv * B * T^2)
 * A row whose teacher mass on every candidate underflows fp32 gets zero loss and
 * gradients and records QSA_ERR_DEVICE.  T == 0 is a no-op.  Constraints: r = 4,
 * the attention shapes of qsa_dense_gqa_prefill, the indexer shapes of
 * qsa_index_topk.
 */
QSA_API size_t qsa_index_distill_workspace_size(int B, int64_t T, int Hkv, int r);
QSA_API qsa_status_t qsa_index_distill(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                       const float *lse, const qsa_bf16_t *q_idx,
                                       const float *w, const qsa_bf16_t *k_pooled, int B,
                                       int64_t T, int Hq, int Hkv, int D, int Hi, int Di,
                                       int r, float scale, float *kl, float *dq_idx, float *dw,
                                       float *dk_pooled, float *dk_idx, void *ws,
                                       size_t ws_bytes, void *stream);

/*
 * Stage-2 indexer loss over the selection [ART: after the dense distillation,
 * the second training stage trains the indexer together with the backbone so
 * that the model adapts to the sparse attention pattern].  The pages give no
 * formula; the reading: stage 1's KL restricted to each row's selected
 * candidate blocks, with the layer's own sparse attention as the teacher.
 *
 * For query t of batch row b at position p = t, c = floor(p / r), and
 * J(t) = { j in sel[b,t,:] : 0 <= j < c } (the selected blocks other than the
 * forced own block):
 *   a(t, j)  = sum over all Hq heads h and the r tokens u of block j of
 *              exp(scale * q[b,t,h] . k[b,u,h/(Hq/Hkv)] - lse[b,t,h])
 *              (lse: the sparse forward's, qsa_sparse_attn_prefill writes it)
 *   pi(t, j) = a(t, j) / sum_{j' in J(t)} a(t, j')          (the teacher)
 *   s(t, j)  = sum_h w[b,t,h] * max(0, q_idx[b,t,h,:] . k_pooled[b,j,:])
 *   kl[b,t]  = KL(pi(t, .) || softmax_{j in J(t)} s(t, .)), 0 when |J(t)| < 2
 * and the gradients of L = sum_{b,t} kl[b,t] as in qsa_index_distill, over J(t):
 * g = softmax(s) - pi; dq_idx, dw per row; dk_pooled summed over rows (fp32
 * atomics: the low-order bits vary from run to run); dk_idx = dk_pooled / r
 * spread over each complete block's tokens, 0 on the trailing partial block.
 *   q, k     [B, T, Hq, D] / [B, T, Hkv, D] bf16; lse [B, T, Hq] fp32 (natural log)
 *   sel      [B, T, budget / r] int32 (qsa_index_topk's output for the same rows)
 *   q_idx [B, T, Hi, Di] bf16, w [B, T, Hi] fp32, k_pooled [B, floor(T/r), Di] bf16
 *            (NULL allowed when T < r)
 *   kl [B, T], dq_idx [B, T, Hi, Di], dw [B, T, Hi], dk_pooled [B, floor(T/r), Di]
 *            fp32 outputs (dk_pooled is overwritten, not accumulated into);
 *            dk_idx [B, T, Di] fp32 or NULL
 *   ws       at least qsa_index_distill_sparse_workspace_size(...) bytes, first
 *            256 bytes zeroed once (status word); it holds the teacher's mass,
 *            4 * Hkv * B * T * (budget / r) bytes
 * A row whose teacher mass on its selected candidates underflows fp32 gets zero
 * loss and gradients and records QSA_ERR_DEVICE.  T == 0 is a no-op.
 * Constraints: r = 4, budget / r <= 1024, the attention shapes of
 * qsa_sparse_attn_prefill, the indexer shapes of qsa_index_topk.
 */
QSA_API size_t qsa_index_distill_sparse_workspace_size(int B, int64_t T, int Hkv, int r,
                                                       int budget);
QSA_API qsa_status_t qsa_index_distill_sparse(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                              const float *lse, const int32_t *sel,
                                              const qsa_bf16_t *q_idx, const float *w,
                                              const qsa_bf16_t *k_pooled, int B, int64_t T,
                                              int Hq, int Hkv, int D, int Hi, int Di, int r,
                                              int budget, float scale, float *kl, float *dq_idx,
                                              float *dw, float *dk_pooled, float *dk_idx,
                                              void *ws, size_t ws_bytes, void *stream);

/*
 * Gated DeltaNet token mixing, the hybrid's other layers [ART: GDN keeps a
 * matrix state and, for each token, writes the error between the token's
 * information and what the memory holds for it, under a decay gate and a write
 * gate; SUM: a fixed-size recurrent state with a decay gate and delta writes].
 * Per (sequence b, head h), state S in R^{dv x dk} (fp32), per token t:
 *   S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,   o_t = S_t q_t
 * (keys, queries and gates as given: normalisation and scaling are the caller's).
 *   q, k [B, T, H, dk] bf16; v [B, T, H, dv] bf16; alpha, beta [B, T, H] fp32;
 *   state_in [B, H, dv, dk] fp32 or NULL (zeros); o [B, T, H, dv] fp32;
 *   state_out [B, H, dv, dk] fp32 (may be state_in).  dk, dv in {64, 128}.
 * T == 0 copies the initial state.  Decode is one token per sequence with the
 * state updated in place: q, k [B, H, dk], v [B, H, dv], alpha, beta [B, H],
 * state [B, H, dv, dk], o [B, H, dv].
 */
QSA_API qsa_status_t qsa_gdn_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                     const qsa_bf16_t *v, const float *alpha, const float *beta,
                                     const float *state_in, int B, int64_t T, int H, int dk,
                                     int dv, float *o, float *state_out, void *stream);
/*
 * The same prefill in chunks of 64 tokens [SUM: GDN, token mixing; the chunked
 * form of the delta rule]: within a chunk, with gamma_t the product of the
 * chunk's decay gates up to t and S0 the entering state, the writes
 * u_t = beta_t (v_t - alpha_t S_{t-1} k_t) solve a unit lower-triangular system
 * (I + A) U = diag(beta) V - diag(beta gamma) K S0^T, A_tj = beta_t
 * (gamma_t / gamma_j) k_t.k_j; the outputs are diag(gamma) Q S0^T + P U,
 * P_tj = (gamma_t / gamma_j) q_t.k_j (j <= t), and the next state gamma_last S0 +
 * U^T diag(gamma_last / gamma) K.  The solves run for all chunks at once; the
 * state products then run chunk after chunk on the tensor cores with fp32
 * operands split into bf16 high and low parts (about 2^-16 relative per
 * product).  Same arguments and layouts as qsa_gdn_prefill, plus a caller
 * workspace of qsa_gdn_prefill_chunked_workspace_size bytes (256-byte aligned;
 * per (sequence, head, chunk) the chunk's solve: 112.5 KiB at dk = dv = 128).
 * Returns QSA_ERR_WORKSPACE if it is missing, too small or misaligned.
 */
QSA_API size_t qsa_gdn_prefill_chunked_workspace_size(int B, int64_t T, int H, int dk, int dv);
QSA_API qsa_status_t qsa_gdn_prefill_chunked(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                             const qsa_bf16_t *v, const float *alpha,
                                             const float *beta, const float *state_in, int B,
                                             int64_t T, int H, int dk, int dv, float *o,
                                             float *state_out, void *ws, size_t ws_bytes,
                                             void *stream);
QSA_API qsa_status_t qsa_gdn_decode(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                    const qsa_bf16_t *v, const float *alpha, const float *beta,
                                    float *state, int B, int H, int dk, int dv, float *o,
                                    void *stream);

/*
 * Measurement aid, not part of the attention path: reads the first `bytes` of
 * the device buffer `buf` (16-byte aligned, >= 16 bytes) `reps` times with
 * 16-byte loads cached in L2 only, on all SMs; `sink` is a device word the
 * kernel may write (to keep its loads live).  Timed around with events over a
 * buffer that fits in L2, it gives the L2-to-SM read bandwidth that kernels
 * with L2-resident sources are rated against.  Bytes read = bytes * reps
 * (rounded down to 16-byte units).
 */
QSA_API qsa_status_t qsa_probe_l2_read(const void *buf, size_t bytes, int reps, void *sink,
                                       void *stream);

/*
 * Synchronises `stream`, reads the status word kernels recorded at the start
 * of `ws`, clears it, and returns it (QSA_OK if nothing was recorded).  The
 * word is sticky: it keeps the first error recorded by any call that used
 * this workspace since the last check.  A new workspace must have its first
 * 256 bytes zeroed once before first use (this function leaves them zero).
 */
QSA_API qsa_status_t qsa_check_device_status(void *ws, void *stream);

/* Static description of a status code. */
QSA_API const char *qsa_status_string(qsa_status_t status);

/* Library version, "major.minor.patch". */
QSA_API const char *qsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
