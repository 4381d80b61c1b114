/*
 * tokengate.h -- C ABI of the B200 (sm_100a) TokenGate pruned-prefill library.
 *
 * The library implements the data-parallel core of the method described in the
 * MarkTechPost article "Researchers from Stanford and UC Berkeley Introduce
 * TokenGate: token-gated attention speeds up long-context prefill by up to
 * 11.3x" (October 2026), called "the TokenGate article" below:
 *
 *   1. tg_gate_score      -- MLP gate scores every prompt token from its residual;
 *   2. tg_select_topk     -- keep the K best document tokens, always keep the question;
 *   3. tg_gather          -- compact the kept tokens' rows;
 *   4. tg_gated_attention -- causal GQA attention over the kept tokens with the
 *                            gate score as a per-key logit bias.
 *
 * Conventions shared by every call
 *   - Tensor arguments are DEVICE pointers owned by the caller, packed row-major
 *     (the last dimension contiguous).  The library never allocates, never
 *     frees and never keeps a pointer after the call returns.
 *   - bf16 tensors are passed as tg_bf16, the raw 16-bit pattern.
 *   - Calls are asynchronous on ``stream`` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronise it.  They can be captured into a
 *     CUDA graph.
 *   - The return value reports errors that the host can detect (shapes,
 *     alignment, null pointers, unsupported sizes, launch failures).  When it
 *     is not TG_OK nothing was launched, with one exception: a call that
 *     launches several kernels (tg_select_topk_varlen, tg_select_fused, the
 *     backward) and whose second or later launch fails returns TG_ERR_CUDA with
 *     the earlier kernels already queued; its outputs and workspace are then
 *     undefined.  tg_last_error_detail() describes the error.
 *   - Conditions only the device can see (an index out of range, a budget
 *     above the document length, a full output, a bounded wait that ran out)
 *     set bits in a sticky per-device status word and never trap.  Read and
 *     clear it with tg_get_device_error().
 *   - Calls on different streams may run concurrently; they share only the
 *     status word, whose bits are OR-ed.  Exception: every
 *     tg_gated_attention_backward_noalloc call on a device uses the same static
 *     scratch array, so those calls must be ordered on the device (one stream,
 *     or streams that wait on each other).
 *   - Host threads may call the library concurrently.  Per-device set-up (kernel
 *     attributes, the device addresses of the status word and of the static
 *     scratch) is done by the first call on each device and kept for the life of
 *     the process, so a device reset (cudaDeviceReset) invalidates it: do not use
 *     the library on a device after resetting that device.
 *   - Every call opens an NVTX range named after it on the calling host thread.
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TG_ABI_VERSION 1

typedef uint16_t tg_bf16;   /* bf16 bit pattern (the high half of an IEEE fp32) */
typedef void *tg_stream;    /* cudaStream_t */

typedef enum {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size */
    TG_ERR_UNSUPPORTED = 2,   /* a size the kernels are not built for */
    TG_ERR_ALIGNMENT = 3,     /* a pointer or row pitch not 16-byte aligned */
    TG_ERR_CUDA = 4           /* a CUDA runtime/driver call failed (launch, attribute) */
} tg_status;

/* Bits of the per-device status word. */
enum {
    TG_DEVERR_TIMEOUT = 1u,    /* a bounded wait inside a kernel gave up; its outputs are invalid */
    TG_DEVERR_INDEX_OOB = 2u,  /* tg_gather met an index outside [0, n); that row was skipped */
    TG_DEVERR_K_GT_NDOC = 4u,  /* budget above the document length; clamped to keep every document token */
    TG_DEVERR_CAPACITY = 8u,   /* kept tokens exceed the output capacity; writes past it were dropped */
    TG_DEVERR_BAD_SEQLENS = 16u /* cu_seqlens not non-decreasing within [0, total], or a
                                   request longer than max_seqlen */
};

/* ABI version of the loaded library (TG_ABI_VERSION it was built with). */
int tg_abi_version(void);

/* Static string naming a status code. */
const char *tg_status_string(tg_status status);

/* Human-readable detail of the last non-TG_OK return on the calling host thread
 * (empty string if none).  The pointer stays valid until that thread's next call. */
const char *tg_last_error_detail(void);

/* Synchronise ``stream``, then read and clear the status word of the current
 * device into *bits (a host pointer).  Returns TG_ERR_CUDA if the
 * synchronisation itself failed (e.g. a sticky CUDA error from another kernel). */
tg_status tg_get_device_error(tg_stream stream, uint32_t *bits);

/* Diagnostics: launch one kernel whose bounded wait on an mbarrier that nothing
 * arrives on runs out after limit_ns (0 < limit_ns <= 2e9), so that the
 * timeout path (TG_DEVERR_TIMEOUT in the status word) can be checked without
 * hanging a GPU.  The paper has no counterpart; it exists for testing. */
tg_status tg_probe_wait_timeout(int64_t limit_ns, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_gate_score -- gate MLP scorer.
 * TokenGate article, "How does TokenGate learned token pruning work?" (gate
 * module): a small MLP scores each token from its post-attention residual at
 * the gate layer.  The scorer is Linear(d -> h), SiLU, Linear(h -> 1):
 *     scores[i] = b2 + sum_j W2[j] * SiLU(b1[j] + sum_k W1[j,k] * hidden[i,k])
 * computed with bf16 inputs, fp32 accumulation and an fp32 result.
 *
 *   hidden  bf16 [n, d]   residual stream at the gate layer
 *   W1      bf16 [h, d]   first layer, nn.Linear layout (row j = hidden unit j)
 *   b1      bf16 [h]
 *   W2      bf16 [h]      second layer weights (one output)
 *   b2      bf16 [1]
 *   scores  fp32 [n]      output
 * Sizes: n >= 0 (n = 0 launches nothing); d a positive multiple of 8;
 * h a multiple of 16 in [16, 256].  hidden, W1 and scores 16-byte aligned.
 * -------------------------------------------------------------------------- */
tg_status tg_gate_score(const tg_bf16 *hidden, int64_t n, int32_t d,
                        const tg_bf16 *W1, const tg_bf16 *b1, const tg_bf16 *W2,
                        const tg_bf16 *b2, int32_t h, float *scores, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_select_topk -- top-K over the document, question always kept.
 * TokenGate article, "How does TokenGate learned token pruning work?": a top-K
 * selector keeps the highest-scoring tokens; only the document part of the
 * prompt is prunable, the question is never pruned.  The generation API's
 * max_kept_prefill_tokens budget ("How do you deploy TokenGate?") is k.
 *
 * Among tokens with doc_mask[i] != 0 the k largest scores are kept, ordered by
 * (score descending, index ascending): ties go to the lower index, -0.0 equals
 * +0.0, NaN ranks below every number.  Every token with doc_mask[i] == 0 is
 * kept.  kept_idx receives the union in ascending order and *n_kept (a device
 * int32) its size, min(k, n_doc) + n_question.
 *
 *   scores    fp32 [n]      the gate scores (read only)
 *   doc_mask  uint8 [n]     1 = document token (prunable), 0 = question token
 *   k         budget, >= 0; k > n_doc keeps every document token and sets
 *             TG_DEVERR_K_GT_NDOC
 *   kept_idx  int32 [cap]   output; entries past *n_kept are left untouched
 *   cap       capacity of kept_idx; writes past it are dropped and set
 *             TG_DEVERR_CAPACITY
 *   n_kept    int32 [1]     output (device)
 * Sizes: 0 <= n < 2^31.  No workspace: intermediate state lives in the
 * shared memory of one thread-block cluster.
 * -------------------------------------------------------------------------- */
tg_status tg_select_topk(const float *scores, const uint8_t *doc_mask, int64_t n, int64_t k,
                         int32_t *kept_idx, int64_t cap, int32_t *n_kept, tg_stream stream);

/* Packed ragged batch: request b owns positions [cu_seqlens[b], cu_seqlens[b+1])
 * of scores/doc_mask and budget k_per_seq[b] (both device int32 arrays).
 * Kept indices are positions in the packed sequence; request b's come out at
 * kept_idx[cu_kept[b] .. cu_kept[b+1]) and cu_kept (device int32 [B+1]) is
 * written with cu_kept[0] = 0.  max_seqlen is a host upper bound on any
 * request's length and total the packed length (the bound cu_seqlens must
 * respect).  Malformed cu_seqlens, or a request longer than max_seqlen, set
 * TG_DEVERR_BAD_SEQLENS (the kept indices are then invalid). */
tg_status tg_select_topk_varlen(const float *scores, const uint8_t *doc_mask,
                                const int32_t *cu_seqlens, int32_t B, int64_t total,
                                const int32_t *k_per_seq, int64_t max_seqlen,
                                int32_t *kept_idx, int64_t cap, int32_t *cu_kept,
                                tg_stream stream);

/* Budget sweep: the same selection for m budgets in one launch (one thread-block
 * cluster per budget), e.g. for the accuracy-versus-budget curves of the TokenGate
 * article ("How does TokenGate perform on benchmarks?") or a training step's random
 * budget ("What is token-gated attention?").  ks: device int32 [m]; budget b's kept
 * indices go to kept_idx[b * stride ...] (capacity stride each) and its count to
 * n_kept[b] (device int32 [m]).  Same order and error bits as tg_select_topk. */
tg_status tg_select_topk_sweep(const float *scores, const uint8_t *doc_mask, int64_t n,
                               const int32_t *ks, int32_t m, int32_t *kept_idx, int64_t stride,
                               int32_t *n_kept, tg_stream stream);

/* Random-K selection: keep k uniformly random document tokens (without replacement)
 * and every question token, ascending -- the random-selector ablation of the
 * TokenGate article ("How does TokenGate perform on benchmarks?": even random-K
 * selection scores well on the co-adapted backbone).  Token i's random key is
 * SplitMix64(seed, i) (Steele, Lea and Flood, 2014): x = seed + (i + 1) * 0x9E3779B97F4A7C15,
 * x = (x ^ x >> 30) * 0xBF58476D1CE4E5B9, x = (x ^ x >> 27) * 0x94D049BB133111EB,
 * x ^= x >> 31; the k document tokens with the largest (x >> 33) are kept, ties to the
 * lower index.  Outputs and error bits as tg_select_topk. */
tg_status tg_select_random_k(const uint8_t *doc_mask, int64_t n, int64_t k, uint64_t seed,
                             int32_t *kept_idx, int64_t cap, int32_t *n_kept, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_select_fused -- tg_gate_score, tg_select_topk and tg_gather as one call.
 * TokenGate article, "How does TokenGate learned token pruning work?": the gate
 * scores every token, the K best document tokens and every question token are
 * kept, and the layers above L run on the kept tokens only.  The results are
 * exactly those of the three calls in sequence on the same arguments:
 *     scores  = tg_gate_score(hidden, W1, b1, W2, b2)                fp32 [n]
 *     kept_idx, *n_kept = tg_select_topk(scores, doc_mask, k, cap)
 *     hidden_k, s_k = tg_gather(hidden, kept_idx, n_rows, n_kept, scores)
 * Faster: the gate's epilogue histograms the top byte of every document token's
 * selection key, so the selector's first radix pass reads those histograms
 * instead of every score, and the three kernels overlap at their boundaries.
 *   workspace: device memory of at least tg_select_fused_workspace(n) bytes
 *   (depends on the current device's SM count), 16-byte aligned, caller-owned;
 *   it holds the per-CTA histograms until the stream reaches the end of the call.
 * Sizes as for the three calls (d a multiple of 8, at most 16384; h a multiple of
 * 16 in [16, 256]; n < 2^31); n_rows <= cap; hidden_k and s_k are required when
 * n_rows > 0.  Device-side conditions set the same status bits as the three calls.
 * -------------------------------------------------------------------------- */
size_t tg_select_fused_workspace(int64_t n);

tg_status tg_select_fused(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1,
                          const tg_bf16 *b1, const tg_bf16 *W2, const tg_bf16 *b2, int32_t h,
                          const uint8_t *doc_mask, int64_t k, float *scores, int32_t *kept_idx,
                          int64_t cap, int32_t *n_kept, tg_bf16 *hidden_k, float *s_k,
                          int64_t n_rows, void *workspace, size_t workspace_bytes,
                          tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_gather -- compaction of the kept tokens.
 * TokenGate article, "How does TokenGate learned token pruning work?" (pruned
 * forward): layers above the gate process only the kept tokens and create no
 * KV entries for pruned ones.
 *     hidden_k[r, :] = hidden[kept_idx[r], :]      s_k[r] = scores[kept_idx[r]]
 * for r < n_rows, further limited to r < *n_kept when n_kept is not NULL (a
 * device int32, e.g. the count written by tg_select_topk).  Rows outside
 * that range are left untouched.
 *
 *   hidden    bf16 [n, d]      kept_idx  int32 [n_rows]   hidden_k bf16 [n_rows, d]
 *   scores    fp32 [n] or NULL s_k       fp32 [n_rows] or NULL (both or neither)
 * Sizes: d a positive multiple of 8, at most 16384; hidden and hidden_k
 * 16-byte aligned.  An index outside [0, n) skips its row and sets TG_DEVERR_INDEX_OOB.
 * -------------------------------------------------------------------------- */
tg_status tg_gather(const tg_bf16 *hidden, int64_t n, int32_t d, const int32_t *kept_idx,
                    int64_t n_rows, const int32_t *n_kept, tg_bf16 *hidden_k,
                    const float *scores, float *s_k, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_gated_attention -- token-gated causal GQA attention over the kept tokens.
 * TokenGate article, "What is token-gated attention?": each kept token's score
 * becomes a bias on the attention logits of every layer above the gate, with a
 * learnable per-head gain and a learnable temperature.  For query row i, query
 * head h and key/value head g = h / (Hq / Hkv):
 *     logit(i, j) = tau * (Q[i,h,:] . Kc[j,g,:]) / sqrt(D) + gain[h] * s[j],  j <= i
 *     O[i,h,:]    = sum_j softmax_j(logit(i, .)) * V[j,g,:]
 * Causality is in compacted order, which is the prompt order because kept
 * indices are ascending.  bf16 inputs, fp32 accumulation, bf16 output.
 *
 *   Q   bf16 [S, Hq, D]    Kc, V  bf16 [S, Hkv, D]    O  bf16 [S, Hq, D]
 *   s   fp32 [S] or NULL   gain   fp32 [Hq]           tau (host float)
 * With s = NULL the call is plain causal GQA attention (no key bias; gain may then
 * also be NULL): the form of the layers below the gate, and the baseline the bias
 * costs are measured against.
 * Sizes: S >= 0; D in {64, 128}; Hq a positive multiple of Hkv; S * Hq < 2^31.
 * Q, Kc, V and O 16-byte aligned.
 * Two kernels serve this call and its varlen / training forms: one with two 128-row
 * query tiles per CTA, and, when that grid (one CTA per 256 query rows, head and
 * request, counted from max_seqlen) would hold at most 1.5 CTAs per SM, a persistent
 * one that works through single query tiles.  Both are deterministic and held to the
 * same tolerance; their outputs are not bitwise equal to each other.
 * -------------------------------------------------------------------------- */
tg_status tg_gated_attention(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                             const float *s, const float *gain, float tau,
                             int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                             tg_bf16 *O, tg_stream stream);

/* The same forward for training: also stores what tg_gated_attention_backward
 * needs.  lse[i * Hq + h] = log sum_{j <= i} exp(logit(i, j)) (natural log), fp32
 * [S, Hq], required.  O32: fp32 [S, Hq, D] or NULL: the output before its bf16
 * rounding; given to the backward, it keeps that rounding out of dO . O (at S =
 * 8704 the rounding otherwise moves the first keys' score gradients by ~10 % of
 * their rms).  Both caller-allocated, 16-byte aligned, written. */
tg_status tg_gated_attention_train(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                   const float *s, const float *gain, float tau,
                                   int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                   tg_bf16 *O, float *lse, float *O32, tg_stream stream);

/* Packed ragged batch: request b owns rows [cu_seqlens[b], cu_seqlens[b+1]) of
 * Q, Kc, V, s and O (cu_seqlens: device int32 [B+1], e.g. cu_kept from
 * tg_select_topk_varlen) and attends causally within itself only.  total is
 * the packed row count and max_seqlen a host upper bound on any request's
 * length (it sizes the grid).  A range outside [0, total], a decreasing one or a
 * request with rows beyond those max_seqlen covers (rounded up to whole tiles) sets
 * TG_DEVERR_BAD_SEQLENS (that request's output is then incomplete; the ranges are
 * clamped into [0, total]). */
tg_status tg_gated_attention_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                    const float *s, const float *gain, float tau,
                                    const int32_t *cu_seqlens, int32_t B, int64_t total,
                                    int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                    tg_bf16 *O, tg_stream stream);

/* The training forward of a packed ragged batch: the outputs of
 * tg_gated_attention_varlen plus lse and O32 as in tg_gated_attention_train, at the
 * packed rows (lse [total, Hq], O32 [total, Hq, D] or NULL).  Rows outside every
 * request are left untouched. */
tg_status tg_gated_attention_train_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                          const float *s, const float *gain, float tau,
                                          const int32_t *cu_seqlens, int32_t B, int64_t total,
                                          int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                          tg_bf16 *O, float *lse, float *O32, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_gated_attention_backward -- gradients of token-gated attention with respect
 * to the key scores, the per-head gains and the temperature: the path by which
 * the gate is trained through the layers above it.
 * TokenGate article, "What is token-gated attention?": the score is a logit bias
 * with a learnable per-head gain, the dot product a learnable temperature.  For a
 * loss L with dL/dO = dO, per head h, query i and key j <= i (g = h / (Hq/Hkv)):
 *     P_ij    = exp(logit(i, j) - lse[i, h])
 *     dl_ij   = P_ij (dO[i,h,:] . V[j,g,:] - dO[i,h,:] . O[i,h,:])
 *     ds[j]   = sum_{h,i} gain[h] dl_ij
 *     dgain[h]= sum_{i,j} s[j] dl_ij
 *     dtau    = sum_{h,i,j} dl_ij (Q[i,h,:] . Kc[j,g,:]) / sqrt(D)
 *
 *   Q, dO, O  bf16 [S, Hq, D]     Kc, V  bf16 [S, Hkv, D]     s fp32 [S]
 *   gain fp32 [Hq]   tau (host)   lse fp32 [S, Hq], O, O32 (fp32 [S, Hq, D] or NULL):
 *   from tg_gated_attention_train with the same inputs.  dO . O is taken from O32
 *   when it is given (recommended), else from O (one of the two must be given).
 *   ds fp32 [S], dgain fp32 [Hq], dtau fp32 [1]: written (overwritten, not added to).
 *   workspace: device memory of at least tg_gated_attention_backward_workspace(S, Hq)
 *   bytes, 16-byte aligned, owned by the caller, contents irrelevant on entry; the
 *   call uses it until the stream reaches the end of the call.
 * Sizes as for tg_gated_attention.  Results are deterministic (fixed summation
 * order).  fp32 arithmetic over the bf16 inputs; the probabilities are recomputed
 * in fp32 from lse.
 * -------------------------------------------------------------------------- */
size_t tg_gated_attention_backward_workspace(int64_t S, int32_t Hq);

tg_status tg_gated_attention_backward(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                      const float *s, const float *gain, float tau,
                                      const tg_bf16 *O, const float *O32, const tg_bf16 *dO,
                                      const float *lse,
                                      int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                      float *ds, float *dgain, float *dtau,
                                      void *workspace, size_t workspace_bytes, tg_stream stream);

/* The backward of a packed ragged batch (the training side of
 * tg_gated_attention_varlen, e.g. a batch of requests each trained under its own
 * budget).  Request b owns packed rows [cu_seqlens[b], cu_seqlens[b+1]) of Q, Kc, V, s,
 * O, O32, dO and lse (cu_seqlens: device int32 [B+1], non-decreasing within [0, total])
 * and attends causally within itself only, so
 *     ds[j]    = the formula above within j's request,
 *     dgain[h] = sum over every request,   dtau = sum over every request.
 * Rows outside every request get ds = 0.  max_seqlen is a host upper bound on any
 * request's length (it sizes the grid).  workspace: at least
 * tg_gated_attention_backward_varlen_workspace(total, B, Hq) bytes (each request's rows
 * padded to whole 128-row blocks), 16-byte aligned, caller-owned.  Malformed cu_seqlens,
 * or a request longer than max_seqlen, set TG_DEVERR_BAD_SEQLENS and leave the gradients
 * undefined.  Sizes and the rest as for tg_gated_attention_backward. */
size_t tg_gated_attention_backward_varlen_workspace(int64_t total, int32_t B, int32_t Hq);

tg_status tg_gated_attention_backward_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                             const float *s, const float *gain, float tau,
                                             const tg_bf16 *O, const float *O32, const tg_bf16 *dO,
                                             const float *lse, const int32_t *cu_seqlens, int32_t B,
                                             int64_t total, int64_t max_seqlen,
                                             int32_t Hq, int32_t Hkv, int32_t D,
                                             float *ds, float *dgain, float *dtau,
                                             void *workspace, size_t workspace_bytes, tg_stream stream);

/* tg_gated_attention_backward_noalloc -- the same backward without a caller
 * workspace and without allocating anything: its scratch is a fixed 4 MiB device
 * array inside the library (one per device), so any S * Hq whose workspace
 * (tg_gated_attention_backward_workspace) exceeds 4,194,304 bytes is rejected
 * with TG_ERR_UNSUPPORTED before any launch.  Calls on one device share that
 * array: they must be ordered (one stream, or streams that wait on each other).
 * Results are bitwise those of tg_gated_attention_backward.  The TokenGate article
 * has no counterpart of this call: it is a deployment convenience of this library. */
tg_status tg_gated_attention_backward_noalloc(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                              const float *s, const float *gain, float tau,
                                              const tg_bf16 *O, const float *O32, const tg_bf16 *dO,
                                              const float *lse, int64_t S, int32_t Hq, int32_t Hkv,
                                              int32_t D, float *ds, float *dgain, float *dtau,
                                              tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_qkv_rope -- Q, K and V of a pruned layer, at the kept tokens' positions.
 * TokenGate article, "How does TokenGate learned token pruning work?" (pruned
 * forward): the layers above the gate run on the kept tokens only, and each kept
 * token stays at its prompt position.  On the article's Qwen3 backbone an
 * attention block projects, normalises each Q / K head and applies the rotary
 * embedding; for kept row i at position p = positions[i]:
 *     y            = W_qkv hidden[i, :]                       (fp32 accumulation)
 *     Q / K head u = y_head / sqrt(mean(y_head^2) + eps) * norm_weight
 *                    (when q_norm / k_norm is NULL that head kind is not normalised)
 *     phi_j        = p * rope_base^(-2j / D),   j < D/2
 *     out_j        = u_j cos phi_j - u_(j+D/2) sin phi_j
 *     out_(j+D/2)  = u_(j+D/2) cos phi_j + u_j sin phi_j
 *     V head       = y_head (no norm, no rotation)
 * One bf16 rounding at the end.
 *
 *   hidden    bf16 [S, d]                     W_qkv  bf16 [(Hq + 2 Hkv) D, d]
 *             (rows: Hq Q heads, then Hkv K heads, then Hkv V heads)
 *   positions int32 [S] (e.g. the kept indices from tg_select_topk)
 *   q_norm, k_norm  bf16 [D] or NULL          eps    host float >= 0
 *   Q bf16 [S, Hq, D]   Kc, V bf16 [S, Hkv, D]   (written, caller-allocated)
 * Sizes: S >= 0; d a positive multiple of 8; D in {64, 128}; rope_base > 1.
 * hidden, W_qkv, Q, Kc and V 16-byte aligned.
 * -------------------------------------------------------------------------- */
tg_status tg_qkv_rope(const tg_bf16 *hidden, int64_t S, int32_t d, const tg_bf16 *W_qkv,
                      const int32_t *positions, double rope_base, const tg_bf16 *q_norm,
                      const tg_bf16 *k_norm, float eps, int32_t Hq, int32_t Hkv, int32_t D,
                      tg_bf16 *Q, tg_bf16 *Kc, tg_bf16 *V, tg_stream stream);

/* --------------------------------------------------------------------------
 * tg_linear -- the output projection of a pruned layer (o_proj), with the
 * residual add fused: y[i, :] = W x[i, :] (+ residual[i, :]).
 * TokenGate article, "How does TokenGate learned token pruning work?" (pruned
 * forward: the layers above the gate run on the kept tokens only).
 *
 *   x  bf16 [M, K]   W  bf16 [N, K] (nn.Linear layout)
 *   residual bf16 [M, N] or NULL   y  bf16 [M, N] (written; may not alias x or W)
 * Sizes: M >= 0; K a positive multiple of 8; N a positive multiple of 32.
 * All pointers 16-byte aligned.  fp32 accumulation, one bf16 rounding.
 * -------------------------------------------------------------------------- */
tg_status tg_linear(const tg_bf16 *x, int64_t M, int32_t K, const tg_bf16 *W, int32_t N,
                    const tg_bf16 *residual, tg_bf16 *y, tg_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H */
