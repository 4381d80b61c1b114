// internal.h -- launchers shared between the library's translation units (not part of
// the C ABI; hidden from the shared object's exports).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "tokengate.h"

#define TG_INTERNAL __attribute__((visibility("hidden")))

namespace tg {

// CTAs of the gate launch for n tokens (two per 256-token tile, at most one pair per
// two SMs); the fused selection keeps one 256-bin histogram per CTA.
TG_INTERNAL int64_t gate_grid(int64_t n);

// tg_gate_score with, when hist_parts is not null, a histogram of the top 8 bits of the
// selector's order key of every document token's score: CTA c writes bins
// hist_parts[c * 256 .. c * 256 + 255] (gate_grid(n) CTAs).
TG_INTERNAL tg_status gate_score_hist(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1,
                                      const tg_bf16 *b1, const tg_bf16 *W2, const tg_bf16 *b2, int32_t h,
                                      float *scores, const uint8_t *doc_mask, uint32_t *hist_parts, tg_stream stream);

// tg_select_topk whose first radix pass sums n_parts such histograms instead of
// histogramming the keys itself.
TG_INTERNAL tg_status select_topk_hist(const float *scores, const uint8_t *doc_mask, int64_t n, int64_t k,
                                       int32_t *kept_idx, int64_t cap, int32_t *n_kept, const uint32_t *hist_parts,
                                       int n_parts, tg_stream stream);

// Token-gated attention in its persistent form (attention_persistent.cu): one CTA per SM
// working through (request, 128-row query tile, head) items.  Arguments as for
// tg_gated_attention_train_varlen (cu_seqlens NULL: one sequence of ``total`` rows; lse
// and O32 may be NULL); validated by the caller.
TG_INTERNAL tg_status gated_attention_persistent(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                                 const float *s, const float *gain, float tau,
                                                 const int32_t *cu_seqlens, int32_t B, int64_t total,
                                                 int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D, tg_bf16 *O,
                                                 float *lse, float *O32, cudaStream_t stream, uint32_t *err);

// Whether an attention call of this size runs the persistent kernel: when the two-tile
// kernel's grid (one CTA per 256 query rows, head and request) would hold at most 1.5
// CTAs per SM, so that its causal triangle leaves SMs idle.
TG_INTERNAL bool attention_uses_persistent(int64_t max_seqlen, int32_t Hq, int32_t B);

}  // namespace tg
