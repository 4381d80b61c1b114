// internal.h -- launchers shared between the library's translation units (not part of
// the C ABI; hidden from the shared object's exports).
#pragma once
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

}  // namespace tg
