// select_fused.cu -- tg_select_fused: the gate -> top-K -> gather chain as one call.
//
// TokenGate article, "How does TokenGate learned token pruning work?": the gate
// scores every token at layer L, the K best document tokens and every question
// token are kept, and the layers above L run on the kept tokens only.  This call
// computes exactly tg_gate_score, tg_select_topk and tg_gather in that order; what
// changes is the work between them:
//   * the gate's epilogue histograms the top byte of the selector's order key of
//     every document token's score, one 256-bin histogram per CTA, stored in the
//     caller's workspace (no zeroing, no global atomics);
//   * the selector's first radix pass sums those histograms (148 x 256 counters at
//     N = 128k) instead of histogramming 131072 keys and reducing them across its
//     cluster;
//   * the three kernels are launched back to back with programmatic stream
//     serialisation, so each one's launch and prologue overlap the previous one's
//     tail; captured in a CUDA graph the chain replays without host gaps.
#include "internal.h"
#include "runtime.h"

extern "C" size_t tg_select_fused_workspace(int64_t n) {
  if (n <= 0) return 0;
  return static_cast<size_t>(tg::gate_grid(n)) * 256 * sizeof(uint32_t);
}

extern "C" tg_status tg_select_fused(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1,
                                     const tg_bf16 *b1, const tg_bf16 *W2, const tg_bf16 *b2, int32_t h,
                                     const uint8_t *doc_mask, int64_t k, float *scores, int32_t *kept_idx,
                                     int64_t cap, int32_t *n_kept, tg_bf16 *hidden_k, float *s_k, int64_t n_rows,
                                     void *workspace, size_t workspace_bytes, tg_stream stream) {
  TG_API_ENTRY();
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (n_rows < 0) return tg::fail(TG_ERR_INVALID_ARG, "n_rows must be >= 0");
  if (n_rows > cap) return tg::fail(TG_ERR_INVALID_ARG, "n_rows must not exceed cap");
  if (d <= 0 || d % 8 != 0 || d > 16384)
    return tg::fail(TG_ERR_UNSUPPORTED, "d must be a positive multiple of 8, at most 16384 (got %d)", d);
  if (n_rows > 0 && (!hidden_k || !s_k)) return tg::fail(TG_ERR_INVALID_ARG, "hidden_k and s_k are required");
  const size_t need = tg_select_fused_workspace(n);
  if (n > 0 && (!workspace || workspace_bytes < need))
    return tg::fail(TG_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu bytes needed", workspace_bytes, need);
  if (n > 0 && !tg::aligned16(workspace)) return tg::fail(TG_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  if (n == 0) {
    // no tokens: nothing kept (the selector writes the count)
    return tg_select_topk(scores, doc_mask, 0, k, kept_idx, cap, n_kept, stream);
  }
  uint32_t *parts = static_cast<uint32_t *>(workspace);
  const int n_parts = static_cast<int>(tg::gate_grid(n));
  tg_status st = tg::gate_score_hist(hidden, n, d, W1, b1, W2, b2, h, scores, doc_mask, parts, stream);
  if (st != TG_OK) return st;
  st = tg::select_topk_hist(scores, doc_mask, n, k, kept_idx, cap, n_kept, parts, n_parts, stream);
  if (st != TG_OK) return st;
  if (n_rows == 0) return TG_OK;
  return tg_gather(hidden, n, d, kept_idx, n_rows, n_kept, hidden_k, scores, s_k, stream);
}
