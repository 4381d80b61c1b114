// gather.cu -- tg_gather: compaction of the kept tokens' rows.
//
// TokenGate article, "How does TokenGate learned token pruning work?" (pruned
// forward): the layers above the gate process only the kept tokens, so their
// residual rows (and gate scores) are gathered into a dense, shorter sequence.
//
// B200 design: the copy is HBM-bound (read + write each kept row once).  Rows
// move through shared memory with the TMA engine's bulk copies
// (cp.async.bulk global->shared with mbarrier completion, then
// cp.async.bulk shared->global), so no thread touches the payload.  Each warp
// runs its own pipeline of ``stages`` row buffers; one lane issues the copies.
// The grid is sized to two CTAs per SM (fewer only when there are fewer rows than
// warps), keeping several MB of copies in flight.
#include <algorithm>

#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kSmemBudget = 96 * 1024;

__global__ void __launch_bounds__(kThreads) gather_rows_kernel(
    const uint8_t *__restrict__ hidden, int64_t n, uint32_t row_bytes, const int32_t *__restrict__ kept_idx,
    int64_t n_rows, const int32_t *__restrict__ n_kept_dev, uint8_t *__restrict__ hidden_k,
    const float *__restrict__ scores, float *__restrict__ s_k, int stages, uint32_t *err) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int abort_flag;
  tg::pdl_wait();
  tg::pdl_trigger();

  int64_t rows = n_rows;
  if (n_kept_dev) {
    const int64_t c = static_cast<int64_t>(*n_kept_dev);
    rows = c < 0 ? 0 : (c < rows ? c : rows);
  }

  // The scores travel with their rows; plain coalesced loads are enough for 4 bytes a row.
  if (scores && s_k) {
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; r < rows;
         r += static_cast<int64_t>(gridDim.x) * kThreads) {
      const int32_t idx = kept_idx[r];
      if (idx >= 0 && idx < n) s_k[r] = scores[idx];
    }
  }

  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;
  uint8_t *buf = smem + static_cast<size_t>(warp) * stages * row_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + static_cast<size_t>(kWarps) * stages * row_bytes) +
                   warp * stages;

  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0) {
    for (int s = 0; s < stages; ++s) tg::mbar_init(tg::smem_addr(&bars[s]), 1);
    tg::fence_mbar_init();
  }
  __syncthreads();
  if (lane != 0) return;

  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  uint32_t phase = 0;
  bool failed = false;
  for (int64_t first = gwarp; first < rows && !failed; first += nwarps * stages) {
    int cnt = 0;
    for (int s = 0; s < stages; ++s) {
      const int64_t r = first + static_cast<int64_t>(s) * nwarps;
      if (r >= rows) break;
      const uint32_t bar = tg::smem_addr(&bars[s]);
      const int32_t idx = kept_idx[r];
      if (idx < 0 || idx >= n) {
        tg::set_device_error(err, TG_DEVERR_INDEX_OOB);
        tg::mbar_arrive(bar);  // complete the phase without a copy
      } else {
        tg::mbar_arrive_expect_tx(bar, row_bytes);
        tg::bulk_load(tg::smem_addr(buf + static_cast<size_t>(s) * row_bytes),
                      hidden + static_cast<size_t>(idx) * row_bytes, row_bytes, bar);
      }
      ++cnt;
    }
    for (int s = 0; s < cnt; ++s) {
      const int64_t r = first + static_cast<int64_t>(s) * nwarps;
      if (!tg::mbar_wait(tg::smem_addr(&bars[s]), phase, &abort_flag)) {
        tg::set_device_error(err, TG_DEVERR_TIMEOUT);
        failed = true;
        break;
      }
      const int32_t idx = kept_idx[r];
      if (idx >= 0 && idx < n)
        tg::bulk_store(hidden_k + static_cast<size_t>(r) * row_bytes,
                       tg::smem_addr(buf + static_cast<size_t>(s) * row_bytes), row_bytes);
    }
    tg::bulk_commit();
    tg::bulk_wait_read_all();  // the stores have read the buffers before they are refilled
    phase ^= 1u;
  }
  tg::bulk_wait_all();
}

}  // namespace

extern "C" tg_status tg_gather(const tg_bf16 *hidden, int64_t n, int32_t d, const int32_t *kept_idx,
                               int64_t n_rows, const int32_t *n_kept, tg_bf16 *hidden_k, const float *scores,
                               float *s_k, tg_stream stream) {
  TG_API_ENTRY();
  if (n < 0 || n_rows < 0) return tg::fail(TG_ERR_INVALID_ARG, "negative n or n_rows");
  if (d <= 0 || d % 8 != 0) return tg::fail(TG_ERR_INVALID_ARG, "d must be a positive multiple of 8 (got %d)", d);
  if (d > 16384) return tg::fail(TG_ERR_UNSUPPORTED, "d above 16384 (got %d)", d);
  if ((scores == nullptr) != (s_k == nullptr)) return tg::fail(TG_ERR_INVALID_ARG, "scores and s_k: both or neither");
  if (n_rows == 0) return TG_OK;
  if (!hidden || !kept_idx || !hidden_k) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (!tg::aligned16(hidden) || !tg::aligned16(hidden_k))
    return tg::fail(TG_ERR_ALIGNMENT, "hidden and hidden_k must be 16-byte aligned");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;

  const uint32_t row_bytes = static_cast<uint32_t>(d) * 2u;
  int stages = static_cast<int>(kSmemBudget / (kWarps * (row_bytes + 8)));
  stages = std::max(1, std::min(stages, 8));
  const size_t smem = static_cast<size_t>(kWarps) * stages * (row_bytes + 8);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(gather_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  }
  // one row per warp before any warp takes a second, so that a short gather still spreads
  // over every SM (up to two CTAs per SM)
  int64_t grid = (n_rows + kWarps - 1) / kWarps;
  grid = std::max<int64_t>(1, std::min<int64_t>(grid, 2LL * tg::sm_count()));
  const cudaError_t e = tg::launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem,
                                      static_cast<cudaStream_t>(stream), reinterpret_cast<const uint8_t *>(hidden), n,
                                      row_bytes, kept_idx, n_rows, n_kept, reinterpret_cast<uint8_t *>(hidden_k),
                                      scores, s_k, stages, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "gather_rows_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("gather_rows_kernel");
}
