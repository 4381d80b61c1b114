// topk.cu -- tg_select_topk / tg_select_topk_varlen: keep the K best document
// tokens, always keep the question, output the kept positions in ascending order.
//
// TokenGate article, "How does TokenGate learned token pruning work?": a top-K
// selector keeps the highest-scoring tokens; only the document part of the prompt
// is prunable and the question is never pruned.  Order: score descending, ties to
// the lower index, -0.0 == +0.0, NaN below every number.
//
// B200 design: the work is memory-trivial (5 bytes a token), so the cost is
// latency.  One request is handled by one 8-CTA thread-block cluster; each CTA
// owns a contiguous chunk of the request and keeps its 32-bit order keys in
// shared memory.  Four 8-bit radix passes find the K-th largest key: every CTA
// builds a shared-memory histogram, the cluster barrier publishes it and every
// CTA sums the eight histograms through distributed shared memory, so all of
// them agree on the digit without touching global memory.  The ordered
// compaction then needs only two more cluster exchanges (tie counts and kept
// counts per CTA) and block-wide prefix sums.  No workspace, no global atomics,
// one launch for a single request.
#include <cooperative_groups.h>

#include <algorithm>

#include "ptx.cuh"
#include "runtime.h"

namespace cg = cooperative_groups;

namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kItems = 8;                   // consecutive positions per thread in a compaction tile
constexpr int kTile = kThreads * kItems;    // 4096 positions per tile
constexpr int kBins = 256;
constexpr int kKeyCap = 16384;              // order keys cached per CTA (64 KB)

// Order key: larger key = earlier in (score desc, NaN last).  0 marks a question
// token (never competes), 1 is NaN, every number maps to >= 0x007FFFFF.
__device__ __forceinline__ uint32_t order_key(float f, bool doc) {
  if (!doc) return 0u;
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 1u;  // NaN
  if (b == 0x80000000u) b = 0u;                      // -0.0 ranks with +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct Scan {
  int *warp_tot;  // [kWarps + 1]
};

// Block-wide exclusive prefix sum of one int per thread (thread order = index order).
// Returns the exclusive prefix; *total receives the block sum.  Contains barriers.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += t;
    }
    if (lane < kWarps) warp_tot[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) warp_tot[kWarps] = wi;
  }
  __syncthreads();
  const int res = warp_tot[warp] + incl - v;
  *total = warp_tot[kWarps];
  __syncthreads();
  return res;
}

struct TopkShared {
  uint32_t hist[kBins];
  uint32_t tot[kBins];
  int warp_tot[kWarps + 1];
  uint32_t sel_digit;
  uint32_t sel_above;
  long long exch[2];          // values other CTAs of the cluster read: [0] ties, [1] kept
  long long red[kWarps];
};

__device__ __forceinline__ void cluster_sum_hist(cg::cluster_group &cluster, TopkShared &sh) {
  if (threadIdx.x < kBins) {
    uint32_t s = 0;
#pragma unroll
    for (int c = 0; c < kCluster; ++c) s += cluster.map_shared_rank(sh.hist, c)[threadIdx.x];
    sh.tot[threadIdx.x] = s;
  }
  __syncthreads();
}

// Pick the digit D of the remaining-th largest candidate from sh.tot (bins scanned from 255 down).
__device__ __forceinline__ void select_digit(TopkShared &sh, uint32_t remaining) {
  if ((threadIdx.x >> 5) == 0) {
    const int lane = threadIdx.x & 31;
    uint32_t c[8];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = sh.tot[255 - 8 * lane - j];
      sum += c[j];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += t;
    }
    const uint32_t excl = incl - sum;
    if (excl < remaining && remaining <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (run + c[j] >= remaining) {
          sh.sel_digit = 255u - 8u * lane - j;
          sh.sel_above = run;
          break;
        }
        run += c[j];
      }
    }
  }
  __syncthreads();
}

__device__ __forceinline__ long long block_sum_ll(long long v, TopkShared &sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, off);
  if (lane == 0) sh.red[warp] = v;
  __syncthreads();
  long long s = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += sh.red[w];
  __syncthreads();
  return s;
}

// One cluster per request.  Single-request mode: cu_seqlens == nullptr, the request is
// [0, n_single) with budget k_single, base 0, and the CTA of rank 0 writes *n_kept.
// Varlen mode: request b = cluster index, range from cu_seqlens, budget k_per_seq[b],
// output offset cu_kept[b] (computed beforehand by seg_offsets_kernel).
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
    topk_cluster_kernel(const float *__restrict__ scores, const uint8_t *__restrict__ mask, int64_t n_single,
                        int64_t k_single, const int32_t *__restrict__ cu_seqlens, const int32_t *__restrict__ k_per_seq,
                        const int32_t *__restrict__ cu_kept, int64_t total, int32_t *__restrict__ kept_idx,
                        int64_t cap, int32_t *__restrict__ n_kept, int use_cache, uint32_t *err) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ TopkShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int seg = static_cast<int>(blockIdx.x) / kCluster;

  int64_t start = 0, end = n_single, k = k_single, base = 0;
  if (cu_seqlens) {
    start = cu_seqlens[seg];
    end = cu_seqlens[seg + 1];
    start = start < 0 ? 0 : (start > total ? total : start);
    end = end < start ? start : (end > total ? total : end);
    k = k_per_seq[seg];
    base = cu_kept[seg];
  }
  if (k < 0) k = 0;
  const int64_t len = end - start;
  const int64_t chunk = (len + kCluster - 1) / kCluster;
  const int64_t lo = start + chunk * rank;
  const int64_t hi = std::min<int64_t>(lo + chunk, end);
  const int m = lo < hi ? static_cast<int>(hi - lo) : 0;
  // The launcher sizes the key cache from its length bound; a request longer than
  // that bound falls back to reading the scores again on every pass.
  if (chunk > kKeyCap) use_cache = 0;

  auto key_at = [&](int i) -> uint32_t {
    if (use_cache) return keys[i];
    return order_key(scores[lo + i], mask[lo + i] != 0);
  };

  // ---- pass 0: order keys, histogram of the top byte, document count
  for (int b = threadIdx.x; b < kBins; b += kThreads) sh.hist[b] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += kThreads) {
    const uint32_t key = order_key(scores[lo + i], mask[lo + i] != 0);
    if (use_cache) keys[i] = key;
    if (key) atomicAdd(&sh.hist[key >> 24], 1u);
  }
  __syncthreads();
  cluster.sync();
  cluster_sum_hist(cluster, sh);
  long long n_doc = 0;
  {
    long long v = threadIdx.x < kBins ? sh.tot[threadIdx.x] : 0;
    n_doc = block_sum_ll(v, sh);
  }
  if (k > n_doc && rank == 0 && threadIdx.x == 0) tg::set_device_error(err, TG_DEVERR_K_GT_NDOC);
  const long long K = k < n_doc ? k : n_doc;

  // mode: 0 = keep no document token, 1 = keep all, 2 = radix threshold
  const int mode = (K == 0) ? 0 : (K == n_doc ? 1 : 2);
  uint32_t T = 0xFFFFFFFFu;  // keep key > T, plus the first need_eq keys == T in index order
  long long need_eq = 0;
  if (mode == 1) {
    T = 0u;  // every document key is > 0
  } else if (mode == 2) {
    uint32_t remaining = static_cast<uint32_t>(K);
    select_digit(sh, remaining);
    uint32_t prefix = sh.sel_digit << 24;
    remaining -= sh.sel_above;
    for (int pass = 1; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      cluster.sync();  // every CTA has finished reading the previous histograms
      for (int b = threadIdx.x; b < kBins; b += kThreads) sh.hist[b] = 0;
      __syncthreads();
      const uint32_t hi_mask = 0xFFFFFFFFu << (shift + 8);
      for (int i = threadIdx.x; i < m; i += kThreads) {
        const uint32_t key = key_at(i);
        if (key && (key & hi_mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 0xFFu], 1u);
      }
      __syncthreads();
      cluster.sync();
      cluster_sum_hist(cluster, sh);
      select_digit(sh, remaining);
      prefix |= sh.sel_digit << shift;
      remaining -= sh.sel_above;
    }
    T = prefix;
    need_eq = remaining;
  }

  // ---- exchange 1: ties (keys == T) per CTA, in index order across the cluster
  long long c_eq = 0;
  if (mode == 2) {
    long long v = 0;
    for (int i = threadIdx.x; i < m; i += kThreads) v += key_at(i) == T;
    c_eq = block_sum_ll(v, sh);
  }
  if (threadIdx.x == 0) sh.exch[0] = c_eq;
  cluster.sync();
  long long tie_base = 0;
  for (int c = 0; c < rank; ++c) tie_base += cluster.map_shared_rank(sh.exch, c)[0];
  long long ties_here = need_eq - tie_base;
  ties_here = ties_here < 0 ? 0 : (ties_here > c_eq ? c_eq : ties_here);

  // ---- exchange 2: kept count per CTA
  long long c_keep = ties_here;
  {
    long long v = 0;
    for (int i = threadIdx.x; i < m; i += kThreads) {
      const uint32_t key = key_at(i);
      v += (key == 0u) || (key > T);
    }
    c_keep += block_sum_ll(v, sh);
  }
  if (threadIdx.x == 0) sh.exch[1] = c_keep;
  cluster.sync();
  long long out_base = base, n_total = 0;
  for (int c = 0; c < kCluster; ++c) {
    const long long v = cluster.map_shared_rank(sh.exch, c)[1];
    if (c < rank) out_base += v;
    n_total += v;
  }
  if (!cu_seqlens && rank == 0 && threadIdx.x == 0) *n_kept = static_cast<int32_t>(n_total);
  if (cu_seqlens && rank == 0 && threadIdx.x == 0) {
    if (static_cast<long long>(cu_kept[seg + 1]) - base != n_total) tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
  }

  // ---- ordered compaction: tiles of kTile positions, kItems consecutive per thread
  long long tie_run = 0, keep_run = 0;
  for (int t0 = 0; t0 < m; t0 += kTile) {
    uint32_t kk[kItems];
    int n_tie = 0;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int i = t0 + threadIdx.x * kItems + j;
      kk[j] = i < m ? key_at(i) : 0xFFFFFFFFu;  // out-of-range marker: never kept, never a tie
      n_tie += (i < m) && (mode == 2) && (kk[j] == T);
    }
    int tie_tot = 0;
    const int tie_excl = block_exclusive_scan(n_tie, sh.warp_tot, &tie_tot);
    bool keep[kItems];
    int n_keep = 0;
    long long trank = tie_run + tie_excl;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int i = t0 + threadIdx.x * kItems + j;
      bool kp = false;
      if (i < m) {
        if (kk[j] == 0u || kk[j] > T) {
          kp = true;
        } else if (mode == 2 && kk[j] == T) {
          kp = (tie_base + trank) < need_eq;
          ++trank;
        }
      }
      keep[j] = kp;
      n_keep += kp;
    }
    int keep_tot = 0;
    const int keep_excl = block_exclusive_scan(n_keep, sh.warp_tot, &keep_tot);
    long long pos = out_base + keep_run + keep_excl;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      if (keep[j]) {
        if (pos < cap) {
          kept_idx[pos] = static_cast<int32_t>(lo + t0 + threadIdx.x * kItems + j);
        } else {
          tg::set_device_error(err, TG_DEVERR_CAPACITY);
        }
        ++pos;
      }
    }
    tie_run += tie_tot;
    keep_run += keep_tot;
  }
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

// Varlen pre-pass (one CTA): kept count of every request, min(k_b, n_doc_b) + question_b,
// then their prefix sums into cu_kept[0..B].  Also validates cu_seqlens.
__global__ void __launch_bounds__(1024) seg_offsets_kernel(const uint8_t *__restrict__ mask,
                                                           const int32_t *__restrict__ cu_seqlens, int32_t B,
                                                           int64_t total, const int32_t *__restrict__ k_per_seq,
                                                           int32_t *__restrict__ cu_kept, uint32_t *err) {
  __shared__ long long red[32];
  __shared__ long long run;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    run = 0;
    cu_kept[0] = 0;
  }
  __syncthreads();
  for (int b = 0; b < B; ++b) {
    int64_t s = cu_seqlens[b], e = cu_seqlens[b + 1];
    if (threadIdx.x == 0 && (s < 0 || e < s || e > total || (b == 0 && s != 0)))
      tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
    s = s < 0 ? 0 : (s > total ? total : s);
    e = e < s ? s : (e > total ? total : e);
    long long cnt = 0;
    for (int64_t i = s + threadIdx.x; i < e; i += blockDim.x) cnt += mask[i] != 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_down_sync(0xFFFFFFFFu, cnt, off);
    if (lane == 0) red[warp] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
      long long n_doc = 0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) n_doc += red[w];
      long long k = k_per_seq[b];
      if (k < 0) k = 0;
      const long long kept = (k < n_doc ? k : n_doc) + ((e - s) - n_doc);
      run += kept;
      cu_kept[b + 1] = static_cast<int32_t>(run);
    }
    __syncthreads();
  }
}

tg_status configure() {
  static bool done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(kKeyCap * sizeof(uint32_t)));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    done[dev] = true;
  }
  return TG_OK;
}

}  // namespace

extern "C" tg_status tg_select_topk(const float *scores, const uint8_t *doc_mask, int64_t n, int64_t k,
                                    int32_t *kept_idx, int64_t cap, int32_t *n_kept, tg_stream stream) {
  tg::clear_detail();
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (k < 0) return tg::fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  if (cap < 0) return tg::fail(TG_ERR_INVALID_ARG, "cap must be >= 0");
  if (!n_kept) return tg::fail(TG_ERR_INVALID_ARG, "n_kept is NULL");
  if (n > 0 && (!scores || !doc_mask)) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (cap > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  const int64_t chunk = (n + kCluster - 1) / kCluster;
  const int use_cache = chunk <= kKeyCap;
  const size_t smem = use_cache ? static_cast<size_t>(kKeyCap) * sizeof(uint32_t) : 0;
  tg_status st = configure();
  if (st != TG_OK) return st;
  topk_cluster_kernel<<<kCluster, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      scores, doc_mask, n, k, nullptr, nullptr, nullptr, n, kept_idx, cap, n_kept, use_cache, err);
  return tg::check_launch("topk_cluster_kernel");
}

extern "C" tg_status tg_select_topk_varlen(const float *scores, const uint8_t *doc_mask, const int32_t *cu_seqlens,
                                           int32_t B, int64_t total, const int32_t *k_per_seq, int64_t max_seqlen,
                                           int32_t *kept_idx, int64_t cap, int32_t *cu_kept, tg_stream stream) {
  tg::clear_detail();
  if (B < 0) return tg::fail(TG_ERR_INVALID_ARG, "B must be >= 0");
  if (total < 0 || total > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "total must be in [0, 2^31)");
  if (max_seqlen < 0 || max_seqlen > total) return tg::fail(TG_ERR_INVALID_ARG, "max_seqlen must be in [0, total]");
  if (cap < 0) return tg::fail(TG_ERR_INVALID_ARG, "cap must be >= 0");
  if (!cu_seqlens || !cu_kept || !k_per_seq) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (total > 0 && (!scores || !doc_mask)) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (cap > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  if (B > 65535) return tg::fail(TG_ERR_UNSUPPORTED, "B above 65535");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  seg_offsets_kernel<<<1, 1024, 0, s>>>(doc_mask, cu_seqlens, B, total, k_per_seq, cu_kept, err);
  tg_status st = tg::check_launch("seg_offsets_kernel");
  if (st != TG_OK || B == 0) return st;
  const int64_t chunk = (max_seqlen + kCluster - 1) / kCluster;
  const int use_cache = chunk <= kKeyCap;
  const size_t smem = use_cache ? static_cast<size_t>(kKeyCap) * sizeof(uint32_t) : 0;
  st = configure();
  if (st != TG_OK) return st;
  topk_cluster_kernel<<<static_cast<unsigned>(B) * kCluster, kThreads, smem, s>>>(
      scores, doc_mask, 0, 0, cu_seqlens, k_per_seq, cu_kept, total, kept_idx, cap, nullptr, use_cache, err);
  return tg::check_launch("topk_cluster_kernel");
}
