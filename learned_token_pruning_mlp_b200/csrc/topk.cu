// topk.cu -- tg_select_topk / tg_select_topk_varlen: keep the K best document
// tokens, always keep the question, output the kept positions in ascending order.
//
// TokenGate article, "How does TokenGate learned token pruning work?": a top-K
// selector keeps the highest-scoring tokens; only the document part of the prompt
// is prunable and the question is never pruned.  Order: score descending, ties to
// the lower index, -0.0 == +0.0, NaN below every number.
//
// B200 design: the work is memory-trivial (5 bytes a token), so the cost is
// latency.  One request is handled by one 8-CTA thread-block cluster of 1024
// threads each (a request of at most 8192 positions by one CTA alone, the same code
// with a cluster of one); every thread owns 16 consecutive positions (loaded with 16-byte
// vector loads) and keeps their 32-bit order keys in registers (131072 positions per
// cluster; longer requests re-derive the keys from the scores on every pass).  Up to
// three radix passes over 11-, 11- and 10-bit digits find the K-th largest key (each
// cluster barrier costs about a microsecond, so fewer, wider passes win: continuous
// scores resolve after two): each CTA builds a shared-memory histogram of the
// remaining candidates, one cluster barrier publishes it, the CTA's threads sum the
// eight CTAs' histograms through distributed shared memory and one warp scans the
// totals, so every CTA agrees on the digit without touching global memory.  A pass
// whose chosen bin holds exactly the keys still needed ends the search early.
// Histograms alternate between two buffers, so one barrier per pass suffices.  When
// the first digit's histogram comes precomputed (tg_select_fused: the gate's epilogue
// counts the top 8 bits), the passes use four 8-bit digits instead.  The ordered
// compaction needs one scan of packed (tie, keep) counts per CTA and one exchange of the
// per-CTA totals.  No workspace, no global atomics, one launch for a single request.
#include <cooperative_groups.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "runtime.h"
#include "select_key.cuh"

namespace cg = cooperative_groups;

namespace {

constexpr int kCluster = 8;                       // CTAs per request above kRound positions
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kItems = 16;                        // consecutive positions per thread
constexpr int kRound = kThreads * kItems;         // positions per CTA per round (16384)
constexpr int kBins = 2048;                       // up to 11-bit digits
constexpr int kPassBins8 = 256;                   // the precomputed first digit: 8 bits
constexpr int kCoarse = 256;                      // coarse bins of the two-level digit search

using tg::order_key;

struct TopkShared {
  uint32_t hist[2][kBins];     // double-buffered per-CTA histograms (read by the cluster)
  uint32_t coarse[2][kCoarse]; // the same histograms folded to 256 coarse bins (read by the cluster)
  uint32_t fine[kBins / kCoarse];  // cluster totals of the chosen coarse bin's fine bins
  uint32_t wsum[kWarps + 1];
  uint32_t sel_digit, sel_above, sel_count, sel_cbin;
  long long exch[2];           // ties (key == T) and certain keeps of this CTA: read by the cluster
  long long bcast[2];          // tie_base, out_base
};

// Block-wide exclusive prefix sum of one value per thread (thread order = index order).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, TopkShared &sh, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) sh.wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = sh.wsum[lane];
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += t;
    }
    sh.wsum[lane] = wi - w;
    if (lane == 31) sh.wsum[kWarps] = wi;
  }
  __syncthreads();
  const uint32_t res = sh.wsum[warp] + incl - v;
  *total = sh.wsum[kWarps];
  return res;
}

// Fold this CTA's histogram of buffer ``buf`` (nbins bins) into 256 coarse bins, g =
// nbins / 256 consecutive bins each (a copy when g = 1).  Runs before the cluster
// barrier that publishes the histograms, so the cluster reads the folded bins.
__device__ __forceinline__ void fold_coarse(TopkShared &sh, int buf, int nbins) {
  const int g = nbins / kCoarse;
  if (threadIdx.x < kCoarse) {
    uint32_t c = 0;
    for (int j = 0; j < g; ++j) c += sh.hist[buf][threadIdx.x * g + j];
    sh.coarse[buf][threadIdx.x] = c;
  }
}

// Find the digit of the remaining-th largest candidate over the whole cluster, in two
// levels so that few distributed-shared-memory reads are needed: the 256 coarse totals
// (8 remote reads by each of 256 threads) locate the coarse bin, then the g fine bins
// of that coarse bin are summed over the eight CTAs.  Publishes sel_digit, sel_above
// (candidates in higher bins) and sel_count (candidates in the chosen bin);
// sel_digit = nbins if none qualifies.  The total lands in wsum[kWarps].
template <int kC>
__device__ __forceinline__ void cluster_select_digit(cg::cluster_group &cluster, TopkShared &sh, int buf,
                                                     int nbins, uint32_t remaining) {
  const int g = nbins / kCoarse;
  const int t = static_cast<int>(threadIdx.x);
  const int cb = kCoarse - 1 - t;  // coarse bins from the top, one per thread of the first 256
  uint32_t cnt = 0;
  if (t < kCoarse) {
#pragma unroll
    for (int r = 0; r < kC; ++r) cnt += cluster.map_shared_rank(&sh.coarse[buf][0], r)[cb];
  }
  if (t == 0) sh.sel_digit = nbins;  // ordered before the writes below by the scan's barriers
  uint32_t total;
  const uint32_t excl = block_excl_scan(cnt, sh, &total);
  if (t < kCoarse && remaining > 0 && excl < remaining && remaining <= excl + cnt) {
    sh.sel_cbin = static_cast<uint32_t>(cb);
    sh.sel_above = excl;
    sh.sel_count = cnt;
    if (g == 1) sh.sel_digit = static_cast<uint32_t>(cb);
  }
  __syncthreads();
  if (g == 1 || sh.sel_digit != static_cast<uint32_t>(nbins) || remaining == 0 || remaining > total) return;
  // the fine bins of the chosen coarse bin: lane group j (kC lanes, one per CTA) sums
  // fine bin cbin * g + g - 1 - j
  const uint32_t cbin = sh.sel_cbin;
  if (t < kC * g) {
    const int j = t / kC, r = t % kC;
    uint32_t c = cluster.map_shared_rank(&sh.hist[buf][0], r)[cbin * g + g - 1 - j];
#pragma unroll
    for (int off = kC / 2; off > 0; off >>= 1) c += __shfl_down_sync(0xFFFFFFFFu, c, off, kC);
    if (r == 0) sh.fine[j] = c;
  }
  __syncthreads();
  if (t == 0) {
    uint32_t run = sh.sel_above;
    for (int j = 0; j < g; ++j) {
      const uint32_t c = sh.fine[j];
      if (run + c >= remaining) {
        sh.sel_digit = cbin * g + g - 1 - j;
        sh.sel_above = run;
        sh.sel_count = c;
        break;
      }
      run += c;
    }
  }
  __syncthreads();
}

// Everything one launch of the cluster kernel needs (passed by value).
struct TopkArgs {
  const float *scores;        // nullptr in random mode
  const uint8_t *mask;
  int64_t n_single;           // single / sweep: the request is [0, n_single)
  int64_t k_single;           // single: the budget
  const int32_t *cu_seqlens;  // varlen: request b = [cu_seqlens[b], cu_seqlens[b+1])
  const int32_t *k_per_seq;   // varlen: budgets
  const int32_t *cu_kept;     // varlen: output offsets (from seg_offsets_kernel)
  int64_t total;              // varlen: packed length
  const int32_t *k_sweep;     // sweep: cluster b selects with budget k_sweep[b]
  int64_t sweep_stride;       // sweep: cluster b writes kept_idx[b * stride ...]
  int32_t *kept_idx;
  int64_t cap;                // capacity per request (per budget in sweep mode)
  int32_t *n_kept;            // single: [1]; sweep: [number of budgets]
  uint64_t seed;              // random mode: key = SplitMix64(seed, position)
  int random;
  const uint32_t *hist_parts; // single mode: n_parts histograms of the keys' top byte (pass 0)
  int n_parts;
  uint32_t *err;
};

// SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
// OOPSLA 2014): the state after n steps from ``seed`` is seed + n * golden gamma, and
// the output mixes it with two multiply-xorshift rounds.  Counter-based, so any
// position's value is computed directly.
__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t index) {
  uint64_t z = seed + (index + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Random-mode order key of a document token: 31 random bits above every number key,
// so the "largest" K keys are a uniformly random K-subset (ties by position).
__device__ __forceinline__ uint32_t random_key(uint64_t seed, int64_t pos, bool doc) {
  return doc ? (0x80000000u | static_cast<uint32_t>(splitmix64(seed, static_cast<uint64_t>(pos)) >> 33)) : 0u;
}

// One cluster per request.  Single-request mode: the request is [0, n_single) with
// budget k_single, base 0, and the CTA of rank 0 writes *n_kept.  Varlen mode: request
// b = cluster index, range from cu_seqlens, budget k_per_seq[b], output offset
// cu_kept[b] (computed beforehand by seg_offsets_kernel).  Sweep mode: every cluster
// selects from [0, n_single) with its own budget k_sweep[b] into its own output block.
// kResident: every CTA's chunk fits one round (<= 16384 positions), keys stay in
// registers; otherwise the keys are re-derived from the scores on every pass.
// kC: CTAs per cluster, 8, or 1 when a request fits one CTA's registers (no cluster
// barrier or distributed-shared-memory read is then paid).
template <bool kResident, int kC>
__global__ void __cluster_dims__(kC, 1, 1) __launch_bounds__(kThreads, 1)
    topk_cluster_kernel(const TopkArgs args) {
  __shared__ TopkShared sh;
  tg::pdl_wait();
  tg::pdl_trigger();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int seg = static_cast<int>(blockIdx.x) / kC;
  const float *__restrict__ scores = args.scores;
  const uint8_t *__restrict__ mask = args.mask;
  const int32_t *__restrict__ cu_seqlens = args.cu_seqlens;
  const int32_t *__restrict__ cu_kept = args.cu_kept;
  int32_t *__restrict__ kept_idx = args.kept_idx;
  uint32_t *err = args.err;
  const int64_t cap = args.cap;
  const int64_t total = args.total;

  int64_t start = 0, end = args.n_single, k = args.k_single, base = 0;
  if (cu_seqlens) {
    start = cu_seqlens[seg];
    end = cu_seqlens[seg + 1];
    start = start < 0 ? 0 : (start > total ? total : start);
    end = end < start ? start : (end > total ? total : end);
    k = args.k_per_seq[seg];
    base = cu_kept[seg];
  } else if (args.k_sweep) {
    k = args.k_sweep[seg];
    base = static_cast<int64_t>(seg) * args.sweep_stride;
  }
  const int64_t cap_end = args.k_sweep ? base + cap : cap;  // writes go below cap_end
  if (k < 0) k = 0;
  const int64_t len = end - start;
  // chunk: a multiple of kItems so that a thread's positions never straddle two CTAs
  const int64_t chunk = ((len + kC - 1) / kC + kItems - 1) / kItems * kItems;
  const int64_t lo = start + chunk * rank;
  const int64_t hi = lo + chunk < end ? lo + chunk : end;
  const int m = lo < hi ? static_cast<int>(hi - lo) : 0;
  const int rounds = kResident ? 1 : (m + kRound - 1) / kRound;
  // the launcher picks the register-resident variant from the caller's length bound; a
  // request longer than that bound cannot be handled by it and is reported
  if (kResident && m > kRound && threadIdx.x == 0) tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);

  // 16-byte vector loads when this CTA's chunk starts aligned (always for a single request
  // with aligned buffers; varlen requests may start anywhere and then use scalar loads)
  const bool vec = !args.random &&
                   ((reinterpret_cast<uintptr_t>(scores + lo) | reinterpret_cast<uintptr_t>(mask + lo)) & 15u) == 0;
  uint32_t keys[kItems];
  // positions past the chunk get key 0 and are excluded from every count by valid()
  auto load_keys = [&](int round) {
    const int i0 = round * kRound + threadIdx.x * kItems;
    if (args.random) {
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        const int i = i0 + e;
        keys[e] = i < m ? random_key(args.seed, lo + i, mask[lo + i] != 0) : 0u;
      }
    } else if (vec && i0 + kItems <= m) {
      float f[kItems];
      const float4 *s4 = reinterpret_cast<const float4 *>(scores + lo + i0);
#pragma unroll
      for (int q = 0; q < kItems / 4; ++q) {
        const float4 v = __ldg(s4 + q);
        f[4 * q] = v.x;
        f[4 * q + 1] = v.y;
        f[4 * q + 2] = v.z;
        f[4 * q + 3] = v.w;
      }
      const uint4 mv = __ldg(reinterpret_cast<const uint4 *>(mask + lo + i0));
      const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
      for (int e = 0; e < kItems; ++e) keys[e] = order_key(f[e], ((mw[e >> 2] >> (8 * (e & 3))) & 0xFFu) != 0);
    } else {
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        const int i = i0 + e;
        keys[e] = i < m ? order_key(scores[lo + i], mask[lo + i] != 0) : 0u;
      }
    }
  };
  auto valid = [&](int round, int e) { return round * kRound + static_cast<int>(threadIdx.x) * kItems + e < m; };

  if (kResident) load_keys(0);
  for (int i = threadIdx.x; i < 2 * kBins; i += kThreads) (&sh.hist[0][0])[i] = 0;
  __syncthreads();

  // ---- radix passes, most significant digit first: 11, 11 and 10 bits, or four 8-bit
  // digits when the first digit's histogram is precomputed.  Pass p histograms the
  // candidates (document keys whose higher digits equal the prefix found so far).
  const bool digits8 = args.hist_parts != nullptr;
  const int n_pass = digits8 ? 4 : 3;
  uint32_t prefix = 0, pmask = 0;
  uint32_t remaining = static_cast<uint32_t>(k < 0x7FFFFFFFLL ? k : 0x7FFFFFFFLL);
  long long n_doc = 0;
  int mode = 2;          // 0 = keep no document token, 1 = keep all, 2 = threshold
  uint32_t T = 0u;       // keep key > T, plus the first need_eq keys == T in index order
  long long need_eq = 0;
  for (int pass = 0; pass < n_pass; ++pass) {
    const int buf = pass & 1;
    const int width = digits8 ? 8 : (pass < 2 ? 11 : 10);
    const int shift = digits8 ? 24 - 8 * pass : (pass == 0 ? 21 : (pass == 1 ? 10 : 0));
    const int nbins = 1 << width;
    const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
    if (pass >= 2) {
      // this buffer was read by every CTA before the cluster barrier of the previous pass
      for (int i = threadIdx.x; i < nbins; i += kThreads) sh.hist[buf][i] = 0;
      __syncthreads();
    }
    if (pass == 0 && digits8) {
      // the first digit's histogram was built by the producer of the scores: sum this
      // CTA's share of its partial histograms (the cluster reduction adds the shares)
      if (threadIdx.x < kPassBins8) {
        uint32_t c = 0;
        for (int p = rank; p < args.n_parts; p += kC)
          c += __ldg(args.hist_parts + p * kPassBins8 + threadIdx.x);
        sh.hist[0][threadIdx.x] = c;
      }
    } else {
      for (int rd = 0; rd < rounds; ++rd) {
        if (!kResident) load_keys(rd);
#pragma unroll
        for (int e = 0; e < kItems; ++e)
          if (keys[e] != 0u && (keys[e] & pmask) == prefix) atomicAdd(&sh.hist[buf][(keys[e] >> shift) & dmask], 1u);
      }
    }
    __syncthreads();
    fold_coarse(sh, buf, nbins);
    __syncthreads();
    cluster.sync();
    cluster_select_digit<kC>(cluster, sh, buf, nbins, remaining);
    if (pass == 0) {
      n_doc = sh.wsum[kWarps];
      if (k > n_doc && rank == 0 && threadIdx.x == 0) tg::set_device_error(err, TG_DEVERR_K_GT_NDOC);
      if (k == 0 || n_doc == 0) { mode = 0; T = 0xFFFFFFFFu; break; }
      if (k >= n_doc) { mode = 1; T = 0u; break; }
    }
    const uint32_t d = sh.sel_digit;
    const uint32_t above = sh.sel_above, cnt = sh.sel_count;
    prefix |= d << shift;
    pmask |= dmask << shift;
    remaining -= above;
    if (cnt == remaining) {
      // every candidate of this bin is kept: threshold just below the bin
      T = prefix ? prefix - 1u : 0u;  // (prefix = 0 would mean every document key is kept)
      need_eq = 0;
      break;
    }
    if (pass == n_pass - 1) {
      T = prefix;
      need_eq = remaining;
    }
  }
  if (mode == 0) need_eq = 0;

  // ---- per-thread counts: ties (key == T, threshold mode only) and certain keeps
  // (question tokens and keys > T), kept as 16-bit masks of the thread's positions.
  // Within one round a CTA holds at most 16384 positions, so the two counts pack into
  // one 32-bit value and one block scan gives both prefixes.
  auto classify = [&](int rd, uint32_t &tie_bits, uint32_t &keep_bits) {
    tie_bits = 0;
    keep_bits = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      const bool v = valid(rd, e);
      tie_bits |= static_cast<uint32_t>(v && mode == 2 && keys[e] == T) << e;
      keep_bits |= static_cast<uint32_t>(v && (keys[e] == 0u || keys[e] > T)) << e;
    }
  };
  uint32_t tie_bits0 = 0, keep_bits0 = 0, excl0 = 0, tot0 = 0;
  long long cta_eq = 0, cta_gtq = 0;
  if (kResident) {
    classify(0, tie_bits0, keep_bits0);
    excl0 = block_excl_scan((static_cast<uint32_t>(__popc(tie_bits0)) << 16) | __popc(keep_bits0), sh, &tot0);
    cta_eq = tot0 >> 16;
    cta_gtq = tot0 & 0xFFFFu;
  } else {
    for (int rd = 0; rd < rounds; ++rd) {
      load_keys(rd);
      uint32_t tb, kb, t;
      classify(rd, tb, kb);
      block_excl_scan((static_cast<uint32_t>(__popc(tb)) << 16) | __popc(kb), sh, &t);
      cta_eq += t >> 16;
      cta_gtq += t & 0xFFFFu;
      __syncthreads();  // the next scan reuses the scan buffer
    }
  }
  if (threadIdx.x == 0) {
    sh.exch[0] = cta_eq;
    sh.exch[1] = cta_gtq;
  }
  cluster.sync();
  if (threadIdx.x < 32) {
    // lane r < 8 reads CTA r's counts; the prefixes over CTAs come from warp shuffles
    const int lane = threadIdx.x;
    long long eq = 0, gtq = 0;
    if (lane < kC) {
      const long long *x = cluster.map_shared_rank(&sh.exch[0], lane);
      eq = x[0];
      gtq = x[1];
    }
    long long eq_incl = eq;
#pragma unroll
    for (int off = 1; off < kC; off <<= 1) {
      const long long t = __shfl_up_sync(0xFFFFFFFFu, eq_incl, off);
      if (lane >= off) eq_incl += t;
    }
    const long long tb = eq_incl - eq;  // ties in CTAs before this lane's CTA
    long long th = need_eq - tb;
    th = th < 0 ? 0 : (th > eq ? eq : th);
    const long long keep = lane < kC ? gtq + th : 0;
    long long keep_incl = keep;
#pragma unroll
    for (int off = 1; off < kC; off <<= 1) {
      const long long t = __shfl_up_sync(0xFFFFFFFFu, keep_incl, off);
      if (lane >= off) keep_incl += t;
    }
    const long long nt = __shfl_sync(0xFFFFFFFFu, keep_incl, kC - 1);
    if (lane == rank) {
      sh.bcast[0] = tb;
      sh.bcast[1] = base + keep_incl - keep;
    }
    if (lane == 0) {
      if (!cu_seqlens && rank == 0) args.n_kept[args.k_sweep ? seg : 0] = static_cast<int32_t>(nt);
      if (cu_seqlens && rank == 0 && static_cast<long long>(cu_kept[seg + 1]) - base != nt)
        tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
    }
  }
  // the last reads of another CTA's shared memory are done: arrive on the cluster
  // barrier now and wait for the others only before leaving (a CTA's shared memory must
  // stay until every reader is through), so the compaction overlaps the barrier
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  __syncthreads();
  const long long tie_base = sh.bcast[0], out_base = sh.bcast[1];

  // ---- ordered compaction.  The ties this CTA keeps are its first ``quota`` ties, so
  // the kept ties before a thread are min(ties before it, quota).
  long long quota = need_eq - tie_base;
  quota = quota < 0 ? 0 : quota;
  long long run_tie = 0, run_gtq = 0;
  for (int rd = 0; rd < rounds; ++rd) {
    uint32_t x = excl0, rt = tot0, tie_bits = tie_bits0, keep_bits = keep_bits0;
    if (!kResident) {
      load_keys(rd);
      classify(rd, tie_bits, keep_bits);
      x = block_excl_scan((static_cast<uint32_t>(__popc(tie_bits)) << 16) | __popc(keep_bits), sh, &rt);
    }
    // kept ties of this thread: the first (quota - ties before it) of its tie positions
    const long long tbefore = run_tie + (x >> 16);
    long long allow = quota - tbefore;
    allow = allow < 0 ? 0 : (allow > 16 ? 16 : allow);
    uint32_t tb = 0, rem = tie_bits;
    for (long long c = 0; c < allow && rem; ++c) {  // keep the lowest ``allow`` tie positions
      tb |= rem & (~rem + 1u);
      rem &= rem - 1u;
    }
    const uint32_t out_bits = keep_bits | tb;
    long long pos = out_base + run_gtq + (x & 0xFFFFu) + (tbefore < quota ? tbefore : quota);
    const int64_t p0 = lo + static_cast<int64_t>(rd) * kRound + static_cast<int64_t>(threadIdx.x) * kItems;
    uint32_t bits = out_bits;
    while (bits) {
      const int e = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < cap_end) {
        kept_idx[pos] = static_cast<int32_t>(p0 + e);
      } else {
        tg::set_device_error(err, TG_DEVERR_CAPACITY);
      }
      ++pos;
    }
    run_tie += rt >> 16;
    run_gtq += rt & 0xFFFFu;
    if (!kResident) __syncthreads();  // the next round's scan reuses the scan buffer
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // every CTA is past its remote reads
}

// Varlen pre-pass (one CTA of 1024 threads): the kept count of every request,
// min(k_b, n_doc_b) + question_b, and their prefix sums into cu_kept[0..B]; it also
// validates cu_seqlens.  For a well-formed batch of at most kSegFast requests one pass
// over the mask suffices: each thread counts the document tokens of a contiguous run of
// 16-byte words (the mask's address decides where whole words start; the bytes before
// and after them are counted singly) and records, for every request boundary inside its
// run, the count up to that boundary; a block scan of the run counts turns those into
// the number of document tokens before every boundary, and the differences of
// consecutive boundaries are the requests' document counts.  A malformed or larger batch
// takes one request at a time.
constexpr int kSegFast = 4096;

__device__ __forceinline__ uint32_t doc_bytes(uint32_t w) { return __popc(__vcmpne4(w, 0u)) >> 3; }
__device__ __forceinline__ uint32_t doc_bytes(const uint4 &v) {
  return doc_bytes(v.x) + doc_bytes(v.y) + doc_bytes(v.z) + doc_bytes(v.w);
}
// document bytes among the first n (0..16) bytes of a 16-byte word
__device__ __forceinline__ uint32_t doc_bytes_prefix(const uint4 &v, int n) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = n - 4 * q;  // bytes of this 32-bit lane to count
    const uint32_t keep = k >= 4 ? 0xFFFFFFFFu : (k <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * k)));
    c += doc_bytes(w[q] & keep);
  }
  return c;
}

// exclusive scan over the 1024 threads of the block (32 warps); *total gets the sum
__device__ __forceinline__ uint32_t seg_excl_scan(uint32_t v, uint32_t *wsum, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = wsum[lane];
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += u;
    }
    wsum[lane] = wi - w;
    if (lane == 31) wsum[32] = wi;
  }
  __syncthreads();
  const uint32_t res = wsum[warp] + incl - v;
  *total = wsum[32];
  __syncthreads();  // wsum may be reused by the next scan
  return res;
}

__global__ void __launch_bounds__(1024) seg_offsets_kernel(const uint8_t *__restrict__ mask,
                                                           const int32_t *__restrict__ cu_seqlens, int32_t B,
                                                           int64_t total, const int32_t *__restrict__ k_per_seq,
                                                           int32_t *__restrict__ cu_kept, uint32_t *err) {
  __shared__ int32_t s_cu[kSegFast + 1];
  __shared__ uint32_t s_pre[kSegFast + 1];  // document tokens before each boundary
  __shared__ uint32_t wsum[33];
  __shared__ uint32_t s_head;
  tg::pdl_wait();
  tg::pdl_trigger();
  const int t = static_cast<int>(threadIdx.x);
  const int nt = static_cast<int>(blockDim.x);
  const int lane = t & 31, warp = t >> 5;

  bool bad = false;
  for (int b = t; b < B; b += nt) {
    const int64_t s = cu_seqlens[b], e = cu_seqlens[b + 1];
    bad = bad || s < 0 || e < s || e > total || (b == 0 && s != 0);
  }
  if (bad) tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
  if (t == 0) cu_kept[0] = 0;
  if (B == 0) return;  // uniform over the block
  if (__syncthreads_or(bad) || B > kSegFast) {
    // one request at a time (ranges clamped into [0, total])
    __shared__ long long red[32];
    __shared__ long long run;
    if (t == 0) run = 0;
    __syncthreads();
    for (int b = 0; b < B; ++b) {
      int64_t s = cu_seqlens[b], e = cu_seqlens[b + 1];
      s = s < 0 ? 0 : (s > total ? total : s);
      e = e < s ? s : (e > total ? total : e);
      // whole 16-byte words where the mask's address is aligned, single bytes around them
      const int64_t a0 = s + static_cast<int64_t>((16u - (reinterpret_cast<uintptr_t>(mask + s) & 15u)) & 15u);
      long long cnt = 0;
      if (a0 + 16 <= e) {
        const int64_t nw = (e - a0) >> 4, a1 = a0 + 16 * nw;
        const uint4 *w = reinterpret_cast<const uint4 *>(mask + a0);
        for (int64_t q = t; q < nw; q += nt) cnt += doc_bytes(__ldg(w + q));
        for (int64_t i = s + t; i < a0; i += nt) cnt += mask[i] != 0;
        for (int64_t i = a1 + t; i < e; i += nt) cnt += mask[i] != 0;
      } else {
        for (int64_t i = s + t; i < e; i += nt) cnt += mask[i] != 0;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cnt += __shfl_down_sync(0xFFFFFFFFu, cnt, off);
      if (lane == 0) red[warp] = cnt;
      __syncthreads();
      if (t == 0) {
        long long n_doc = 0;
        for (int w = 0; w < nt / 32; ++w) n_doc += red[w];
        long long k = k_per_seq[b];
        if (k < 0) k = 0;
        run += (k < n_doc ? k : n_doc) + ((e - s) - n_doc);
        cu_kept[b + 1] = static_cast<int32_t>(run);
      }
      __syncthreads();
    }
    return;
  }

  // ---- one pass: requests cover [0, E), well formed
  for (int b = t; b <= B; b += nt) s_cu[b] = cu_seqlens[b];
  __syncthreads();
  const int64_t E = s_cu[B];
  const int64_t a_mis = static_cast<int64_t>((16u - (reinterpret_cast<uintptr_t>(mask) & 15u)) & 15u);
  const int64_t A0 = a_mis < E ? a_mis : E;  // whole words start where the mask's address is aligned
  const int64_t nw = (E - A0) >> 4, A1 = A0 + 16 * nw;
  if (warp == 0) {
    const bool d = lane < A0 && mask[lane] != 0;
    const uint32_t h = __popc(__ballot_sync(0xFFFFFFFFu, d));
    if (lane == 0) s_head = h;
  }
  // this thread's run of words and the boundaries inside it
  const int64_t per = (nw + nt - 1) / nt;
  const int64_t w0 = static_cast<int64_t>(t) * per < nw ? static_cast<int64_t>(t) * per : nw;
  const int64_t w1 = w0 + per < nw ? w0 + per : nw;
  int b_first = B + 1;
  {
    int lo = 0, hi = B + 1;  // first boundary >= the run's first position
    const int64_t p0 = A0 + 16 * w0;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s_cu[mid] < p0) lo = mid + 1;
      else hi = mid;
    }
    b_first = lo;
  }
  int b_end = b_first;
  uint32_t local = 0;
  const uint4 *mw = reinterpret_cast<const uint4 *>(mask + A0);
  // eight loads in flight at a time (the run's words are independent)
  for (int64_t wb = w0; wb < w1; wb += 8) {
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = wb + i < w1 ? __ldg(mw + wb + i) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (wb + i >= w1) break;
      const int64_t ws = A0 + 16 * (wb + i);
      while (b_end <= B && s_cu[b_end] < ws + 16) {
        s_pre[b_end] = local + doc_bytes_prefix(v[i], static_cast<int>(s_cu[b_end] - ws));
        ++b_end;
      }
      local += doc_bytes(v[i]);
    }
  }
  uint32_t words_total;
  const uint32_t before = seg_excl_scan(local, wsum, &words_total);
  const uint32_t head = s_head;
  for (int b = b_first; b < b_end; ++b) s_pre[b] += head + before;
  // boundaries before the first whole word or at / after the end of the last one
  for (int b = t; b <= B; b += nt) {
    const int64_t x = s_cu[b];
    if (x < A0 || x >= A1) {
      uint32_t c = 0;
      if (x < A0) {
        for (int64_t i = 0; i < x; ++i) c += mask[i] != 0;
      } else {
        c = head + words_total;
        for (int64_t i = A1; i < x; ++i) c += mask[i] != 0;
      }
      s_pre[b] = c;
    }
  }
  __syncthreads();
  // kept counts of four consecutive requests per thread, then their prefix sums
  uint32_t kept[4], sum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int b = 4 * t + q;
    kept[q] = 0;
    if (b < B) {
      const uint32_t n_doc = s_pre[b + 1] - s_pre[b];
      const uint32_t len = static_cast<uint32_t>(s_cu[b + 1] - s_cu[b]);
      const int32_t kb = k_per_seq[b];
      const uint32_t k = kb < 0 ? 0u : static_cast<uint32_t>(kb);
      kept[q] = (k < n_doc ? k : n_doc) + (len - n_doc);
    }
    sum += kept[q];
  }
  uint32_t all;
  uint32_t run = seg_excl_scan(sum, wsum, &all);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int b = 4 * t + q;
    run += kept[q];
    if (b < B) cu_kept[b + 1] = static_cast<int32_t>(run);
  }
}

// CTAs per request for requests of at most ``len`` positions: one for up to half a
// CTA's register tile (measured: 4096 positions 11.5 us against 12.5 us in a cluster,
// 16384 positions 13.1 us against 12.6 us), else a cluster of kCluster
constexpr int64_t kLoneCta = kRound / 2;
int cluster_for(int64_t len) { return len <= kLoneCta ? 1 : kCluster; }

// chunk per CTA for a request of ``len`` positions in clusters of kc CTAs (as the kernel
// computes it)
int64_t chunk_of(int64_t len, int kc) { return ((len + kc - 1) / kc + kItems - 1) / kItems * kItems; }

// ``n_seg`` clusters (requests, or budgets in sweep mode) of cluster_for(len_bound) CTAs
cudaError_t launch_cluster(int64_t len_bound, unsigned n_seg, cudaStream_t s, const TopkArgs &a) {
  const int kc = cluster_for(len_bound);
  const bool resident = chunk_of(len_bound, kc) <= kRound;
  const dim3 grid(n_seg * static_cast<unsigned>(kc));
  // a lone CTA always holds its request in registers (len_bound <= kLoneCta < kRound)
  if (kc == 1) return tg::launch_pdl(topk_cluster_kernel<true, 1>, grid, dim3(kThreads), 0, s, a);
  if (resident) return tg::launch_pdl(topk_cluster_kernel<true, kCluster>, grid, dim3(kThreads), 0, s, a);
  return tg::launch_pdl(topk_cluster_kernel<false, kCluster>, grid, dim3(kThreads), 0, s, a);
}

}  // namespace

extern "C" tg_status tg_select_topk(const float *scores, const uint8_t *doc_mask, int64_t n, int64_t k,
                                    int32_t *kept_idx, int64_t cap, int32_t *n_kept, tg_stream stream) {
  TG_API_ENTRY();
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (k < 0) return tg::fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  if (cap < 0) return tg::fail(TG_ERR_INVALID_ARG, "cap must be >= 0");
  if (!n_kept) return tg::fail(TG_ERR_INVALID_ARG, "n_kept is NULL");
  if (n > 0 && (!scores || !doc_mask)) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (cap > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  TopkArgs a = {};
  a.scores = scores;
  a.mask = doc_mask;
  a.n_single = n;
  a.k_single = k;
  a.total = n;
  a.kept_idx = kept_idx;
  a.cap = cap;
  a.n_kept = n_kept;
  a.err = err;
  const cudaError_t e = launch_cluster(n, 1, static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "topk_cluster_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("topk_cluster_kernel");
}

tg_status tg::select_topk_hist(const float *scores, const uint8_t *doc_mask, int64_t n, int64_t k, int32_t *kept_idx,
                               int64_t cap, int32_t *n_kept, const uint32_t *hist_parts, int n_parts,
                               tg_stream stream) {
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (k < 0) return tg::fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  if (cap < 0) return tg::fail(TG_ERR_INVALID_ARG, "cap must be >= 0");
  if (!n_kept) return tg::fail(TG_ERR_INVALID_ARG, "n_kept is NULL");
  if (n > 0 && (!scores || !doc_mask)) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (cap > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  if (n > 0 && (!hist_parts || n_parts <= 0)) return tg::fail(TG_ERR_INVALID_ARG, "no first-pass histograms");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  TopkArgs a = {};
  a.scores = scores;
  a.mask = doc_mask;
  a.n_single = n;
  a.k_single = k;
  a.total = n;
  a.kept_idx = kept_idx;
  a.cap = cap;
  a.n_kept = n_kept;
  a.hist_parts = hist_parts;
  a.n_parts = n_parts;
  a.err = err;
  const cudaError_t e = launch_cluster(n, 1, static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "topk_cluster_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("topk_cluster_kernel");
}

extern "C" tg_status tg_select_random_k(const uint8_t *doc_mask, int64_t n, int64_t k, uint64_t seed,
                                        int32_t *kept_idx, int64_t cap, int32_t *n_kept, tg_stream stream) {
  TG_API_ENTRY();
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (k < 0) return tg::fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  if (cap < 0) return tg::fail(TG_ERR_INVALID_ARG, "cap must be >= 0");
  if (!n_kept) return tg::fail(TG_ERR_INVALID_ARG, "n_kept is NULL");
  if (n > 0 && !doc_mask) return tg::fail(TG_ERR_INVALID_ARG, "doc_mask is NULL");
  if (cap > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  TopkArgs a = {};
  a.mask = doc_mask;
  a.n_single = n;
  a.k_single = k;
  a.total = n;
  a.kept_idx = kept_idx;
  a.cap = cap;
  a.n_kept = n_kept;
  a.seed = seed;
  a.random = 1;
  a.err = err;
  const cudaError_t e = launch_cluster(n, 1, static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "topk_cluster_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("topk_cluster_kernel");
}

extern "C" tg_status tg_select_topk_sweep(const float *scores, const uint8_t *doc_mask, int64_t n,
                                          const int32_t *ks, int32_t m, int32_t *kept_idx, int64_t stride,
                                          int32_t *n_kept, tg_stream stream) {
  TG_API_ENTRY();
  if (n < 0 || n > 0x7FFFFFFFLL) return tg::fail(TG_ERR_INVALID_ARG, "n must be in [0, 2^31) (got %lld)", (long long)n);
  if (m < 0 || m > 65535) return tg::fail(TG_ERR_INVALID_ARG, "the number of budgets must be in [0, 65535]");
  if (stride < 0 || (m > 0 && stride > 0x7FFFFFFFLL / m))
    return tg::fail(TG_ERR_INVALID_ARG, "stride must be >= 0 and m * stride < 2^31");
  if (m == 0) return TG_OK;
  if (!ks || !n_kept) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (n > 0 && (!scores || !doc_mask)) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (stride > 0 && !kept_idx) return tg::fail(TG_ERR_INVALID_ARG, "kept_idx is NULL");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  TopkArgs a = {};
  a.scores = scores;
  a.mask = doc_mask;
  a.n_single = n;
  a.total = n;
  a.k_sweep = ks;
  a.sweep_stride = stride;
  a.kept_idx = kept_idx;
  a.cap = stride;
  a.n_kept = n_kept;
  a.err = err;
  const cudaError_t e =
      launch_cluster(n, static_cast<unsigned>(m), static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "topk_cluster_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("topk_cluster_kernel");
}

extern "C" tg_status tg_select_topk_varlen(const float *scores, const uint8_t *doc_mask, const int32_t *cu_seqlens,
                                           int32_t B, int64_t total, const int32_t *k_per_seq, int64_t max_seqlen,
                                           int32_t *kept_idx, int64_t cap, int32_t *cu_kept, tg_stream stream) {
  TG_API_ENTRY();
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
  cudaError_t e = tg::launch_pdl(seg_offsets_kernel, dim3(1), dim3(1024), 0, s, doc_mask, cu_seqlens, B, total,
                                 k_per_seq, cu_kept, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "seg_offsets_kernel launch: %s", cudaGetErrorString(e));
  tg_status st = tg::check_launch("seg_offsets_kernel");
  if (st != TG_OK || B == 0) return st;
  TopkArgs a = {};
  a.scores = scores;
  a.mask = doc_mask;
  a.cu_seqlens = cu_seqlens;
  a.k_per_seq = k_per_seq;
  a.cu_kept = cu_kept;
  a.total = total;
  a.kept_idx = kept_idx;
  a.cap = cap;
  a.err = err;
  // the register-resident variant is chosen when max_seqlen fits it; a request longer
  // than max_seqlen then sets TG_DEVERR_BAD_SEQLENS
  e = launch_cluster(max_seqlen, static_cast<unsigned>(B), s, a);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "topk_cluster_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("topk_cluster_kernel");
}
