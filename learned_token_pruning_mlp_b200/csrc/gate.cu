// gate.cu -- tg_gate_score: the MLP gate that scores every prompt token.
//
// TokenGate article, "How does TokenGate learned token pruning work?" (gate
// module): a small MLP scores each token from its post-attention residual at the
// gate layer.  Scorer: Linear(d -> h), SiLU, Linear(h -> 1):
//     s_i = b2 + sum_j W2_j * SiLU(b1_j + W1[j,:] . x_i)
//
// B200 design.  At d = 2048, h = 256 the first layer is 2*d*h = 1 MFLOP per token
// against 2*d = 4 KB of residual read once from HBM: 256 flop/B, right on the
// B200 ridge (measured bf16 peak / measured HBM bandwidth ~ 250 flop/B).  CUDA-core
// FMAs would be ~20x too slow, so the contraction runs on tcgen05.  A single-SM
// M=128 x N=256 MMA reads 12 KB of operands from shared memory per 128 clocks while
// TMA writes as much again, more than shared memory delivers, so the kernel runs on
// CTA pairs (cta_group::2):
//   * a 2-CTA cluster owns 256-token tiles: each CTA stages its 128 tokens x 64
//     columns of the residual and its half (h/2 rows) of the matching 64-column
//     slice of W1 (6 stages of 32 KB, 128-byte swizzle, K-major), both TMA loads
//     completing on the pair leader's barrier;
//   * the leader's warp 1 issues one tcgen05.mma.cta_group::2 (M = 256, N = h) per
//     16 columns; each CTA's TMEM holds its 128 rows x h fp32 accumulator,
//     double-buffered so the epilogue of tile t overlaps the MMAs of t+1.  W1 is
//     now staged once per 256 tokens instead of once per 128;
//   * warps 4-7 of each CTA read their accumulator rows with tcgen05.ld (one token
//     per thread) and apply +b1, SiLU, the dot with W2 and +b2 in registers, writing
//     one fp32 per token.  The hidden activations never leave the SM.
// The residual is streamed with an L2 evict-first hint and W1 (re-read by every
// tile) with evict-last, so W1 stays L2-resident while the residual passes through.
// For the fused selection (tg_select_fused) the epilogue also histograms the top 8
// bits of the selector's order key of each document token's score (warp-aggregated
// shared-memory atomics) and every CTA stores its 256 bins: the selector's first
// radix pass then sums those instead of reading the scores.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "runtime.h"
#include "select_key.cuh"

namespace {

constexpr int kBlockM = 128;      // tokens per CTA (256 per pair)
constexpr int kBlockK = 64;       // bf16 elements in one 128-byte swizzled row
constexpr int kStages = 6;
constexpr int kThreads = 256;
constexpr int kMaxH = 256;
constexpr uint32_t kTileABytes = kBlockM * kBlockK * 2;  // 16 KB

struct GateCtl {
  uint64_t full[kStages];      // used in the leader: both CTAs' loads complete here
  uint64_t empty[kStages];     // each CTA's own copy, signalled by the leader's MMA commit
  uint64_t acc_full[2];        // each CTA's own copy
  uint64_t acc_empty[2];       // used in the leader: 128 epilogue threads of each CTA
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float b1[kMaxH];
  float w2[kMaxH];
  uint32_t hist[256];          // top-byte histogram of the document tokens' order keys
};

constexpr size_t smem_bytes(int h) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(kStages) * (kTileABytes + static_cast<size_t>(h / 2) * 128) +
         sizeof(GateCtl);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gate_score_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __nv_bfloat16 *__restrict__ b1, const __nv_bfloat16 *__restrict__ W2,
                      const __nv_bfloat16 *__restrict__ b2, float *__restrict__ scores, int64_t n, int d, int h,
                      uint32_t tmem_cols, const uint8_t *__restrict__ doc_mask, uint32_t *__restrict__ hist_parts,
                      uint32_t *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kTileABytes;
  const uint32_t tile_b_bytes = static_cast<uint32_t>(h / 2) * 128u;  // this CTA's half of the W1 slice
  GateCtl *ctl = reinterpret_cast<GateCtl *>(sB + kStages * tile_b_bytes);

  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tg::cluster_ctarank();       // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1;
  const int64_t n_pairs = gridDim.x >> 1;
  const int64_t num_tiles = (n + 2 * kBlockM - 1) / (2 * kBlockM);
  const int ksteps = (d + kBlockK - 1) / kBlockK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tg::mbar_init(tg::smem_addr(&ctl->acc_full[a]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->acc_empty[a]), 2 * 128);
    }
    tg::mbar_init(tg::smem_addr(&ctl->drain), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
    tg::prefetch_tmap(&tm_x);
    tg::prefetch_tmap(&tm_w);
  }
  if (warp == 2) {
    tg::tmem_alloc_pair(tg::smem_addr(&ctl->tmem_base), tmem_cols);
    tg::tmem_relinquish_pair();
  }
  // barriers of both CTAs initialised and TMEM allocated before any cross-CTA traffic
  tg::tc_fence_before();
  __syncthreads();
  tg::cluster_sync_all();
  tg::tc_fence_after();
  // the prologue above overlaps the previous kernel; global memory only from here on
  tg::pdl_wait();
  tg::pdl_trigger();
  if (warp >= 4) {
    for (int j = threadIdx.x - 128; j < h; j += 128) {
      ctl->b1[j] = __bfloat162float(b1[j]);
      ctl->w2[j] = __bfloat162float(W2[j]);
    }
    if (hist_parts)
      for (int j = threadIdx.x - 128; j < 256; j += 128) ctl->hist[j] = 0;
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
  }
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int *abort_flag = &ctl->abort_flag;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    const uint64_t pol_x = tg::l2_policy_evict_first();
    const uint64_t pol_w = tg::l2_policy_evict_last();
    uint32_t it = 0;
    for (int64_t tile = pair; tile < num_tiles; tile += n_pairs) {
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!tg::mbar_wait(tg::smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag)) goto producer_done;
        const uint32_t full = tg::smem_addr(&ctl->full[s]);
        if (leader) tg::mbar_arrive_expect_tx(full, 2u * (kTileABytes + tile_b_bytes));
        const uint32_t lbar = tg::pair_leader_addr(full);
        tg::tma_load_2d_pair(tg::smem_addr(sA + s * kTileABytes), &tm_x, lbar, ks * kBlockK,
                             static_cast<int32_t>(tile * 2 * kBlockM + rank * kBlockM), pol_x);
        tg::tma_load_2d_pair(tg::smem_addr(sB + s * tile_b_bytes), &tm_w, lbar, ks * kBlockK,
                             static_cast<int32_t>(rank * (h / 2)), pol_w);
      }
    }
  producer_done:;
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    const uint32_t idesc = tg::idesc_bf16_f32(2 * kBlockM, h, false, false);
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int64_t tile = pair; tile < num_tiles && ok; tile += n_pairs, ++tc) {
      const uint32_t acc = tc & 1u, aph = (tc >> 1) & 1u;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->acc_empty[acc]), aph ^ 1u, abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(h);
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!tg::mbar_wait(tg::smem_addr(&ctl->full[s]), ph, abort_flag)) {
          ok = false;
          break;
        }
        tg::tc_fence_after();
        const uint64_t adesc = tg::smem_desc_sw128(tg::smem_addr(sA + s * kTileABytes), 16, 1024);
        const uint64_t bdesc = tg::smem_desc_sw128(tg::smem_addr(sB + s * tile_b_bytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kBlockK / 16; ++kk) {
          // advance 16 bf16 = 32 bytes along K inside the 128-byte swizzled rows
          tg::mma_bf16_ss_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, (ks | kk) != 0);
        }
        tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->empty[s]), 0x3);
      }
      if (ok) tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->acc_full[acc]), 0x3);
    }
    if (*abort_flag) {
      // let every MMA already issued finish before TMEM is released
      tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->drain), 0x1);
      int local_abort = 0;
      tg::mbar_wait(tg::smem_addr(&ctl->drain), 0, &local_abort, 100000000ull);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp - 4;  // TMEM lanes 32*quarter .. 32*quarter+31
    const float bias2 = __bfloat162float(b2[0]);
    uint32_t tc = 0;
    for (int64_t tile = pair; tile < num_tiles; tile += n_pairs, ++tc) {
      const uint32_t acc = tc & 1u, aph = (tc >> 1) & 1u;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->acc_full[acc]), aph, abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t taddr = tmem_base + acc * static_cast<uint32_t>(h) + (static_cast<uint32_t>(quarter * 32) << 16);
      float sum = 0.f;
      for (int c = 0; c < h; c += 16) {
        uint32_t r[16];
        tg::tmem_ld16(taddr + static_cast<uint32_t>(c), r);
        tg::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float z = __uint_as_float(r[j]) + ctl->b1[c + j];
          const float a = __fdividef(z, 1.0f + __expf(-z));
          sum = fmaf(ctl->w2[c + j], a, sum);
        }
      }
      tg::tc_fence_before();
      tg::mbar_arrive_remote(tg::smem_addr(&ctl->acc_empty[acc]), 0u);  // the leader's copy
      const int64_t row = tile * 2 * kBlockM + rank * kBlockM + quarter * 32 + lane;
      const float score = sum + bias2;
      if (row < n) scores[row] = score;
      if (hist_parts) {
        // lanes with the same top byte add once, with the group's size
        const uint32_t key = row < n ? tg::order_key(score, doc_mask[row] != 0) : 0u;
        const unsigned live = __ballot_sync(0xFFFFFFFFu, key != 0u);
        if (key != 0u) {
          const unsigned peers = __match_any_sync(live, key >> 24);
          if (lane == __ffs(peers) - 1) atomicAdd(&ctl->hist[key >> 24], static_cast<uint32_t>(__popc(peers)));
        }
      }
    }
    if (hist_parts) {
      asm volatile("bar.sync 1, 128;" ::: "memory");  // every epilogue warp has added its tiles
      for (int j = threadIdx.x - 128; j < 256; j += 128) hist_parts[blockIdx.x * 256 + j] = ctl->hist[j];
    }
  }

  // every MMA, remote arrive and peer TMEM access is done before either CTA frees TMEM
  tg::tc_fence_before();
  __syncthreads();
  tg::cluster_sync_all();
  if (threadIdx.x == 0 && ctl->abort_flag) tg::set_device_error(err, TG_DEVERR_TIMEOUT);
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc_pair(tmem_base, tmem_cols);
  }
}

}  // namespace

int64_t tg::gate_grid(int64_t n) {
  const int64_t num_tiles = (n + 2 * kBlockM - 1) / (2 * kBlockM);
  return 2 * std::min<int64_t>(num_tiles, tg::sm_count() / 2);
}

tg_status tg::gate_score_hist(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1, const tg_bf16 *b1,
                              const tg_bf16 *W2, const tg_bf16 *b2, int32_t h, float *scores, const uint8_t *doc_mask,
                              uint32_t *hist_parts, tg_stream stream) {
  if (n < 0) return tg::fail(TG_ERR_INVALID_ARG, "n must be >= 0");
  if (d <= 0 || d % 8 != 0) return tg::fail(TG_ERR_INVALID_ARG, "d must be a positive multiple of 8 (got %d)", d);
  if (h < 16 || h > kMaxH || h % 16 != 0)
    return tg::fail(TG_ERR_UNSUPPORTED, "h must be a multiple of 16 in [16, 256] (got %d)", h);
  if (n == 0) return TG_OK;
  if (!hidden || !W1 || !b1 || !W2 || !b2 || !scores) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (hist_parts && !doc_mask) return tg::fail(TG_ERR_INVALID_ARG, "doc_mask is NULL");
  if (!tg::aligned16(hidden) || !tg::aligned16(W1) || !tg::aligned16(scores))
    return tg::fail(TG_ERR_ALIGNMENT, "hidden, W1 and scores must be 16-byte aligned");
  if (n > (int64_t(1) << 31) * kBlockM) return tg::fail(TG_ERR_UNSUPPORTED, "n too large");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;

  CUtensorMap tm_x, tm_w;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d) * 2};
    const uint32_t box[2] = {kBlockK, kBlockM};
    if (!tg::encode_tmap(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, hidden, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(h)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d) * 2};
    const uint32_t box[2] = {kBlockK, static_cast<uint32_t>(h / 2)};
    if (!tg::encode_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W1, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  uint32_t tmem_cols = 32;
  while (tmem_cols < 2u * static_cast<uint32_t>(h)) tmem_cols <<= 1;

  const size_t smem = smem_bytes(h);
  static tg::PerDevice configured;
  const tg_status setup = tg::once_per_device(configured, [&](int) -> tg_status {
    const cudaError_t e = cudaFuncSetAttribute(gate_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem_bytes(kMaxH)));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TG_OK;
  });
  if (setup != TG_OK) return setup;
  const cudaError_t e = tg::launch_pdl(gate_score_kernel, dim3(static_cast<unsigned>(gate_grid(n))), dim3(kThreads), smem,
                                      static_cast<cudaStream_t>(stream), tm_x, tm_w,
                                      reinterpret_cast<const __nv_bfloat16 *>(b1),
                                      reinterpret_cast<const __nv_bfloat16 *>(W2),
                                      reinterpret_cast<const __nv_bfloat16 *>(b2), scores, n, d, h, tmem_cols, doc_mask,
                                      hist_parts, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "gate_score_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("gate_score_kernel");
}

extern "C" tg_status tg_gate_score(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1, const tg_bf16 *b1,
                                   const tg_bf16 *W2, const tg_bf16 *b2, int32_t h, float *scores, tg_stream stream) {
  TG_API_ENTRY();
  return tg::gate_score_hist(hidden, n, d, W1, b1, W2, b2, h, scores, nullptr, nullptr, stream);
}
