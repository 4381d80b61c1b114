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
// FMAs would be ~20x too slow, so the contraction runs on tcgen05:
//   * persistent grid, one CTA per SM, tiles of 128 tokens (MMA M = 128, N = h);
//   * warp 0 streams 128x64 residual tiles and the matching 64-wide slice of W1
//     through a 4-stage TMA pipeline (128-byte swizzle, K-major operands);
//   * warp 1 issues tcgen05.mma (one thread) into a TMEM accumulator of h fp32
//     columns, double-buffered so the epilogue of tile t overlaps the MMAs of t+1;
//   * warps 4-7 read the accumulator rows with tcgen05.ld (one token per thread)
//     and apply +b1, SiLU, the dot with W2 and +b2 in registers, writing one fp32
//     per token.  The hidden activations never leave the SM.
// The residual is streamed with an L2 evict-first hint and W1 (re-read by every
// tile) with evict-last, so W1 stays L2-resident while the residual passes through.
#include <algorithm>

#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kBlockM = 128;
constexpr int kBlockK = 64;  // bf16 elements in one 128-byte swizzled row
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr int kMaxH = 256;
constexpr uint32_t kTileABytes = kBlockM * kBlockK * 2;

struct GateCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float b1[kMaxH];
  float w2[kMaxH];
};

constexpr size_t smem_bytes(int h) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(kStages) * (kTileABytes + static_cast<size_t>(h) * 128) +
         sizeof(GateCtl);
}

__global__ void __launch_bounds__(kThreads, 1)
    gate_score_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __nv_bfloat16 *__restrict__ b1, const __nv_bfloat16 *__restrict__ W2,
                      const __nv_bfloat16 *__restrict__ b2, float *__restrict__ scores, int64_t n, int d, int h,
                      uint32_t tmem_cols, uint32_t *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kTileABytes;
  const uint32_t tile_b_bytes = static_cast<uint32_t>(h) * 128u;
  GateCtl *ctl = reinterpret_cast<GateCtl *>(sB + kStages * tile_b_bytes);

  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;
  const int64_t num_tiles = (n + kBlockM - 1) / kBlockM;
  const int ksteps = (d + kBlockK - 1) / kBlockK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tg::mbar_init(tg::smem_addr(&ctl->acc_full[a]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->acc_empty[a]), 128);
    }
    tg::mbar_init(tg::smem_addr(&ctl->drain), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
    tg::prefetch_tmap(&tm_x);
    tg::prefetch_tmap(&tm_w);
  }
  if (warp == 2) {
    tg::tmem_alloc(tg::smem_addr(&ctl->tmem_base), tmem_cols);
    tg::tmem_relinquish();
  }
  if (warp >= 4) {
    for (int j = threadIdx.x - 128; j < h; j += 128) {
      ctl->b1[j] = __bfloat162float(b1[j]);
      ctl->w2[j] = __bfloat162float(W2[j]);
    }
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int *abort_flag = &ctl->abort_flag;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    const uint64_t pol_x = tg::l2_policy_evict_first();
    const uint64_t pol_w = tg::l2_policy_evict_last();
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!tg::mbar_wait(tg::smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag)) goto producer_done;
        const uint32_t full = tg::smem_addr(&ctl->full[s]);
        tg::mbar_arrive_expect_tx(full, kTileABytes + tile_b_bytes);
        tg::tma_load_2d_hint(tg::smem_addr(sA + s * kTileABytes), &tm_x, full, ks * kBlockK,
                             static_cast<int32_t>(tile * kBlockM), pol_x);
        tg::tma_load_2d_hint(tg::smem_addr(sB + s * tile_b_bytes), &tm_w, full, ks * kBlockK, 0, pol_w);
      }
    }
  producer_done:;
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = tg::idesc_bf16_f32(kBlockM, h, false, false);
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tc) {
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
          tg::mma_bf16_ss(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, (ks | kk) != 0);
        }
        tg::mma_commit(tg::smem_addr(&ctl->empty[s]));
      }
      if (ok) tg::mma_commit(tg::smem_addr(&ctl->acc_full[acc]));
    }
    if (*abort_flag) {
      // let every MMA already issued finish before TMEM is released
      tg::mma_commit(tg::smem_addr(&ctl->drain));
      int local_abort = 0;
      tg::mbar_wait(tg::smem_addr(&ctl->drain), 0, &local_abort, 100000000ull);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp - 4;  // TMEM lanes 32*quarter .. 32*quarter+31
    const float bias2 = __bfloat162float(b2[0]);
    uint32_t tc = 0;
    for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
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
      tg::mbar_arrive(tg::smem_addr(&ctl->acc_empty[acc]));
      const int64_t row = tile * kBlockM + quarter * 32 + lane;
      if (row < n) scores[row] = sum + bias2;
    }
  }

  tg::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ctl->abort_flag) tg::set_device_error(err, TG_DEVERR_TIMEOUT);
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace

extern "C" tg_status tg_gate_score(const tg_bf16 *hidden, int64_t n, int32_t d, const tg_bf16 *W1, const tg_bf16 *b1,
                                   const tg_bf16 *W2, const tg_bf16 *b2, int32_t h, float *scores, tg_stream stream) {
  tg::clear_detail();
  if (n < 0) return tg::fail(TG_ERR_INVALID_ARG, "n must be >= 0");
  if (d <= 0 || d % 8 != 0) return tg::fail(TG_ERR_INVALID_ARG, "d must be a positive multiple of 8 (got %d)", d);
  if (h < 16 || h > kMaxH || h % 16 != 0)
    return tg::fail(TG_ERR_UNSUPPORTED, "h must be a multiple of 16 in [16, 256] (got %d)", h);
  if (n == 0) return TG_OK;
  if (!hidden || !W1 || !b1 || !W2 || !b2 || !scores) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
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
    const uint32_t box[2] = {kBlockK, static_cast<uint32_t>(h)};
    if (!tg::encode_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W1, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  uint32_t tmem_cols = 32;
  while (tmem_cols < 2u * static_cast<uint32_t>(h)) tmem_cols <<= 1;

  const size_t smem = smem_bytes(h);
  static bool configured[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(gate_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem_bytes(kMaxH)));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    configured[dev] = true;
  }
  const int64_t num_tiles = (n + kBlockM - 1) / kBlockM;
  const int grid = static_cast<int>(std::min<int64_t>(num_tiles, tg::sm_count()));
  gate_score_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      tm_x, tm_w, reinterpret_cast<const __nv_bfloat16 *>(b1), reinterpret_cast<const __nv_bfloat16 *>(W2),
      reinterpret_cast<const __nv_bfloat16 *>(b2), scores, n, d, h, tmem_cols, err);
  return tg::check_launch("gate_score_kernel");
}
