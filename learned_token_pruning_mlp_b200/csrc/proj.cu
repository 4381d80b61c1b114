// proj.cu -- the projections around token-gated attention in a pruned layer:
//   tg_qkv_rope : [Q K V] = hidden_k W_qkv^T, then (optionally) a per-head RMS norm of
//                 the Q and K heads and the rotary position embedding of Q and K at
//                 each kept token's original prompt position;
//   tg_linear   : y = x W^T (+ residual), the output projection.
//
// TokenGate article, "How does TokenGate learned token pruning work?" (pruned
// forward): the layers above the gate process only the kept tokens.  Those tokens
// keep their prompt positions, so the rotary angles use the kept indices, not the
// compacted row numbers.
//
// B200 design: one CTA-pair tcgen05 GEMM (cta_group::2, 256 x 256 output tiles,
// each CTA staging 128 rows of x and its half of the weight slice through 6 TMA
// stages of 32 KB, double-buffered TMEM accumulators), persistent over tiles with
// consecutive tiles sharing the same 256 rows of x.  The elementwise work sits in the
// epilogue, run by two warpgroups per CTA (each thread owns one row, i.e. one TMEM
// lane, and half of the tile's columns):
//   * output projection: + residual, whose row slice each thread loads into registers
//     before the accumulator is ready;
//   * QKV: a 256-column tile holds whole heads of one kind (Q, K or V).  The tile is
//     four (head, 32-pair chunk) units; each warpgroup takes the two units that share
//     one chunk of rotary indices j, so each thread forms 32 angles per tile and
//     applies them to two heads.  The angle p * base^(-2j/D) is reduced modulo one
//     turn exactly with a 64-bit fixed-point product (integer pipe), then sin/cos run
//     in fp32.  The per-head norm takes the head's mean square in a first pass over
//     TMEM.  Q, K and V go straight into their [S, H, D] buffers.
#include <algorithm>
#include <cmath>

#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kBM = 128;         // rows per CTA (256 per pair)
constexpr int kBN = 256;         // output columns per pair tile
constexpr int kBK = 64;          // bf16 elements in one 128-byte swizzled row
constexpr int kStages = 6;
constexpr int kThreads = 384;  // warps 0-3: TMA, MMA, TMEM alloc, idle; 4-11: two epilogue warpgroups
constexpr uint32_t kTileABytes = kBM * kBK * 2;          // 16 KB
constexpr uint32_t kTileBBytes = (kBN / 2) * kBK * 2;    // 16 KB (this CTA's half)

struct ProjCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float q_norm[128];
  float k_norm[128];
};

constexpr size_t kSmem = 1024 + kStages * static_cast<size_t>(kTileABytes + kTileBBytes) + sizeof(ProjCtl);

// Epilogue description (passed by value).
struct ProjOut {
  // plain: y[M, N] bf16 (+ residual [M, N]).  qkv: Q [M, Hq*D], K [M, Hkv*D], V [M, Hkv*D] bf16.
  __nv_bfloat16 *y;
  const __nv_bfloat16 *residual;
  const __nv_bfloat16 *q_norm;  // [D] or null
  const __nv_bfloat16 *k_norm;  // [D] or null
  float eps;
  __nv_bfloat16 *q;
  __nv_bfloat16 *k;
  __nv_bfloat16 *v;
  const int32_t *pos;     // rotary position of every row
  int32_t q_cols;         // Hq * D
  int32_t k_cols;         // Hkv * D
  // base^(-2j/D) / (2 pi) modulo 1 as a 64-bit binary fraction, j < D/2: the rotary
  // angle of position p in turns is (p * turn[j] mod 2^64) / 2^64
  uint64_t turn[64];
};

// Round 32 fp32 values to bf16 and write them as four 16-byte stores.
__device__ __forceinline__ void store_row32(__nv_bfloat16 *dst, const float *v) {
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    pk[e] = *reinterpret_cast<const uint32_t *>(&b);
  }
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
}

// kHD = 0: plain projection; kHD = 64 / 128: QKV projection with head dim kHD.
template <int kHD>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, int64_t M,
                     int32_t N, int32_t K, const __grid_constant__ ProjOut out, uint32_t *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kTileABytes;
  ProjCtl *ctl = reinterpret_cast<ProjCtl *>(sB + kStages * kTileBBytes);

  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tg::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int n_pairs = static_cast<int>(gridDim.x >> 1);
  const int m_tiles = static_cast<int>((M + 2 * kBM - 1) / (2 * kBM));
  const int n_tiles = (N + kBN - 1) / kBN;
  const int num_tiles = m_tiles * n_tiles;  // below 2^31 (checked on the host)
  const int ksteps = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tg::mbar_init(tg::smem_addr(&ctl->acc_full[a]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->acc_empty[a]), 2 * 256);
    }
    tg::mbar_init(tg::smem_addr(&ctl->drain), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
    tg::prefetch_tmap(&tm_a);
    tg::prefetch_tmap(&tm_b);
  }
  if (warp == 2) {
    tg::tmem_alloc_pair(tg::smem_addr(&ctl->tmem_base), 512);
    tg::tmem_relinquish_pair();
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::cluster_sync_all();
  tg::tc_fence_after();
  tg::pdl_wait();
  tg::pdl_trigger();
  if (kHD > 0 && warp >= 4) {
    for (int j = threadIdx.x - 128; j < kHD; j += 256) {
      ctl->q_norm[j] = out.q_norm ? __bfloat162float(out.q_norm[j]) : 1.f;
      ctl->k_norm[j] = out.k_norm ? __bfloat162float(out.k_norm[j]) : 1.f;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");  // the two epilogue warpgroups
  }
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int *abort_flag = &ctl->abort_flag;

  // Register split for the QKV epilogue (32 angles and two 32-wide TMEM rows live per
  // thread): the launch gives 384 threads x 168 registers; 128 x 80 + 256 x 208 =
  // 63488 <= 384 x 168, so the increase never waits (the launcher checks the launch
  // count).
  // Each warpgroup changes its budget inside its own branch.
  if (warp < 4) {
  if constexpr (kHD > 0) asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    const uint64_t pol_a = tg::l2_policy_evict_last();  // x rows are reused by every N tile
    const uint64_t pol_b = tg::l2_policy_evict_last();  // the weights by every M tile
    uint32_t it = 0;
    for (int t = pair; t < num_tiles; t += n_pairs) {
      const int mt = t / n_tiles;
      const int nt = static_cast<int>(t % n_tiles);
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!tg::mbar_wait(tg::smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag)) goto producer_done;
        const uint32_t full = tg::smem_addr(&ctl->full[s]);
        if (leader) tg::mbar_arrive_expect_tx(full, 2u * (kTileABytes + kTileBBytes));
        const uint32_t lbar = tg::pair_leader_addr(full);
        tg::tma_load_2d_pair(tg::smem_addr(sA + s * kTileABytes), &tm_a, lbar, ks * kBK,
                             static_cast<int32_t>(mt * 2 * kBM + rank * kBM), pol_a);
        tg::tma_load_2d_pair(tg::smem_addr(sB + s * kTileBBytes), &tm_b, lbar, ks * kBK,
                             static_cast<int32_t>(nt * kBN + rank * (kBN / 2)), pol_b);
      }
    }
  producer_done:;
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    constexpr uint32_t idesc = tg::idesc_bf16_f32(2 * kBM, kBN, false, false);
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int t = pair; t < num_tiles && ok; t += n_pairs, ++tc) {
      const uint32_t acc = tc & 1u, aph = (tc >> 1) & 1u;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->acc_empty[acc]), aph ^ 1u, abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(kBN);
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!tg::mbar_wait(tg::smem_addr(&ctl->full[s]), ph, abort_flag)) {
          ok = false;
          break;
        }
        tg::tc_fence_after();
        const uint64_t adesc = tg::smem_desc_sw128(tg::smem_addr(sA + s * kTileABytes), 16, 1024);
        const uint64_t bdesc = tg::smem_desc_sw128(tg::smem_addr(sB + s * kTileBBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          tg::mma_bf16_ss_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, (ks | kk) != 0);
        tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->empty[s]), 0x3);
      }
      if (ok) tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->acc_full[acc]), 0x3);
    }
    if (*abort_flag) {
      tg::mma_commit_pair_multicast(tg::smem_addr(&ctl->drain), 0x1);
      int local_abort = 0;
      tg::mbar_wait(tg::smem_addr(&ctl->drain), 0, &local_abort, 100000000ull);
    }
  }
  } else {
    if constexpr (kHD > 0) asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. 32*quarter+31
    const int group = (warp - 4) >> 2;     // 0 or 1: which half of the tile's work
    uint32_t tc = 0;
    for (int t = pair; t < num_tiles; t += n_pairs, ++tc) {
      const int mt = t / n_tiles;
      const int nt = static_cast<int>(t % n_tiles);
      const uint32_t acc = tc & 1u, aph = (tc >> 1) & 1u;
      const int64_t row = mt * 2 * kBM + rank * kBM + quarter * 32 + lane;
      const bool row_ok = row < M;
      const int n0 = nt * kBN;
      // the residual slice this thread adds (its row, the group's 128 columns), loaded into
      // registers before the accumulator is ready so the loads overlap the tile's MMAs
      uint4 res[kHD == 0 ? 16 : 1];
      if constexpr (kHD == 0) {
        const int c0 = n0 + group * (kBN / 2);
        if (out.residual && row_ok) {
          const uint4 *src = reinterpret_cast<const uint4 *>(out.residual + row * static_cast<int64_t>(N) + c0);
#pragma unroll
          for (int q = 0; q < 16; ++q) res[q] = c0 + 8 * q < N ? src[q] : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      int32_t p = 0;
      if constexpr (kHD > 0) p = row_ok ? out.pos[row] : 0;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->acc_full[acc]), aph, abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t taddr = tmem_base + acc * static_cast<uint32_t>(kBN) + (static_cast<uint32_t>(quarter * 32) << 16);
      if constexpr (kHD == 0) {
#pragma unroll
        for (int c = 0; c < kBN / 64; ++c) {
          const int cc = group * (kBN / 64) + c;  // 32-column chunk of the tile
          uint32_t r[32];
          tg::tmem_ld32(taddr + cc * 32, r);
          tg::tmem_ld_wait();
          const int col = n0 + cc * 32;
          if (row_ok && col < N) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
            if (out.residual) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 u = res[4 * c + q];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[e]);
                  v[8 * q + 2 * e] += __low2float(b);
                  v[8 * q + 2 * e + 1] += __high2float(b);
                }
              }
            }
            store_row32(out.y + row * static_cast<int64_t>(N) + col, v);
          }
          __syncwarp();
        }
      } else {
        constexpr int kHalf = kHD / 2;
        // units (head, chunk) of this warpgroup: two heads sharing rotary chunk jc
        const int jc = kHD == 128 ? group : 0;                // chunk of 32 rotary indices
        const int hA = kHD == 128 ? 0 : group;                // head offsets inside the tile
        const int hB = kHD == 128 ? 1 : group + 2;
        const int colA = n0 + hA * kHD, colB = n0 + hB * kHD;
        // the 32 angles of this chunk, in turns, reduced exactly, then sin/cos
        float cs[32], sn[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint64_t prod = static_cast<uint64_t>(static_cast<int64_t>(p)) * out.turn[32 * jc + e];
          const uint32_t hi = static_cast<uint32_t>(prod >> 32);
          float f = __uint_as_float(0x3F800000u | (hi >> 9)) - 1.0f;  // [0, 1) turns
          f = f >= 0.5f ? f - 1.0f : f;                              // [-1/2, 1/2) turns
          __sincosf(f * 6.28318530717958647692f, &sn[e], &cs[e]);
        }
#pragma unroll 1
        for (int u = 0; u < 2; ++u) {
          const int col = u == 0 ? colA : colB;  // warp-uniform
          if (col >= N) break;
          const uint32_t hcol = static_cast<uint32_t>(col - n0);
          __nv_bfloat16 *dst;
          int64_t ld;
          const float *nw = nullptr;
          const bool is_v = col >= out.q_cols + out.k_cols;
          if (col < out.q_cols) {
            dst = out.q + col;
            ld = out.q_cols;
            nw = out.q_norm ? ctl->q_norm : nullptr;
          } else if (!is_v) {
            dst = out.k + (col - out.q_cols);
            ld = out.k_cols;
            nw = out.k_norm ? ctl->k_norm : nullptr;
          } else {
            dst = out.v + (col - out.q_cols - out.k_cols);
            ld = out.k_cols;
          }
          float rn = 1.f;
          if (nw) {  // mean square of the whole head
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < kHD / 32; ++c) {
              uint32_t r[32];
              tg::tmem_ld32(taddr + hcol + 32 * c, r);
              tg::tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
            }
            rn = rsqrtf(ss * (1.0f / kHD) + out.eps);
          }
          uint32_t lo[32], hi[32];
          tg::tmem_ld32(taddr + hcol + 32 * jc, lo);
          tg::tmem_ld32(taddr + hcol + kHalf + 32 * jc, hi);
          tg::tmem_ld_wait();
          float a[32], b[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            a[e] = __uint_as_float(lo[e]);
            b[e] = __uint_as_float(hi[e]);
          }
          if (nw) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              a[e] = a[e] * rn * nw[32 * jc + e];
              b[e] = b[e] * rn * nw[kHalf + 32 * jc + e];
            }
          }
          if (!is_v) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x0 = a[e], x1 = b[e];
              a[e] = x0 * cs[e] - x1 * sn[e];
              b[e] = x1 * cs[e] + x0 * sn[e];
            }
          }
          if (row_ok) {
            __nv_bfloat16 *drow = dst + row * ld;
            store_row32(drow + 32 * jc, a);
            store_row32(drow + kHalf + 32 * jc, b);
          }
          __syncwarp();
        }
      }
      tg::tc_fence_before();
      tg::mbar_arrive_remote(tg::smem_addr(&ctl->acc_empty[acc]), 0u);
    }
  }

  tg::tc_fence_before();
  __syncthreads();
  tg::cluster_sync_all();
  if (threadIdx.x == 0 && ctl->abort_flag) tg::set_device_error(err, TG_DEVERR_TIMEOUT);
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc_pair(tmem_base, 512);
  }
}

template <int kHD>
tg_status launch_proj(const tg_bf16 *x, int64_t M, int32_t K, const tg_bf16 *W, int32_t N, const ProjOut &out,
                      cudaStream_t stream, const char *name) {
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  CUtensorMap tm_a, tm_b;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {kBK, kBM};
    if (!tg::encode_tmap(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {kBK, kBN / 2};
    if (!tg::encode_tmap(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  static tg::PerDevice configured;
  const tg_status setup = tg::once_per_device(configured, [&](int) -> tg_status {
    const cudaError_t e =
        cudaFuncSetAttribute(proj_gemm_kernel<kHD>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (kHD > 0) {
      // the register split in the kernel assumes 168 registers per thread at launch
      cudaFuncAttributes fa;
      const cudaError_t ea = cudaFuncGetAttributes(&fa, proj_gemm_kernel<kHD>);
      if (ea != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(ea));
      if (fa.numRegs != 168)
        return tg::fail(TG_ERR_UNSUPPORTED, "%s built with %d registers per thread; the warpgroup register split "
                        "needs 168", name, fa.numRegs);
    }
    return TG_OK;
  });
  if (setup != TG_OK) return setup;
  const int64_t tiles = ((M + 2 * kBM - 1) / (2 * kBM)) * ((N + kBN - 1) / kBN);
  if (tiles > 0x7FFFFFFF) return tg::fail(TG_ERR_UNSUPPORTED, "%s: more than 2^31 - 1 output tiles", name);
  const int64_t pairs = std::min<int64_t>(tiles, tg::sm_count() / 2);
  const cudaError_t e = tg::launch_pdl(proj_gemm_kernel<kHD>, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads),
                                      kSmem, stream, tm_a, tm_b, M, N, K, out, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "%s launch: %s", name, cudaGetErrorString(e));
  return tg::check_launch(name);
}

}  // namespace

extern "C" tg_status tg_linear(const tg_bf16 *x, int64_t M, int32_t K, const tg_bf16 *W, int32_t N,
                               const tg_bf16 *residual, tg_bf16 *y, tg_stream stream) {
  TG_API_ENTRY();
  if (M < 0 || K <= 0 || N <= 0) return tg::fail(TG_ERR_INVALID_ARG, "M >= 0, K > 0, N > 0 required");
  if (K % 8 != 0) return tg::fail(TG_ERR_UNSUPPORTED, "K must be a multiple of 8 (got %d)", K);
  if (N % 32 != 0) return tg::fail(TG_ERR_UNSUPPORTED, "N must be a multiple of 32 (got %d)", N);
  if (M > (int64_t(1) << 31) - 1) return tg::fail(TG_ERR_UNSUPPORTED, "M must be below 2^31");
  if (M == 0) return TG_OK;
  if (!x || !W || !y) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (!tg::aligned16(x) || !tg::aligned16(W) || !tg::aligned16(y) || (residual && !tg::aligned16(residual)))
    return tg::fail(TG_ERR_ALIGNMENT, "x, W, residual and y must be 16-byte aligned");
  ProjOut out = {};
  out.y = reinterpret_cast<__nv_bfloat16 *>(y);
  out.residual = reinterpret_cast<const __nv_bfloat16 *>(residual);
  return launch_proj<0>(x, M, K, W, N, out, static_cast<cudaStream_t>(stream), "proj_gemm_kernel<linear>");
}

extern "C" tg_status tg_qkv_rope(const tg_bf16 *hidden, int64_t S, int32_t d, const tg_bf16 *W_qkv,
                                 const int32_t *positions, double rope_base, const tg_bf16 *q_norm,
                                 const tg_bf16 *k_norm, float eps, int32_t Hq, int32_t Hkv, int32_t D, tg_bf16 *Q,
                                 tg_bf16 *Kc, tg_bf16 *V, tg_stream stream) {
  TG_API_ENTRY();
  if (S < 0 || d <= 0) return tg::fail(TG_ERR_INVALID_ARG, "S >= 0 and d > 0 required");
  if (d % 8 != 0) return tg::fail(TG_ERR_UNSUPPORTED, "d must be a multiple of 8 (got %d)", d);
  if (D != 64 && D != 128) return tg::fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (Hq <= 0 || Hkv <= 0) return tg::fail(TG_ERR_INVALID_ARG, "Hq and Hkv must be positive");
  if (!(rope_base > 1.0) || !std::isfinite(rope_base)) return tg::fail(TG_ERR_INVALID_ARG, "rope_base must be > 1");
  if (!(eps >= 0.f) || !std::isfinite(eps)) return tg::fail(TG_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (S > (int64_t(1) << 31) - 1) return tg::fail(TG_ERR_UNSUPPORTED, "S must be below 2^31");
  const int64_t N = static_cast<int64_t>(Hq + 2 * static_cast<int64_t>(Hkv)) * D;
  if (N > 0x7FFFFFFF) return tg::fail(TG_ERR_UNSUPPORTED, "too many heads");
  if (S == 0) return TG_OK;
  if (!hidden || !W_qkv || !positions || !Q || !Kc || !V) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (!tg::aligned16(hidden) || !tg::aligned16(W_qkv) || !tg::aligned16(Q) || !tg::aligned16(Kc) || !tg::aligned16(V))
    return tg::fail(TG_ERR_ALIGNMENT, "hidden, W_qkv, Q, Kc and V must be 16-byte aligned");
  ProjOut out = {};
  out.q = reinterpret_cast<__nv_bfloat16 *>(Q);
  out.k = reinterpret_cast<__nv_bfloat16 *>(Kc);
  out.v = reinterpret_cast<__nv_bfloat16 *>(V);
  out.pos = positions;
  out.q_norm = reinterpret_cast<const __nv_bfloat16 *>(q_norm);
  out.k_norm = reinterpret_cast<const __nv_bfloat16 *>(k_norm);
  out.eps = eps;
  out.q_cols = Hq * D;
  out.k_cols = Hkv * D;
  // base^(-2j/D) / (2 pi) modulo 1 as a 64-bit binary fraction (x86 long double
  // carries 64 significant bits, so the table is exact to about 2^-64 turns)
  const long double two_pi = 6.283185307179586476925286766559005768L;
  for (int j = 0; j < D / 2; ++j) {
    long double g = std::pow(static_cast<long double>(rope_base), -2.0L * j / D) / two_pi;
    g -= std::floor(g);
    const long double scaled = std::ldexp(g, 64);
    out.turn[j] = scaled >= 18446744073709551615.0L ? ~uint64_t(0) : static_cast<uint64_t>(scaled);
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64) return launch_proj<64>(hidden, S, d, W_qkv, static_cast<int32_t>(N), out, st, "proj_gemm_kernel<qkv64>");
  return launch_proj<128>(hidden, S, d, W_qkv, static_cast<int32_t>(N), out, st, "proj_gemm_kernel<qkv128>");
}
