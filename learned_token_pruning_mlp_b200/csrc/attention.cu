// attention.cu -- tg_gated_attention / tg_gated_attention_varlen: token-gated
// causal GQA attention over the kept tokens.
//
// TokenGate article, "What is token-gated attention?": each kept token's gate
// score becomes a bias on the attention logits of the layers above the gate,
// with a learnable per-head gain and a learnable temperature.  For query row i,
// head h, KV head g = h / (Hq/Hkv):
//     logit(i,j) = tau * Q[i,h].K[j,g] / sqrt(D) + gain[h] * s[j]   (j <= i)
//     O[i,h]     = softmax_j(logit(i,.)) V[., g]
// Without scores (s = NULL) the call is plain causal GQA attention: the kernel
// instantiation without the bias step runs (tau = 0 keeps it, with a block of zeros).
//
// Two kernels.  When the grid below would hold at most 1.5 CTAs per SM (a short
// sequence: S = 2560 with 16 heads is 160 CTAs on 148 SMs) the call runs the persistent
// kernel of attention_persistent.cu instead, one CTA per SM working through single
// query tiles, which fills the SMs and balances the causal triangle; longer sequences
// run the kernel below, whose CTAs share each K/V tile between two query tiles.
//
// B200 design (flash-style, one CTA per pair of 128-row query tiles of one head):
//   * TMEM (512 columns): S_0, S_1 (128 fp32 columns each, one per query tile),
//     O_0, O_1 (D columns each).  The bf16 probabilities P_t are written back over
//     the first 64 columns of S_t and fed to the PV product straight from TMEM.
//   * The key bias rides on the tensor core: with c_j = gain_h*log2(e)*s_j / scale
//     (scale = tau*log2(e)/sqrt(D)), one extra K=16 MMA step multiplies a constant
//     [1, 1, 1, 0...] block of Q by a [c0, c1, c2, 0...] block of K (c_j split into
//     three bf16 parts, exact to 2^-24 relative), so S'_ij = q_i.k_j + c_j and the
//     base-2 logit is scale * S'_ij: the softmax needs one FMA per logit, as without
//     a bias.  tau < 0 negates the A operand (so the largest logit is still the
//     largest S'); tau = 0 skips the Q.K steps.
//   * warp 0 (one lane) loads Q once and streams K/V tiles of 128 keys through a
//     TMA pipeline (128-byte swizzle).  K and V stages are freed apart: a K stage as
//     soon as the S' products of its tile complete, a V stage when its PV products do,
//     so each K load has a whole KV step to land before its product is issued (with
//     one release per K/V pair, the next K load could only start once the tile after
//     it had been multiplied, and the tensor core waited on it every step); warp 3
//     writes the c_j block of each tile into
//     shared memory from plain loads of the scores (request offsets need not be
//     16-byte aligned, which a TMA copy would require).
//   * warp 1 (one lane) issues every tcgen05.mma: S_t = [1 Q] [c K]^T (K-major
//     operands in shared memory) and O_t += P_t V_j (P from TMEM, V MN-major in
//     shared memory).  The MMAs of one thread execute in issue order, so S_t(j+1) may
//     be issued right after O_t += P_t(j) V_j even though it overwrites P_t(j).
//   * warps 4-7 and 8-11 are the softmax warpgroups of tile 0 and tile 1 (one query
//     row per thread): tcgen05.ld of the S' row, causal mask on the diagonal tile,
//     exp2 of one packed f32x2 FMA per pair against the running max with the tile's
//     max taken in the same pass, bf16 pack, 8-way sum of the rounded weights with
//     mixed-precision adds (so normalisation matches the weights the PV product
//     uses), tcgen05.st of P.  While one warpgroup works on its softmax the tensor core
//     works on the other tile's products.
//   * The running max is only moved when it grows by more than 2^8 for some row of
//     the warp (decided per warp: TMEM access is warp-collective); then O_t is
//     rescaled in TMEM after P is stored (S_t(j) completing orders this after O_t's
//     previous product).  Otherwise exponentials are taken against the stale max,
//     which stays exact in fp32 and loses nothing in bf16.
//   * The epilogue divides O by the row sum and converts it to bf16; a whole tile is
//     staged in shared memory (over its finished Q tile) and written by one tensor
//     store, a partial tile row by row.  For training it also stores each row's
//     log-sum-exp (natural log), from which
//     the backward recomputes the probabilities, and optionally the output before its
//     bf16 rounding (fp32), from which the backward forms dO . O.
//   * CTAs are ordered heaviest first (the longest causal rows), which the hardware
//     block scheduler turns into a longest-processing-time schedule.
#include <algorithm>
#include <cmath>

#include "internal.h"
#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kBM = 128;   // query rows per tile
constexpr int kBN = 128;   // keys per KV tile
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kHalfBytes = kBM * 64 * 2;  // one 128-row x 64-column swizzled block (16 KB)
constexpr uint32_t kExtBytes = kBM * 16 * 2;   // one 128-row x 16-column unswizzled block (4 KB)
constexpr uint32_t kExtLBO = kExtBytes / 2;    // columns 8..15 follow columns 0..7
constexpr uint32_t kExtSBO = 128;              // 8 rows x 16 bytes per core matrix

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kTileBytes = kHalfBytes * kHalves;  // 128 rows x D bf16
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr size_t kSmem = 1024 + 2 * kTileBytes + 2 * static_cast<size_t>(kStages) * kTileBytes +
                                  (1 + kStages) * static_cast<size_t>(kExtBytes) + 256;
};

struct AttnCtl {
  uint64_t q_full;
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t k_empty[4];
  uint64_t v_empty[4];
  uint64_t bias_full[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_final;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// kBias: the key-bias step is part of every S' product (with scores, or with tau = 0
// where it is the whole product); without it the kernel is plain causal attention.
template <int D, bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    gated_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                           const float *__restrict__ key_scores,
                           const float *__restrict__ gain, float scale_log2, const int32_t *__restrict__ cu_seqlens,
                           int64_t S_single, int64_t total, int n_mblocks, int B, int Hq, int Hkv,
                           __nv_bfloat16 *__restrict__ O, float *__restrict__ lse, float *__restrict__ O32,
                           uint32_t *err) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                                  // [2][tile]
  uint8_t *sK = sQ + 2 * C::kTileBytes;                // [NS][tile]
  uint8_t *sV = sK + NS * C::kTileBytes;               // [NS][tile]
  uint8_t *sQx = sV + NS * C::kTileBytes;              // [128 x 16] block of ones (columns 0..2)
  uint8_t *sKx = sQx + kExtBytes;                      // [NS][128 x 16] blocks of c_j (columns 0..2)
  AttnCtl *ctl = reinterpret_cast<AttnCtl *>(sKx + NS * kExtBytes);
  tg::pdl_wait();
  tg::pdl_trigger();

  // ---- work unit: heaviest query blocks first, then request, then head
  const int per_mb = Hq * B;
  const int mb = n_mblocks - 1 - static_cast<int>(blockIdx.x) / per_mb;
  const int rest = static_cast<int>(blockIdx.x) % per_mb;
  const int b = rest / Hq;
  const int h = rest % Hq;
  const int g = h / (Hq / Hkv);
  int64_t seg_start = 0, len = S_single;
  if (cu_seqlens) {
    int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
    // one CTA per request reports a malformed range or a request past the grid's rows
    // (longer than max_seqlen), whose remaining rows no CTA computes
    if (threadIdx.x == 0 && h == 0 && mb == n_mblocks - 1 &&
        (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > static_cast<int64_t>(n_mblocks) * 2 * kBM))
      tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
    s0 = s0 < 0 ? 0 : (s0 > total ? total : s0);
    s1 = s1 < s0 ? s0 : (s1 > total ? total : s1);
    seg_start = s0;
    len = s1 - s0;
  }
  const int64_t row0 = static_cast<int64_t>(mb) * 2 * kBM;
  if (row0 >= len) return;  // uniform over the CTA
  const int n0 = 2 * mb + 1;                              // KV tiles of query tile 0 (its diagonal is tile 2mb)
  const int n1 = (row0 + kBM < len) ? 2 * mb + 2 : 0;     // query tile 1 (0 = beyond the request)
  const int n_kv = n1 ? n1 : n0;

  // ---- logit scaling: base-2 logit = eff * S', S' = (+/-)(q.k + c_j)
  const bool skip_qk = (scale_log2 == 0.f);
  const float eff = skip_qk ? 1.f : fabsf(scale_log2);
  const bool has_bias = key_scores != nullptr;  // kBias without scores: a block of zeros
  const float cmul = has_bias ? gain[h] * kLog2e / (skip_qk ? 1.f : scale_log2) : 0.f;

  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;

  // constant [1, 1] columns of the extended Q block, zeros elsewhere (also in the c_j blocks)
  for (uint32_t w = threadIdx.x; w < (1 + NS) * kExtBytes / 4; w += kThreads) {
    uint32_t v = 0;
    if (w < kExtLBO / 4 && (w & 3u) == 0) v = 0x3F803F80u;  // bf16 1.0 in columns 0, 1 of each row
    if (w < kExtLBO / 4 && (w & 3u) == 1) v = 0x00003F80u;  // and in column 2
    reinterpret_cast<uint32_t *>(sQx)[w] = v;
  }
  tg::fence_proxy_async_smem();

  if (threadIdx.x == 0) {
    tg::mbar_init(tg::smem_addr(&ctl->q_full), 1);
    for (int s = 0; s < NS; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->k_full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->v_full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->k_empty[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->v_empty[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->bias_full[s]), 32);
    }
    for (int t = 0; t < 2; ++t) {
      tg::mbar_init(tg::smem_addr(&ctl->s_full[t]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->p_full[t]), 128);
    }
    tg::mbar_init(tg::smem_addr(&ctl->o_final), 1);
    tg::mbar_init(tg::smem_addr(&ctl->drain), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
    tg::prefetch_tmap(&tm_q);
    tg::prefetch_tmap(&tm_k);
    tg::prefetch_tmap(&tm_v);
    tg::prefetch_tmap(&tm_o);
  }
  if (warp == 2) {
    tg::tmem_alloc(tg::smem_addr(&ctl->tmem_base), 512);
    tg::tmem_relinquish();
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int *abort_flag = &ctl->abort_flag;

  // Register split: the launch gives 384 threads x 168 registers; the loader/MMA
  // warpgroup needs few, the two softmax warpgroups hold a 128-wide S row each.
  // 128 x 64 + 256 x 216 = 63488 <= 384 x 168, so the increase never waits (the
  // launcher checks the launch count).  Each warpgroup changes its budget inside its
  // own branch.
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    const int nq = n1 ? 2 : 1;
    const uint32_t qbar = tg::smem_addr(&ctl->q_full);
    tg::mbar_arrive_expect_tx(qbar, nq * C::kTileBytes);
    for (int t = 0; t < nq; ++t)
      for (int hf = 0; hf < C::kHalves; ++hf)
        tg::tma_load_3d(tg::smem_addr(sQ + t * C::kTileBytes + hf * kHalfBytes), &tm_q, qbar, hf * 64, h,
                        static_cast<int32_t>(seg_start + row0 + t * kBM));
    for (int j = 0; j < n_kv; ++j) {
      const int s = j % NS;
      const uint32_t ph = (j / NS) & 1;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->k_empty[s]), ph ^ 1u, abort_flag)) break;
      const int32_t krow = static_cast<int32_t>(seg_start + static_cast<int64_t>(j) * kBN);
      const uint32_t kb = tg::smem_addr(&ctl->k_full[s]);
      tg::mbar_arrive_expect_tx(kb, C::kTileBytes);
      for (int hf = 0; hf < C::kHalves; ++hf)
        tg::tma_load_3d(tg::smem_addr(sK + s * C::kTileBytes + hf * kHalfBytes), &tm_k, kb, hf * 64, g, krow);
      if (!tg::mbar_wait(tg::smem_addr(&ctl->v_empty[s]), ph ^ 1u, abort_flag)) break;
      const uint32_t vb = tg::smem_addr(&ctl->v_full[s]);
      tg::mbar_arrive_expect_tx(vb, C::kTileBytes);
      for (int hf = 0; hf < C::kHalves; ++hf)
        tg::tma_load_3d(tg::smem_addr(sV + s * C::kTileBytes + hf * kHalfBytes), &tm_v, vb, hf * 64, g, krow);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ key-bias block writer
    for (int j = 0; j < n_kv; ++j) {
      const int s = j % NS;
      const uint32_t ph = (j / NS) & 1;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->k_empty[s]), ph ^ 1u, abort_flag)) break;
#pragma unroll
      for (int e = 0; e < kBN / 32; ++e) {
        const int r = e * 32 + lane;
        const int64_t kv = static_cast<int64_t>(j) * kBN + r;
        const float c = has_bias && kv < len ? cmul * key_scores[seg_start + kv] : 0.f;
        // c_j in three bf16 parts (their sum is c_j to 2^-24 relative)
        const __nv_bfloat16 p0 = __float2bfloat16_rn(c);
        const float r1 = c - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
        uint8_t *row = sKx + s * kExtBytes + r * 16;  // row r, columns 0..2
        *reinterpret_cast<__nv_bfloat162 *>(row) = __halves2bfloat162(p0, p1);
        *reinterpret_cast<__nv_bfloat16 *>(row + 4) = p2;
      }
      tg::fence_proxy_async_smem();
      tg::mbar_arrive(tg::smem_addr(&ctl->bias_full[s]));
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = tg::idesc_bf16_f32(kBM, kBN, false, false) | (scale_log2 < 0.f ? (1u << 13) : 0u);
    constexpr uint32_t idesc_o = tg::idesc_bf16_f32(kBM, D, false, true);
    bool ok = tg::mbar_wait(tg::smem_addr(&ctl->q_full), 0, abort_flag);

    // Shared-memory descriptors, built once: a descriptor is two 32-bit words, and the
    // operand of each K step differs from its tile's by a constant offset added to the
    // start-address field of the low word (16-byte units, 14 bits; shared addresses stay
    // below 2^18 bytes, so the add never carries out of the field).  This keeps the
    // issuing thread's instruction count per MMA low: it shares its SM sub-partition
    // with two softmax warps.
    const uint64_t dsw = tg::smem_desc_sw128(tg::smem_addr(sQ), 16, 1024);
    const uint32_t hi_sw = static_cast<uint32_t>(dsw >> 32);
    const uint32_t q_lo0 = static_cast<uint32_t>(dsw);
    const uint32_t k_lo0 = static_cast<uint32_t>(tg::smem_desc_sw128(tg::smem_addr(sK), 16, 1024));
    const uint64_t dv = tg::smem_desc_sw128(tg::smem_addr(sV), kHalfBytes, 1024);
    const uint32_t v_lo0 = static_cast<uint32_t>(dv), hi_v = static_cast<uint32_t>(dv >> 32);
    const uint64_t dqx = tg::smem_desc_noswz(tg::smem_addr(sQx), kExtLBO, kExtSBO);
    const uint64_t dkx = tg::smem_desc_noswz(tg::smem_addr(sKx), kExtLBO, kExtSBO);
    const uint32_t kx_lo0 = static_cast<uint32_t>(dkx), hi_x = static_cast<uint32_t>(dkx >> 32);
    constexpr uint32_t kTileUnits = C::kTileBytes >> 4;

    auto issue_s = [&](int t, int j) {
      const uint32_t s = static_cast<uint32_t>(j % NS);
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(t * kBN);
      if constexpr (kBias) tg::mma_bf16_ss(d_tmem, dqx, tg::desc_words(kx_lo0 + s * (kExtBytes >> 4), hi_x), idesc_s, 0u);
      if (!skip_qk) {
        const uint32_t q_lo = q_lo0 + static_cast<uint32_t>(t) * kTileUnits, k_lo = k_lo0 + s * kTileUnits;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
          tg::mma_bf16_ss(d_tmem, tg::desc_words(q_lo + off, hi_sw), tg::desc_words(k_lo + off, hi_sw), idesc_s,
                          (kBias || kk > 0) ? 1u : 0u);
        }
      }
      tg::mma_commit(tg::smem_addr(&ctl->s_full[t]));
    };
    auto issue_pv = [&](int t, int j) {
      const uint32_t s = static_cast<uint32_t>(j % NS);
      const uint32_t d_tmem = tmem_base + 256u + static_cast<uint32_t>(t * D);
      const uint32_t p_tmem = tmem_base + static_cast<uint32_t>(t * kBN);
      const uint32_t v_lo = v_lo0 + s * kTileUnits;
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        // 16 keys = 16 rows of V (2 swizzle groups of 8 rows, 2048 bytes); D blocks 16 KB apart
        const uint64_t bd = tg::desc_words(v_lo + static_cast<uint32_t>(kk) * (2048u >> 4), hi_v);
        tg::mma_bf16_ts(d_tmem, p_tmem + kk * 8u, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
      }
    };
    auto wait_k = [&](int j) {
      return tg::mbar_wait(tg::smem_addr(&ctl->k_full[j % NS]), (j / NS) & 1u, abort_flag) &&
             tg::mbar_wait(tg::smem_addr(&ctl->bias_full[j % NS]), (j / NS) & 1u, abort_flag);
    };

    if (ok && (ok = wait_k(0))) {
      tg::tc_fence_after();
      issue_s(0, 0);
      if (n1) issue_s(1, 0);
      tg::mma_commit(tg::smem_addr(&ctl->k_empty[0]));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const int s = j % NS;
      if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->v_full[s]), (j / NS) & 1u, abort_flag))) break;
      bool next_k_ready = false;
      if (j < n0) {
        if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->p_full[0]), j & 1u, abort_flag))) break;
        tg::tc_fence_after();
        issue_pv(0, j);
        if (j + 1 < n0) {
          if (!(ok = wait_k(j + 1))) break;
          next_k_ready = true;
          tg::tc_fence_after();
          issue_s(0, j + 1);
        }
      }
      if (j < n1) {
        if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->p_full[1]), j & 1u, abort_flag))) break;
        tg::tc_fence_after();
        issue_pv(1, j);
      }
      tg::mma_commit(tg::smem_addr(&ctl->v_empty[s]));  // V_j's last product
      if (j + 1 < n1) {
        if (!next_k_ready && !(ok = wait_k(j + 1))) break;
        tg::tc_fence_after();
        issue_s(1, j + 1);
      }
      if (j + 1 < n_kv) tg::mma_commit(tg::smem_addr(&ctl->k_empty[(j + 1) % NS]));  // K_{j+1}'s last product
    }
    if (ok) tg::mma_commit(tg::smem_addr(&ctl->o_final));
    if (*abort_flag) {
      tg::mma_commit(tg::smem_addr(&ctl->drain));
      int local_abort = 0;
      tg::mbar_wait(tg::smem_addr(&ctl->drain), 0, &local_abort, 100000000ull);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;" ::: "memory");
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;          // query tile of this warpgroup
    const int quarter = warp & 3;           // TMEM lane quarter
    const int r = quarter * 32 + lane;      // row within the tile
    const int n_t = t ? n1 : n0;
    const int64_t rt = row0 + t * kBM;      // first row of the tile (request-relative)
    const int diag = static_cast<int>(rt / kBN);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_taddr = tmem_base + static_cast<uint32_t>(t * kBN) + lane_off;
    const uint32_t o_taddr = tmem_base + 256u + static_cast<uint32_t>(t * D) + lane_off;
    const uint64_t eff2 = tg::f2_pack(eff, eff);
    float m = -INFINITY, l = 0.f;           // running max of S' (S' units) and row sum
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->s_full[t]), j & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tg::tc_fence_after();
      uint32_t x[kBN];
      // the S' row of this tile from TMEM, causal mask on the diagonal tile
      auto load_row = [&]() {
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tg::tmem_ld32(s_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));
        tg::tmem_ld_wait();
        if (j == diag) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c > r) x[c] = __float_as_uint(-INFINITY);
        }
      };
      float acc[8], mx[8];
      // exp2(eff S' - eff m) for the row, packed to bf16 in place (pair c into x[c]) and
      // summed as rounded; with want_max, the row's max is taken from the same reads
      auto exp_pass = [&](float m_used, bool want_max) {
        const float nms = -m_used * eff;
        const uint64_t nms2 = tg::f2_pack(nms, nms);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          acc[k] = 0.f;
          mx[k] = -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < kBN / 2; ++c) {
          const float s0 = __uint_as_float(x[2 * c]), s1 = __uint_as_float(x[2 * c + 1]);
          if (want_max) mx[c & 7] = tg::fmax3(mx[c & 7], s0, s1);
          const uint64_t arg = tg::f2_fma(tg::f2_pack(s0, s1), eff2, nms2);
          float a0, a1;
          tg::f2_unpack(arg, a0, a1);
          const uint32_t pb = pack_bf16x2(tg::ex2_approx(a0), tg::ex2_approx(a1));
          x[c] = pb;  // in place: x[c] is no longer needed once read above
          // the row sum adds the same bf16-rounded weights the PV product uses, so every
          // output row is an exact convex combination of its value rows
          tg::add_bf16x2_to_f32(acc[(2 * c) & 7], acc[(2 * c + 1) & 7], pb);
        }
      };
      auto row_max = [&]() {
        return fmaxf(tg::fmax3(mx[0], mx[1], mx[2]), tg::fmax3(tg::fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
      };
      load_row();
      float alpha = 1.f;
      bool rescale;
      if (j == 0) {
        // first tile: the max first (there is no running max to use yet); 8 running maxima
        // over the 64 pairs of the row
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN / 2; ++c)
          mx[c & 7] = tg::fmax3(mx[c & 7], __uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1]));
        const float m_new = fmaxf(m, row_max());
        // taken per warp: the TMEM loads and stores of the rescale are warp-collective
        rescale = __any_sync(0xFFFFFFFFu, (m_new - m) * eff > kRescaleLog2);
        if (rescale) {
          alpha = tg::ex2_approx((m - m_new) * eff);
          m = m_new;
        }
        exp_pass(m, false);
      } else {
        // exponentials against the running max, the tile's max taken in the same pass (the
        // max then costs no time of its own: the pass waits on the MUFU); only when the max
        // grows past the rescale threshold is the row read again from TMEM and redone
        exp_pass(m, true);
        const float m_new = fmaxf(m, row_max());
        rescale = __any_sync(0xFFFFFFFFu, (m_new - m) * eff > kRescaleLog2);
        if (rescale) {
          alpha = tg::ex2_approx((m - m_new) * eff);
          m = m_new;
          load_row();
          exp_pass(m, false);
        }
      }
      tg::tmem_st32(s_taddr, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tg::tmem_st32(s_taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
      l = fmaf(l, alpha, ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
      if (rescale && j > 0) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tg::tmem_ld32(o_taddr + c * 32, o);
          tg::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tg::tmem_st32(o_taddr + c * 32, o);
        }
      }
      tg::tmem_st_wait();
      tg::tc_fence_before();
      tg::mbar_arrive(tg::smem_addr(&ctl->p_full[t]));
    }
    // A whole tile of bf16 output leaves through shared memory and a tensor store:
    // the rows are staged in the 128-byte-swizzled layout the tensor map expects, over
    // this tile's Q buffer (every product has completed), and written as full 128-byte
    // lines.  A partial tile (its rows past the end of the request may belong to the
    // next one) and the fp32 copy are stored row by row.
    const bool staged = !O32 && rt + kBM <= len;  // uniform over the warpgroup
    uint8_t *stage = sQ + t * C::kTileBytes;
    if (ok && n_t > 0 && tg::mbar_wait_warp(tg::smem_addr(&ctl->o_final), 0, abort_flag)) {
      tg::tc_fence_after();
      const float inv_l = 1.0f / l;
      const int64_t row = rt + r;
      // base-2 log of sum_j 2^(eff S'_j) is eff m + log2 l (m the max the weights used)
      if (lse && row < len) lse[(seg_start + row) * Hq + h] = (m * eff + __log2f(l)) * 0.6931471805599453f;
      __nv_bfloat16 *orow = O + ((seg_start + row) * Hq + h) * static_cast<int64_t>(D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tg::tmem_ld32(o_taddr + c * 32, o);
        tg::tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (staged) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = (c & 1) * 4 + q;  // 16-byte chunk within the 64-column half c / 2
            *reinterpret_cast<uint4 *>(stage + (c >> 1) * kHalfBytes + r * 128 + ((ch ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
          continue;
        }
        if (O32 && row < len) {
          float4 *d32 = reinterpret_cast<float4 *>(O32 + ((seg_start + row) * Hq + h) * static_cast<int64_t>(D) + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d32[q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                 __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
        }
        if (row < len) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
    }
    if (staged) {
      // every warp of the warpgroup arrives here, also after a failed wait (no store then)
      tg::fence_proxy_async_smem();
      if (t == 0) asm volatile("bar.sync 1, 128;" ::: "memory");  // this warpgroup's rows are staged
      else asm volatile("bar.sync 2, 128;" ::: "memory");
      if (quarter == 0 && lane == 0 && !*abort_flag) {
        for (int hf = 0; hf < C::kHalves; ++hf)
          tg::tma_store_3d(&tm_o, tg::smem_addr(stage + hf * kHalfBytes), hf * 64, h,
                           static_cast<int32_t>(seg_start + rt));
        tg::bulk_commit();
        tg::bulk_wait_read_all();  // the staging buffer is read before the CTA exits
      }
    }
  }

  tg::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ctl->abort_flag) tg::set_device_error(err, TG_DEVERR_TIMEOUT);
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem_base, 512);
  }
}

template <int D, bool kBias>
tg_status launch_kernel(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain, float tau,
                 const int32_t *cu_seqlens, int32_t B, int64_t total, int64_t max_seqlen, int32_t Hq, int32_t Hkv,
                 tg_bf16 *O, float *lse, float *O32, cudaStream_t stream, uint32_t *err) {
  using C = Cfg<D>;
  CUtensorMap tm_q, tm_k, tm_v, tm_o;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(Hq), static_cast<uint64_t>(total)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hq) * D * 2};
    const uint32_t box[3] = {64, 1, kBM};
    if (!tg::encode_tmap(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
    // O has Q's shape; its map serves the tensor stores of whole output tiles
    if (!tg::encode_tmap(&tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, O, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(Hkv), static_cast<uint64_t>(total)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hkv) * D * 2};
    const uint32_t box[3] = {64, 1, kBN};
    if (!tg::encode_tmap(&tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Kc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
    if (!tg::encode_tmap(&tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  static tg::PerDevice configured;
  const tg_status setup = tg::once_per_device(configured, [&](int) -> tg_status {
    const cudaError_t e = cudaFuncSetAttribute(gated_attention_kernel<D, kBias>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    // the warpgroup register split in the kernel assumes 168 registers per thread at launch
    cudaFuncAttributes fa;
    const cudaError_t ea = cudaFuncGetAttributes(&fa, gated_attention_kernel<D, kBias>);
    if (ea != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(ea));
    if (fa.numRegs != 168)
      return tg::fail(TG_ERR_UNSUPPORTED, "gated_attention_kernel built with %d registers per thread; the register "
                      "split needs 168", fa.numRegs);
    return TG_OK;
  });
  if (setup != TG_OK) return setup;
  const float scale_log2 = tau / std::sqrt(static_cast<float>(D)) * kLog2e;
  const int n_mblocks = static_cast<int>((max_seqlen + 2 * kBM - 1) / (2 * kBM));
  const int64_t grid = static_cast<int64_t>(n_mblocks) * Hq * B;
  if (grid == 0) return TG_OK;
  if (grid > 0x7FFFFFFFLL) return tg::fail(TG_ERR_UNSUPPORTED, "grid too large");
  const cudaError_t e = tg::launch_pdl(gated_attention_kernel<D, kBias>, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                                      C::kSmem, stream, tm_q, tm_k, tm_v, tm_o, s, gain, scale_log2, cu_seqlens,
                                      cu_seqlens ? int64_t(0) : total, total, n_mblocks, B, Hq, Hkv,
                                      reinterpret_cast<__nv_bfloat16 *>(O), lse, O32, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "gated_attention_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("gated_attention_kernel");
}

template <int D>
tg_status launch(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain, float tau,
                 const int32_t *cu_seqlens, int32_t B, int64_t total, int64_t max_seqlen, int32_t Hq, int32_t Hkv,
                 tg_bf16 *O, float *lse, float *O32, cudaStream_t stream, uint32_t *err) {
  if (tg::attention_uses_persistent(max_seqlen, Hq, B))
    return tg::gated_attention_persistent(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, D, O,
                                          lse, O32, stream, err);
  // plain causal attention leaves the bias step out; with tau = 0 it is the whole product
  if (s || tau == 0.f)
    return launch_kernel<D, true>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                                  stream, err);
  return launch_kernel<D, false>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                                 stream, err);
}

tg_status validate(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain,
                   float tau, int64_t total, int32_t Hq, int32_t Hkv, int32_t D, tg_bf16 *O) {
  if (total < 0) return tg::fail(TG_ERR_INVALID_ARG, "sequence length must be >= 0");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
    return tg::fail(TG_ERR_INVALID_ARG, "Hq must be a positive multiple of Hkv (got %d, %d)", Hq, Hkv);
  if (D != 64 && D != 128) return tg::fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (!std::isfinite(tau)) return tg::fail(TG_ERR_INVALID_ARG, "tau must be finite");
  if (total * Hq >= 0x7FFFFFFFLL) return tg::fail(TG_ERR_UNSUPPORTED, "S * Hq must be below 2^31");
  if (total == 0) return TG_OK;
  if (!Q || !Kc || !V || !O) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (s && !gain) return tg::fail(TG_ERR_INVALID_ARG, "gain is NULL");
  if (!tg::aligned16(Q) || !tg::aligned16(Kc) || !tg::aligned16(V) || !tg::aligned16(O))
    return tg::fail(TG_ERR_ALIGNMENT, "Q, Kc, V and O must be 16-byte aligned");
  return TG_OK;
}

}  // namespace

namespace tg {

bool attention_uses_persistent(int64_t max_seqlen, int32_t Hq, int32_t B) {
  const int64_t two_tile_ctas = (max_seqlen + 2 * kBM - 1) / (2 * kBM) * Hq * B;
  return 2 * two_tile_ctas <= 3 * static_cast<int64_t>(sm_count());
}

}  // namespace tg

extern "C" tg_status tg_gated_attention(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s,
                                        const float *gain, float tau, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                        tg_bf16 *O, tg_stream stream) {
  TG_API_ENTRY();
  tg_status st = validate(Q, Kc, V, s, gain, tau, S, Hq, Hkv, D, O);
  if (st != TG_OK || S == 0) return st;
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128>(Q, Kc, V, s, gain, tau, nullptr, 1, S, S, Hq, Hkv, O, nullptr, nullptr, cs, err)
                  : launch<64>(Q, Kc, V, s, gain, tau, nullptr, 1, S, S, Hq, Hkv, O, nullptr, nullptr, cs, err);
}

extern "C" tg_status tg_gated_attention_train(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s,
                                              const float *gain, float tau, int64_t S, int32_t Hq, int32_t Hkv,
                                              int32_t D, tg_bf16 *O, float *lse, float *O32, tg_stream stream) {
  TG_API_ENTRY();
  tg_status st = validate(Q, Kc, V, s, gain, tau, S, Hq, Hkv, D, O);
  if (st != TG_OK || S == 0) return st;
  if (!lse) return tg::fail(TG_ERR_INVALID_ARG, "lse is NULL");
  if (O32 && !tg::aligned16(O32)) return tg::fail(TG_ERR_ALIGNMENT, "O32 must be 16-byte aligned");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128>(Q, Kc, V, s, gain, tau, nullptr, 1, S, S, Hq, Hkv, O, lse, O32, cs, err)
                  : launch<64>(Q, Kc, V, s, gain, tau, nullptr, 1, S, S, Hq, Hkv, O, lse, O32, cs, err);
}

extern "C" tg_status tg_gated_attention_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s,
                                               const float *gain, float tau, const int32_t *cu_seqlens, int32_t B,
                                               int64_t total, int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                               tg_bf16 *O, tg_stream stream) {
  TG_API_ENTRY();
  if (B < 0) return tg::fail(TG_ERR_INVALID_ARG, "B must be >= 0");
  if (max_seqlen < 0 || max_seqlen > total) return tg::fail(TG_ERR_INVALID_ARG, "max_seqlen must be in [0, total]");
  if (B > 0 && !cu_seqlens) return tg::fail(TG_ERR_INVALID_ARG, "cu_seqlens is NULL");
  tg_status st = validate(Q, Kc, V, s, gain, tau, total, Hq, Hkv, D, O);
  if (st != TG_OK || total == 0 || B == 0) return st;
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, nullptr, nullptr, cs, err)
                  : launch<64>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, nullptr, nullptr, cs, err);
}

extern "C" tg_status tg_gated_attention_train_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                                     const float *s, const float *gain, float tau,
                                                     const int32_t *cu_seqlens, int32_t B, int64_t total,
                                                     int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                                     tg_bf16 *O, float *lse, float *O32, tg_stream stream) {
  TG_API_ENTRY();
  if (B < 0) return tg::fail(TG_ERR_INVALID_ARG, "B must be >= 0");
  if (max_seqlen < 0 || max_seqlen > total) return tg::fail(TG_ERR_INVALID_ARG, "max_seqlen must be in [0, total]");
  if (B > 0 && !cu_seqlens) return tg::fail(TG_ERR_INVALID_ARG, "cu_seqlens is NULL");
  tg_status st = validate(Q, Kc, V, s, gain, tau, total, Hq, Hkv, D, O);
  if (st != TG_OK || total == 0 || B == 0) return st;
  if (!lse) return tg::fail(TG_ERR_INVALID_ARG, "lse is NULL");
  if (O32 && !tg::aligned16(O32)) return tg::fail(TG_ERR_ALIGNMENT, "O32 must be 16-byte aligned");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32, cs, err)
                  : launch<64>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32, cs, err);
}
