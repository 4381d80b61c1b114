// attention_persistent.cu -- token-gated causal GQA attention, persistent form for
// short sequences (few query tiles per head), behind tg_gated_attention and its
// varlen / training forms.  attention.cu chooses between this kernel and the two-tile
// kernel there by the size of the two-tile grid (see tg::attention_uses_persistent).
//
// TokenGate article, "What is token-gated attention?": each kept token's gate score
// becomes a bias on the attention logits of the layers above the gate, with a learnable
// per-head gain and a learnable temperature:
//     logit(i,j) = tau * Q[i,h].K[j,g] / sqrt(D) + gain[h] * s[j]   (j <= i)
//     O[i,h]     = softmax_j(logit(i,.)) V[., g]
//
// Why a second kernel: the two-tile kernel gives each CTA two 128-row query tiles of one
// head, so a short sequence launches fewer CTAs than there are SMs (S = 1536 with 16 heads
// is 96 CTAs on 148 SMs) and the causal triangle leaves the CTAs unevenly loaded.  Here one
// CTA per SM works through a list of (request, 128-row query tile, head) items, heaviest
// first, dealt to the CTAs in alternating directions (CTA c takes items c, 2G-1-c, 2G+c,
// ...), which keeps the per-SM totals within about one item of each other.
//   * TMEM (512 columns): two S buffers (128 fp32 columns each), O (D columns) and two Q
//     buffers (D / 2 columns of bf16 pairs each).  Step t of a CTA (its t-th KV tile over
//     all its items) computes S into buffer t % 2, so S(t+1) = Q K(t+1)^T runs on the
//     tensor core while the softmax works on S(t).  The bf16 probabilities are written over
//     their S buffer and feed the PV product from TMEM; S(t+2) is issued into that buffer
//     once PV(t) has completed.
//   * The key bias rides on the tensor core as in the two-tile kernel: with
//     c_j = gain_h*log2(e)*s_j / scale (scale = tau*log2(e)/sqrt(D)), one extra K=16 MMA
//     step multiplies a constant [1, 1, 1, 0...] block by a [c0, c1, c2, 0...] block
//     (c_j split into three bf16 parts), so S'_ij = q_i.k_j + c_j and the base-2 logit is
//     scale * S'_ij.  tau < 0 negates the A operand; tau = 0 skips the Q.K steps.
//   * warp 0 (one lane) streams the K tiles and warp 2 (one lane, after allocating TMEM)
//     the V tiles by TMA (128-byte swizzle); K and V stages are freed apart.  Warp 3 writes
//     the c_j block of each K stage from plain loads of the scores, then one lane issues
//     S(t) = [1 Q] [c K]^T (Q from TMEM, K from shared memory).  Warp 1 (one lane) issues
//     the PV products, so neither issuer's waits leave the tensor core idle while the
//     other has work queued.
//   * warps 4-7 and 8-11 are the softmax: one query row per thread, warps 4-7 over keys
//     0-63 of each S tile and warps 8-11 over keys 64-127, so each SM sub-partition runs
//     two softmax warps on the same rows and their exponentials keep the MUFU busy (one
//     warp alone leaves it idle between dependent instructions).  The two warps of a TMEM
//     lane quarter swap their halves' tile maxima through shared memory at a named
//     barrier once per tile.  Exponentials are taken against the running max with the
//     tile's max found in the same pass; the running max only moves when it grows by more
//     than 2^8 for some row of the warp (both warps of a pair see the same maxima and
//     vote alike), and then each warp rescales its half of O's columns once the previous
//     PV product has completed.  Each half keeps the sum of its bf16-rounded weights (so
//     normalisation matches the weights the PV product uses); the epilogue adds the two.
//   * warps 12-15 (epilogue): load each item's Q rows from global memory straight into
//     its TMEM buffer two items ahead, then divide O by the row sum and convert to bf16; a
//     whole tile is staged in shared memory and written by one tensor store, a partial
//     tile row by row.  For training also each row's log-sum-exp (natural log) and
//     optionally the output before its bf16 rounding (fp32).
//   * Every wait is bounded (a timeout sets the device status word and the kernel
//     drains its tensor-core work and returns); a failure seen by one softmax warp reaches
//     its partner at their next shared barrier, so neither waits there alone.
#include <algorithm>
#include <cmath>

#include "internal.h"
#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kBM = 128;   // query rows per tile
constexpr int kBN = 128;   // keys per KV tile
constexpr int kThreads = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kHalfBytes = kBM * 64 * 2;  // one 128-row x 64-column swizzled block (16 KB)
constexpr uint32_t kExtBytes = kBM * 16 * 2;   // one 128-row x 16-column unswizzled block (4 KB)
constexpr uint32_t kExtLBO = kExtBytes / 2;    // columns 8..15 follow columns 0..7
constexpr uint32_t kExtSBO = 128;              // 8 rows x 16 bytes per core matrix
// Register budgets after the split (per thread): the loader / MMA / bias warpgroup, each
// softmax warpgroup (64 S values per row) and the epilogue.  128 x (72 + 2 x 152 + 128) =
// 64512 registers, within the 512 x 128 = 65536 a launch of 512 threads at 128 registers
// each holds (the launcher checks the count), so the increases never wait.
constexpr int kRegsLow = 72, kRegsSoftmax = 152, kRegsEpilogue = 128;

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kTileBytes = kHalfBytes * kHalves;  // 128 rows x D bf16
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr size_t kSmem = 1024 + kTileBytes + 2 * static_cast<size_t>(kStages) * kTileBytes +
                                  (1 + kStages) * static_cast<size_t>(kExtBytes) + 10 * kBM * sizeof(float) + 512;
  // TMEM columns: two S buffers, O, two Q buffers (bf16 pairs: D / 2 columns each)
  static constexpr uint32_t kTmemO = 2 * kBN;
  static constexpr uint32_t kTmemQ = 2 * kBN + D;
};

struct AttnCtl {
  uint64_t q_full[2];   // the item's Q tile is in its TMEM buffer
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t k_empty[4];
  uint64_t v_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];  // PV(t) has completed (buffer t % 2: one phase per product into it)
  uint64_t o_final;
  uint64_t o_empty;
  uint64_t l_full[2];
  uint64_t l_empty[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Named barrier of ``count`` threads that also returns whether ``pred`` held for any of them.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// One work item: a 128-row query tile of one head of one request.
struct Item {
  int64_t seg_start;  // first row of the request in the packed tensors
  int64_t len;        // rows of the request
  int64_t rt;         // first row of the tile, request-relative
  int h, g;           // query head and its KV head
  int n;              // KV tiles 0..n-1; the last one holds the diagonal
  bool valid;
};

// The items of one CTA in order.  Work w in [0, n_mt * Hq * B): query tile
// mt = n_mt - 1 - w / (Hq * B) (heaviest first), then request, then head; CTA c takes
// w = r * G + c in even rounds r and r * G + G - 1 - c in odd ones.  Items of requests
// shorter than the tile's start are skipped the same way by every role.
struct Sched {
  const int32_t *cu_seqlens;
  int64_t S_single, total;
  int n_mt, B, Hq, group, G, c;
  int r;

  __device__ Item next() {
    const int per_mt = Hq * B;
    const int64_t n_work = static_cast<int64_t>(n_mt) * per_mt;
    while (static_cast<int64_t>(r) * G < n_work) {
      const int pos = (r & 1) ? (G - 1 - c) : c;
      const int64_t w = static_cast<int64_t>(r) * G + pos;
      ++r;
      if (w >= n_work) continue;
      const int mt = n_mt - 1 - static_cast<int>(w / per_mt);
      const int rest = static_cast<int>(w % per_mt);
      const int b = rest / Hq;
      Item it;
      it.h = rest % Hq;
      it.g = it.h / group;
      it.seg_start = 0;
      it.len = S_single;
      if (cu_seqlens) {
        int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        s0 = s0 < 0 ? 0 : (s0 > total ? total : s0);
        s1 = s1 < s0 ? s0 : (s1 > total ? total : s1);
        it.seg_start = s0;
        it.len = s1 - s0;
      }
      it.rt = static_cast<int64_t>(mt) * kBM;
      if (it.rt >= it.len) continue;
      it.n = mt + 1;
      it.valid = true;
      return it;
    }
    Item none;
    none.valid = false;
    none.n = 0;
    return none;
  }
};

// kBias: the key-bias step is part of every S' product (with scores, or with tau = 0
// where it is the whole product); without it the kernel is plain causal attention.
template <int D, bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    gated_attention_persistent_kernel(const __nv_bfloat16 *__restrict__ Qg, const __grid_constant__ CUtensorMap tm_k,
                                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                                      const float *__restrict__ key_scores, const float *__restrict__ gain,
                                      float scale_log2, const int32_t *__restrict__ cu_seqlens, int64_t S_single,
                                      int64_t total, int n_mt, int B, int Hq, int Hkv, __nv_bfloat16 *__restrict__ O,
                                      float *__restrict__ lse, float *__restrict__ O32, uint32_t *err) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sStage = smem;                              // [tile] staged output tile
  uint8_t *sK = sStage + C::kTileBytes;                // [NS][tile]
  uint8_t *sV = sK + NS * C::kTileBytes;               // [NS][tile]
  uint8_t *sQx = sV + NS * C::kTileBytes;              // [128 x 16] block of ones (columns 0..2)
  uint8_t *sKx = sQx + kExtBytes;                      // [NS][128 x 16] blocks of c_j (columns 0..2)
  float *sL = reinterpret_cast<float *>(sKx + NS * kExtBytes);  // [2 items][2 halves][128] partial row sums
  float *sM = sL + 4 * kBM;                                      // [2][128] row maxima (base-2 logit units)
  float *sXm = sM + 2 * kBM;                                     // [2 steps][2 halves][128] partial tile maxima
  AttnCtl *ctl = reinterpret_cast<AttnCtl *>(sXm + 4 * kBM);
  tg::pdl_wait();
  tg::pdl_trigger();

  const Sched sched0{cu_seqlens, S_single, total, n_mt, B, Hq, Hq / Hkv, static_cast<int>(gridDim.x),
                     static_cast<int>(blockIdx.x), 0};

  // ---- logit scaling: base-2 logit = eff * S', S' = (+/-)(q.k + c_j)
  const bool skip_qk = (scale_log2 == 0.f);
  const float eff = skip_qk ? 1.f : fabsf(scale_log2);
  const bool has_bias = key_scores != nullptr;  // kBias without scores: a block of zeros

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
    for (int b = 0; b < 2; ++b) {
      tg::mbar_init(tg::smem_addr(&ctl->q_full[b]), 128);
      tg::mbar_init(tg::smem_addr(&ctl->s_full[b]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->p_full[b]), 256);
      tg::mbar_init(tg::smem_addr(&ctl->l_full[b]), 256);
      tg::mbar_init(tg::smem_addr(&ctl->l_empty[b]), 128);
    }
    tg::mbar_init(tg::smem_addr(&ctl->o_final), 1);
    tg::mbar_init(tg::smem_addr(&ctl->o_empty), 128);
    for (int s = 0; s < NS; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->k_full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->v_full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->k_empty[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->v_empty[s]), 1);
    }
    tg::mbar_init(tg::smem_addr(&ctl->pv_done[0]), 1);
    tg::mbar_init(tg::smem_addr(&ctl->pv_done[1]), 1);
    tg::mbar_init(tg::smem_addr(&ctl->drain[0]), 1);
    tg::mbar_init(tg::smem_addr(&ctl->drain[1]), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
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

  // Register split (kRegsLow / kRegsSoftmax / kRegsEpilogue): the loader/MMA warpgroup
  // needs few, each softmax warpgroup holds half an S row per thread, the epilogue one
  // 32-column slice of O.  Each warpgroup changes its budget inside its own branch.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow) : "memory");
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- K producer
      Sched sc = sched0;
      uint32_t t = 0;
      bool ok = true;
      for (Item it = sc.next(); it.valid && ok; it = sc.next()) {
        for (int j = 0; j < it.n; ++j, ++t) {
          const int s = static_cast<int>(t % NS);
          const uint32_t ph = (t / NS) & 1u;
          if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->k_empty[s]), ph ^ 1u, abort_flag))) break;
          const uint32_t kb = tg::smem_addr(&ctl->k_full[s]);
          tg::mbar_arrive_expect_tx(kb, C::kTileBytes);
          const int32_t krow = static_cast<int32_t>(it.seg_start + static_cast<int64_t>(j) * kBN);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tg::tma_load_3d(tg::smem_addr(sK + s * C::kTileBytes + hf * kHalfBytes), &tm_k, kb, hf * 64, it.g, krow);
        }
      }
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------------------- V producer
      Sched sc = sched0;
      uint32_t t = 0;
      bool ok = true;
      for (Item it = sc.next(); it.valid && ok; it = sc.next()) {
        for (int j = 0; j < it.n; ++j, ++t) {
          const int s = static_cast<int>(t % NS);
          const uint32_t ph = (t / NS) & 1u;
          if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->v_empty[s]), ph ^ 1u, abort_flag))) break;
          const uint32_t vb = tg::smem_addr(&ctl->v_full[s]);
          tg::mbar_arrive_expect_tx(vb, C::kTileBytes);
          const int32_t krow = static_cast<int32_t>(it.seg_start + static_cast<int64_t>(j) * kBN);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tg::tma_load_3d(tg::smem_addr(sV + s * C::kTileBytes + hf * kHalfBytes), &tm_v, vb, hf * 64, it.g, krow);
        }
      }
    } else if (warp == 3) {
      // ---------------------------------------------------------- key-bias blocks and S products
      // Per step: the warp writes the c_j block of the K stage (once the stage is free),
      // then one lane issues S(t) = [1 Q] [c K]^T into S buffer t % 2 once K(t) has
      // landed and PV(t - 2), the last reader of that buffer, has completed.  The PV
      // products are issued by another warp, so neither issuer's waits leave the
      // tensor core idle while the other has work queued.
      const uint32_t idesc_s = tg::idesc_bf16_f32(kBM, kBN, false, false) | (scale_log2 < 0.f ? (1u << 13) : 0u);
      const uint64_t dsw = tg::smem_desc_sw128(tg::smem_addr(sK), 16, 1024);
      const uint32_t hi_sw = static_cast<uint32_t>(dsw >> 32);
      const uint32_t k_lo0 = static_cast<uint32_t>(dsw);
      const uint64_t dqx = tg::smem_desc_noswz(tg::smem_addr(sQx), kExtLBO, kExtSBO);
      const uint64_t dkx = tg::smem_desc_noswz(tg::smem_addr(sKx), kExtLBO, kExtSBO);
      const uint32_t kx_lo0 = static_cast<uint32_t>(dkx), hi_x = static_cast<uint32_t>(dkx >> 32);
      constexpr uint32_t kTileUnits = C::kTileBytes >> 4;
      Sched sc = sched0;
      uint32_t t = 0;
      int k = 0;
      bool ok = true;
      for (Item it = sc.next(); it.valid && ok; it = sc.next(), ++k) {
        const float cmul = has_bias ? gain[it.h] * kLog2e / (skip_qk ? 1.f : scale_log2) : 0.f;
        for (int j = 0; j < it.n; ++j, ++t) {
          const uint32_t st = t % NS;
          const uint32_t ph = (t / NS) & 1u;
          if (!(ok = tg::mbar_wait_warp(tg::smem_addr(&ctl->k_empty[st]), ph ^ 1u, abort_flag))) break;
#pragma unroll
          for (int e = 0; e < kBN / 32; ++e) {
            const int r = e * 32 + lane;
            const int64_t kv = static_cast<int64_t>(j) * kBN + r;
            const float c = has_bias && kv < it.len ? cmul * key_scores[it.seg_start + kv] : 0.f;
            // c_j in three bf16 parts (their sum is c_j to 2^-24 relative)
            const __nv_bfloat16 p0 = __float2bfloat16_rn(c);
            const float r1 = c - __bfloat162float(p0);
            const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
            const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
            uint8_t *row = sKx + st * kExtBytes + r * 16;  // row r, columns 0..2
            *reinterpret_cast<__nv_bfloat162 *>(row) = __halves2bfloat162(p0, p1);
            *reinterpret_cast<__nv_bfloat16 *>(row + 4) = p2;
          }
          tg::fence_proxy_async_smem();
          __syncwarp();
          int good = 1;
          if (lane == 0) {
            good = (j > 0 || tg::mbar_wait(tg::smem_addr(&ctl->q_full[k & 1]), (k >> 1) & 1u, abort_flag)) &&
                   tg::mbar_wait(tg::smem_addr(&ctl->k_full[st]), ph, abort_flag) &&
                   (t < 2 || tg::mbar_wait(tg::smem_addr(&ctl->pv_done[t & 1u]), ((t >> 1) - 1u) & 1u, abort_flag));
            if (good) {
              tg::tc_fence_after();
              const uint32_t d_tmem = tmem_base + (t & 1u) * kBN;
              if constexpr (kBias)
                tg::mma_bf16_ss(d_tmem, dqx, tg::desc_words(kx_lo0 + st * (kExtBytes >> 4), hi_x), idesc_s, 0u);
              if (!skip_qk) {
                // Q from TMEM (8 columns = 16 bf16 per K step), K from shared memory
                const uint32_t q_tmem = tmem_base + C::kTmemQ + static_cast<uint32_t>(k & 1) * (D / 2);
                const uint32_t k_lo = k_lo0 + st * kTileUnits;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
                  tg::mma_bf16_ts(d_tmem, q_tmem + kk * 8u, tg::desc_words(k_lo + off, hi_sw), idesc_s,
                                  (kBias || kk > 0) ? 1u : 0u);
                }
              }
              tg::mma_commit(tg::smem_addr(&ctl->s_full[t & 1u]));
              tg::mma_commit(tg::smem_addr(&ctl->k_empty[st]));
            }
          }
          if (!(ok = __shfl_sync(0xFFFFFFFFu, good, 0) != 0)) break;
        }
      }
      if (lane == 0 && *abort_flag) {
        tg::mma_commit(tg::smem_addr(&ctl->drain[1]));
        int local_abort = 0;
        tg::mbar_wait(tg::smem_addr(&ctl->drain[1]), 0, &local_abort, 100000000ull);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- PV products
      constexpr uint32_t idesc_o = tg::idesc_bf16_f32(kBM, D, false, true);
      // Shared-memory descriptors, built once: a descriptor is two 32-bit words, and the
      // operand of each K step differs from its tile's by a constant offset added to the
      // start-address field of the low word (16-byte units, 14 bits; shared addresses stay
      // below 2^18 bytes, so the add never carries out of the field).
      const uint64_t dv = tg::smem_desc_sw128(tg::smem_addr(sV), kHalfBytes, 1024);
      const uint32_t v_lo0 = static_cast<uint32_t>(dv), hi_v = static_cast<uint32_t>(dv >> 32);
      constexpr uint32_t kTileUnits = C::kTileBytes >> 4;
      bool ok = true;
      Sched p_sc = sched0;
      int p_k = 0;
      uint32_t p_t = 0;
      for (Item it = p_sc.next(); it.valid && ok; it = p_sc.next(), ++p_k) {
        const uint32_t o_tmem = tmem_base + C::kTmemO;
        for (int j = 0; j < it.n; ++j, ++p_t) {
          if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->p_full[p_t & 1u]), (p_t >> 1) & 1u, abort_flag))) break;
          if (j == 0 && p_k >= 1 &&
              !(ok = tg::mbar_wait(tg::smem_addr(&ctl->o_empty), static_cast<uint32_t>(p_k - 1) & 1u, abort_flag)))
            break;
          const uint32_t sv = p_t % NS;
          if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->v_full[sv]), (p_t / NS) & 1u, abort_flag))) break;
          tg::tc_fence_after();
          const uint32_t p_tmem = tmem_base + (p_t & 1u) * kBN;
          const uint32_t v_lo = v_lo0 + sv * kTileUnits;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // 16 keys = 16 rows of V (2 swizzle groups of 8 rows, 2048 bytes); D blocks 16 KB apart
            const uint64_t bd = tg::desc_words(v_lo + static_cast<uint32_t>(kk) * (2048u >> 4), hi_v);
            tg::mma_bf16_ts(o_tmem, p_tmem + kk * 8u + (kk >= kBN / 32 ? 32u : 0u), bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          tg::mma_commit(tg::smem_addr(&ctl->v_empty[sv]));
          tg::mma_commit(tg::smem_addr(&ctl->pv_done[p_t & 1u]));  // frees S buffer p_t % 2 for S(p_t + 2)
          if (j == it.n - 1) tg::mma_commit(tg::smem_addr(&ctl->o_final));
        }
      }
      if (*abort_flag) {
        tg::mma_commit(tg::smem_addr(&ctl->drain[0]));
        int local_abort = 0;
        tg::mbar_wait(tg::smem_addr(&ctl->drain[0]), 0, &local_abort, 100000000ull);
      }
    }
  } else if (warp < 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax) : "memory");
    // ------------------------------------------------------------ softmax
    // Warps 4-7 take keys 0-63 of every S tile, warps 8-11 keys 64-127, one query row per
    // thread; the two warps of a TMEM lane quarter (same rows, same sub-partition) share
    // the MUFU and swap their halves' maxima through shared memory once per tile.
    const int half = (warp - 4) >> 2;
    const int quarter = warp & 3;           // TMEM lane quarter
    const int r = quarter * 32 + lane;      // row within the tile
    const int pair_bar = 2 + quarter;       // named barrier of this quarter's two warps
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t col0 = static_cast<uint32_t>(half * (kBN / 2));
    const uint64_t eff2 = tg::f2_pack(eff, eff);
    Sched sc = sched0;
    uint32_t t = 0;
    int k = 0;
    bool ok = true;     // this warp's waits so far
    bool stop = false;  // either warp of the pair failed (known to both at the barrier)
    for (Item it = sc.next(); it.valid && !stop; it = sc.next(), ++k) {
      const uint32_t o_taddr = tmem_base + C::kTmemO + lane_off + static_cast<uint32_t>(half * (D / 2));
      float m = -INFINITY, l = 0.f;         // running max of S' (S' units) and this half's row sum
      for (int j = 0; j < it.n; ++j, ++t) {
        ok = ok && tg::mbar_wait_warp(tg::smem_addr(&ctl->s_full[t & 1u]), (t >> 1) & 1u, abort_flag);
        const uint32_t s_taddr = tmem_base + (t & 1u) * kBN + lane_off + col0;
        const bool diag = (j == it.n - 1);
        uint32_t x[kBN / 2];
        auto load_row = [&]() {
          tg::tmem_ld32(s_taddr, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
          tg::tmem_ld32(s_taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
          tg::tmem_ld_wait();
          if (diag) {
#pragma unroll
            for (int c = 0; c < kBN / 2; ++c)
              if (static_cast<int>(col0) + c > r) x[c] = __float_as_uint(-INFINITY);
          }
        };
        uint64_t acc2[4];
        float mx[8];
        auto exp_pass = [&](float m_used, bool want_max) {
          const float nms = -m_used * eff;
          const uint64_t nms2 = tg::f2_pack(nms, nms);
#pragma unroll
          for (int q = 0; q < 4; ++q) acc2[q] = 0ull;
#pragma unroll
          for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
          for (int c = 0; c < kBN / 4; ++c) {
            const float s0 = __uint_as_float(x[2 * c]), s1 = __uint_as_float(x[2 * c + 1]);
            if (want_max) mx[c & 7] = tg::fmax3(mx[c & 7], s0, s1);
            const uint64_t arg = tg::f2_fma(tg::f2_pack(s0, s1), eff2, nms2);
            float a0, a1;
            tg::f2_unpack(arg, a0, a1);
            const uint32_t pb = pack_bf16x2(tg::ex2_approx(a0), tg::ex2_approx(a1));
            x[c] = pb;
            acc2[c & 3] = tg::f2_add(acc2[c & 3], tg::f2_pack(__uint_as_float(pb << 16), __uint_as_float(pb & 0xFFFF0000u)));
          }
        };
        auto row_max = [&]() {
          return fmaxf(tg::fmax3(mx[0], mx[1], mx[2]), tg::fmax3(tg::fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
        };
        float pm = -INFINITY;  // this half's max of the tile
        if (ok) {
          tg::tc_fence_after();
          load_row();
          if (j == 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBN / 4; ++c)
              mx[c & 7] = tg::fmax3(mx[c & 7], __uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1]));
          } else {
            exp_pass(m, true);
          }
          pm = row_max();
        }
        float *xm = sXm + (t & 1u) * 2 * kBM;
        xm[half * kBM + r] = pm;
        if (bar_red_or(pair_bar, 64, !ok)) {
          stop = true;
          break;
        }
        const float tile_max = fmaxf(pm, xm[(half ^ 1) * kBM + r]);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = tile_max;
          exp_pass(m, false);
        } else {
          const float m_new = fmaxf(m, tile_max);
          // the same vote in both warps of the pair: they see the same row maxima
          rescale = __any_sync(0xFFFFFFFFu, (m_new - m) * eff > kRescaleLog2);
          if (rescale) {
            alpha = tg::ex2_approx((m - m_new) * eff);
            m = m_new;
            load_row();
            exp_pass(m, false);
          }
        }
        // P of this half's 64 keys over the first 32 of its S columns
        tg::tmem_st32(s_taddr, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
        float sum_lo, sum_hi, sum_lo2, sum_hi2;
        tg::f2_unpack(tg::f2_add(acc2[0], acc2[1]), sum_lo, sum_hi);
        tg::f2_unpack(tg::f2_add(acc2[2], acc2[3]), sum_lo2, sum_hi2);
        l = fmaf(l, alpha, (sum_lo + sum_hi) + (sum_lo2 + sum_hi2));
        if (rescale) {
          // O holds the products up to step t - 1: wait for the last of them; this warp
          // rescales its half of O's columns
          ok = tg::mbar_wait_warp(tg::smem_addr(&ctl->pv_done[(t - 1) & 1u]), ((t - 1) >> 1) & 1u, abort_flag);
          if (ok) {
            tg::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              uint32_t o[32];
              tg::tmem_ld32(o_taddr + c * 32, o);
              tg::tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tg::tmem_st32(o_taddr + c * 32, o);
            }
          }
        }
        tg::tmem_st_wait();
        tg::tc_fence_before();
        tg::mbar_arrive(tg::smem_addr(&ctl->p_full[t & 1u]));
      }
      if (stop) break;
      // the row's partial sum and max for the epilogue (its buffer is free once the
      // epilogue two items back has read it); a failed wait here stops the pair at its
      // next barrier
      if (k >= 2) ok = ok && tg::mbar_wait(tg::smem_addr(&ctl->l_empty[k & 1]), ((k >> 1) & 1u) ^ 1u, abort_flag);
      sL[((k & 1) * 2 + half) * kBM + r] = l;
      if (half == 0) sM[(k & 1) * kBM + r] = m * eff;
      tg::mbar_arrive(tg::smem_addr(&ctl->l_full[k & 1]));
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue) : "memory");
    // ------------------------------------------------------------ epilogue (and Q into TMEM)
    // Each item's Q tile goes straight from global memory into its TMEM buffer (row r by
    // thread r), two items ahead, so the S products read Q from TMEM and only K from
    // shared memory.  A whole tile of bf16 output leaves through shared memory and a
    // tensor store (rows staged in the 128-byte-swizzled layout the tensor map expects,
    // written as full 128-byte lines); a partial tile (its rows past the end of the
    // request may belong to the next one) and the fp32 copy are stored row by row.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const bool leader = (warp == 12 && lane == 0);
    // CTA 0 reports a malformed request range or a request past the grid's rows (longer
    // than max_seqlen), whose remaining rows no item covers
    if (cu_seqlens && blockIdx.x == 0 && warp == 12) {
      for (int b = lane; b < B; b += 32) {
        const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        if (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > static_cast<int64_t>(n_mt) * kBM)
          tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
      }
    }
    auto load_q = [&](const Item &qi, int buf) {
      const uint32_t q_taddr = tmem_base + C::kTmemQ + static_cast<uint32_t>(buf * (D / 2)) + lane_off;
      const int64_t row = qi.rt + r;
      const bool in = row < qi.len;  // rows past the request get zeros (their outputs are never stored)
      const uint4 *src = reinterpret_cast<const uint4 *>(Qg + ((qi.seg_start + (in ? row : 0)) * Hq + qi.h) *
                                                                   static_cast<int64_t>(D));
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = in ? __ldg(src + c * 8 + q) : make_uint4(0u, 0u, 0u, 0u);
          w[4 * q] = v.x;
          w[4 * q + 1] = v.y;
          w[4 * q + 2] = v.z;
          w[4 * q + 3] = v.w;
        }
        tg::tmem_st32(q_taddr + c * 32, w);
      }
      tg::tmem_st_wait();
      tg::tc_fence_before();
      tg::mbar_arrive(tg::smem_addr(&ctl->q_full[buf]));
    };
    Sched q_sc = sched0;
    Item q_it = q_sc.next();
    for (int b = 0; b < 2 && q_it.valid; ++b, q_it = q_sc.next()) load_q(q_it, b);
    Sched sc = sched0;
    int k = 0;
    for (Item it = sc.next(); it.valid; it = sc.next(), ++k) {
      bool ok = tg::mbar_wait_warp(tg::smem_addr(&ctl->o_final), static_cast<uint32_t>(k) & 1u, abort_flag);
      ok = ok && tg::mbar_wait_warp(tg::smem_addr(&ctl->l_full[k & 1]), (k >> 1) & 1u, abort_flag);
      // stop together: the warpgroup shares named barriers below
      if (bar_red_or(1, 128, !ok || *abort_flag)) break;
      tg::tc_fence_after();
      const float l = sL[(k & 1) * 2 * kBM + r] + sL[((k & 1) * 2 + 1) * kBM + r];
      const float m2 = sM[(k & 1) * kBM + r];
      tg::mbar_arrive(tg::smem_addr(&ctl->l_empty[k & 1]));
      const uint32_t o_taddr = tmem_base + C::kTmemO + lane_off;
      const int64_t row = it.rt + r;
      const int h = it.h;
      const float inv_l = 1.0f / l;
      // base-2 log of sum_j 2^(eff S'_j) is eff m + log2 l (m the max the weights used)
      if (lse && row < it.len) lse[(it.seg_start + row) * Hq + h] = (m2 + __log2f(l)) * 0.6931471805599453f;
      const bool staged = !O32 && it.rt + kBM <= it.len;  // uniform over the warpgroup
      __nv_bfloat16 *orow = O + ((it.seg_start + row) * Hq + h) * static_cast<int64_t>(D);
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
            *reinterpret_cast<uint4 *>(sStage + (c >> 1) * kHalfBytes + r * 128 + ((ch ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
          continue;
        }
        if (O32 && row < it.len) {
          float4 *d32 = reinterpret_cast<float4 *>(O32 + ((it.seg_start + row) * Hq + h) * static_cast<int64_t>(D) + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d32[q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                 __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
        }
        if (row < it.len) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      // O may take the next item
      tg::tc_fence_before();
      tg::mbar_arrive(tg::smem_addr(&ctl->o_empty));
      if (staged) {
        tg::fence_proxy_async_smem();
        bar_sync(1, 128);  // every row of the tile is staged
        if (leader) {
          for (int hf = 0; hf < C::kHalves; ++hf)
            tg::tma_store_3d(&tm_o, tg::smem_addr(sStage + hf * kHalfBytes), hf * 64, h,
                             static_cast<int32_t>(it.seg_start + it.rt));
          tg::bulk_commit();
          tg::bulk_wait_read_all();  // the staging buffer is read before the next item's rows go there
        }
      }
      // the item two ahead takes this item's Q buffer (every S product of this item has completed)
      if (q_it.valid) {
        load_q(q_it, k & 1);
        q_it = q_sc.next();
      }
    }
    if (leader) tg::bulk_wait_all();
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
tg_status launch_kernel(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain,
                        float tau, const int32_t *cu_seqlens, int32_t B, int64_t total, int64_t max_seqlen, int32_t Hq,
                        int32_t Hkv, tg_bf16 *O, float *lse, float *O32, cudaStream_t stream, uint32_t *err) {
  using C = Cfg<D>;
  CUtensorMap tm_k, tm_v, tm_o;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(Hq), static_cast<uint64_t>(total)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hq) * D * 2};
    const uint32_t box[3] = {64, 1, kBM};
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
    const cudaError_t e = cudaFuncSetAttribute(gated_attention_persistent_kernel<D, kBias>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    // the warpgroup register split must fit the registers the launch allocates
    cudaFuncAttributes fa;
    const cudaError_t ea = cudaFuncGetAttributes(&fa, gated_attention_persistent_kernel<D, kBias>);
    if (ea != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(ea));
    if (fa.numRegs * kThreads < 128 * (kRegsLow + 2 * kRegsSoftmax + kRegsEpilogue))
      return tg::fail(TG_ERR_UNSUPPORTED, "gated_attention_persistent_kernel built with %d registers per thread; "
                      "the register split needs %d", fa.numRegs,
                      128 * (kRegsLow + 2 * kRegsSoftmax + kRegsEpilogue) / kThreads);
    return TG_OK;
  });
  if (setup != TG_OK) return setup;
  const float scale_log2 = tau / std::sqrt(static_cast<float>(D)) * kLog2e;
  const int64_t n_mt = (max_seqlen + kBM - 1) / kBM;
  const int64_t n_work = n_mt * Hq * B;
  if (n_work == 0) return TG_OK;
  if (n_work > 0x7FFFFFFFLL) return tg::fail(TG_ERR_UNSUPPORTED, "too many query tiles");
  const int64_t grid = std::min<int64_t>(n_work, tg::sm_count());
  const cudaError_t e =
      tg::launch_pdl(gated_attention_persistent_kernel<D, kBias>, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                     C::kSmem, stream, reinterpret_cast<const __nv_bfloat16 *>(Q), tm_k, tm_v, tm_o, s, gain, scale_log2,
                     cu_seqlens, cu_seqlens ? int64_t(0) : total, total, static_cast<int>(n_mt), B, Hq, Hkv,
                     reinterpret_cast<__nv_bfloat16 *>(O), lse, O32, err);
  if (e != cudaSuccess)
    return tg::fail(TG_ERR_CUDA, "gated_attention_persistent_kernel launch: %s", cudaGetErrorString(e));
  return tg::check_launch("gated_attention_persistent_kernel");
}

template <int D>
tg_status launch(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain, float tau,
                 const int32_t *cu_seqlens, int32_t B, int64_t total, int64_t max_seqlen, int32_t Hq, int32_t Hkv,
                 tg_bf16 *O, float *lse, float *O32, cudaStream_t stream, uint32_t *err) {
  // plain causal attention leaves the bias step out; with tau = 0 it is the whole product
  if (s || tau == 0.f)
    return launch_kernel<D, true>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                                  stream, err);
  return launch_kernel<D, false>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                                 stream, err);
}

}  // namespace

namespace tg {

tg_status gated_attention_persistent(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s,
                                     const float *gain, float tau, const int32_t *cu_seqlens, int32_t B,
                                     int64_t total, int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                     tg_bf16 *O, float *lse, float *O32, cudaStream_t stream, uint32_t *err) {
  return D == 128 ? launch<128>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                                stream, err)
                  : launch<64>(Q, Kc, V, s, gain, tau, cu_seqlens, B, total, max_seqlen, Hq, Hkv, O, lse, O32,
                               stream, err);
}

}  // namespace tg
