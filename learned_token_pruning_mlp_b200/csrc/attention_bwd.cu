// attention_bwd.cu -- tg_gated_attention_backward: gradients of token-gated attention
// with respect to the key scores s, the per-head gains and the temperature (the path
// by which the gate learns through the layers above it).
//
// TokenGate article, "What is token-gated attention?": the gate score of every kept
// token is a bias on the attention logits, scaled by a learnable per-head gain, and
// the dot product carries a learnable temperature.  For a loss L with dL/dO = dO,
// per head h (KV head g = h / (Hq/Hkv)), query i and key j <= i:
//     P_ij    = exp(l_ij - lse_i)           lse_i from the forward
//     dP_ij   = dO_i . V_j,   Delta_i = dO_i . O_i,   dl_ij = P_ij (dP_ij - Delta_i)
//     ds_j    = sum_{h,i} gain_h dl_ij
//     dgain_h = sum_{i,j} s_j dl_ij
//     dtau    = sum_{h,i,j} dl_ij (q_i . k_j) / sqrt(D)
//
// B200 design, three kernels on the caller's stream (programmatic launches):
//   1. prep: Delta_i = dO_i . O_i (from the forward's fp32 output when the caller has
//      it, else from the bf16 output) and the base-2 lse of every (row, head), negated,
//      into per-head vectors of the workspace padded to a multiple of 128 rows
//      (padding: -lse = -inf and -Delta = 0, so padding queries contribute nothing).
//   2. main, one CTA per (128-key block, head), heaviest (first) key blocks first.
//      Keys sit on the TMEM lanes, so each thread owns one key and every sum over
//      queries is a register sum.  Per 128-query block, from the diagonal on:
//          S^T  = K Q^T    and    dP^T = V dO^T
//      (tcgen05, M = 128 keys, N = 128 queries, K = D, operands K-major in shared
//      memory) go to one of two TMEM buffers while four warpgroups (32 query columns
//      each) form p = exp2(S c + b_j - lse2_i) with c = tau log2(e) / sqrt(D) and
//      b_j = gain_h log2(e) s_j, dl = p (dP - Delta_i), and accumulate sum_i dl and
//      sum_i dl S with packed f32x2 arithmetic.  dP - Delta_i comes out of the tensor
//      core: one extra K step multiplies a block of ones on V's side by -Delta_i in three
//      bf16 parts on dO's side (written per step by warp 3 from the prep's vector).  Q and dO stream through a TMA
//      pipeline, the lse / Delta vectors through bulk copies.
//   3. reduce: ds, dgain and dtau from the per-(head, key) column sums and the
//      per-CTA temperature partials, each summed in a fixed order, so the result is
//      deterministic.
// Packed ragged batches (cu_seqlens): each request attends within itself only, so its
// rows get their own span of every per-head workspace vector, padded to whole 128-row
// blocks; a CTA works on (key block, request, head) and the reduction maps packed rows
// back to their request's span.  dgain and dtau sum over every request.
#include <algorithm>
#include <cmath>

#include "ptx.cuh"
#include "runtime.h"

namespace {

constexpr int kBK = 128;          // keys per CTA (TMEM lanes)
constexpr int kBQ = 128;          // queries per step (TMEM columns of S^T and dP^T)
constexpr int kThreads = 640;     // warps 0-3: TMA, MMA, TMEM alloc, -Delta blocks; 4-19: four warpgroups
constexpr int kAux = 4;           // stages of the lse / Delta vectors
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kHalfBytes = 128 * 64 * 2;  // 128 rows x 64 bf16 columns, 128-byte swizzle
constexpr uint32_t kExtBytes = 128 * 16 * 2;   // one 128-row x 16-column unswizzled block (4 KB)
constexpr uint32_t kExtLBO = kExtBytes / 2;    // columns 8..15 follow columns 0..7
constexpr uint32_t kExtSBO = 128;              // 8 rows x 16 bytes per core matrix

template <int D>
struct BwdCfg {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kTileBytes = kHalfBytes * kHalves;  // 128 rows x D bf16
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr size_t kSmem = 1024 + 2 * static_cast<size_t>(kTileBytes) +
                                  2 * static_cast<size_t>(kStages) * kTileBytes + (1 + kStages) * static_cast<size_t>(kExtBytes) +
                                  kAux * 2 * kBQ * 4 + 3 * kBK * 4 + 512;
};

struct BwdCtl {
  uint64_t kv_full;
  uint64_t q_full[4];
  uint64_t q_empty[4];
  uint64_t ext_full[4];   // the -Delta block of Q / dO stage s is written
  uint64_t aux_full[kAux];
  uint64_t aux_empty[kAux];
  uint64_t s_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float tau_part[16];
};

// Workspace (fp32), ``stride`` rows per head (a multiple of 128): -lse2 [Hq][stride],
// -Delta [Hq][stride], colsum [Hq][stride], tau partials [Hq][stride / 128].
struct Workspace {
  float *nlse2, *ndelta, *colsum, *taup;
  int64_t stride;
};

__host__ __device__ inline int64_t padded_rows(int64_t S) { return (S + kBK - 1) / kBK * kBK; }

// Workspace rows per head: one sequence of S rows, or a packed batch of ``total`` rows in
// B requests (each request padded to whole blocks: at most total + 127 B rows).
inline int64_t ws_stride(int64_t total, int32_t B) { return B <= 1 ? padded_rows(total) : padded_rows(total) + kBK * B; }

inline size_t workspace_bytes_stride(int64_t stride, int32_t Hq) {
  const size_t floats = static_cast<size_t>(Hq) * (3 * static_cast<size_t>(stride) + static_cast<size_t>(stride / kBK));
  return (floats * 4 + 255) / 256 * 256;
}

inline size_t workspace_bytes(int64_t S, int32_t Hq) { return workspace_bytes_stride(padded_rows(S), Hq); }

inline Workspace carve(void *base, int64_t stride, int32_t Hq) {
  const size_t sp = static_cast<size_t>(stride);
  float *f = static_cast<float *>(base);
  return Workspace{f, f + Hq * sp, f + 2 * Hq * sp, f + 3 * Hq * sp, stride};
}

// The requests of a packed batch.  Request b owns packed rows [s0, s0 + len) of Q, K, V,
// dO, O, lse and s, and rows [p0, p0 + padded_rows(len)) of every per-head workspace
// vector.  Without cu_seqlens there is one request of ``total`` rows at p0 = 0.
struct Segs {
  const int32_t *cu;  // device int32 [B + 1], or nullptr
  int B;
  int64_t total;
  int64_t max_len;    // host bound on a request's length (it sizes the grids)
};
struct Seg {
  int64_t s0, len, p0;
  bool valid;  // cu_seqlens non-decreasing within [0, total] up to this request, length <= max_len
};

__device__ inline Seg seg_of(const Segs &sg, int64_t stride, int b) {
  Seg r{0, sg.total, 0, true};
  if (!sg.cu) return r;
  int64_t prev = sg.cu[0], p = 0;
  bool ok = prev >= 0 && prev <= sg.total;
  for (int i = 0; i < b && ok; ++i) {
    const int64_t nx = sg.cu[i + 1];
    ok = nx >= prev && nx <= sg.total;
    p += padded_rows(nx - prev);
    prev = nx;
  }
  const int64_t e = ok ? static_cast<int64_t>(sg.cu[b + 1]) : prev;
  ok = ok && e >= prev && e <= sg.total && e - prev <= sg.max_len && p + padded_rows(e - prev) <= stride;
  r.s0 = prev;
  r.len = ok ? e - prev : 0;
  r.p0 = p;
  r.valid = ok;
  return r;
}

// ------------------------------------------------------------------------------ prep
// One warp per (row, head) of the padded range, the whole range in one grid: Delta =
// dO . O (fp32), from the fp32 output with one 16-byte load per lane (D = 128) when it
// is given, and the lse converted to base 2; both stored negated, per head.
// Warps cover (request, padded row of the request, head); rows past a request's length
// are its padding.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16 *__restrict__ O,
                                                            const float *__restrict__ O32,
                                                            const __nv_bfloat16 *__restrict__ dO,
                                                            const float *__restrict__ lse, Segs sg, int64_t Lpad,
                                                            int Hq, Workspace ws, uint32_t *err) {
  tg::pdl_wait();
  tg::pdl_trigger();
  constexpr int kPer = D / 32;  // elements per lane (2 or 4)
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= static_cast<int64_t>(sg.B) * Lpad * Hq) return;  // whole warps
  const int h = static_cast<int>(w % Hq);
  const int64_t lr = (w / Hq) % Lpad;
  const int b = static_cast<int>(w / Hq / Lpad);
  const Seg sgm = seg_of(sg, ws.stride, b);
  if (!sgm.valid) {
    if (lane == 0 && lr == 0 && h == 0) tg::set_device_error(err, TG_DEVERR_BAD_SEQLENS);
    return;
  }
  if (lr >= padded_rows(sgm.len)) return;
  const int64_t i = sgm.s0 + lr;  // packed row (a real one when lr < len)
  float nd = 0.f, nl = -INFINITY;
  if (lr < sgm.len) {
    const int64_t off = (i * Hq + h) * D + lane * kPer;
    float o[kPer], d[kPer];
    if constexpr (kPer == 4) {
      const uint2 dv = *reinterpret_cast<const uint2 *>(dO + off);
      const __nv_bfloat162 d01 = *reinterpret_cast<const __nv_bfloat162 *>(&dv.x);
      const __nv_bfloat162 d23 = *reinterpret_cast<const __nv_bfloat162 *>(&dv.y);
      d[0] = __low2float(d01);
      d[1] = __high2float(d01);
      d[2] = __low2float(d23);
      d[3] = __high2float(d23);
    } else {
      const __nv_bfloat162 d01 = *reinterpret_cast<const __nv_bfloat162 *>(dO + off);
      d[0] = __low2float(d01);
      d[1] = __high2float(d01);
    }
    if (O32) {
      if constexpr (kPer == 4) {
        const float4 ov = *reinterpret_cast<const float4 *>(O32 + off);
        o[0] = ov.x;
        o[1] = ov.y;
        o[2] = ov.z;
        o[3] = ov.w;
      } else {
        const float2 ov = *reinterpret_cast<const float2 *>(O32 + off);
        o[0] = ov.x;
        o[1] = ov.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < kPer; e += 2) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(O + off + e);
        o[e] = __low2float(a);
        o[e + 1] = __high2float(a);
      }
    }
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc = fmaf(o[e], d[e], acc);
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, sh);
    nd = -acc;
    nl = -lse[i * Hq + h] * kLog2e;
  }
  if (lane == 0) {
    ws.ndelta[h * ws.stride + sgm.p0 + lr] = nd;
    ws.nlse2[h * ws.stride + sgm.p0 + lr] = nl;
  }
}

// ------------------------------------------------------------------------------ main
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const float *__restrict__ key_scores, const float *__restrict__ gain, float c_log2, Segs sg,
                    int Hq, int Hkv, Workspace ws, uint32_t *err) {
  using C = BwdCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem;
  uint8_t *sV = sK + C::kTileBytes;
  uint8_t *sQ = sV + C::kTileBytes;                  // [NS][tile]
  uint8_t *sdO = sQ + NS * C::kTileBytes;            // [NS][tile]
  uint8_t *sVx = sdO + NS * C::kTileBytes;          // [128 x 16]: ones in columns 0..2 (V's extra K step)
  uint8_t *sDx = sVx + kExtBytes;                    // [NS][128 x 16]: -Delta in three bf16 parts (dO's)
  float *sL = reinterpret_cast<float *>(sDx + NS * kExtBytes);      // [kAux][kBQ]  -lse2
  float *sDl = sL + kAux * kBQ;                                      // [kAux][kBQ]  -Delta
  float *sCs = sDl + kAux * kBQ;                                     // [3][kBK] warpgroups 1-3's column sums
  BwdCtl *ctl = reinterpret_cast<BwdCtl *>(sCs + 3 * kBK);

  // (key block, request, head); key blocks ascending: the longest ones first
  const int per_kb = sg.B * Hq;
  const int kb = static_cast<int>(blockIdx.x) / per_kb;
  const int b = (static_cast<int>(blockIdx.x) % per_kb) / Hq;
  const int h = static_cast<int>(blockIdx.x) % Hq;
  const int g = h / (Hq / Hkv);
  const Seg sgm = seg_of(sg, ws.stride, b);
  const int n_kb = static_cast<int>(padded_rows(sgm.len) / kBK);
  if (!sgm.valid || kb >= n_kb) return;              // uniform over the CTA, before any set-up
  const int n_steps = n_kb - kb;                     // query blocks kb .. n_kb-1
  const int64_t s0 = sgm.s0;
  const int64_t wrow0 = h * ws.stride + sgm.p0;      // the request's span of this head's vectors
  const int warp = tg::warp_id();
  const int lane = threadIdx.x & 31;

  // V's extra K step: ones in columns 0..2 of every row (bf16 1.0 = 0x3F80), zeros
  // elsewhere, also in dO's blocks (their columns 0..2 are written per step)
  for (uint32_t w = threadIdx.x; w < (1 + NS) * kExtBytes / 4; w += kThreads) {
    uint32_t v = 0;
    if (w < kExtLBO / 4 && (w & 3u) == 0) v = 0x3F803F80u;
    if (w < kExtLBO / 4 && (w & 3u) == 1) v = 0x00003F80u;
    reinterpret_cast<uint32_t *>(sVx)[w] = v;
  }
  tg::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    tg::mbar_init(tg::smem_addr(&ctl->kv_full), 1);
    for (int s = 0; s < NS; ++s) {
      tg::mbar_init(tg::smem_addr(&ctl->q_full[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->q_empty[s]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->ext_full[s]), 1);
    }
    for (int a = 0; a < kAux; ++a) {
      tg::mbar_init(tg::smem_addr(&ctl->aux_full[a]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->aux_empty[a]), 17);  // 16 dl warps and the -Delta block writer
    }
    for (int b = 0; b < 2; ++b) {
      tg::mbar_init(tg::smem_addr(&ctl->s_full[b]), 1);
      tg::mbar_init(tg::smem_addr(&ctl->tmem_empty[b]), 512);
    }
    tg::mbar_init(tg::smem_addr(&ctl->drain), 1);
    ctl->abort_flag = 0;
    tg::fence_mbar_init();
    tg::prefetch_tmap(&tm_q);
    tg::prefetch_tmap(&tm_k);
    tg::prefetch_tmap(&tm_v);
    tg::prefetch_tmap(&tm_do);
  }
  if (warp == 2) {
    tg::tmem_alloc(tg::smem_addr(&ctl->tmem_base), 512);
    tg::tmem_relinquish();
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  tg::pdl_wait();
  tg::pdl_trigger();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int *abort_flag = &ctl->abort_flag;

  // 640 threads at 96 registers each: a dl thread holds 32 columns of S^T and of dP^T,
  // so no warpgroup needs more than the launch gives (four warpgroups per step keep
  // four dl warps on every SM sub-partition to hide the exponentials' latency).
  if (warp < 4) {
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA / bulk producer
    const uint32_t kvb = tg::smem_addr(&ctl->kv_full);
    tg::mbar_arrive_expect_tx(kvb, 2 * C::kTileBytes);
    for (int hf = 0; hf < C::kHalves; ++hf) {
      tg::tma_load_3d(tg::smem_addr(sK + hf * kHalfBytes), &tm_k, kvb, hf * 64, g,
                      static_cast<int32_t>(s0 + kb * kBK));
      tg::tma_load_3d(tg::smem_addr(sV + hf * kHalfBytes), &tm_v, kvb, hf * 64, g,
                      static_cast<int32_t>(s0 + kb * kBK));
    }
    for (int n = 0; n < n_steps; ++n) {
      const int qblk = (kb + n) * kBQ;  // request-relative
      const int32_t qrow = static_cast<int32_t>(s0 + qblk);
      const int s = n % NS;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->q_empty[s]), ((n / NS) & 1) ^ 1, abort_flag)) break;
      const uint32_t qf = tg::smem_addr(&ctl->q_full[s]);
      tg::mbar_arrive_expect_tx(qf, 2 * C::kTileBytes);
      for (int hf = 0; hf < C::kHalves; ++hf) {
        tg::tma_load_3d(tg::smem_addr(sQ + s * C::kTileBytes + hf * kHalfBytes), &tm_q, qf, hf * 64, h, qrow);
        tg::tma_load_3d(tg::smem_addr(sdO + s * C::kTileBytes + hf * kHalfBytes), &tm_do, qf, hf * 64, h, qrow);
      }
      const int a = n % kAux;
      if (!tg::mbar_wait(tg::smem_addr(&ctl->aux_empty[a]), ((n / kAux) & 1) ^ 1, abort_flag)) break;
      const uint32_t af = tg::smem_addr(&ctl->aux_full[a]);
      tg::mbar_arrive_expect_tx(af, 2 * kBQ * 4);
      tg::bulk_load(tg::smem_addr(sL + a * kBQ), ws.nlse2 + wrow0 + qblk, kBQ * 4, af);
      tg::bulk_load(tg::smem_addr(sDl + a * kBQ), ws.ndelta + wrow0 + qblk, kBQ * 4, af);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ -Delta blocks
    // dP^T - Delta comes out of the tensor core: one extra K step multiplies V's block of
    // ones by dO's block holding each query's -Delta split into three bf16 parts (their
    // sum is -Delta to 2^-24), so the dl loop reads dP - Delta directly.
    for (int n = 0; n < n_steps; ++n) {
      const int s = n % NS, a = n % kAux;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->q_empty[s]), ((n / NS) & 1) ^ 1, abort_flag)) break;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->aux_full[a]), (n / kAux) & 1, abort_flag)) break;
#pragma unroll
      for (int e = 0; e < kBQ / 32; ++e) {
        const int q = e * 32 + lane;
        const float v = sDl[a * kBQ + q];
        const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
        uint8_t *row = sDx + s * kExtBytes + q * 16;  // row q, columns 0..2
        *reinterpret_cast<__nv_bfloat162 *>(row) = __halves2bfloat162(p0, p1);
        *reinterpret_cast<__nv_bfloat16 *>(row + 4) = p2;
      }
      tg::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tg::mbar_arrive(tg::smem_addr(&ctl->ext_full[s]));
        tg::mbar_arrive(tg::smem_addr(&ctl->aux_empty[a]));
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = tg::idesc_bf16_f32(kBK, kBQ, false, false);
    // shared-memory descriptors built once; each K step adds its constant offset to the
    // start-address field of the low word (16-byte units; shared addresses stay below
    // 2^18 bytes, so the add never carries out of the 14-bit field)
    const uint64_t dk = tg::smem_desc_sw128(tg::smem_addr(sK), 16, 1024);
    const uint32_t hi = static_cast<uint32_t>(dk >> 32), k_lo = static_cast<uint32_t>(dk);
    const uint32_t v_lo = static_cast<uint32_t>(tg::smem_desc_sw128(tg::smem_addr(sV), 16, 1024));
    const uint32_t q_lo0 = static_cast<uint32_t>(tg::smem_desc_sw128(tg::smem_addr(sQ), 16, 1024));
    const uint32_t do_lo0 = static_cast<uint32_t>(tg::smem_desc_sw128(tg::smem_addr(sdO), 16, 1024));
    const uint64_t dvx = tg::smem_desc_noswz(tg::smem_addr(sVx), kExtLBO, kExtSBO);
    const uint64_t ddx = tg::smem_desc_noswz(tg::smem_addr(sDx), kExtLBO, kExtSBO);
    const uint32_t dx_lo0 = static_cast<uint32_t>(ddx), hi_x = static_cast<uint32_t>(ddx >> 32);
    constexpr uint32_t kTileUnits = C::kTileBytes >> 4;
    bool ok = tg::mbar_wait(tg::smem_addr(&ctl->kv_full), 0, abort_flag);
    for (int n = 0; n < n_steps && ok; ++n) {
      const int s = n % NS;
      const int buf = n & 1;
      if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->q_full[s]), (n / NS) & 1, abort_flag))) break;
      if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->tmem_empty[buf]), ((n >> 1) & 1) ^ 1, abort_flag))) break;
      if (!(ok = tg::mbar_wait(tg::smem_addr(&ctl->ext_full[s]), (n / NS) & 1, abort_flag))) break;
      tg::tc_fence_after();
      const uint32_t d_s = tmem_base + static_cast<uint32_t>(buf * 256);
      const uint32_t q_lo = q_lo0 + static_cast<uint32_t>(s) * kTileUnits;
      const uint32_t do_lo = do_lo0 + static_cast<uint32_t>(s) * kTileUnits;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
        tg::mma_bf16_ss(d_s, tg::desc_words(k_lo + off, hi), tg::desc_words(q_lo + off, hi), idesc, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
        tg::mma_bf16_ss(d_s + kBQ, tg::desc_words(v_lo + off, hi), tg::desc_words(do_lo + off, hi), idesc,
                        kk > 0 ? 1u : 0u);
      }
      tg::mma_bf16_ss(d_s + kBQ, dvx, tg::desc_words(dx_lo0 + static_cast<uint32_t>(s) * (kExtBytes >> 4), hi_x), idesc, 1u);
      tg::mma_commit(tg::smem_addr(&ctl->s_full[buf]));
      tg::mma_commit(tg::smem_addr(&ctl->q_empty[s]));
    }
    if (*abort_flag) {
      tg::mma_commit(tg::smem_addr(&ctl->drain));
      int local_abort = 0;
      tg::mbar_wait(tg::smem_addr(&ctl->drain), 0, &local_abort, 100000000ull);
    }
  }
  } else {
    // ------------------------------------------------------------ dl and its sums
    const int grp = (warp - 4) >> 2;       // query columns 32*grp .. 32*grp+31
    const int quarter = warp & 3;          // TMEM lane quarter
    const int r = quarter * 32 + lane;     // key within the block
    const int64_t j = static_cast<int64_t>(kb) * kBK + r;  // request-relative key
    const float bj = j < sgm.len ? gain[h] * kLog2e * key_scores[s0 + j] : -INFINITY;
    const uint64_t bj2 = tg::f2_pack(bj, bj);
    const uint64_t c2 = tg::f2_pack(c_log2, c_log2);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint64_t cs2 = tg::f2_pack(0.f, 0.f), ta2 = tg::f2_pack(0.f, 0.f);
    for (int n = 0; n < n_steps; ++n) {
      const int buf = n & 1;
      const int a = n % kAux;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->s_full[buf]), (n >> 1) & 1, abort_flag)) break;
      if (!tg::mbar_wait_warp(tg::smem_addr(&ctl->aux_full[a]), (n / kAux) & 1, abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t t_s = tmem_base + static_cast<uint32_t>(buf * 256 + 32 * grp) + lane_off;
      uint32_t sx[32], dp[32];
      tg::tmem_ld32(t_s, sx);
      tg::tmem_ld32(t_s + kBQ, dp);
      tg::tmem_ld_wait();
      tg::tc_fence_before();
      tg::mbar_arrive(tg::smem_addr(&ctl->tmem_empty[buf]));
      const uint64_t *nl = reinterpret_cast<const uint64_t *>(sL + a * kBQ + 32 * grp);
      const bool diag = n == 0;  // query block == key block: keep query >= key
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint64_t s2 = tg::f2_pack(__uint_as_float(sx[2 * c]), __uint_as_float(sx[2 * c + 1]));
        const uint64_t x2 = tg::f2_fma(s2, c2, tg::f2_add(bj2, nl[c]));
        float x0, x1;
        tg::f2_unpack(x2, x0, x1);
        if (diag) {
          const int q0 = 32 * grp + 2 * c;
          if (q0 < r) x0 = -INFINITY;
          if (q0 + 1 < r) x1 = -INFINITY;
        }
        const uint64_t p2 = tg::f2_pack(tg::ex2_approx(x0), tg::ex2_approx(x1));
        const uint64_t d2 = tg::f2_pack(__uint_as_float(dp[2 * c]), __uint_as_float(dp[2 * c + 1]));  // dP - Delta
        const uint64_t dl2 = tg::f2_mul(p2, d2);
        cs2 = tg::f2_add(cs2, dl2);
        ta2 = tg::f2_fma(dl2, s2, ta2);
      }
      __syncwarp();
      if (lane == 0) tg::mbar_arrive(tg::smem_addr(&ctl->aux_empty[a]));
    }
    float cs0, cs1, ta0, ta1;
    tg::f2_unpack(cs2, cs0, cs1);
    tg::f2_unpack(ta2, ta0, ta1);
    float colsum = cs0 + cs1;
    float tacc = ta0 + ta1;
    if (grp > 0) sCs[(grp - 1) * kBK + r] = colsum;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tacc += __shfl_xor_sync(0xFFFFFFFFu, tacc, off);
    if (lane == 0) ctl->tau_part[warp - 4] = tacc;
    asm volatile("bar.sync 1, 512;" ::: "memory");  // the four warpgroups
    if (grp == 0) {
      ws.colsum[wrow0 + j] = ((colsum + sCs[r]) + sCs[kBK + r]) + sCs[2 * kBK + r];
      if (r == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 16; ++w) t += ctl->tau_part[w];
        ws.taup[h * (ws.stride / kBK) + sgm.p0 / kBK + kb] = t;
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

// ------------------------------------------------------------------------------ reduce
// Blocks [0, nb_ds): ds for 256 packed keys each; blocks nb_ds + h: dgain[h]; the last
// block: dtau.  Every sum runs in a fixed order (requests in order), so the result is
// deterministic.  Rows outside every request (a batch that does not cover [0, total))
// get ds = 0; a malformed batch leaves the outputs undefined (flagged by the prep).
__global__ void __launch_bounds__(256) attn_bwd_reduce_kernel(Workspace ws, const float *__restrict__ key_scores,
                                                              const float *__restrict__ gain, Segs sg, int Hq,
                                                              int nb_ds, float inv_sqrt_d, float *__restrict__ ds,
                                                              float *__restrict__ dgain, float *__restrict__ dtau) {
  tg::pdl_wait();
  tg::pdl_trigger();
  __shared__ float red[256];
  const int blk = static_cast<int>(blockIdx.x);
  const int t = threadIdx.x;
  if (blk < nb_ds) {
    const int64_t j = static_cast<int64_t>(blk) * 256 + t;
    if (j < sg.total) {
      float acc = 0.f;
      for (int b = 0; b < sg.B; ++b) {  // the request that holds packed row j
        const Seg sgm = seg_of(sg, ws.stride, b);
        if (!sgm.valid) break;
        if (j >= sgm.s0 && j < sgm.s0 + sgm.len) {
          const int64_t wr = sgm.p0 + (j - sgm.s0);
          for (int h = 0; h < Hq; ++h) acc = fmaf(gain[h], ws.colsum[h * ws.stride + wr], acc);
          break;
        }
      }
      ds[j] = acc;
    }
    return;
  }
  const int h = blk - nb_ds;  // h == Hq: the temperature
  float acc = 0.f;
  for (int b = 0; b < sg.B; ++b) {
    const Seg sgm = seg_of(sg, ws.stride, b);
    if (!sgm.valid) break;
    if (h < Hq) {
      const float *cs = ws.colsum + h * ws.stride + sgm.p0;
      for (int64_t jl = t; jl < sgm.len; jl += 256) acc = fmaf(key_scores[sgm.s0 + jl], cs[jl], acc);
    } else {
      const int64_t nkb = padded_rows(sgm.len) / kBK;
      for (int64_t i = t; i < nkb * Hq; i += 256)
        acc += ws.taup[(i / nkb) * (ws.stride / kBK) + sgm.p0 / kBK + (i % nkb)];
    }
  }
  red[t] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w) red[t] += red[t + w];
    __syncthreads();
  }
  if (t == 0) {
    if (h < Hq)
      dgain[h] = red[0];
    else
      dtau[0] = red[0] * inv_sqrt_d;
  }
}

bool tmap3(CUtensorMap *m, const void *base, int D, int heads, int64_t rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(heads), static_cast<uint64_t>(rows)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(heads) * D * 2};
  const uint32_t box[3] = {64, 1, 128};
  return tg::encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int D>
tg_status launch_bwd(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain,
                     float tau, const tg_bf16 *O, const float *O32, const tg_bf16 *dO, const float *lse,
                     const Segs &sg, int32_t Hq, int32_t Hkv, const Workspace &ws, cudaStream_t stream,
                     uint32_t *err) {
  using C = BwdCfg<D>;
  const int64_t S = sg.total;
  const int64_t Lpad = padded_rows(sg.max_len);
  const int n_kb = static_cast<int>(Lpad / kBK);
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  if (!tmap3(&tm_q, Q, D, Hq, S) || !tmap3(&tm_k, Kc, D, Hkv, S) || !tmap3(&tm_v, V, D, Hkv, S) ||
      !tmap3(&tm_do, dO, D, Hq, S))
    return TG_ERR_CUDA;
  static tg::PerDevice configured;
  const tg_status setup = tg::once_per_device(configured, [&](int) -> tg_status {
    const cudaError_t e =
        cudaFuncSetAttribute(attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TG_OK;
  });
  if (setup != TG_OK) return setup;
  const int64_t prep_warps = static_cast<int64_t>(sg.B) * Lpad * Hq;  // checked by the caller
  const unsigned prep_grid = static_cast<unsigned>((prep_warps + 7) / 8);
  cudaError_t e = tg::launch_pdl(attn_bwd_prep_kernel<D>, dim3(prep_grid), dim3(256), 0, stream,
                                 reinterpret_cast<const __nv_bfloat16 *>(O), O32,
                                 reinterpret_cast<const __nv_bfloat16 *>(dO), lse, sg, Lpad, static_cast<int>(Hq), ws,
                                 err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "attn_bwd_prep_kernel launch: %s", cudaGetErrorString(e));
  const float c_log2 = tau / std::sqrt(static_cast<float>(D)) * kLog2e;
  const int64_t grid = static_cast<int64_t>(n_kb) * sg.B * Hq;
  e = tg::launch_pdl(attn_bwd_kernel<D>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), C::kSmem, stream, tm_q,
                     tm_k, tm_v, tm_do, s, gain, c_log2, sg, static_cast<int>(Hq), static_cast<int>(Hkv), ws, err);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "attn_bwd_kernel launch: %s", cudaGetErrorString(e));
  return TG_OK;
}

// Scratch of the allocation-free entry point: a fixed device array in this module's
// global memory, 4 MiB (enough for S * Hq up to about 349,000 padded rows, e.g. the
// 128k workload's layer, S = 8704 with 16 heads, which needs 1.7 MB).
constexpr size_t kStaticScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

tg_status launch_reduce(const Workspace &ws, const float *s, const float *gain, const Segs &sg, int32_t Hq, int32_t D,
                        float *ds, float *dgain, float *dtau, cudaStream_t stream) {
  const int nb_ds = static_cast<int>((sg.total + 255) / 256);
  const cudaError_t e =
      tg::launch_pdl(attn_bwd_reduce_kernel, dim3(static_cast<unsigned>(nb_ds + Hq + 1)), dim3(256), 0, stream, ws, s,
                     gain, sg, static_cast<int>(Hq), nb_ds, 1.0f / std::sqrt(static_cast<float>(D)), ds, dgain, dtau);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "attn_bwd_reduce_kernel launch: %s", cudaGetErrorString(e));
  return TG_OK;
}

// The backward of one sequence (cu_seqlens = nullptr, B = 1) or of a packed batch.
tg_status backward_impl(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V, const float *s, const float *gain,
                        float tau, const tg_bf16 *O, const float *O32, const tg_bf16 *dO, const float *lse,
                        const int32_t *cu_seqlens, int32_t B, int64_t S, int64_t max_len, int32_t Hq, int32_t Hkv,
                        int32_t D, float *ds, float *dgain, float *dtau, void *workspace, size_t workspace_size,
                        tg_stream stream) {
  if (S < 0) return tg::fail(TG_ERR_INVALID_ARG, "S must be >= 0");
  if (B < 1) return tg::fail(TG_ERR_INVALID_ARG, "B must be >= 1");
  if (max_len < 0 || max_len > S) return tg::fail(TG_ERR_INVALID_ARG, "max_seqlen must be in [0, total]");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return tg::fail(TG_ERR_INVALID_ARG, "Hq must be a positive multiple of Hkv");
  if (D != 64 && D != 128) return tg::fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (!std::isfinite(tau)) return tg::fail(TG_ERR_INVALID_ARG, "tau must be finite");
  const int64_t stride = cu_seqlens ? ws_stride(S, B) : padded_rows(S);
  if (stride * Hq > (int64_t(1) << 31) - 1 || padded_rows(max_len) * B * Hq > (int64_t(1) << 31) - 1)
    return tg::fail(TG_ERR_UNSUPPORTED, "S * Hq must be below 2^31");
  if (!gain || !dgain || !dtau) return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  if (S > 0 && (!Q || !Kc || !V || !s || (!O && !O32) || !dO || !lse || !ds || !workspace))
    return tg::fail(TG_ERR_INVALID_ARG, "null pointer");
  const size_t need = workspace_bytes_stride(stride, Hq);
  if (S > 0 && workspace_size < need)
    return tg::fail(TG_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu bytes needed", workspace_size, need);
  if (S > 0 && (!tg::aligned16(Q) || !tg::aligned16(Kc) || !tg::aligned16(V) || !tg::aligned16(dO) ||
                !tg::aligned16(O) || !tg::aligned16(O32) || !tg::aligned16(workspace)))
    return tg::fail(TG_ERR_ALIGNMENT, "Q, Kc, V, O, O32, dO and workspace must be 16-byte aligned");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Segs sg{cu_seqlens, cu_seqlens ? B : 1, S, cu_seqlens ? max_len : S};
  const Workspace ws = S > 0 ? carve(workspace, stride, Hq) : Workspace{nullptr, nullptr, nullptr, nullptr, stride};
  if (S > 0 && max_len > 0) {
    const tg_status r = D == 64 ? launch_bwd<64>(Q, Kc, V, s, gain, tau, O, O32, dO, lse, sg, Hq, Hkv, ws, st, err)
                                : launch_bwd<128>(Q, Kc, V, s, gain, tau, O, O32, dO, lse, sg, Hq, Hkv, ws, st, err);
    if (r != TG_OK) return r;
  }
  // with no work the reduction still writes the (zero) gradients: its loops find no rows
  const Segs sg_reduce = (S > 0 && max_len > 0) ? sg : Segs{nullptr, 0, S, 0};
  const tg_status r = launch_reduce(ws, s, gain, sg_reduce, Hq, D, ds, dgain, dtau, st);
  if (r != TG_OK) return r;
  return tg::check_launch("tg_gated_attention_backward");
}

}  // namespace

extern "C" size_t tg_gated_attention_backward_workspace(int64_t S, int32_t Hq) {
  if (S < 0 || Hq <= 0) return 0;
  return workspace_bytes(S, Hq);
}

extern "C" size_t tg_gated_attention_backward_varlen_workspace(int64_t total, int32_t B, int32_t Hq) {
  if (total < 0 || B < 1 || Hq <= 0) return 0;
  return workspace_bytes_stride(ws_stride(total, B), Hq);
}

extern "C" tg_status tg_gated_attention_backward(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                                 const float *s, const float *gain, float tau, const tg_bf16 *O,
                                                 const float *O32, const tg_bf16 *dO, const float *lse, int64_t S,
                                                 int32_t Hq,
                                                 int32_t Hkv, int32_t D, float *ds, float *dgain, float *dtau,
                                                 void *workspace, size_t workspace_size, tg_stream stream) {
  TG_API_ENTRY();
  return backward_impl(Q, Kc, V, s, gain, tau, O, O32, dO, lse, nullptr, 1, S, S, Hq, Hkv, D, ds, dgain, dtau,
                       workspace, workspace_size, stream);
}

extern "C" tg_status tg_gated_attention_backward_varlen(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                                        const float *s, const float *gain, float tau, const tg_bf16 *O,
                                                        const float *O32, const tg_bf16 *dO, const float *lse,
                                                        const int32_t *cu_seqlens, int32_t B, int64_t total,
                                                        int64_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                                        float *ds, float *dgain, float *dtau, void *workspace,
                                                        size_t workspace_size, tg_stream stream) {
  TG_API_ENTRY();
  if (B < 1) return tg::fail(TG_ERR_INVALID_ARG, "B must be >= 1");
  if (!cu_seqlens) return tg::fail(TG_ERR_INVALID_ARG, "cu_seqlens is NULL");
  return backward_impl(Q, Kc, V, s, gain, tau, O, O32, dO, lse, cu_seqlens, B, total, max_seqlen, Hq, Hkv, D, ds,
                       dgain, dtau, workspace, workspace_size, stream);
}

extern "C" tg_status tg_gated_attention_backward_noalloc(const tg_bf16 *Q, const tg_bf16 *Kc, const tg_bf16 *V,
                                                         const float *s, const float *gain, float tau,
                                                         const tg_bf16 *O, const float *O32, const tg_bf16 *dO,
                                                         const float *lse, int64_t S, int32_t Hq, int32_t Hkv,
                                                         int32_t D, float *ds, float *dgain, float *dtau,
                                                         tg_stream stream) {
  TG_API_ENTRY();
  if (S < 0) return tg::fail(TG_ERR_INVALID_ARG, "S must be >= 0");
  if (Hq <= 0) return tg::fail(TG_ERR_INVALID_ARG, "Hq must be positive");
  if (padded_rows(S) * Hq > (int64_t(1) << 31) - 1) return tg::fail(TG_ERR_UNSUPPORTED, "S * Hq must be below 2^31");
  const size_t need = workspace_bytes(S, Hq);
  if (need > kStaticScratchBytes)
    return tg::fail(TG_ERR_UNSUPPORTED,
                    "S = %lld with Hq = %d needs %zu bytes of scratch; the static scratch of this entry point holds "
                    "%zu bytes (use tg_gated_attention_backward with a caller workspace)",
                    static_cast<long long>(S), Hq, need, kStaticScratchBytes);
  void *scratch = nullptr;
  if (S > 0) {
    // The array's device address (host code may not use the symbol itself), looked up
    // by the first call on each device with that device current, under the library's
    // set-up lock, and read without the lock afterwards.
    static std::atomic<void *> addr[tg::kMaxDevices];
    static tg::PerDevice looked_up;
    int dev = 0;
    const tg_status st = tg::once_per_device(
        looked_up,
        [&](int d) -> tg_status {
          void *p = nullptr;
          const cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_scratch);
          if (e != cudaSuccess || !p)
            return tg::fail(TG_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
          addr[d].store(p, std::memory_order_relaxed);  // published by the set-up flag's release
          return TG_OK;
        },
        &dev);
    if (st != TG_OK) return st;
    scratch = addr[dev].load(std::memory_order_relaxed);
  }
  return tg_gated_attention_backward(Q, Kc, V, s, gain, tau, O, O32, dO, lse, S, Hq, Hkv, D, ds, dgain, dtau, scratch,
                                     kStaticScratchBytes, stream);
}
