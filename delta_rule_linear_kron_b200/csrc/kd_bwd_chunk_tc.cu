// kd_bwd_chunk_tc.cu -- the backward's per-chunk tensor-core kernels for bf16
// q, k, v, dO and d_k = d_v = 128: one CTA per chunk, all chunks in parallel,
// one launch before the reverse chain (bwd_pre_tc) and one after it
// (bwd_post_tc).
//
// Notation, per chunk (positions t, i, s < 64; key channel j; value channel r):
//   L = cumulative log decay inside the chunk, gamma = e^L, Lambda = L at the
//   chunk end; K+ = k o gamma, K- = k / gamma, K^e = k o e^{Lambda - L},
//   Q+ = q o gamma;  G_K = K+ K-^T and G_V = V V^T (the decayed key Gram and
//   the value Gram of the chunk form: KronLSTM digest, "무엇과 다른가";
//   Gated DeltaNet-2 article, "기술 상세").  Saved by the forward: u, b0,
//   P = tril(Q+ K-^T) and the chunk-start state S0.  From the reverse chain:
//   g and dS (gradient of the chunk-end state); db0 = -beta o g.
//
// Reverse mode of the chunk form (derived here; the pages only ask that the
// gradient reach every gate: Gated DeltaNet-2 article, "핵심 기여"):
//   dP    = (dO V^T) o 1u^T on i <= t
//   dG_K  = diag(db0) E_V,  E_V = strict lower part of G_V o 1u^T
//   dG_V' = diag(db0) E_K + (diag(db0) E_K)^T,  E_K likewise from G_K
//   dbeta = -g o (b0 + M u),  M = tril(G_K o G_V, -1);   dc = g
//   du_intra[i] = sum_{t >= i} P[t,i] (dO_t . v_i)       (input of the chain)
// Everything but the db0 scalings is known before the chain runs, so
// bwd_pre_tc computes it (du_intra, M u, and E_V, E_K, dP, P diag(u) as bf16
// MMA operand tiles) and bwd_post_tc applies db0 while building its operands.
//
// bwd_post_tc: with the gates factored out, every state and intra-chunk
// product of the gradient is one of five tensor-memory accumulators, all
// transposed (TMEM lane = channel, column = position t):
//   QT = (dO S0 + dP K-)^T                  dq = gamma o QT
//   XA = (V S0 + E_V K-)^T                  XB = (V dS')^T,  dS' = dS diag(e^Lambda)
//   R2 = (dP^T Q+ + dG_K^T K+)^T            (as [Q+; db0 o K+]^T [dP; E_V])
//   dk = gamma o db0 o XA + u o e^{-L} o XB + e^{-L} o R2
//   VT = S0 (db0 o K+)^T + [dO; V]^T [P diag(u); dG_V'],  VD = dS' K-^T
//   dv = VT + VD diag(u)
//   dL = q o dq + k o (gamma o db0 o XA - u o e^{-L} o XB - e^{-L} o R2),
//        plus, on the last position, sum_r dS[r,j] (S0 e^Lambda + V^T diag(u) K^e)[r,j]
//   dlogf = reverse cumulative sum of dL over the chunk.
// Chunks whose |L| reaches kPostSafe (so that e^{-L} times a bf16 value could
// lose precision to subnormals) are flagged and recomputed exactly by the
// CUDA-core kernels.
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;

// |L| bound of the factorised post-chain products: e^{-40} keeps dS' = dS e^Lambda
// well inside bf16's normal range for any |dS| above 1e-20.
constexpr float kPostSafe = 40.0f;

__device__ __forceinline__ float bf(const unsigned char* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
__device__ __forceinline__ void put_bf(unsigned char* p, float x) {
  *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
// 16 bf16 values into row `row` (columns c0..c0+15) of a 128-byte-swizzled tile
__device__ __forceinline__ void put_row16(unsigned char* tile, int row, int c0, int rows, const float (&x)[16]) {
#pragma unroll
  for (int h8 = 0; h8 < 2; ++h8) {
    __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v8[i] = __float2bfloat16_rn(x[8 * h8 + i]);
    *reinterpret_cast<uint4*>(tile + tc::sw128_off(row, c0 + 8 * h8, rows, 2)) = *reinterpret_cast<const uint4*>(v8);
  }
}

// Cumulative log decay of key channel j, split between two threads: half 0
// holds positions 0..31, half 1 positions 32..63 (all 256 threads call it).
__device__ __forceinline__ void split_prefix(const float* lg, int j, int half, float* xch, float (&Lr)[32]) {
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    acc += lg[(32 * half + i) * D + j];
    Lr[i] = acc;
  }
  if (half == 0) xch[j] = acc;
  __syncthreads();
  const float off = half ? xch[j] : 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) Lr[i] += off;
}

// ---------------------------------------------------------------------------
// bwd_pre_tc
// ---------------------------------------------------------------------------
struct PreCfg {
  static constexpr uint32_t KPM = 0;         // tf32 [K+; K-]: per 32-channel K block (16 KB) rows 0-63 K+, 64-127 K-
  static constexpr uint32_t VD = 65536;      // [V; dO] bf16, 2 K blocks x 128 rows (TMA, 128-byte swizzle)
  static constexpr uint32_t KR = 98304;      // k bf16 [64][128] (TMA)
  static constexpr uint32_t LG = 114688;     // logf fp32 [64][128] (TMA)
  static constexpr uint32_t PS = 147456;     // P fp32 [64][64]
  static constexpr uint32_t US = 163840;     // u [64]
  static constexpr uint32_t XCH = US + 256;  // prefix exchange [128]
  static constexpr uint32_t QR = 165888;     // q bf16 [64][128] (TMA)
  static constexpr uint32_t QT = 182272;     // Q+^T bf16 [j][t], 128 rows x 128 B, 128-byte swizzle (staging)
  static constexpr uint32_t BYTES = QT + 16384 + 1024;
  static constexpr uint32_t LOAD_BYTES = 32768 + 16384 + 32768 + 16384 + 256 + 16384;
  // output staging in the KPM area once the MMAs are done
  static constexpr uint32_t OT1 = 0, OPU = 16384, OEK = 24576;
};

__global__ void __launch_bounds__(256, 1) bwd_pre_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_logf,
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp, int H, int NC,
    const float* __restrict__ wP, const float* __restrict__ wu, float* __restrict__ wdu, float* __restrict__ wMu,
    __nv_bfloat16* __restrict__ wT1, __nv_bfloat16* __restrict__ wPU, __nv_bfloat16* __restrict__ wEK,
    __nv_bfloat16* __restrict__ wQpT, int ahead, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C;
  const size_t ch = blockIdx.x;

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, PreCfg::LOAD_BYTES);
    tc::tma_load_4d(sm + PreCfg::VD, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::VD + 16384, &tm_v, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::VD + 8192, &tm_do, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::VD + 24576, &tm_do, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::KR, &tm_k, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::LG, &tm_logf, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PreCfg::QR, &tm_q, 0, h, t0, b, &ld_bar);
    tc::bulk_g2s(sm + PreCfg::PS, wP + ch * C * C, 16384u, &ld_bar);
    tc::bulk_g2s(sm + PreCfg::US, wu + ch * C, 256u, &ld_bar);
    const size_t nx = ch + (size_t)ahead;
    if (nx < gridDim.x) {  // the chunk this SM most likely runs next: its tiles into L2
      const int nn = static_cast<int>(nx % NC), un = static_cast<int>(nx / NC), tn = nn * C;
      tc::tma_prefetch_l2_4d(&tm_v, 0, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_v, 64, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_do, 0, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_do, 64, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_k, 0, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_logf, 0, un % H, tn, un / H);
      tc::tma_prefetch_l2_4d(&tm_q, 0, un % H, tn, un / H);
      tc::prefetch_l2(wP + nx * C * C, 16384u);
    }
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 256);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);

  // K+ and K- (fp32, read as tf32), and Q+ (bf16, transposed for the reverse
  // chain's dO^T Q+ MMA); thread (j, half) covers 32 positions.  K+ and Q+
  // carry decays e^L <= 1 and are always finite; chunks with extreme decays
  // may overflow K- here: their E_K and M u are never used (the post-chain
  // kernel hands such chunks to the exact path).
  {
    const int j = tid & 127, half = tid >> 7;
    float Lr[32];
    split_prefix(reinterpret_cast<const float*>(sm + PreCfg::LG), j, half,
                 reinterpret_cast<float*>(sm + PreCfg::XCH), Lr);
    const unsigned char* kr = sm + PreCfg::KR;
    const unsigned char* qr = sm + PreCfg::QR;
    __align__(16) __nv_bfloat16 q8[8];  // eight consecutive positions of Q+^T row j: one 16-byte store
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * half + i;
      const float kk = bf(kr + (t * D + j) * 2);
      const float gm = expf(Lr[i]);
      *reinterpret_cast<float*>(sm + PreCfg::KPM + tc::sw128_off(t, j, 128, 4)) = kk * gm;
      *reinterpret_cast<float*>(sm + PreCfg::KPM + tc::sw128_off(64 + t, j, 128, 4)) = kk * expf(-Lr[i]);
      q8[i & 7] = __float2bfloat16_rn(bf(qr + (t * D + j) * 2) * gm);
      if ((i & 7) == 7)
        *reinterpret_cast<uint4*>(sm + PreCfg::QT + tc::sw128_off(j, t - 7, 128, 2)) = *reinterpret_cast<const uint4*>(q8);
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    // K+ (rows 0-63 of each 32-channel block) and the Q+^T tile out for the reverse chain
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) tc::tma_store_4d(&tm_kp, sm + PreCfg::KPM + kb * 16384, 32 * kb, h, t0, b);
    tc::bulk_s2g(wQpT + ch * (D * C), sm + PreCfg::QT, 16384u);
    tc::bulk_commit();
    const uint32_t IDT = tc::idesc(128, 64, 2), IDB = tc::idesc(128, 64, 1);
    // cols 0-63: [K+; K-] K-^T (rows 0-63: G_K)
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
      tc::mma_tf32_ss(tmem + 0, tc::desc_sw128(tc::smem_u32(sm + PreCfg::KPM + o)),
                      tc::desc_sw128(tc::smem_u32(sm + PreCfg::KPM + o + 8192)), IDT, ks > 0 ? 1u : 0u);
    }
    // cols 64-127: [V; dO] V^T (rows 0-63: G_V, rows 64-127: dO V^T);
    // cols 128-191: [V; dO] dO^T (rows 0-63: V dO^T)
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
      const uint64_t a = tc::desc_sw128(tc::smem_u32(sm + PreCfg::VD + o));
      tc::mma_bf16_ss(tmem + 64, a, tc::desc_sw128(tc::smem_u32(sm + PreCfg::VD + o)), IDB, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + 128, a, tc::desc_sw128(tc::smem_u32(sm + PreCfg::VD + o + 8192)), IDB,
                      ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  if (tid == 0) tc::bulk_wait_read();  // the K+ stores have read the area the staging below reuses
  __syncthreads();

  const float* us = reinterpret_cast<const float*>(sm + PreCfg::US);
  const float* Ps = reinterpret_cast<const float*>(sm + PreCfg::PS);
  unsigned char* o = sm + PreCfg::KPM;
  const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
  if (warp < 2) {
    // row t of G_K and G_V: E_K, E_V (rows 64.. of T1) and (M u)_t
    const int t = warp * 32 + lane;
    float mu = 0.f;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float gk[16], gv[16], ek[16], ev[16];
      tc::tmem_ld16(lanes + 16 * c16, gk);
      tc::tmem_ld16(lanes + 64 + 16 * c16, gv);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int i = 16 * c16 + ii;
        const bool low = i < t;
        const float ui = us[i];
        ek[ii] = low ? ui * gk[ii] : 0.f;
        ev[ii] = low ? ui * gv[ii] : 0.f;
        mu = fmaf(ek[ii], gv[ii], mu);
      }
      put_row16(o + PreCfg::OEK, t, 16 * c16, 64, ek);
      put_row16(o + PreCfg::OT1, 64 + t, 16 * c16, 128, ev);
    }
    wMu[ch * C + t] = mu;
  } else if (warp < 4) {
    // row t of dO V^T: dP (rows 0-63 of T1)
    const int t = (warp - 2) * 32 + lane;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float x[16];
      tc::tmem_ld16(lanes + 64 + 16 * c16, x);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int i = 16 * c16 + ii;
        x[ii] = i <= t ? us[i] * x[ii] : 0.f;
      }
      put_row16(o + PreCfg::OT1, t, 16 * c16, 128, x);
    }
  } else if (warp < 6) {
    // row i of V dO^T: du_intra[i] = sum_{t >= i} P[t,i] (dO_t . v_i)
    const int i = (warp - 4) * 32 + lane;
    float du = 0.f;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float x[16];
      tc::tmem_ld16(lanes + 128 + 16 * c16, x);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int t = 16 * c16 + ii;
        if (t >= i) du = fmaf(Ps[t * C + i], x[ii], du);
      }
    }
    wdu[ch * C + i] = du;
  } else {
    // P diag(u) as a bf16 tile [i][t] (thread = column t)
    const int t = tid - 192;
    const float ut = us[t];
#pragma unroll 8
    for (int i = 0; i < C; ++i) put_bf(o + PreCfg::OPU + tc::sw128_off(i, t, 64, 2), Ps[i * C + t] * ut);
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  if (tid == 0) {
    tc::bulk_s2g(wT1 + ch * (2 * C * C), o + PreCfg::OT1, 16384u);
    tc::bulk_s2g(wPU + ch * (C * C), o + PreCfg::OPU, 8192u);
    tc::bulk_s2g(wEK + ch * (C * C), o + PreCfg::OEK, 8192u);
    tc::bulk_commit();
    tc::bulk_wait_read();
  }
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// bwd_post_tc
// ---------------------------------------------------------------------------
struct PostCfg {
  static constexpr uint32_t S0T = 0;          // S0 bf16 [r][j], 2 K blocks x 128 rows
  static constexpr uint32_t DST = 32768;      // dS, scaled in place to dS' = dS diag(e^Lambda)
  static constexpr uint32_t DOV = 65536;      // [dO; V] bf16 (TMA)
  static constexpr uint32_t A4 = 98304;       // [q; k] (TMA), then [Q+; db0 o K+] in place
  static constexpr uint32_t KM = 131072;      // K- bf16 [t][j], 2 K blocks x 64 rows
  static constexpr uint32_t T1 = 147456;      // [dP; E_V] bf16, 128 rows x 64
  static constexpr uint32_t B7 = 163840;      // [P diag(u); dG_V'] bf16, 128 rows x 64
  static constexpr uint32_t EK = 180224;      // E_K bf16, 64 rows x 64
  static constexpr uint32_t LG = 188416;      // logf fp32 [64][128] (TMA)
  static constexpr uint32_t SMALL = 221184;   // u, db0 [64]; xch, lam, csum [2], ek [2], tail [128] (floats)
  static constexpr uint32_t BYTES = SMALL + (2 * 64 + 7 * 128) * 4 + 1024;
  static constexpr uint32_t LOAD_A = 32768 + 32768 + 8192;          // logf, q and k, E_K
  static constexpr uint32_t LOAD_B = 3 * 32768 + 16384 + 8192;      // S0, dS, [dO; V], T1, P diag(u)
  // tensor-memory columns of the accumulators
  static constexpr uint32_t C_A = 0, C_XB = 128, C_R2 = 192, C_VT = 256, C_VD = 320;
  // output staging once the MMAs are done
  static constexpr uint32_t OQ = 0, OK = 16384, OV = 32768, OL = 65536;
};

__global__ void __launch_bounds__(256, 1) bwd_post_tc(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_logf, const __grid_constant__ CUtensorMap tm_dq,
    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
    const __grid_constant__ CUtensorMap tm_dlogf, const float* __restrict__ beta, int H, int T, int NC,
    const float* __restrict__ wu, const float* __restrict__ wb0, const float* __restrict__ wg,
    const float* __restrict__ wMu, const __nv_bfloat16* __restrict__ wS0b, const __nv_bfloat16* __restrict__ wdSb,
    const __nv_bfloat16* __restrict__ wT1, const __nv_bfloat16* __restrict__ wPU,
    const __nv_bfloat16* __restrict__ wEK, float* __restrict__ dbeta, float* __restrict__ dc,
    int* __restrict__ flags, const float* __restrict__ a_log, float* __restrict__ dapart, int* __restrict__ err) {
  using Cf = PostCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t bar_a, bar_b, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  float* us = reinterpret_cast<float*>(sm + Cf::SMALL);
  float* db0s = us + 64;
  float* xch = db0s + 64;    // [128]
  float* lam = xch + 128;    // [128] Lambda_j
  float* csp = lam + 128;    // [2][128] sum_r dS'[r,j] S0[r,j] (in the first half; the second is zero)
  float* ekp = csp + 256;    // [2][128] sum_t k o u o e^{-L} o XB by position half
  float* tail = ekp + 256;   // [128] sum of dL over positions 32..63
  __shared__ float dred[8];  // gated inputs: per-warp parts of this chunk's da_log term
  __shared__ float csred[8][D];  // per-warp parts of sum_r dS'[r,j] S0[r,j]

  if (tid == 0) {
    tc::mbar_init(&bar_a, 1);
    tc::mbar_init(&bar_b, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&bar_a, Cf::LOAD_A);
    tc::tma_load_4d(sm + Cf::LG, &tm_logf, 0, h, t0, b, &bar_a);
    tc::tma_load_4d(sm + Cf::A4, &tm_q, 0, h, t0, b, &bar_a);
    tc::tma_load_4d(sm + Cf::A4 + 16384, &tm_q, 64, h, t0, b, &bar_a);
    tc::tma_load_4d(sm + Cf::A4 + 8192, &tm_k, 0, h, t0, b, &bar_a);
    tc::tma_load_4d(sm + Cf::A4 + 24576, &tm_k, 64, h, t0, b, &bar_a);
    tc::bulk_g2s(sm + Cf::EK, wEK + ch * (C * C), 8192u, &bar_a);
    tc::mbar_expect_tx(&bar_b, Cf::LOAD_B);
    tc::bulk_g2s(sm + Cf::S0T, wS0b + ch * (D * D), 32768u, &bar_b);
    tc::bulk_g2s(sm + Cf::DST, wdSb + ch * (D * D), 32768u, &bar_b);
    tc::tma_load_4d(sm + Cf::DOV, &tm_do, 0, h, t0, b, &bar_b);
    tc::tma_load_4d(sm + Cf::DOV + 16384, &tm_do, 64, h, t0, b, &bar_b);
    tc::tma_load_4d(sm + Cf::DOV + 8192, &tm_v, 0, h, t0, b, &bar_b);
    tc::tma_load_4d(sm + Cf::DOV + 24576, &tm_v, 64, h, t0, b, &bar_b);
    tc::bulk_g2s(sm + Cf::T1, wT1 + ch * (2 * C * C), 16384u, &bar_b);
    tc::bulk_g2s(sm + Cf::B7, wPU + ch * (C * C), 8192u, &bar_b);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 512);
  // per position: g, beta, u and the chain's two dbeta terms, loaded now and
  // used after the tiles land (their round trip overlaps the tile loads)
  float gt = 0.f, bt = 0.f, ut = 0.f, b0t = 0.f, mut = 0.f;
  const size_t gi = ((size_t)b * T + t0 + tid) * H + h;
  if (tid < C) {
    gt = wg[ch * C + tid];
    bt = tid < nv ? beta[gi] : 0.f;
    ut = wu[ch * C + tid];
    b0t = wb0[ch * C + tid];
    mut = wMu[ch * C + tid];
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&bar_a, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  if (tid < C) {  // read after the prefix's barrier below
    us[tid] = ut;
    db0s[tid] = -bt * gt;
    if (tid < nv) {
      dc[gi] = gt;
      dbeta[gi] = -gt * (b0t + mut);
    }
  }
  // gated inputs: logf (formed by the forward's preparation kernel) with the
  // exponent a = e^{a_log}, for the epilogue's df~ and da_log
  const float ga = a_log ? expf(a_log[h]) : 0.f, inv_ga = a_log ? expf(-a_log[h]) : 0.f;

  // decay prefix: thread (j, half) holds L for positions 32*half .. +31
  const int j = tid & 127, half = tid >> 7;
  float Lr[32];
  split_prefix(reinterpret_cast<const float*>(sm + Cf::LG), j, half, xch, Lr);
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(Lr[i]));
  if (half) lam[j] = Lr[31];
  const bool unsafe = __syncthreads_or(!(mx < kPostSafe)) != 0;

  __nv_bfloat162 qk[32];  // raw (q, k) of this thread's positions, for dL
  if (!unsafe) {
    // Q+ and db0 o K+ in place, K-
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * half + i;
      unsigned char* pq = sm + Cf::A4 + tc::sw128_off(t, j, 128, 2);
      unsigned char* pk = sm + Cf::A4 + tc::sw128_off(64 + t, j, 128, 2);
      const __nv_bfloat16 qb = *reinterpret_cast<const __nv_bfloat16*>(pq);
      const __nv_bfloat16 kb = *reinterpret_cast<const __nv_bfloat16*>(pk);
      qk[i] = __halves2bfloat162(qb, kb);
      const float gm = expf(Lr[i]), ig = expf(-Lr[i]), kk = __bfloat162float(kb);
      put_bf(pq, __bfloat162float(qb) * gm);
      put_bf(pk, db0s[t] * kk * gm);
      put_bf(sm + Cf::KM + tc::sw128_off(t, j, 64, 2), kk * ig);
    }
    // dG_V' into rows 64..127 of B7: [i][t] = db0_i E_K[i,t] + db0_t E_K[t,i]
    {
      const int i = tid >> 2, tb = (tid & 3) * 16;
      const float di = db0s[i];
      float x[16];
#pragma unroll
      for (int tt = 0; tt < 16; ++tt) {
        const int t = tb + tt;
        x[tt] = di * bf(sm + Cf::EK + tc::sw128_off(i, t, 64, 2)) + db0s[t] * bf(sm + Cf::EK + tc::sw128_off(t, i, 64, 2));
      }
      put_row16(sm + Cf::B7, 64 + i, tb, 128, x);
    }
  }
  tc::mbar_wait<false>(&bar_b, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  if (!unsafe) {
    // dS' = dS diag(e^Lambda) in place, with the sums of dS' o S0 over r: a
    // thread takes eight channels (one 16-byte swizzle chunk) of eight rows;
    // the two row groups of a warp meet by a shuffle, the warps below in order
    const int g = tid & 15, rg = tid >> 4, lane = tid & 31;
    float e8[8], acc8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      e8[c] = expf(lam[8 * g + c]);
      acc8[c] = 0.f;
    }
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const uint32_t off = tc::sw128_off(8 * rg + rr, 8 * g, 128, 2);
      uint4 dv = *reinterpret_cast<const uint4*>(sm + Cf::DST + off);
      const uint4 sv = *reinterpret_cast<const uint4*>(sm + Cf::S0T + off);
      __nv_bfloat162* dp = reinterpret_cast<__nv_bfloat162*>(&dv);
      const __nv_bfloat162* sp = reinterpret_cast<const __nv_bfloat162*>(&sv);
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float2 d2 = __bfloat1622float2(dp[c2]);
        const float2 s2 = __bfloat1622float2(sp[c2]);
        d2.x *= e8[2 * c2];
        d2.y *= e8[2 * c2 + 1];
        acc8[2 * c2] = fmaf(d2.x, s2.x, acc8[2 * c2]);
        acc8[2 * c2 + 1] = fmaf(d2.y, s2.y, acc8[2 * c2 + 1]);
        dp[c2] = __floats2bfloat162_rn(d2.x, d2.y);
      }
      *reinterpret_cast<uint4*>(sm + Cf::DST + off) = dv;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) acc8[c] += __shfl_xor_sync(0xffffffffu, acc8[c], 16);
    if (lane < 16) {
#pragma unroll
      for (int c = 0; c < 8; ++c) csred[warp][8 * g + c] = acc8[c];
    }
    tc::fence_proxy_async();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (!unsafe && tid < D) {  // read by the epilogue, after its barriers
    float cs = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) cs += csred[w][tid];
    csp[tid] = cs;
    csp[128 + tid] = 0.f;
  }

  if (!unsafe) {
    if (tid == 0) {
      auto smd = [&](uint32_t off) { return tc::smem_u32(sm + off); };
      const uint32_t ID_A = tc::idesc(128, 128, 1) | (1u << 15);             // A MN-major
      const uint32_t ID_MN = tc::idesc(128, 64, 1) | (1u << 15);             // A MN-major
      const uint32_t ID_MM = tc::idesc(128, 64, 1) | (1u << 15) | (1u << 16);  // A and B MN-major
      const uint32_t ID_KK = tc::idesc(128, 64, 1);                          // both K-major
      // QT | XA = S0^T [dO; V]^T + K-^T [dP; E_V]^T
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_A, tc::desc_sw128_mn(smd(Cf::S0T + ks * 2048), 16384u),
                        tc::desc_sw128(smd(Cf::DOV + (ks / 4) * 16384 + (ks % 4) * 32)), ID_A, ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_A, tc::desc_sw128_mn(smd(Cf::KM + ks * 2048), 8192u),
                        tc::desc_sw128(smd(Cf::T1 + ks * 32)), ID_A, 1u);
      // XB = dS'^T V^T
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_XB, tc::desc_sw128_mn(smd(Cf::DST + ks * 2048), 16384u),
                        tc::desc_sw128(smd(Cf::DOV + (ks / 4) * 16384 + 8192 + (ks % 4) * 32)), ID_MN,
                        ks > 0 ? 1u : 0u);
      // R2 = [Q+; db0 o K+]^T [dP; E_V]
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_R2, tc::desc_sw128_mn(smd(Cf::A4 + ks * 2048), 16384u),
                        tc::desc_sw128_mn(smd(Cf::T1 + ks * 2048), 8192u), ID_MM, ks > 0 ? 1u : 0u);
      // VT = S0 (db0 o K+)^T + [dO; V]^T [P diag(u); dG_V']
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_VT, tc::desc_sw128(smd(Cf::S0T + (ks / 4) * 16384 + (ks % 4) * 32)),
                        tc::desc_sw128(smd(Cf::A4 + (ks / 4) * 16384 + 8192 + (ks % 4) * 32)), ID_KK,
                        ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_VT, tc::desc_sw128_mn(smd(Cf::DOV + ks * 2048), 16384u),
                        tc::desc_sw128_mn(smd(Cf::B7 + ks * 2048), 8192u), ID_MM, 1u);
      // VD = dS' K-^T
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss(tmem + Cf::C_VD, tc::desc_sw128(smd(Cf::DST + (ks / 4) * 16384 + (ks % 4) * 32)),
                        tc::desc_sw128(smd(Cf::KM + (ks / 4) * 8192 + (ks % 4) * 32)), ID_KK, ks > 0 ? 1u : 0u);
      tc::mma_commit(&mma_bar);
    }
    tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
    tc::tc_after_sync();

    // epilogue: lane j (or r) of every accumulator, positions 32*half .. +31
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
    unsigned char* oq = sm + Cf::OQ;
    unsigned char* ok = sm + Cf::OK;
    unsigned char* ov = sm + Cf::OV;
    float* ol = reinterpret_cast<float*>(sm + Cf::OL);
    float dL[32];
    float ekj = 0.f;
#pragma unroll
    for (int c16 = 0; c16 < 2; ++c16) {
      const int tb = 32 * half + 16 * c16;
      float qt[16], xa[16], xb[16], r2[16];
      tc::tmem_ld16(lanes + Cf::C_A + tb, qt);
      tc::tmem_ld16(lanes + Cf::C_A + 64 + tb, xa);
      tc::tmem_ld16(lanes + Cf::C_XB + tb, xb);
      tc::tmem_ld16(lanes + Cf::C_R2 + tb, r2);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int i = 16 * c16 + ii, t = tb + ii;
        const float gm = expf(Lr[i]), ig = expf(-Lr[i]);
        const float qq = __low2float(qk[i]), kk = __high2float(qk[i]);
        const float dq = gm * qt[ii];
        const float a = gm * db0s[t] * xa[ii];
        const float bb = us[t] * ig * xb[ii];
        const float cc = ig * r2[ii];
        dL[i] = fmaf(qq, dq, kk * (a - bb - cc));
        ekj = fmaf(kk, bb, ekj);
        put_bf(oq + tc::sw128_off(t, j, 64, 2), dq);
        put_bf(ok + tc::sw128_off(t, j, 64, 2), a + bb + cc);
      }
      float vt[16], vd[16];
      tc::tmem_ld16(lanes + Cf::C_VT + tb, vt);
      tc::tmem_ld16(lanes + Cf::C_VD + tb, vd);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int t = tb + ii;
        put_bf(ov + tc::sw128_off(t, j, 64, 2), fmaf(us[t], vd[ii], vt[ii]));  // lane j is value channel r
      }
    }
    // dlogf: reverse cumulative sum over the chunk, plus the chunk-end term
    float run = 0.f;
#pragma unroll
    for (int i = 31; i >= 0; --i) {
      run += dL[i];
      dL[i] = run;
    }
    ekp[half * 128 + j] = ekj;
    if (half) tail[j] = run;
    __syncthreads();
    const float add = ekp[j] + ekp[128 + j] + csp[j] + csp[128 + j] + (half ? 0.f : tail[j]);
    if (a_log) {
      // gated inputs: df~ = dlogf a sigma(-f~), and this chunk's part of
      // da_log = sum dlogf logf (d logf / d a_log = logf), reduced in a fixed order
      const float* lgs = reinterpret_cast<const float*>(sm + Cf::LG);
      float dap = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float lf = lgs[(32 * half + i) * D + j], dl = dL[i] + add;
        dap = fmaf(dl, lf, dap);
        ol[(32 * half + i) * D + j] = dl * dlogf_dfpre(lf, ga, inv_ga);
      }
      dap = warp_sum(dap);
      if ((tid & 31) == 0) dred[warp] = dap;
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) ol[(32 * half + i) * D + j] = dL[i] + add;
    }
    tc::fence_proxy_async();
    __syncthreads();
    if (a_log && tid == 0) {
      float s2 = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s2 += dred[w];
      dapart[ch] = s2;
    }
    if (tid == 0) {
      tc::tma_store_4d(&tm_dq, oq, 0, h, t0, b);
      tc::tma_store_4d(&tm_dq, oq + 8192, 64, h, t0, b);
      tc::tma_store_4d(&tm_dk, ok, 0, h, t0, b);
      tc::tma_store_4d(&tm_dk, ok + 8192, 64, h, t0, b);
      tc::tma_store_4d(&tm_dv, ov, 0, h, t0, b);
      tc::tma_store_4d(&tm_dv, ov + 8192, 64, h, t0, b);
      tc::tma_store_4d(&tm_dlogf, ol, 0, h, t0, b);
      tc::bulk_commit();
      tc::bulk_wait_read();
    }
  }
  if (tid == 0) flags[ch] = unsafe ? 1 : 0;
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_bwd_pre_tc(const BwdArgs& a, int* err, int sms, cudaStream_t st) {
  const Layout& L = a.L;
  CUtensorMap tm_v, tm_do, tm_k, tm_logf, tm_q, tm_kp;
  if (!make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_do, a.dO, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_logf, a.logf, 4, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_kp, ws_ptr<float>(a.ws, L.Kp), 4, L.B, L.T, L.H, D, 32, true))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_pre_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PreCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "bwd_pre_tc");
  bwd_pre_tc<<<(unsigned)L.chunks, 256, PreCfg::BYTES, st>>>(
      tm_v, tm_do, tm_k, tm_logf, tm_q, tm_kp, L.H, L.NC, ws_ptr<float>(a.fws, L.P),
      ws_ptr<float>(a.fws, L.u), ws_ptr<float>(a.ws, L.du), ws_ptr<float>(a.ws, L.Mu),
      ws_ptr<__nv_bfloat16>(a.ws, L.T1), ws_ptr<__nv_bfloat16>(a.ws, L.PU), ws_ptr<__nv_bfloat16>(a.ws, L.EK),
      ws_ptr<__nv_bfloat16>(a.ws, L.QpT), sms, err);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_bwd_post_tc(const BwdArgs& a, int* err, cudaStream_t st) {
  const Layout& L = a.L;
  CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_logf, tm_dq, tm_dk, tm_dv, tm_dlogf;
  if (!make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_do, a.dO, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_logf, a.logf, 4, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_dq, a.dq, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_dk, a.dk, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_dv, a.dv, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_dlogf, a.dlogf, 4, L.B, L.T, L.H, D, 128, false))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(bwd_post_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PostCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "bwd_post_tc");
  bwd_post_tc<<<(unsigned)L.chunks, 256, PostCfg::BYTES, st>>>(
      tm_q, tm_k, tm_v, tm_do, tm_logf, tm_dq, tm_dk, tm_dv, tm_dlogf, a.beta, L.H, L.T, L.NC,
      ws_ptr<float>(a.fws, L.u), ws_ptr<float>(a.fws, L.b0), ws_ptr<float>(a.ws, L.g), ws_ptr<float>(a.ws, L.Mu),
      ws_ptr<__nv_bfloat16>(a.fws, L.S0b), ws_ptr<__nv_bfloat16>(a.ws, L.dSCb), ws_ptr<__nv_bfloat16>(a.ws, L.T1),
      ws_ptr<__nv_bfloat16>(a.ws, L.PU), ws_ptr<__nv_bfloat16>(a.ws, L.EK), a.dbeta, a.dc,
      ws_ptr<int>(a.ws, L.bflags), a.a_log, ws_ptr<float>(a.ws, L.dapart), err);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
