// kd_bwd_tc.cu -- tensor-core reverse chain for bf16 q,k,v,dO and
// d_k = d_v = 128.
//
// Reverse-mode of the chunk recurrence (derived here; the pages only ask for a
// gate-aware backward: Gated DeltaNet-2 article, "핵심 기여").  Walking the
// chunks from last to first with dS = dL/d(chunk-end state):
//   du   = du_intra + rowdot(V, dS K^e^T),  du_intra[i] = sum_{t>=i} P[t,i] (dO_t . v_i)
//   g    = A^T du,   db0 = -beta o g
//   dS  <- dS diag(gamma_C) + dO^T Q+ + V^T diag(db0) K+
// The cluster / warp-role structure follows the forward chain (kd_fwd_tc.cu):
// CTA c of an R-CTA cluster keeps the key-channel slice dS[:, J_c] in tensor
// memory; the per-chunk du partial sums are all-reduced over the cluster.
//   MMA 1 (tf32, A = dS slice from TMEM):  Z_c = dS[:,J_c] K^e[:,J_c]^T
//   MMA 3 (bf16, off the critical path):   dO^T Q+[:,J_c]
//   MMA 2 (bf16):                          V^T (db0 o K+[:,J_c])
// dO and V reach shared memory by TMA in the 128-byte-swizzled layout that the
// MMAs read directly as MN-major A operands.  Each chunk's dS (before the
// chunk's update) and g are written out for the parallel gradient kernels.
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;

template <int R>
struct BChainCfg {
  static constexpr int NJ = D / R;
  static constexpr int KB1 = (NJ * 4 + 127) / 128;
  static constexpr int TPC = 128 / NJ;
  static constexpr int SEG = C / TPC;
  static constexpr int KPS = NJ + 1;
  static constexpr int D1_COL = 0, S_COL = 64, D2_COL = 64 + NJ, D3_COL = 64 + 2 * NJ;
  static constexpr uint32_t TMEM_COLS = (64 + 3 * NJ) <= 128 ? 128u : 256u;
  static constexpr uint32_t up1k(uint32_t x) { return (x + 1023u) / 1024u * 1024u; }
  // operand buffer (two): K^e slice (tf32, B of MMA 1), K+ slice (fp32), Q+^T slice (bf16, B of MMA 3), gamma_C
  static constexpr uint32_t OP_B1 = 0;
  static constexpr uint32_t OP_BQ = OP_B1 + KB1 * 8192;          // NJ rows x 128 B
  static constexpr uint32_t OP_KP = OP_BQ + up1k(NJ * 128);      // fp32 [64][KPS]
  static constexpr uint32_t OP_GC = OP_KP + 64 * KPS * 4;
  static constexpr uint32_t OP_SZ = up1k(OP_GC + NJ * 4);
  // raw staging (two): V and dO as two swizzled 64-channel halves, A, du_intra, k/q/logf slices
  static constexpr uint32_t ST_V = 0, ST_DO = 16384, ST_A = 32768, ST_DU = 49152;
  static constexpr uint32_t ST_K = ST_DU + 256, ST_Q = ST_K + 64 * NJ * 2, ST_L = ST_Q + 64 * NJ * 2;
  static constexpr uint32_t ST_SZ = up1k(ST_L + 64 * NJ * 4);
  static constexpr uint32_t LOAD_BYTES = 3 * 16384 + 256 + 64 * NJ * 8;
  static constexpr uint32_t OPS = 0, STG = OPS + 2 * OP_SZ;
  static constexpr uint32_t B2 = STG + 2 * ST_SZ;                 // db0 o K+ slice, bf16, NJ rows x 128 B
  static constexpr uint32_t SM = B2 + up1k(NJ * 128);
  static constexpr uint32_t SM_BS = SM;                           // beta [2][64]
  static constexpr uint32_t SM_DU = SM_BS + 2 * 64 * 4;           // du [64]
  static constexpr uint32_t SM_GP = SM_DU + 64 * 4;               // g partial sums [2][64]
  static constexpr uint32_t SM_DB = SM_GP + 2 * 64 * 4;           // db0 [64]
  static constexpr uint32_t SM_MINE = SM_DB + 64 * 4;
  static constexpr uint32_t SM_XRED = SM_MINE + 64 * 4;
  static constexpr uint32_t SM_RECV = SM_XRED + 4 * 64 * 4;
  static constexpr uint32_t SM_SEG = SM_RECV + 2 * R * 64 * 4;
  static constexpr uint32_t SM_END = SM_SEG + TPC * NJ * 4;
  static constexpr uint32_t BYTES = SM_END + 1024;
};

__device__ __forceinline__ void bar_chain() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_prod() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(b)) : "memory");
}
// element (t, r) of a [64 positions][128 channels] bf16 tile stored as two
// 128-byte-swizzled 64-channel halves (the TMA layout)
__device__ __forceinline__ float tile_bf16(const unsigned char* base, int t, int r) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + tc::sw128_off(t, r, 64, 2)));
}

template <int R>
__global__ void __launch_bounds__(256, 1) bwd_chain_tc(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
    const __grid_constant__ CUtensorMap tm_logf, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ beta,
    const float* __restrict__ dST, float* __restrict__ dS0, int H, int T, int NC,
    const float* __restrict__ wA, const float* __restrict__ wdu, __nv_bfloat16* __restrict__ wdSCb,
    float* __restrict__ wg, int* __restrict__ err) {
  using Cf = BChainCfg<R>;
  constexpr int NJ = Cf::NJ;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t raw_full[2], op_full[2], freeb[2], s_ready, s_saved, x_bar[2], mma_bar, mma3_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_rank();
  const int unit = blockIdx.x / R;
  const int b = unit / H, h = unit % H;
  const int j0 = static_cast<int>(rank) * NJ;

  float* bs = reinterpret_cast<float*>(sm + Cf::SM_BS);
  float* dus = reinterpret_cast<float*>(sm + Cf::SM_DU);
  float* gp = reinterpret_cast<float*>(sm + Cf::SM_GP);
  float* db0 = reinterpret_cast<float*>(sm + Cf::SM_DB);
  float* mine = reinterpret_cast<float*>(sm + Cf::SM_MINE);
  float* xred = reinterpret_cast<float*>(sm + Cf::SM_XRED);
  float* recv = reinterpret_cast<float*>(sm + Cf::SM_RECV);
  float* segs = reinterpret_cast<float*>(sm + Cf::SM_SEG);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&raw_full[i], 1);
      tc::mbar_init(&op_full[i], 1);
      tc::mbar_init(&freeb[i], 1);
      tc::mbar_init(&x_bar[i], 1);
    }
    tc::mbar_init(&s_ready, 1);
    tc::mbar_init(&s_saved, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init(&mma3_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, Cf::TMEM_COLS);
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t my_lanes = tc::tmem_lane_addr(tmem, warp, 0);

  if (warp >= 4) {
    // =========================== producer warps ===========================
    const int p = tid - 128;
    auto issue = [&](int k) {  // k-th chunk processed = chunk NC-1-k
      const int n = NC - 1 - k;
      unsigned char* st = sm + Cf::STG + (k & 1) * Cf::ST_SZ;
      uint64_t* bar = &raw_full[k & 1];
      const size_t ch = (size_t)unit * NC + n;
      tc::fence_proxy_async();
      tc::mbar_expect_tx(bar, Cf::LOAD_BYTES);
      tc::tma_load_4d(st + Cf::ST_V, &tm_v, 0, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_V + 8192, &tm_v, 64, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_DO, &tm_do, 0, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_DO + 8192, &tm_do, 64, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_K, &tm_k, j0, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_Q, &tm_q, j0, h, n * C, b, bar);
      tc::tma_load_4d(st + Cf::ST_L, &tm_logf, j0, h, n * C, b, bar);
      tc::bulk_g2s(st + Cf::ST_A, wA + ch * C * C, 64u * 64u * 4u, bar);
      tc::bulk_g2s(st + Cf::ST_DU, wdu + ch * C, 256u, bar);
    };
    if (p == 0) {
      issue(0);
      if (NC > 1) issue(1);
    }
    for (int k = 0; k < NC; ++k) {
      const int n = NC - 1 - k, pb = k & 1;
      unsigned char* st = sm + Cf::STG + pb * Cf::ST_SZ;
      unsigned char* op = sm + Cf::OPS + pb * Cf::OP_SZ;
      if (k >= 2) {
        tc::mbar_wait<false>(&freeb[pb], (uint32_t)(((k - 2) >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
        if (p == 0) issue(k);
      }
      const float bt = (p < C && n * C + p < T) ? beta[((size_t)b * T + n * C + p) * H + h] : 0.f;
      tc::mbar_wait<false>(&raw_full[pb], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      if (p < C) bs[pb * 64 + p] = bt;
      {
        const int j = p % NJ, seg = p / NJ;
        const float* lrow = reinterpret_cast<const float*>(st + Cf::ST_L);
        float lp[Cf::SEG];
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < Cf::SEG; ++i) {
          acc += lrow[(seg * Cf::SEG + i) * NJ + j];
          lp[i] = acc;
        }
        segs[seg * NJ + j] = acc;
        bar_prod();
        float pre = 0.f, tot = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < Cf::TPC; ++s2) {
          const float x = segs[s2 * NJ + j];
          if (s2 < seg) pre += x;
          tot += x;
        }
        float* KP = reinterpret_cast<float*>(op + Cf::OP_KP);
        if (seg == 0) reinterpret_cast<float*>(op + Cf::OP_GC)[j] = expf(tot);
#pragma unroll
        for (int i = 0; i < Cf::SEG; ++i) {
          const int t = seg * Cf::SEG + i;
          const float L = pre + lp[i];
          const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + Cf::ST_K + (t * NJ + j) * 2));
          const float qq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + Cf::ST_Q + (t * NJ + j) * 2));
          const float g = expf(L);
          *reinterpret_cast<float*>(op + Cf::OP_B1 + tc::sw128_off(t, j, 64, 4)) = kk * expf(tot - L);
          KP[t * Cf::KPS + j] = kk * g;
          *reinterpret_cast<__nv_bfloat16*>(op + Cf::OP_BQ + tc::sw128_off(j, t, NJ, 2)) = __float2bfloat16_rn(qq * g);
        }
      }
      tc::fence_proxy_async();
      bar_prod();
      if (p == 0) mbar_arrive(&op_full[pb]);
      // save dS of this chunk (gradient of its end state) once the chain has it,
      // as the bf16 tile [r][j] the post-chain kernel's MMAs read
      tc::mbar_wait<false>(&s_ready, (uint32_t)(k & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        const size_t ch = (size_t)unit * NC + n;
        unsigned char* a = reinterpret_cast<unsigned char*>(wdSCb + ch * D * D);
#pragma unroll
        for (int jj = 0; jj < NJ; jj += 16) {
          float x[16];
          tc::tmem_ld16(my_lanes + Cf::S_COL + jj, x);
          tc::tmem_ld_wait();
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v8[i] = __float2bfloat16_rn(x[8 * h8 + i]);
            *reinterpret_cast<uint4*>(a + tc::sw128_off(p, j0 + jj + 8 * h8, 128, 2)) = *reinterpret_cast<const uint4*>(v8);
          }
        }
      }
      tc::tc_before_sync();
      bar_prod();
      if (p == 0) mbar_arrive(&s_saved);
    }
  } else {
    // ============================= chain warps ============================
    const int r = tid;
    {
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = dST ? dST[(size_t)unit * D * D + (size_t)r * D + j0 + jj + i] : 0.f;
        tc::tmem_st16(my_lanes + Cf::S_COL + jj, x);
      }
      tc::tmem_st_wait();
      tc::tc_before_sync();
      bar_chain();
      if (tid == 0) mbar_arrive(&s_ready);
    }
    int mma_par = 0, mma3_par = 0;
    const uint32_t ID1 = tc::idesc(128, 64, 2);
    const uint32_t IDB = tc::idesc(128, NJ, 1) | (1u << 15);  // bf16, A MN-major
    for (int k = 0; k < NC; ++k) {
      const int n = NC - 1 - k, pb = k & 1;
      const unsigned char* st = sm + Cf::STG + pb * Cf::ST_SZ;
      const unsigned char* op = sm + Cf::OPS + pb * Cf::OP_SZ;
      const size_t ch = (size_t)unit * NC + n;
      tc::mbar_wait<false>(&op_full[pb], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::tc_after_sync();
      if (tid == 0) {
        // MMA 1: Z_c = dS[:,J_c] K^e[:,J_c]^T  (M=128 rows r, N=64 positions, K=NJ)
#pragma unroll
        for (int ks = 0; ks < NJ / 8; ++ks) {
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(op + Cf::OP_B1 + (ks / 4) * 8192 + (ks % 4) * 32));
          tc::mma_tf32_ts(tmem + Cf::D1_COL, tmem + Cf::S_COL + ks * 8, bd, ID1, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mma_bar);
        // MMA 3: dO^T Q+[:,J_c]  (M=128, N=NJ, K=64): not needed until the update
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128_mn(tc::smem_u32(st + Cf::ST_DO + ks * 2048), 8192u);
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(op + Cf::OP_BQ + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::D3_COL, ad, bd, IDB, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mma3_bar);
      }
      tc::mbar_wait<false>(&mma_bar, (uint32_t)mma_par, err, tc::kErrTimeoutMma, &abort_flag);
      mma_par ^= 1;
      tc::tc_after_sync();
      // du_c[t] = sum_r V[t,r] Z_c[r,t]
      {
        float x[64];
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
          float y16[16];
          tc::tmem_ld16(my_lanes + Cf::D1_COL + 16 * c16, y16);
#pragma unroll
          for (int i = 0; i < 16; ++i) x[16 * c16 + i] = y16[i];
        }
        tc::tmem_ld_wait();
        float lo[32], hi[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          lo[t] = x[t] * tile_bf16(st + Cf::ST_V, t, r);
          hi[t] = x[32 + t] * tile_bf16(st + Cf::ST_V, 32 + t, r);
        }
        warp_transpose_reduce<32>(lo, lane);
        warp_transpose_reduce<32>(hi, lane);
        xred[warp * 64 + lane] = lo[0];
        xred[warp * 64 + 32 + lane] = hi[0];
      }
      bar_chain();
      if (tid < C) mine[tid] = xred[tid] + xred[64 + tid] + xred[128 + tid] + xred[192 + tid];
      bar_chain();
      {
        float* rv = recv + pb * R * 64;
        if (tid == 0) tc::mbar_expect_tx(&x_bar[pb], R * 64u * 4u);
        if (tid < 16 * R) {
          const int peer = tid / 16, q4 = tid % 16;
          const float4 val = *reinterpret_cast<const float4*>(mine + 4 * q4);
          const uint32_t raddr = tc::mapa(tc::smem_u32(rv + rank * 64 + 4 * q4), (uint32_t)peer);
          const uint32_t rbar = tc::mapa(tc::smem_u32(&x_bar[pb]), (uint32_t)peer);
          tc::st_async_v4(raddr, val, rbar);
        }
        tc::mbar_wait<true>(&x_bar[pb], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutCluster, &abort_flag);
        if (tid < C) {
          float s = reinterpret_cast<const float*>(st + Cf::ST_DU)[tid];
#pragma unroll
          for (int c2 = 0; c2 < R; ++c2) s += rv[c2 * 64 + tid];
          dus[tid] = s;
        }
      }
      bar_chain();
      // g = A^T du (two threads per column), db0 = -beta o g
      {
        const int i = tid & 63, half = tid >> 6;
        const float* Acol = reinterpret_cast<const float*>(st + Cf::ST_A) + i;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int t = 32 * half; t < 32 * half + 32; t += 4) {
          a0 = fmaf(Acol[t * 64], dus[t], a0);
          a1 = fmaf(Acol[(t + 1) * 64], dus[t + 1], a1);
          a2 = fmaf(Acol[(t + 2) * 64], dus[t + 2], a2);
          a3 = fmaf(Acol[(t + 3) * 64], dus[t + 3], a3);
        }
        gp[half * 64 + i] = (a0 + a1) + (a2 + a3);
      }
      bar_chain();
      if (tid < C) {
        const float g = gp[tid] + gp[64 + tid];
        db0[tid] = -bs[pb * 64 + tid] * g;
        if (rank == 0) wg[ch * C + tid] = g;
      }
      bar_chain();
      // B2[j][t] = db0_t K+[t, j]  (bf16, N = NJ rows, K = 64)
      {
        const int t = tid & 63, jh = tid >> 6;
        const float d = db0[t];
        const float* KP = reinterpret_cast<const float*>(op + Cf::OP_KP);
#pragma unroll
        for (int i = 0; i < NJ / 2; ++i) {
          const int j = jh * (NJ / 2) + i;
          *reinterpret_cast<__nv_bfloat16*>(sm + Cf::B2 + tc::sw128_off(j, t, NJ, 2)) =
              __float2bfloat16_rn(d * KP[t * Cf::KPS + j]);
        }
      }
      tc::fence_proxy_async();
      tc::tc_before_sync();
      bar_chain();
      tc::tc_after_sync();
      if (tid == 0) {
        // MMA 2: V^T B2  (A = V, MN-major; M=128, N=NJ, K=64)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128_mn(tc::smem_u32(st + Cf::ST_V + ks * 2048), 8192u);
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(sm + Cf::B2 + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::D2_COL, ad, bd, IDB, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mma_bar);
      }
      tc::mbar_wait<false>(&mma_bar, (uint32_t)mma_par, err, tc::kErrTimeoutMma, &abort_flag);
      mma_par ^= 1;
      tc::mbar_wait<false>(&mma3_bar, (uint32_t)mma3_par, err, tc::kErrTimeoutMma, &abort_flag);
      mma3_par ^= 1;
      tc::mbar_wait<false>(&s_saved, (uint32_t)(k & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        const float* gC = reinterpret_cast<const float*>(op + Cf::OP_GC);
#pragma unroll
        for (int jj = 0; jj < NJ; jj += 16) {
          float s[16], d2[16], d3[16];
          tc::tmem_ld16(my_lanes + Cf::S_COL + jj, s);
          tc::tmem_ld16(my_lanes + Cf::D2_COL + jj, d2);
          tc::tmem_ld16(my_lanes + Cf::D3_COL + jj, d3);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) s[i] = fmaf(s[i], gC[jj + i], d2[i] + d3[i]);
          tc::tmem_st16(my_lanes + Cf::S_COL + jj, s);
        }
        tc::tmem_st_wait();
      }
      tc::tc_before_sync();
      bar_chain();
      if (tid == 0) {
        mbar_arrive(&freeb[pb]);
        mbar_arrive(&s_ready);
      }
    }
    if (dS0) {
      tc::tc_after_sync();
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float x[16];
        tc::tmem_ld16(my_lanes + Cf::S_COL + jj, x);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) dS0[(size_t)unit * D * D + (size_t)r * D + j0 + jj + i] = x[i];
      }
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
}

template <int R>
cudaError_t launch_bchain(const BwdArgs& a, int* err, cudaStream_t st) {
  const Layout& L = a.L;
  constexpr int NJ = BChainCfg<R>::NJ;
  CUtensorMap tm_k, tm_q, tm_logf, tm_v, tm_do;
  if (!make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, NJ, false) ||
      !make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, NJ, false) ||
      !make_tmap_bthd(&tm_logf, a.logf, 4, L.B, L.T, L.H, D, NJ, false) ||
      !make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_do, a.dO, 2, L.B, L.T, L.H, D, 64, true))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)BChainCfg<R>::BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.B * L.H * R);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = BChainCfg<R>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(st, "bwd_chain_tc");
  e = cudaLaunchKernelEx(&cfg, bwd_chain_tc<R>, tm_k, tm_q, tm_logf, tm_v, tm_do, a.beta, a.dST, a.dS0,
                         L.H, L.T, L.NC, ws_ptr<float>(a.fws, L.A), ws_ptr<float>(a.ws, L.du),
                         ws_ptr<__nv_bfloat16>(a.ws, L.dSCb), ws_ptr<float>(a.ws, L.g), err);
  prof_end(st);
  return e;
}

}  // namespace

cudaError_t launch_bwd_tc(const BwdArgs& a, int* err, int sms, cudaStream_t st) {
  const Layout& L = a.L;
  cudaError_t e;
  if (a.phases & kPhaseLocal) {
    if ((e = launch_bwd_pre_tc(a, err, st)) != cudaSuccess) return e;
  }
  if (!(a.phases & kPhaseCarry)) return cudaSuccess;
  const int R = choose_cluster(L.B * L.H, sms);
  e = (R == 8) ? launch_bchain<8>(a, err, st) : launch_bchain<4>(a, err, st);
  if (e != cudaSuccess) return e;
  if ((e = launch_bwd_post_tc(a, err, st)) != cudaSuccess) return e;
  // chunks outside the factorised decay range: exact CUDA-core recomputation
  return launch_bwd_simt_stages(a, kStageCC | kStageState | kStageIntra, ws_ptr<int>(a.ws, L.bflags), st);
}

}  // namespace kd
