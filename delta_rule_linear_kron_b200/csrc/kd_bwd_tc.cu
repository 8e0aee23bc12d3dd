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
    __nv_bfloat16* __restrict__ wdSCbt, float* __restrict__ wg, int* __restrict__ err) {
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
      // as the two bf16 tiles the state-product kernel's MMAs read
      tc::mbar_wait<false>(&s_ready, (uint32_t)(k & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        const size_t ch = (size_t)unit * NC + n;
        unsigned char* a = reinterpret_cast<unsigned char*>(wdSCb + ch * D * D);
        unsigned char* tt = reinterpret_cast<unsigned char*>(wdSCbt + ch * D * D);
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
#pragma unroll
          for (int i = 0; i < 16; ++i)
            *reinterpret_cast<__nv_bfloat16*>(tt + tc::sw128_off(j0 + jj + i, p, 128, 2)) = __float2bfloat16_rn(x[i]);
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

// du_intra[i] = sum_{t>=i} P[t,i] (dO_t . v_i) for every chunk, in parallel
__global__ void __launch_bounds__(256) bwd_du_intra(const __nv_bfloat16* __restrict__ v,
                                                    const __nv_bfloat16* __restrict__ dO, int H, int T,
                                                    int NC, const float* __restrict__ wP,
                                                    float* __restrict__ wdu) {
  extern __shared__ float sm_du[];
  float* Ds = sm_du;                   // [64][129]
  float* Vs = Ds + C * (D + 1);        // [64][129]
  float* Ps = Vs + C * (D + 1);        // [64][65]
  const int tid = threadIdx.x;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  for (int e = tid; e < C * D; e += 256) {
    const int t = e / D, r = e % D;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + r;
    Ds[t * (D + 1) + r] = t < nv ? __bfloat162float(dO[g]) : 0.f;
    Vs[t * (D + 1) + r] = t < nv ? __bfloat162float(v[g]) : 0.f;
  }
  for (int e = tid; e < C * C; e += 256) Ps[(e / C) * (C + 1) + e % C] = wP[ch * C * C + e];
  __syncthreads();
  const int i = tid >> 2, q = tid & 3;  // 4 threads per column i
  float acc = 0.f;
  for (int t = i + q; t < C; t += 4) {
    float d = 0.f;
    for (int r = 0; r < D; ++r) d = fmaf(Ds[t * (D + 1) + r], Vs[i * (D + 1) + r], d);
    acc = fmaf(Ps[t * (C + 1) + i], d, acc);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (q == 0) wdu[ch * C + i] = acc;
}

// ---------------------------------------------------------------------------
// State products of the backward, one CTA per chunk, all chunks in parallel:
//   dO S0, V S0, V dS (C x dk) and K+ S0^T, K^e dS^T (C x dv), as four bf16
//   tcgen05 MMAs (M=128, N=128, K=128) into the 512 tensor-memory columns:
//     P1 = [dO; V] x S0^T-tile   -> rows 0-63: dO S0,  rows 64-127: V S0
//     P2 = [dO; V] x dS^T-tile   -> rows 64-127: V dS
//     P3 = [K+; K^e] x S0-tile   -> rows 0-63: K+ S0^T
//     P4 = [K+; K^e] x dS-tile   -> rows 64-127: K^e dS^T
// and combines them with the gates into the per-token accumulators the
// intra-chunk gradient kernel consumes:
//   accq = (dO S0) o gamma
//   acck = db0 (V S0) o gamma + u (V dS) o e^{L_C-L}
//   accL = (dO S0) o Q+ + db0 (V S0) o K+ - u (V dS) o K^e   (+ chunk-end terms on the last row)
//   accv = db0 (K+ S0^T) + u (K^e dS^T)
// ---------------------------------------------------------------------------
struct StCfg {
  static constexpr uint32_t OPA = 0;            // [dO; V] bf16, 2 K blocks x 128 rows x 128 B
  static constexpr uint32_t OPK = 32768;        // [K+; K^e] bf16, same shape
  static constexpr uint32_t S0T = 65536;        // chunk-start state, [j][r] tile
  static constexpr uint32_t DST = 98304;        // dS, [j][r] tile
  static constexpr uint32_t S0R = 131072;       // chunk-start state, [r][j] tile
  static constexpr uint32_t DSR = 163840;       // dS, [r][j] tile
  static constexpr uint32_t SMALL = 196608;     // u, db0, colsum, ek partials, L_C
  static constexpr uint32_t BYTES = SMALL + (64 + 64 + 128 + 4 * 64 + 128) * 4 + 1024;
  // epilogue reuse of the operand area (after the MMAs): L, EX1, EX2 as fp32 [64][129]
  static constexpr uint32_t LS = 0, EX1 = 65536, EX2 = 131072;
};

__global__ void __launch_bounds__(256, 1) bwd_state_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const float* __restrict__ beta,
    const float* __restrict__ logf, int H, int T, int NC, const float* __restrict__ wu,
    const float* __restrict__ wg, const __nv_bfloat16* __restrict__ wS0b, const __nv_bfloat16* __restrict__ wS0bt,
    const __nv_bfloat16* __restrict__ wdSCb, const __nv_bfloat16* __restrict__ wdSCbt,
    float* __restrict__ waccq, float* __restrict__ wacck, float* __restrict__ waccL,
    float* __restrict__ waccv, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  float* us = reinterpret_cast<float*>(sm + StCfg::SMALL);
  float* db0 = us + 64;
  float* csum = db0 + 64;          // [128] sum_r dS[r,j] S0[r,j]
  float* ekp = csum + 128;         // [4][64] per-warp column sums
  float* lC = ekp + 256;           // [128] L at the chunk end

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, 32768u + 4u * 32768u);
    tc::tma_load_4d(sm + StCfg::OPA, &tm_do, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + StCfg::OPA + 16384, &tm_do, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + StCfg::OPA + 8192, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + StCfg::OPA + 16384 + 8192, &tm_v, 64, h, t0, b, &ld_bar);
    tc::bulk_g2s(sm + StCfg::S0T, wS0bt + ch * D * D, 32768u, &ld_bar);
    tc::bulk_g2s(sm + StCfg::DST, wdSCbt + ch * D * D, 32768u, &ld_bar);
    tc::bulk_g2s(sm + StCfg::S0R, wS0b + ch * D * D, 32768u, &ld_bar);
    tc::bulk_g2s(sm + StCfg::DSR, wdSCb + ch * D * D, 32768u, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 512);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;

  float Lr[C];  // threads 0..127: decay prefix of channel j = tid
  if (tid < 128) {
    const int j = tid;
    float L = 0.f;
#pragma unroll
    for (int t = 0; t < C; ++t) {
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + j;
      L += t < nv ? logf[g] : 0.f;
      Lr[t] = L;
    }
    lC[j] = L;
#pragma unroll
    for (int t = 0; t < C; ++t) {
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + j;
      const float kk = t < nv ? __bfloat162float(k[g]) : 0.f;
      *reinterpret_cast<__nv_bfloat16*>(sm + StCfg::OPK + tc::sw128_off(t, j, 128, 2)) =
          __float2bfloat16_rn(kk * expf(Lr[t]));
      *reinterpret_cast<__nv_bfloat16*>(sm + StCfg::OPK + tc::sw128_off(64 + t, j, 128, 2)) =
          __float2bfloat16_rn(kk * expf(L - Lr[t]));
    }
  } else {
    const int i = tid - 128;
    if (i < C) {
      us[i] = wu[ch * C + i];
      const float bt = i < nv ? beta[((size_t)b * T + t0 + i) * H + h] : 0.f;
      db0[i] = -bt * wg[ch * C + i];
    }
  }
  tc::fence_proxy_async();
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    const uint32_t ID = tc::idesc(128, 128, 1);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks / 4) * 16384 + (ks % 4) * 32;
      const uint64_t a1 = tc::desc_sw128(tc::smem_u32(sm + StCfg::OPA + off));
      const uint64_t a2 = tc::desc_sw128(tc::smem_u32(sm + StCfg::OPK + off));
      tc::mma_bf16_ss(tmem + 0, a1, tc::desc_sw128(tc::smem_u32(sm + StCfg::S0T + off)), ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + 128, a1, tc::desc_sw128(tc::smem_u32(sm + StCfg::DST + off)), ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + 256, a2, tc::desc_sw128(tc::smem_u32(sm + StCfg::S0R + off)), ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + 384, a2, tc::desc_sw128(tc::smem_u32(sm + StCfg::DSR + off)), ID, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  // meanwhile: sum_r dS[r,j] S0[r,j] from the [r][j] tiles (threads 128..255, j = tid - 128)
  if (tid >= 128) {
    const int j = tid - 128;
    float acc = 0.f;
#pragma unroll 8
    for (int r = 0; r < D; ++r) {
      const uint32_t o = tc::sw128_off(r, j, 128, 2);
      acc = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + StCfg::S0R + o)),
                 __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + StCfg::DSR + o)), acc);
    }
    csum[j] = acc;
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  __syncthreads();  // every operand read is done: the operand area is free
  float* Ls = reinterpret_cast<float*>(sm + StCfg::LS);
  float* EX1 = reinterpret_cast<float*>(sm + StCfg::EX1);
  float* EX2 = reinterpret_cast<float*>(sm + StCfg::EX2);
  if (tid < 128) {
#pragma unroll
    for (int t = 0; t < C; ++t) Ls[t * 129 + tid] = Lr[t];
  }
  __syncthreads();

  const int quad = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
  const int row = quad * 32 + lane;              // D row (TMEM lane)
  const int c0 = half * 64;                      // first column of this thread
  const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
  if (row < 64) {
    const int t = row;
    const float dbt = db0[t];
    const __nv_bfloat16* qrow = q + (((size_t)b * T + t0 + t) * H + h) * D;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float dq[16], kps[16];
      tc::tmem_ld16(lanes + 0 + c0 + 16 * c16, dq);
      tc::tmem_ld16(lanes + 256 + c0 + 16 * c16, kps);
      tc::tmem_ld_wait();
      __align__(16) __nv_bfloat16 qv[16];
      if (t < nv) {
        *reinterpret_cast<uint4*>(qv) = *reinterpret_cast<const uint4*>(qrow + c0 + 16 * c16);
        *reinterpret_cast<uint4*>(qv + 8) = *reinterpret_cast<const uint4*>(qrow + c0 + 16 * c16 + 8);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) qv[i] = __float2bfloat16_rn(0.f);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = c0 + 16 * c16 + i;
        const float gm = expf(Ls[t * 129 + j]);
        waccq[(ch * C + t) * D + j] = dq[i] * gm;
        EX1[t * 129 + j] = dq[i] * __bfloat162float(qv[i]) * gm;
        EX2[t * 129 + j] = dbt * kps[i];   // column j here is the value channel r
      }
    }
  }
  __syncthreads();
  if (row >= 64) {
    const int t = row - 64;
    const float dbt = db0[t], ut = us[t];
    const __nv_bfloat16* krow = k + (((size_t)b * T + t0 + t) * H + h) * D;
    float ekv[64];
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float vs[16], vd[16], ked[16];
      tc::tmem_ld16(lanes + 0 + c0 + 16 * c16, vs);
      tc::tmem_ld16(lanes + 128 + c0 + 16 * c16, vd);
      tc::tmem_ld16(lanes + 384 + c0 + 16 * c16, ked);
      tc::tmem_ld_wait();
      __align__(16) __nv_bfloat16 kv[16];
      if (t < nv) {
        *reinterpret_cast<uint4*>(kv) = *reinterpret_cast<const uint4*>(krow + c0 + 16 * c16);
        *reinterpret_cast<uint4*>(kv + 8) = *reinterpret_cast<const uint4*>(krow + c0 + 16 * c16 + 8);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) kv[i] = __float2bfloat16_rn(0.f);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = c0 + 16 * c16 + i;
        const float L = Ls[t * 129 + j];
        const float gm = expf(L), eC = expf(lC[j] - L);
        const float kk = __bfloat162float(kv[i]);
        const float dKp = dbt * vs[i], dKe = ut * vd[i];
        const size_t o = (ch * C + t) * D + j;
        wacck[o] = dKp * gm + dKe * eC;
        const float dl = EX1[t * 129 + j] + dKp * kk * gm - dKe * kk * eC;
        ekv[16 * c16 + i] = dKe * kk * eC;
        if (t == C - 1) EX1[t * 129 + j] = dl;  // finished below with the chunk-end terms
        else waccL[o] = dl;
        waccv[o] = EX2[t * 129 + j] + ut * ked[i];
      }
    }
    // column sums of dKe o K^e over this warp's 32 positions
    float lo[32], hi[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      lo[i] = ekv[i];
      hi[i] = ekv[32 + i];
    }
    warp_transpose_reduce<32>(lo, lane);
    warp_transpose_reduce<32>(hi, lane);
    // warps 2,3 (half 0) and 6,7 (half 1): slot = (quad - 2) + 2 * half
    const int slot = (quad - 2) + 2 * half;
    ekp[slot * 64 + lane] = lo[0];
    ekp[slot * 64 + 32 + lane] = hi[0];
  }
  __syncthreads();
  if (tid < 128) {
    const int j = tid, hf = j >> 6, jj = j & 63;
    const float ek = ekp[(2 * hf) * 64 + jj] + ekp[(2 * hf + 1) * 64 + jj];
    waccL[(ch * C + (C - 1)) * D + j] = EX1[(C - 1) * 129 + j] + ek + expf(lC[j]) * csum[j];
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Intra-chunk gradient products, one CTA per chunk, all chunks in parallel.
// With the gates factored out, the six C x C by C x d products are three
// bf16 MMAs (M=128, N=128) whose right operands are MN-major views of tiles
// the kernel already holds:
//   R1 = [dP; dG_K] K-            -> rows 0-63: dP K-,  rows 64-127: dG_K K-
//   R2 = [dP^T | dG_K^T] [Q+; K+] -> rows 0-63: dP^T Q+ + dG_K^T K+
//   R3 = [u P^T | dG_V'] [dO; V]  -> rows 0-63: u o (P^T dO) + dG_V' V
// (dG_V' = dG_V + dG_V^T).  Then, with gamma = e^L:
//   dq = accq + gamma o R1top
//   dk = acck + gamma o R1bot + R2 / gamma
//   dv = accv + R3
//   dL = accL + q o gamma o R1top + k o gamma o R1bot - k o R2 / gamma
//   dlogf_t = sum_{s >= t} dL_s
// Chunks whose decay range leaves the factorised form's range are flagged
// and recomputed by the exact CUDA-core kernel.
// ---------------------------------------------------------------------------
struct InCfg {
  static constexpr uint32_t A1 = 0;         // [dP; dG_K], 128 rows x K=64
  static constexpr uint32_t A2 = 16384;     // [dP^T | dG_K^T ; 0], 128 rows x K=128
  static constexpr uint32_t A3 = 49152;     // [u P^T | dG_V' ; 0], 128 rows x K=128
  static constexpr uint32_t B1 = 81920;     // K- [i][j], MN-major (K = 64 rows), 2 N blocks
  static constexpr uint32_t B2 = 98304;     // [Q+; K+], MN-major (K = 128 rows)
  static constexpr uint32_t B3 = 131072;    // [dO; V], MN-major (K = 128 rows), by TMA
  static constexpr uint32_t LS = 163840;    // L fp32 [64][129]
  static constexpr uint32_t SMALL = LS + 64 * 129 * 4;  // u [64]
  static constexpr uint32_t BYTES = SMALL + 256 + 1024;
  // epilogue reuse of the A tiles: EX (gamma o dG_K K-) and dL, fp32 [64][129]
  static constexpr uint32_t EX = 0, DL = 40960;
};

__global__ void __launch_bounds__(256, 1) bwd_intra_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const float* __restrict__ logf,
    int H, int T, int NC, const float* __restrict__ wP, const float* __restrict__ wu,
    const float* __restrict__ wdP, const float* __restrict__ wdGK, const float* __restrict__ wdGVs,
    const float* __restrict__ waccq, const float* __restrict__ wacck, const float* __restrict__ waccL,
    const float* __restrict__ waccv, __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
    __nv_bfloat16* __restrict__ dv, float* __restrict__ dlogf, int* __restrict__ flags, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, unsafe;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  float* Ls = reinterpret_cast<float*>(sm + InCfg::LS);
  float* us = reinterpret_cast<float*>(sm + InCfg::SMALL);

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    unsafe = 0;
    tc::mbar_expect_tx(&ld_bar, 32768u);
    tc::tma_load_4d(sm + InCfg::B3, &tm_do, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + InCfg::B3 + 16384, &tm_do, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + InCfg::B3 + 8192, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + InCfg::B3 + 16384 + 8192, &tm_v, 64, h, t0, b, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 512);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;

  if (tid < 128) {
    // decay prefix of channel j; Q+, K+ (B2) and K- (B1)
    const int j = tid;
    float L = 0.f, mx = 0.f;
#pragma unroll 4
    for (int t = 0; t < C; ++t) {
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + j;
      const bool ok = t < nv;
      L += ok ? logf[g] : 0.f;
      mx = fmaxf(mx, fabsf(L));
      Ls[t * 129 + j] = L;
      const float qq = ok ? __bfloat162float(q[g]) : 0.f, kk = ok ? __bfloat162float(k[g]) : 0.f;
      const float gm = expf(L), ig = expf(-L);
      *reinterpret_cast<__nv_bfloat16*>(sm + InCfg::B2 + tc::sw128_off(t, j, 128, 2)) = __float2bfloat16_rn(qq * gm);
      *reinterpret_cast<__nv_bfloat16*>(sm + InCfg::B2 + tc::sw128_off(64 + t, j, 128, 2)) = __float2bfloat16_rn(kk * gm);
      *reinterpret_cast<__nv_bfloat16*>(sm + InCfg::B1 + tc::sw128_off(t, j, 64, 2)) = __float2bfloat16_rn(kk * ig);
    }
    if (!(mx < kSafeLogRange)) atomicOr(&unsafe, 1);
  } else {
    // C x C operand tiles (bf16) from the adjoint kernel's fp32 matrices
    const int p = tid - 128;
    const float* dPc = wdP + ch * C * C;
    const float* dGc = wdGK + ch * C * C;
    const float* dVc = wdGVs + ch * C * C;
    if (p < C) us[p] = wu[ch * C + p];
    for (int e = p; e < C * C; e += 128) {
      const int r = e / C, c = e % C;  // element [r][c] of the row-major sources
      const float dpv = dPc[e], dgv = dGc[e];
      auto st2 = [&](uint32_t base, int row, int kk, float x) {
        *reinterpret_cast<__nv_bfloat16*>(sm + base + tc::sw128_off(row, kk, 128, 2)) = __float2bfloat16_rn(x);
      };
      st2(InCfg::A1, r, c, dpv);            // dP[t][i]
      st2(InCfg::A1, 64 + r, c, dgv);       // dG_K[t][i]
      st2(InCfg::A2, c, r, dpv);            // dP^T[t][s] = dP[s][t]
      st2(InCfg::A2, c, 64 + r, dgv);       // dG_K^T
      st2(InCfg::A3, r, 64 + c, dVc[e]);    // dG_V'[i][t]
    }
  }
  __syncthreads();
  if (tid >= 128) {
    const int p = tid - 128;
    const float* Pc = wP + ch * C * C;
    for (int e = p; e < C * C; e += 128) {
      const int t = e / C, i = e % C;
      *reinterpret_cast<__nv_bfloat16*>(sm + InCfg::A3 + tc::sw128_off(i, t, 128, 2)) =
          __float2bfloat16_rn(us[i] * Pc[e]);   // u_i P[t][i]
    }
  } else {
    // zero rows 64..127 of A2 and A3 (both K blocks)
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int e = tid; e < 2 * 2 * 512; e += 128) {
      const int tile = e / 1024, rem = e % 1024, kb = rem / 512, w = rem % 512;
      reinterpret_cast<uint4*>(sm + (tile ? InCfg::A3 : InCfg::A2) + kb * 16384 + 8192)[w] = z;
    }
  }
  tc::fence_proxy_async();
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    const uint32_t ID = tc::idesc(128, 128, 1) | (1u << 16);  // bf16, B MN-major
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      tc::mma_bf16_ss(tmem + 0, tc::desc_sw128(tc::smem_u32(sm + InCfg::A1 + ks * 32)),
                      tc::desc_sw128_mn(tc::smem_u32(sm + InCfg::B1 + ks * 2048), 8192u), ID, ks > 0 ? 1u : 0u);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t ao = (ks / 4) * 16384 + (ks % 4) * 32;
      tc::mma_bf16_ss(tmem + 128, tc::desc_sw128(tc::smem_u32(sm + InCfg::A2 + ao)),
                      tc::desc_sw128_mn(tc::smem_u32(sm + InCfg::B2 + ks * 2048), 16384u), ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + 256, tc::desc_sw128(tc::smem_u32(sm + InCfg::A3 + ao)),
                      tc::desc_sw128_mn(tc::smem_u32(sm + InCfg::B3 + ks * 2048), 16384u), ID, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  __syncthreads();  // operand tiles A1..A3 are free from here
  const bool is_unsafe = unsafe != 0;
  if (tid == 0) flags[ch] = is_unsafe ? 1 : 0;
  if (!is_unsafe) {
    float* EX = reinterpret_cast<float*>(sm + InCfg::EX);
    float* DLs = reinterpret_cast<float*>(sm + InCfg::DL);
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane, c0 = half * 64;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
    if (row >= 64) {  // gamma o (dG_K K-)
      const int t = row - 64;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float x[16];
        tc::tmem_ld16(lanes + 0 + c0 + 16 * c16, x);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = c0 + 16 * c16 + i;
          EX[t * 129 + j] = x[i] * expf(Ls[t * 129 + j]);
        }
      }
    }
    __syncthreads();
    if (row < 64) {
      const int t = row;
      const size_t tok = (((size_t)b * T + t0 + t) * H + h) * D;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float r1[16], r2[16], r3[16];
        tc::tmem_ld16(lanes + 0 + c0 + 16 * c16, r1);
        tc::tmem_ld16(lanes + 128 + c0 + 16 * c16, r2);
        tc::tmem_ld16(lanes + 256 + c0 + 16 * c16, r3);
        tc::tmem_ld_wait();
        const int jb = c0 + 16 * c16;
        __align__(16) __nv_bfloat16 qv[16], kv[16];
        if (t < nv) {
          *reinterpret_cast<uint4*>(qv) = *reinterpret_cast<const uint4*>(q + tok + jb);
          *reinterpret_cast<uint4*>(qv + 8) = *reinterpret_cast<const uint4*>(q + tok + jb + 8);
          *reinterpret_cast<uint4*>(kv) = *reinterpret_cast<const uint4*>(k + tok + jb);
          *reinterpret_cast<uint4*>(kv + 8) = *reinterpret_cast<const uint4*>(k + tok + jb + 8);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) qv[i] = kv[i] = __float2bfloat16_rn(0.f);
        }
        const size_t ao = (ch * C + t) * D + jb;
        float aq[16], ak[16], aL[16], av[16];
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          *reinterpret_cast<float4*>(aq + 4 * i4) = *reinterpret_cast<const float4*>(waccq + ao + 4 * i4);
          *reinterpret_cast<float4*>(ak + 4 * i4) = *reinterpret_cast<const float4*>(wacck + ao + 4 * i4);
          *reinterpret_cast<float4*>(aL + 4 * i4) = *reinterpret_cast<const float4*>(waccL + ao + 4 * i4);
          *reinterpret_cast<float4*>(av + 4 * i4) = *reinterpret_cast<const float4*>(waccv + ao + 4 * i4);
        }
        __align__(16) __nv_bfloat16 oq[16], ok[16], ov[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = jb + i;
          const float L = Ls[t * 129 + j];
          const float gm = expf(L), ig = expf(-L);
          const float qq = __bfloat162float(qv[i]), kk = __bfloat162float(kv[i]);
          const float qP = gm * r1[i], kG1 = EX[t * 129 + j], kP2 = r2[i] * ig;
          oq[i] = __float2bfloat16_rn(aq[i] + qP);
          ok[i] = __float2bfloat16_rn(ak[i] + kG1 + kP2);
          ov[i] = __float2bfloat16_rn(av[i] + r3[i]);
          DLs[t * 129 + j] = aL[i] + qq * qP + kk * kG1 - kk * kP2;
        }
        if (t < nv) {
          *reinterpret_cast<uint4*>(dq + tok + jb) = *reinterpret_cast<const uint4*>(oq);
          *reinterpret_cast<uint4*>(dq + tok + jb + 8) = *reinterpret_cast<const uint4*>(oq + 8);
          *reinterpret_cast<uint4*>(dk + tok + jb) = *reinterpret_cast<const uint4*>(ok);
          *reinterpret_cast<uint4*>(dk + tok + jb + 8) = *reinterpret_cast<const uint4*>(ok + 8);
          *reinterpret_cast<uint4*>(dv + tok + jb) = *reinterpret_cast<const uint4*>(ov);
          *reinterpret_cast<uint4*>(dv + tok + jb + 8) = *reinterpret_cast<const uint4*>(ov + 8);
        }
      }
    }
    __syncthreads();
    if (tid < 128) {
      const int j = tid;
      float acc = 0.f;
      for (int t = C - 1; t >= 0; --t) {
        acc += DLs[t * 129 + j];
        if (t < nv) dlogf[(((size_t)b * T + t0 + t) * H + h) * D + j] = acc;
      }
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// C x C adjoints of the backward, one CTA per chunk, all chunks in parallel:
//   K+ K-^T (tf32) -> decayed key Gram G_K;  [V; dO] V^T (bf16) -> G_V, dO V^T
//   dP = (dO V^T) o u (i <= t);  dM = -(beta o g) u^T (i < t)
//   dG_K = dM o G_V;  dG_V' = dM o G_K + (dM o G_K)^T
//   dbeta = -g o (b0 + M u),  dc = g
// Chunks outside the factorised decay range take exact per-element Grams.
// ---------------------------------------------------------------------------
struct CcCfg {
  static constexpr uint32_t AK = 0;         // [K+; unused] tf32, 4 K blocks x 128 rows x 128 B
  static constexpr uint32_t BKM = 65536;    // K- tf32, 4 K blocks x 64 rows x 128 B
  static constexpr uint32_t AVD = 98304;    // [V; dO] bf16, 2 K blocks x 128 rows x 128 B
  static constexpr uint32_t LS = 131072;    // L fp32 [64][129]
  static constexpr uint32_t GV = LS + 64 * 129 * 4;   // dG_V fp32 [64][65]
  static constexpr uint32_t SMALL = GV + 64 * 65 * 4; // u, g, beta, b0 [64] each
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
};

__global__ void __launch_bounds__(256, 1) bwd_cc_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __nv_bfloat16* __restrict__ k, const float* __restrict__ beta, const float* __restrict__ logf, int H,
    int T, int NC, const float* __restrict__ wu, const float* __restrict__ wb0, const float* __restrict__ wg,
    float* __restrict__ dbeta, float* __restrict__ dc, float* __restrict__ wdP, float* __restrict__ wdGK,
    float* __restrict__ wdGVs, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, unsafe;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  float* Ls = reinterpret_cast<float*>(sm + CcCfg::LS);
  float* GVs = reinterpret_cast<float*>(sm + CcCfg::GV);
  float* us = reinterpret_cast<float*>(sm + CcCfg::SMALL);
  float* gs = us + 64;
  float* bs = gs + 64;
  float* b0s = bs + 64;

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    unsafe = 0;
    tc::mbar_expect_tx(&ld_bar, 32768u);
    tc::tma_load_4d(sm + CcCfg::AVD, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CcCfg::AVD + 16384, &tm_v, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CcCfg::AVD + 8192, &tm_do, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CcCfg::AVD + 16384 + 8192, &tm_do, 64, h, t0, b, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 128);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  if (tid < 128) {
    const int j = tid;
    float L = 0.f, mx = 0.f;
#pragma unroll 4
    for (int t = 0; t < C; ++t) {
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + j;
      const bool ok = t < nv;
      L += ok ? logf[g] : 0.f;
      mx = fmaxf(mx, fabsf(L));
      Ls[t * 129 + j] = L;
      const float kk = ok ? __bfloat162float(k[g]) : 0.f;
      *reinterpret_cast<float*>(sm + CcCfg::AK + tc::sw128_off(t, j, 128, 4)) = kk * expf(L);
      *reinterpret_cast<float*>(sm + CcCfg::BKM + tc::sw128_off(t, j, 64, 4)) = kk * expf(-L);
    }
    if (!(mx < kSafeLogRange)) atomicOr(&unsafe, 1);
  } else {
    const int i = tid - 128;
    if (i < C) {
      us[i] = wu[ch * C + i];
      gs[i] = wg[ch * C + i];
      b0s[i] = wb0[ch * C + i];
      bs[i] = i < nv ? beta[((size_t)b * T + t0 + i) * H + h] : 0.f;
    }
  }
  tc::fence_proxy_async();
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    const uint32_t IDT = tc::idesc(128, 64, 2), IDB = tc::idesc(128, 64, 1);
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      const uint32_t kb = ks / 4, w = (ks % 4) * 32;
      tc::mma_tf32_ss(tmem + 0, tc::desc_sw128(tc::smem_u32(sm + CcCfg::AK + kb * 16384 + w)),
                      tc::desc_sw128(tc::smem_u32(sm + CcCfg::BKM + kb * 8192 + w)), IDT, ks > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
      const uint64_t vd = tc::desc_sw128(tc::smem_u32(sm + CcCfg::AVD + o));
      tc::mma_bf16_ss(tmem + 64, vd, vd, IDB, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  const bool is_unsafe = unsafe != 0;
  if (warp < 4) {
    const int row = warp * 32 + lane;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
    if (row < 64) {
      const int t = row;
      const float bg = -bs[t] * gs[t];
      float* dgk = wdGK + ch * C * C + t * C;
      float brow = 0.f;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float gk[16], gv[16];
        tc::tmem_ld16(lanes + 16 * c16, gk);
        tc::tmem_ld16(lanes + 64 + 16 * c16, gv);
        tc::tmem_ld_wait();
        if (is_unsafe) {  // exact decay weights for this row
#pragma unroll 1
          for (int ii = 0; ii < 16; ++ii) {
            const int i = 16 * c16 + ii;
            float x = 0.f;
            if (i < t) {
              const size_t gt = (((size_t)b * T + t0 + t) * H + h) * D, gi = (((size_t)b * T + t0 + i) * H + h) * D;
              for (int j = 0; j < D; ++j)
                x = fmaf(__bfloat162float(k[gt + j]) * __bfloat162float(k[gi + j]),
                         expf(Ls[t * 129 + j] - Ls[i * 129 + j]), x);
            }
            gk[ii] = x;
          }
        }
        float o[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int i = 16 * c16 + ii;
          const bool low = i < t;
          const float mm = low ? gk[ii] * gv[ii] : 0.f;
          brow = fmaf(mm, us[i], brow);
          const float dM = low ? bg * us[i] : 0.f;
          o[ii] = dM * gv[ii];
          GVs[t * 65 + i] = dM * gk[ii];
        }
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4)
          *reinterpret_cast<float4*>(dgk + 16 * c16 + 4 * i4) = make_float4(o[4 * i4], o[4 * i4 + 1], o[4 * i4 + 2], o[4 * i4 + 3]);
      }
      if (t < nv) {
        const size_t g = ((size_t)b * T + t0 + t) * H + h;
        dc[g] = gs[t];
        dbeta[g] = -gs[t] * (b0s[t] + brow);
      }
    } else {
      const int t = row - 64;
      float* dp = wdP + ch * C * C + t * C;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float dov[16];
        tc::tmem_ld16(lanes + 64 + 16 * c16, dov);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          float4 v4;
          const int i = 16 * c16 + 4 * i4;
          v4.x = i <= t ? us[i] * dov[4 * i4] : 0.f;
          v4.y = i + 1 <= t ? us[i + 1] * dov[4 * i4 + 1] : 0.f;
          v4.z = i + 2 <= t ? us[i + 2] * dov[4 * i4 + 2] : 0.f;
          v4.w = i + 3 <= t ? us[i + 3] * dov[4 * i4 + 3] : 0.f;
          *reinterpret_cast<float4*>(dp + i) = v4;
        }
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    wdGVs[ch * C * C + e] = GVs[t * 65 + i] + GVs[i * 65 + t];
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
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
                         ws_ptr<__nv_bfloat16>(a.ws, L.dSCb), ws_ptr<__nv_bfloat16>(a.ws, L.dSCbt),
                         ws_ptr<float>(a.ws, L.g), err);
  prof_end(st);
  return e;
}

}  // namespace

cudaError_t launch_bwd_tc(const BwdArgs& a, int* err, int sms, cudaStream_t st) {
  const Layout& L = a.L;
  constexpr int kDuSmem = (2 * C * (D + 1) + C * (C + 1)) * 4;
  cudaError_t e = cudaFuncSetAttribute(bwd_du_intra, cudaFuncAttributeMaxDynamicSharedMemorySize, kDuSmem);
  if (e != cudaSuccess) return e;
  prof_begin(st, "bwd_du_intra");
  bwd_du_intra<<<(unsigned)L.chunks, 256, kDuSmem, st>>>(
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.dO), L.H, L.T, L.NC,
      ws_ptr<float>(a.fws, L.P), ws_ptr<float>(a.ws, L.du));
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int R = choose_cluster(L.B * L.H, sms);
  e = (R == 8) ? launch_bchain<8>(a, err, st) : launch_bchain<4>(a, err, st);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_v, tm_do;
  if (!make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_do, a.dO, 2, L.B, L.T, L.H, D, 64, true))
    return cudaErrorInvalidValue;
  if ((e = cudaFuncSetAttribute(bwd_state_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)StCfg::BYTES)) != cudaSuccess)
    return e;
  prof_begin(st, "bwd_state_tc");
  bwd_state_tc<<<(unsigned)L.chunks, 256, StCfg::BYTES, st>>>(
      tm_v, tm_do, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k), a.beta,
      a.logf, L.H, L.T, L.NC, ws_ptr<float>(a.fws, L.u), ws_ptr<float>(a.ws, L.g),
      ws_ptr<__nv_bfloat16>(a.fws, L.S0b), ws_ptr<__nv_bfloat16>(a.fws, L.S0bt),
      ws_ptr<__nv_bfloat16>(a.ws, L.dSCb), ws_ptr<__nv_bfloat16>(a.ws, L.dSCbt), ws_ptr<float>(a.ws, L.accq),
      ws_ptr<float>(a.ws, L.acck), ws_ptr<float>(a.ws, L.accL), ws_ptr<float>(a.ws, L.accv), err);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // C x C adjoints, then the intra-chunk products
  if ((e = cudaFuncSetAttribute(bwd_cc_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CcCfg::BYTES)) !=
      cudaSuccess)
    return e;
  prof_begin(st, "bwd_cc_tc");
  bwd_cc_tc<<<(unsigned)L.chunks, 256, CcCfg::BYTES, st>>>(
      tm_v, tm_do, static_cast<const __nv_bfloat16*>(a.k), a.beta, a.logf, L.H, L.T, L.NC,
      ws_ptr<float>(a.fws, L.u), ws_ptr<float>(a.fws, L.b0), ws_ptr<float>(a.ws, L.g), a.dbeta, a.dc,
      ws_ptr<float>(a.ws, L.dP), ws_ptr<float>(a.ws, L.dGK), ws_ptr<float>(a.ws, L.dGVs), err);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int* flags = ws_ptr<int>(a.ws, L.bflags);
  if ((e = cudaFuncSetAttribute(bwd_intra_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)InCfg::BYTES)) != cudaSuccess)
    return e;
  prof_begin(st, "bwd_intra_tc");
  bwd_intra_tc<<<(unsigned)L.chunks, 256, InCfg::BYTES, st>>>(
      tm_v, tm_do, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k), a.logf, L.H,
      L.T, L.NC, ws_ptr<float>(a.fws, L.P), ws_ptr<float>(a.fws, L.u), ws_ptr<float>(a.ws, L.dP),
      ws_ptr<float>(a.ws, L.dGK), ws_ptr<float>(a.ws, L.dGVs), ws_ptr<float>(a.ws, L.accq),
      ws_ptr<float>(a.ws, L.acck), ws_ptr<float>(a.ws, L.accL), ws_ptr<float>(a.ws, L.accv),
      static_cast<__nv_bfloat16*>(a.dq), static_cast<__nv_bfloat16*>(a.dk), static_cast<__nv_bfloat16*>(a.dv),
      a.dlogf, flags, err);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // chunks outside the factorised decay range: exact CUDA-core recomputation
  return launch_bwd_simt_stages(a, kStageIntra, flags, st);
}

}  // namespace kd
