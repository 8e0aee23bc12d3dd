// kd_bchain_tc.cu -- the backward's reverse chunk chain on tensor cores
// (bf16 q, k, v, dO and d_k = d_v = 128).
//
// Reverse mode of the chunk recurrence (derived here; the pages only ask for a
// gate-aware backward: Gated DeltaNet-2 article, "핵심 기여").  Chunks are
// processed last to first; step k handles chunk n = NC-1-k.  Z_k is the
// gradient of the state at the end of that chunk (Z_0 = dS_T), and
//   du_k = du_intra + rowdot(V_n, Z_k K^e_n^T)
//   g_k  = A_n^T du_k,   db0_k = -beta_n o g_k
//   Z_{k+1} = W_k + V_n^T diag(db0_k) K+_n,   W_k = Z_k diag(gamma_C,n) + dO_n^T Q+_n.
// W_k does not depend on db0_k, and the forward's cross-chunk matrix
// H_{n+1} = (V_{n+1} V_n^T) o (K+_{n+1} K^e_n^T) carries the rest, so the erase
// read of step k needs only the state one step earlier:
//   rowdot(V_n, Z_k K^e_n^T) = rowdot(V_n, W_{k-1} K^e_n^T) + H_{n+1}^T db0_{k-1}.
// The same two loops as the forward chain (kd_fchain_tc.cu) follow:
//   short: db0_{k-1} -> db0_k, two 64 x 64 matrix-vector products;
//   long:  db0_k -> update MMA -> Z_{k+1}, W_{k+1} -> lookahead MMA and column
//          dot -> cluster all-reduce -> du_{k+2}, spanning two steps;
// each on its own warps.
//
// One cluster of R CTAs per (b, h); CTA c owns the key-channel slice J_c of
// the state (W in tensor memory as the A operand of the lookahead MMA).
// Warp roles (320 threads):
//   warps 0-3  vector warps: du, g, db0 (every CTA computes the same values
//              from the all-reduced column dots), the update operand
//              diag(db0) K+ in bf16 hi + lo, g written out for the per-chunk
//              gradient kernel.
//   warps 4-7  state warps (thread r = tensor-memory lane r): Z and W, the
//              save of Z as each chunk's end-state gradient (bf16 tile), dS0,
//              the column dot and the send of its partial sums.
//   warp 8     issuer: every tcgen05 MMA (lookahead, dO^T Q+, update).
//   warp 9     producer: the early ring (dO, Q+^T, K^e; two slots), the late
//              ring (V^T, K+, gamma; three slots) and the vector ring (A,
//              H_{n+1}, du_intra, beta; two slots).
// All waits are bounded as in the forward chain.
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;
// Steps ahead of the shared-memory rings whose operands the producer pulls
// into L2, so that the ring's own copies are L2 hits.
constexpr int kL2Ahead = 3;

template <int R>
struct BcCfg {
  static constexpr int NJ = D / R;
  static constexpr int KBJ = (R == 8) ? 2 : 0;
  // tensor memory: X' (64), W (NJ), dO^T Q+ (NJ), the update accumulators [2] (NJ each)
  static constexpr int X_COL = 0, W_COL = 64, M3_COL = 64 + NJ, D2_COL = 64 + 2 * NJ;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t up1k(uint32_t x) { return (x + 1023u) / 1024u * 1024u; }
  // early ring (2 slots): dO [t][r] bf16 (two 64-channel swizzled halves, 16 KB),
  // the 32-channel K^e block (tf32, 8 KB), Q+^T slice [NJ][64] bf16 (K-major)
  static constexpr uint32_t E_DO = 0, E_KE = 16384, E_QP = 24576;
  static constexpr uint32_t E_SZ = up1k(E_QP + NJ * 128);
  static constexpr uint32_t E_BYTES = 16384 + 8192 + NJ * 128;
  // late ring (3 slots): V^T [r][t] bf16 (16 KB), K+ slice fp32 [64][NJ], gamma_C slice
  static constexpr uint32_t L_V = 0, L_KP = 16384, L_GC = 16384 + 64 * NJ * 4;
  static constexpr uint32_t L_SZ = up1k(L_GC + NJ * 4);
  static constexpr uint32_t L_BYTES = 16384 + 64 * NJ * 4 + NJ * 4;
  // vector ring (2 slots): A [64][64], H_{n+1} [64][64], du_intra [64], beta [64]
  static constexpr uint32_t EARLY = 0, LATE = 2 * E_SZ, AUX = LATE + 3 * L_SZ;
  static constexpr uint32_t AX_A = 0, AX_H = 16384, AX_DU = 32768, AX_B = 32768 + 256;
  static constexpr uint32_t AUX_SZ = up1k(AX_B + 256);
  static constexpr uint32_t B2 = AUX + 2 * AUX_SZ;  // diag(db0) K+ [2][hi, lo][NJ rows x 128 B]
  static constexpr uint32_t B2_SZ = 2 * NJ * 128;
  static constexpr uint32_t SM = B2 + 2 * B2_SZ;
  static constexpr uint32_t SM_RECV = SM;                        // [4][R][64]
  static constexpr uint32_t SM_XRED = SM_RECV + 4 * R * 64 * 4;  // [4][64]
  static constexpr uint32_t SM_MINE = SM_XRED + 4 * 64 * 4;      // [64]
  static constexpr uint32_t SM_DB = SM_MINE + 64 * 4;            // db0 [2][64]
  static constexpr uint32_t SM_DU = SM_DB + 2 * 64 * 4;          // du [64]
  static constexpr uint32_t SM_HP = SM_DU + 64 * 4;              // H^T db0 halves [2][64]
  static constexpr uint32_t SM_GP = SM_HP + 2 * 64 * 4;          // A^T du halves [2][64]
  static constexpr uint32_t SM_END = SM_GP + 2 * 64 * 4;
  static constexpr uint32_t BYTES = SM_END + 1024;
};

__device__ __forceinline__ void bar_u() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_s() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  int dummy_abort = 0;
  tc::mbar_wait<false>(b, parity, nullptr, 0, &dummy_abort);
}
// 16 values of row r (columns j..j+15) into a bf16 [r][j] 128-byte-swizzled K-major tile
__device__ __forceinline__ void save_bf16_tile(__nv_bfloat16* rj, size_t ch, int r, int j, const float (&x)[16]) {
  unsigned char* a = reinterpret_cast<unsigned char*>(rj + ch * D * D);
#pragma unroll
  for (int h8 = 0; h8 < 2; ++h8) {
    __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v8[i] = __float2bfloat16_rn(x[8 * h8 + i]);
    *reinterpret_cast<uint4*>(a + tc::sw128_off(r, j + 8 * h8, 128, 2)) = *reinterpret_cast<const uint4*>(v8);
  }
}

template <int R>
__global__ void __launch_bounds__(320, 1) bwd_chain_tc(
    const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_ke,
    const __grid_constant__ CUtensorMap tm_kp, const float* __restrict__ beta, const float* __restrict__ dST,
    float* __restrict__ dS0, int H, int T, int NC, const float* __restrict__ wA, const float* __restrict__ wHx,
    const float* __restrict__ wGC, const __nv_bfloat16* __restrict__ wVt, const __nv_bfloat16* __restrict__ wQpT,
    const float* __restrict__ wdu, __nv_bfloat16* __restrict__ wdSCb, float* __restrict__ wg,
    int* __restrict__ err) {
  using Cf = BcCfg<R>;
  constexpr int NJ = Cf::NJ;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t e_full[2], e_free[2], l_full[3], l_free[3], aux_full[2], aux_free[2], x_bar[4], b2_full[2],
      mma1_bar, mma2_bar[2], s_ready, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_rank();
  const int unit = blockIdx.x / R;
  const int b = unit / H, h = unit % H;
  const int j0 = static_cast<int>(rank) * NJ;
  const int jb = j0 & ~31;

  float* recv = reinterpret_cast<float*>(sm + Cf::SM_RECV);
  float* xred = reinterpret_cast<float*>(sm + Cf::SM_XRED);
  float* mine = reinterpret_cast<float*>(sm + Cf::SM_MINE);
  float* db0s = reinterpret_cast<float*>(sm + Cf::SM_DB);
  float* dus = reinterpret_cast<float*>(sm + Cf::SM_DU);
  float* hp = reinterpret_cast<float*>(sm + Cf::SM_HP);
  float* gp = reinterpret_cast<float*>(sm + Cf::SM_GP);
  auto early = [&](int k) { return sm + Cf::EARLY + (k & 1) * Cf::E_SZ; };
  auto late = [&](int k) { return sm + Cf::LATE + (k % 3) * Cf::L_SZ; };
  auto auxp = [&](int k) { return sm + Cf::AUX + (k & 1) * Cf::AUX_SZ; };
  auto chunk_of = [&](int k) { return NC - 1 - k; };

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&e_full[i], 1);
      tc::mbar_init(&e_free[i], 1);
      tc::mbar_init(&aux_full[i], 2);
      tc::mbar_init(&aux_free[i], 1);
      tc::mbar_init(&b2_full[i], 128);
      tc::mbar_init(&mma2_bar[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      tc::mbar_init(&l_full[i], 1);
      tc::mbar_init(&l_free[i], 1);
    }
    for (int i = 0; i < 4; ++i) tc::mbar_init(&x_bar[i], 1);
    tc::mbar_init(&mma1_bar, 1);
    tc::mbar_init(&s_ready, 1);
    tc::mbar_init(&drain_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, Cf::TMEM_COLS);
  tc::tc_before_sync();
  __syncthreads();
  if (tid == 0)
    for (int i = 0; i < 4 && i < NC; ++i) tc::mbar_expect_tx(&x_bar[i], R * 64u * 4u);
  __syncthreads();
  tc::cluster_sync();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp < 4) {
    // ============================== vector warps ==============================
    // column i of A and H (column reads are conflict-free: a warp reads 32
    // consecutive columns of one row); the two row halves meet in shared memory
    const int i = tid & 63, half = tid >> 6;
    for (int k = 0; k < NC; ++k) {
      const int n = chunk_of(k);
      const size_t ch = (size_t)unit * NC + n;
      const int xs = k & 3;
      tc::mbar_wait<true>(&x_bar[xs], (uint32_t)((k >> 2) & 1), err, tc::kErrTimeoutCluster, &abort_flag);
      tc::mbar_wait<false>(&aux_full[k & 1], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      const unsigned char* ax = auxp(k);
      if (k > 0) {
        // H_{n+1}^T db0_{k-1}
        const float* Hc = reinterpret_cast<const float*>(ax + Cf::AX_H) + 32 * half * 64 + i;
        const float* dp = db0s + ((k - 1) & 1) * 64 + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          a0 = fmaf(Hc[t * 64], dp[t], a0);
          a1 = fmaf(Hc[(t + 1) * 64], dp[t + 1], a1);
          a2 = fmaf(Hc[(t + 2) * 64], dp[t + 2], a2);
          a3 = fmaf(Hc[(t + 3) * 64], dp[t + 3], a3);
        }
        hp[half * 64 + i] = (a0 + a1) + (a2 + a3);
      }
      bar_u();
      if (tid < C) {
        float s = reinterpret_cast<const float*>(ax + Cf::AX_DU)[i];
        const float* rv = recv + xs * R * 64;
#pragma unroll
        for (int c2 = 0; c2 < R; ++c2) s += rv[c2 * 64 + i];
        if (k > 0) s += hp[i] + hp[64 + i];
        dus[i] = s;
      }
      bar_u();  // every thread has read recv[xs]: arm it for step k + 4
      if (tid == 0 && k + 4 < NC) tc::mbar_expect_tx(&x_bar[xs], R * 64u * 4u);
      {
        // A^T du
        const float* Ac = reinterpret_cast<const float*>(ax + Cf::AX_A) + 32 * half * 64 + i;
        const float* dp = dus + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          a0 = fmaf(Ac[t * 64], dp[t], a0);
          a1 = fmaf(Ac[(t + 1) * 64], dp[t + 1], a1);
          a2 = fmaf(Ac[(t + 2) * 64], dp[t + 2], a2);
          a3 = fmaf(Ac[(t + 3) * 64], dp[t + 3], a3);
        }
        gp[half * 64 + i] = (a0 + a1) + (a2 + a3);
      }
      bar_u();
      float* dbk = db0s + (k & 1) * 64;
      if (tid < C) {
        const float g = gp[i] + gp[64 + i];
        dbk[i] = -reinterpret_cast<const float*>(ax + Cf::AX_B)[i] * g;
        if (rank == 0) wg[ch * C + i] = g;
      }
      bar_u();
      if (tid == 0) mbar_arrive(&aux_free[k & 1]);
      // ---- B2 = diag(db0_k) K+_n slice, bf16 hi + lo, into buffer k & 1
      if (k >= 2)
        tc::mbar_wait<false>(&mma2_bar[k & 1], (uint32_t)(((k - 2) >> 1) & 1), err, tc::kErrTimeoutMma,
                             &abort_flag);
      tc::mbar_wait<false>(&l_full[k % 3], (uint32_t)((k / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      {
        constexpr int TQ = 128 / NJ, TPT = C / TQ;
        const int jl = tid % NJ, tq = tid / NJ;
        const float* KP = reinterpret_cast<const float*>(late(k) + Cf::L_KP);
        unsigned char* b2 = sm + Cf::B2 + (k & 1) * Cf::B2_SZ;
#pragma unroll
        for (int g8 = 0; g8 < TPT; g8 += 8) {
          __align__(16) __nv_bfloat16 hi8[8], lo8[8];
#pragma unroll
          for (int ii = 0; ii < 8; ++ii) {
            const int tt = tq * TPT + g8 + ii;
            const float x = dbk[tt] * KP[tt * NJ + jl];
            hi8[ii] = __float2bfloat16_rn(x);
            lo8[ii] = __float2bfloat16_rn(x - __bfloat162float(hi8[ii]));
          }
          const uint32_t off = tc::sw128_off(jl, tq * TPT + g8, NJ, 2);
          *reinterpret_cast<uint4*>(b2 + off) = *reinterpret_cast<const uint4*>(hi8);
          *reinterpret_cast<uint4*>(b2 + NJ * 128 + off) = *reinterpret_cast<const uint4*>(lo8);
        }
      }
      tc::fence_proxy_async();
      mbar_arrive(&b2_full[k & 1]);
    }
    if (tid == 0)
      for (int m = NC - 1; m >= 0 && m >= NC - 4; --m) mbar_drain(&x_bar[m & 3], (uint32_t)((m >> 2) & 1));
  } else if (warp < 8) {
    // ============================== state warps ==============================
    const int r = tid - 128;
    const uint32_t my_lanes = tc::tmem_lane_addr(tmem, warp, 0);
    // column dot of the lookahead MMA of step m: sum_r V_n[i,r] X'[r,i] over this CTA's rows
    auto column_dot_send = [&](int m) {
      tc::mbar_wait<false>(&l_full[m % 3], (uint32_t)((m / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::mbar_wait<false>(&mma1_bar, (uint32_t)(m & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        float x[64];
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
          float y16[16];
          tc::tmem_ld16(my_lanes + Cf::X_COL + 16 * c16, y16);
#pragma unroll
          for (int q = 0; q < 16; ++q) x[16 * c16 + q] = y16[q];
        }
        tc::tmem_ld_wait();
        const unsigned char* vt = late(m) + Cf::L_V;
        float lo[32], hi[32];
#pragma unroll
        for (int g8 = 0; g8 < 8; ++g8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(vt + tc::sw128_off(r, 8 * g8, 128, 2));
          const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int tt = 8 * g8 + q;
            if (tt < 32) lo[tt] = x[tt] * __bfloat162float(e[q]);
            else hi[tt - 32] = x[tt] * __bfloat162float(e[q]);
          }
        }
        warp_transpose_reduce<32>(lo, lane);
        warp_transpose_reduce<32>(hi, lane);
        xred[(warp & 3) * 64 + lane] = lo[0];
        xred[(warp & 3) * 64 + 32 + lane] = hi[0];
      }
      tc::tc_before_sync();
      bar_s();
      if (r < C) mine[r] = (xred[r] + xred[64 + r]) + (xred[128 + r] + xred[192 + r]);
      bar_s();
      if (r < 16 * R) {
        const int peer = r / 16, q4 = r % 16;
        const float4 val = *reinterpret_cast<const float4*>(mine + 4 * q4);
        float* rv = recv + (m & 3) * R * 64;
        const uint32_t raddr = tc::mapa(tc::smem_u32(rv + rank * 64 + 4 * q4), (uint32_t)peer);
        const uint32_t rbar = tc::mapa(tc::smem_u32(&x_bar[m & 3]), (uint32_t)peer);
        tc::st_async_v4(raddr, val, rbar);
      }
    };
    // W <- Z diag(gamma_C of step m's chunk) + dO^T Q+ (z: this thread's Z row slice)
    auto make_w = [&](int m, const float* z) {
      tc::mbar_wait<false>(&l_full[m % 3], (uint32_t)((m / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      const float* gC = reinterpret_cast<const float*>(late(m) + Cf::L_GC);
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float m3[16], w[16];
        tc::tmem_ld16(my_lanes + Cf::M3_COL + jj, m3);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) w[q] = fmaf(z[jj + q], gC[jj + q], m3[q]);
        tc::tmem_st16(my_lanes + Cf::W_COL + jj, w);
      }
      tc::tmem_st_wait();
    };
    {
      // Z_0 = dS_T: into tensor memory (the A operand of step 0's lookahead) and
      // saved as the last chunk's end-state gradient
      float z[NJ];
      const size_t chl = (size_t)unit * NC + chunk_of(0);
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float x[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          x[q] = dST ? dST[(size_t)unit * D * D + (size_t)r * D + j0 + jj + q] : 0.f;
          z[jj + q] = x[q];
        }
        tc::tmem_st16(my_lanes + Cf::W_COL + jj, x);
        save_bf16_tile(wdSCb, chl, r, j0 + jj, x);
      }
      tc::tmem_st_wait();
      tc::tc_before_sync();
      bar_s();
      if (r == 0) mbar_arrive(&s_ready);  // phase 0: Z_0 in place of W
      column_dot_send(0);                 // waits for the lookahead MMA and dO^T Q+ of step 0
      make_w(0, z);                       // W_0 = Z_0 diag(gamma) + dO^T Q+
      tc::tc_before_sync();
      bar_s();
      if (r == 0) mbar_arrive(&s_ready);  // phase 1: W_0
      if (NC > 1) column_dot_send(1);
    }
    for (int k = 0; k < NC; ++k) {
      tc::mbar_wait<false>(&mma2_bar[k & 1], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      // ---- Z_{k+1} = W_k + dS_k; saved as the next chunk's end-state gradient
      //      (or written out as dS0); then W_{k+1} = Z_{k+1} diag(gamma) + dO^T Q+
      float z[NJ];
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float w[16], d2[16];
        tc::tmem_ld16(my_lanes + Cf::W_COL + jj, w);
        tc::tmem_ld16(my_lanes + Cf::D2_COL + (k & 1) * NJ + jj, d2);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          w[q] += d2[q];
          z[jj + q] = w[q];
        }
        if (k + 1 < NC) {
          save_bf16_tile(wdSCb, (size_t)unit * NC + chunk_of(k + 1), r, j0 + jj, w);
        } else if (dS0) {
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4)
            *reinterpret_cast<float4*>(dS0 + (size_t)unit * D * D + (size_t)r * D + j0 + jj + 4 * i4) =
                make_float4(w[4 * i4], w[4 * i4 + 1], w[4 * i4 + 2], w[4 * i4 + 3]);
        }
      }
      if (k + 1 < NC) make_w(k + 1, z);
      tc::tc_before_sync();
      bar_s();
      if (r == 0) mbar_arrive(&s_ready);  // phase k + 2: W_{k+1}
      if (k + 2 < NC) column_dot_send(k + 2);
    }
  } else if (warp == 8) {
    // ================================ issuer ================================
    const uint32_t ID1 = tc::idesc(128, 64, 2);                 // tf32: M = 128 rows r, N = 64 positions
    const uint32_t IDB = tc::idesc(128, NJ, 1) | (1u << 15);    // bf16, A MN-major: M = 128 rows r, N = NJ
    const uint32_t ID2 = tc::idesc(128, NJ, 1);                 // bf16, both K-major
    // lookahead X' = W K^e_n^T and M3 = dO_n^T Q+_n of step m, one commit for both
    auto issue_x = [&](int m) {
      tc::mbar_wait<false>(&e_full[m & 1], (uint32_t)((m >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* es = early(m);
#pragma unroll
        for (int ks = 0; ks < NJ / 8; ++ks) {
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(es + Cf::E_KE + (Cf::KBJ * (rank & 1) + ks) * 32));
          tc::mma_tf32_ts(tmem + Cf::X_COL, tmem + Cf::W_COL + ks * 8, bd, ID1, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128_mn(tc::smem_u32(es + Cf::E_DO + ks * 2048), 8192u);
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(es + Cf::E_QP + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::M3_COL, ad, bd, IDB, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mma1_bar);
        tc::mma_commit(&e_free[m & 1]);  // the early slot may be refilled once these MMAs are done
      }
      __syncwarp();
    };
    tc::mbar_wait<false>(&s_ready, 0u, err, tc::kErrTimeoutMma, &abort_flag);  // Z_0
    tc::tc_after_sync();
    issue_x(0);
    if (NC > 1) {
      tc::mbar_wait<false>(&s_ready, 1u, err, tc::kErrTimeoutMma, &abort_flag);  // W_0
      tc::tc_after_sync();
      issue_x(1);
    }
    for (int k = 0; k < NC; ++k) {
      if (k >= 1 && k + 1 < NC) {
        tc::mbar_wait<false>(&s_ready, (uint32_t)((k + 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);  // W_k
        tc::tc_after_sync();
        issue_x(k + 1);
      }
      tc::mbar_wait<false>(&b2_full[k & 1], (uint32_t)((k >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::mbar_wait<false>(&l_full[k % 3], (uint32_t)((k / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* vt = late(k) + Cf::L_V;
        const unsigned char* b2 = sm + Cf::B2 + (k & 1) * Cf::B2_SZ;
        // dS_k = V_n^T (B2hi + B2lo)^T  (M = 128 rows r, N = NJ, K = 64 positions)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128(tc::smem_u32(vt + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::D2_COL + (k & 1) * NJ, ad, tc::desc_sw128(tc::smem_u32(b2 + ks * 32)), ID2,
                          ks > 0 ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::D2_COL + (k & 1) * NJ, ad,
                          tc::desc_sw128(tc::smem_u32(b2 + NJ * 128 + ks * 32)), ID2, 1u);
        }
        tc::mma_commit(&mma2_bar[k & 1]);
        tc::mma_commit(&l_free[k % 3]);  // the late slot may be refilled once this MMA is done
      }
      __syncwarp();
    }
    if (lane == 0) tc::mma_commit(&drain_bar);
    __syncwarp();
    mbar_drain(&drain_bar, 0u);
  } else {
    // =============================== producer ===============================
    auto early_load = [&](int k) {
      const int si = k & 1, n = chunk_of(k);
      if (k >= 2)
        tc::mbar_wait<false>(&e_free[si], (uint32_t)(((k - 2) >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      if (lane == 0) {
        unsigned char* es = early(k);
        const size_t ch = (size_t)unit * NC + n;
        tc::fence_proxy_async();
        tc::mbar_expect_tx(&e_full[si], Cf::E_BYTES);
        tc::tma_load_4d(es + Cf::E_DO, &tm_do, 0, h, n * C, b, &e_full[si]);
        tc::tma_load_4d(es + Cf::E_DO + 8192, &tm_do, 64, h, n * C, b, &e_full[si]);
        tc::tma_load_4d(es + Cf::E_KE, &tm_ke, jb, h, n * C, b, &e_full[si]);
        tc::bulk_g2s(es + Cf::E_QP, wQpT + ch * (D * C) + (size_t)j0 * C, NJ * 128u, &e_full[si]);
        if (k + kL2Ahead < NC) {
          const int np = chunk_of(k + kL2Ahead);
          tc::tma_prefetch_l2_4d(&tm_do, 0, h, np * C, b);
          tc::tma_prefetch_l2_4d(&tm_do, 64, h, np * C, b);
          tc::tma_prefetch_l2_4d(&tm_ke, jb, h, np * C, b);
          tc::prefetch_l2(wQpT + (ch - kL2Ahead) * (D * C) + (size_t)j0 * C, NJ * 128u);
        }
      }
      __syncwarp();
    };
    auto late_load = [&](int k) {
      const int si = k % 3, n = chunk_of(k);
      if (k >= 3)
        tc::mbar_wait<false>(&l_free[si], (uint32_t)((k / 3 - 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      if (lane == 0) {
        unsigned char* ls = late(k);
        const size_t ch = (size_t)unit * NC + n;
        tc::fence_proxy_async();
        tc::mbar_expect_tx(&l_full[si], Cf::L_BYTES);
        tc::bulk_g2s(ls + Cf::L_V, wVt + ch * (D * C), 16384u, &l_full[si]);
        tc::tma_load_4d(ls + Cf::L_KP, &tm_kp, j0, h, n * C, b, &l_full[si]);
        tc::bulk_g2s(ls + Cf::L_GC, wGC + ch * D + j0, NJ * 4u, &l_full[si]);
        if (k + kL2Ahead < NC) {
          tc::prefetch_l2(wVt + (ch - kL2Ahead) * (D * C), 16384u);
          tc::tma_prefetch_l2_4d(&tm_kp, j0, h, chunk_of(k + kL2Ahead) * C, b);
        }
      }
      __syncwarp();
    };
    auto aux_load = [&](int k) {
      const int ai = k & 1, n = chunk_of(k);
      if (k >= 2)
        tc::mbar_wait<false>(&aux_free[ai], (uint32_t)(((k - 2) >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      unsigned char* ax = auxp(k);
      const size_t ch = (size_t)unit * NC + n;
      if (lane == 0) {
        tc::fence_proxy_async();
        tc::mbar_expect_tx(&aux_full[ai], k >= 1 ? 33024u : 16640u);
        tc::bulk_g2s(ax + Cf::AX_A, wA + ch * C * C, 16384u, &aux_full[ai]);
        if (k >= 1) tc::bulk_g2s(ax + Cf::AX_H, wHx + (ch + 1) * C * C, 16384u, &aux_full[ai]);  // H_{n+1}
        tc::bulk_g2s(ax + Cf::AX_DU, wdu + ch * C, 256u, &aux_full[ai]);
        if (k + kL2Ahead < NC) {
          tc::prefetch_l2(wA + (ch - kL2Ahead) * C * C, 16384u);
          tc::prefetch_l2(wHx + (ch - kL2Ahead + 1) * C * C, 16384u);
        }
      }
      float* bs = reinterpret_cast<float*>(ax + Cf::AX_B);
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int p = lane + 32 * k2;
        bs[p] = (n * C + p < T) ? beta[((size_t)b * T + n * C + p) * H + h] : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&aux_full[ai]);
      __syncwarp();
    };
    for (int k = 0; k < 2 && k < NC; ++k) early_load(k);
    for (int k = 0; k < 3 && k < NC; ++k) late_load(k);
    for (int k = 0; k < 2 && k < NC; ++k) aux_load(k);
    for (int k = 0; k < NC; ++k) {
      if (k + 2 < NC) early_load(k + 2);
      if (k + 2 < NC) aux_load(k + 2);
      if (k + 3 < NC) late_load(k + 3);
    }
    if (lane == 0) {
      for (int m = NC - 1; m >= 0 && m >= NC - 2; --m) mbar_drain(&e_full[m & 1], (uint32_t)((m >> 1) & 1));
      for (int m = NC - 1; m >= 0 && m >= NC - 3; --m) mbar_drain(&l_full[m % 3], (uint32_t)((m / 3) & 1));
      for (int m = NC - 1; m >= 0 && m >= NC - 2; --m) mbar_drain(&aux_full[m & 1], (uint32_t)((m >> 1) & 1));
    }
    __syncwarp();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
}

template <int R>
cudaError_t launch_bchain_r(const BwdArgs& a, int* err, cudaStream_t st) {
  const Layout& L = a.L;
  constexpr int NJ = BcCfg<R>::NJ;
  CUtensorMap tm_do, tm_ke, tm_kp;
  if (!make_tmap_bthd(&tm_do, a.dO, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_ke, const_cast<float*>(ws_ptr<const float>(a.fws, L.Ke)), 4, L.B, L.T, L.H, D, 32,
                      true) ||
      !make_tmap_bthd(&tm_kp, ws_ptr<float>(a.ws, L.Kp), 4, L.B, L.T, L.H, D, NJ, false))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)BcCfg<R>::BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.B * L.H * R);
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = BcCfg<R>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(st, "bwd_chain_tc");
  e = cudaLaunchKernelEx(&cfg, bwd_chain_tc<R>, tm_do, tm_ke, tm_kp, a.beta, a.dST, a.dS0, L.H, L.T, L.NC,
                         ws_ptr<const float>(a.fws, L.A), ws_ptr<const float>(a.fws, L.Hx),
                         ws_ptr<const float>(a.fws, L.GC), ws_ptr<const __nv_bfloat16>(a.fws, L.Vt),
                         (const __nv_bfloat16*)ws_ptr<__nv_bfloat16>(a.ws, L.QpT),
                         (const float*)ws_ptr<float>(a.ws, L.du), ws_ptr<__nv_bfloat16>(a.ws, L.dSCb),
                         ws_ptr<float>(a.ws, L.g), err);
  prof_end(st);
  return e;
}

}  // namespace

cudaError_t launch_bwd_chain_tc(const BwdArgs& a, int R, int* err, cudaStream_t st) {
  return R == 8 ? launch_bchain_r<8>(a, err, st) : launch_bchain_r<4>(a, err, st);
}

// The tensor-core backward: per-chunk adjoints (bwd_pre_tc), the reverse
// chain, the per-chunk gradients (bwd_post_tc), then the exact CUDA-core
// stages for chunks flagged outside the factorised decay range.
// Gated or fused inputs: the forward's preparation kernel kept the prologue's
// outputs (logf; for fused inputs the normalised q, k, v and the gated beta,
// c) in the forward's workspace, and the backward reads them there.  a_log
// stays set: the post-chain kernels write df~ and da_log parts in place of dlogf.
BwdArgs plain_view(const BwdArgs& a) {
  BwdArgs p = a;
  const Layout& L = a.L;
  if (a.a_log) p.logf = ws_ptr<const float>(a.fws, L.glogf);
  if (a.pro.norm) {
    p.q = ws_ptr<const __nv_bfloat16>(a.fws, L.fq);
    p.k = ws_ptr<const __nv_bfloat16>(a.fws, L.fk);
    p.v = ws_ptr<const __nv_bfloat16>(a.fws, L.fv);
  }
  if (a.pro.bscale > 0.f) {
    p.beta = ws_ptr<const float>(a.fws, L.fbeta);
    p.c = ws_ptr<const float>(a.fws, L.fc);
  }
  p.pro = Pro{};
  return p;
}

cudaError_t launch_bwd_tc(const BwdArgs& in, int* err, int sms, cudaStream_t st) {
  const BwdArgs a = plain_view(in);
  const Layout& L = a.L;
  cudaError_t e;
  if (a.phases & kPhaseLocal) {
    if ((e = launch_bwd_pre_tc(a, err, sms, st)) != cudaSuccess) return e;
  }
  if (!(a.phases & kPhaseCarry)) return cudaSuccess;
  if ((e = launch_bwd_chain_tc(a, choose_cluster(L.B * L.H, sms), err, st)) != cudaSuccess) return e;
  if ((e = launch_bwd_post_tc(a, err, st)) != cudaSuccess) return e;
  // chunks outside the factorised decay range: exact CUDA-core recomputation
  return launch_bwd_simt_stages(a, kStageCC | kStageState | kStageIntra, ws_ptr<int>(a.ws, L.bflags), st);
}


}  // namespace kd
