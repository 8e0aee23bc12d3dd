// kd_fwd_tc.cu -- tensor-core (tcgen05/TMEM) forward for bf16 q,k,v and
// d_k = d_v = 128.
//
// Chunk form as in kd_fwd_simt.cu (KronLSTM digest, "무엇과 다른가": the
// DeltaNet chunk-parallel scheme applies; Gated DeltaNet-2 article, "방법론" /
// "기술 상세": WY form, C = 64, forward substitution):
//   b0 = rowdot(V, S0 K+^T), u = y - A (beta o b0),
//   S  <- S diag(gamma_C) + V^T diag(u) K^e,
//   O  = Q+ S0^T + P diag(u) V.
//
// Kernels:
//  1. prep (kd_fwd_simt.cu, fwd_prep_simt): A = (I + diag(beta) M)^{-1}, y.
//  2. fwd_chain_tc: the sequential chain.  One thread-block cluster of R CTAs
//     per (b,h); CTA c owns the key-channel slice J_c (dk/R columns) of the
//     state, kept in tensor memory as the A operand of the MMAs:
//       X_c = S[:,J_c] K+[:,J_c]^T            (tcgen05, A from TMEM)
//       b0_c[t] = sum_r V[t,r] X_c[r,t]       (column sum over TMEM lanes)
//       b0 = sum_c b0_c                       (distributed shared memory:
//                                              st.async + mbarrier tx count)
//       u = y - A (beta o b0)                 (every CTA, identical order)
//       dS_c = V^T (diag(u) K^e[:,J_c])       (tcgen05)
//       S[:,J_c] <- S[:,J_c] diag(gamma_C) + dS_c
//     The next chunk's rows are fetched with bulk async copies while the
//     current chunk runs.  Each chunk-start state slice is written to global
//     memory in the 128-byte-swizzled K-major tile layout the output kernel's
//     MMA reads directly.
//  3. fwd_out_tc: one CTA per chunk, all chunks in parallel:
//       O^T = S0 Q+^T + V^T (diag(u) P^T)  with P = tril(Q+ K-^T) (tcgen05).
//     Chunks whose log-decay range makes k/gamma leave the fp32 range are
//     flagged and recomputed exactly by fwd_out_fixup.
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;

template <int R>
struct ChainCfg {
  static constexpr int NJ = D / R;                    // key channels per CTA
  static constexpr int KBJ = (R == 8) ? 2 : 0;        // K steps of the K~ block that precede this CTA's channels (odd R=8 ranks)
  // tensor memory columns: X' (64), state slice, update
  static constexpr int D1_COL = 0, S_COL = 64, D2_COL = 64 + NJ;
  static constexpr uint32_t TMEM_COLS = (64 + 2 * NJ) <= 128 ? 128u : 256u;
  static constexpr uint32_t up1k(uint32_t x) { return (x + 1023u) / 1024u * 1024u; }
  // chunk slot (ring of three), all written by TMA / bulk copies
  static constexpr uint32_t SL_V = 0;                          // V^T bf16 [r][t], K-major, 128-byte swizzle (16 KB)
  static constexpr uint32_t SL_B1 = 16384;                     // K~, the 32-channel block holding this CTA's channels:
                                                               //   tf32 [t][32], 128-byte swizzle (8 KB)
  static constexpr uint32_t SL_KE = SL_B1 + 8192;              // K^e slice fp32 [64][NJ]
  static constexpr uint32_t SL_GC = SL_KE + 64 * NJ * 4;       // gamma_C slice [NJ]
  static constexpr uint32_t SL_Y = SL_GC + 128;                // y [64]
  static constexpr uint32_t SL_SZ = up1k(SL_Y + 256);
  static constexpr uint32_t LOAD_BYTES = 16384 + 8192 + 64 * NJ * 4 + NJ * 4 + 256;
  // per-chunk matrices of the u recursion (ring of two): A, H
  static constexpr uint32_t AUX = 3 * SL_SZ;
  static constexpr uint32_t AUX_SZ = 32768;
  static constexpr uint32_t B2 = AUX + 2 * AUX_SZ;             // diag(u) K^e slice, bf16 hi / lo, NJ rows x 128 B each
  static constexpr uint32_t SM = B2 + 2 * NJ * 128;            // small arrays (floats)
  static constexpr uint32_t SM_BS = SM;                        // beta [3][64]
  static constexpr uint32_t SM_W = SM_BS + 3 * 64 * 4;         // beta o b0 [64]
  static constexpr uint32_t SM_U = SM_W + 64 * 4;              // u [64] (previous chunk's until replaced)
  static constexpr uint32_t SM_UP = SM_U + 64 * 4;             // partial sums [2][64]
  static constexpr uint32_t SM_MINE = SM_UP + 2 * 64 * 4;      // own c partial [64]
  static constexpr uint32_t SM_XRED = SM_MINE + 64 * 4;        // per-warp partials [4][64]
  static constexpr uint32_t SM_RECV = SM_XRED + 4 * 64 * 4;    // [2][R][64]
  static constexpr uint32_t SM_END = SM_RECV + 2 * R * 64 * 4;
  static constexpr uint32_t BYTES = SM_END + 1024;             // + alignment slack
};

// Writes 16 state values (row r, columns j..j+15) of one chunk into the bf16
// tile the backward's MMAs read: [r][j] (rows r, K = j), 128-byte-swizzled
// K-major, 32 KB.  The backward also reads it transposed, as an MN-major operand.
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

// named barriers: 1 = the 4 chain warps, 2 = the 4 producer warps;
// 3 = chain -> issuer "update operand ready", 4 = chain -> issuer "state updated"
// (the chain warps arrive, the issuer warp waits: 160 threads)
__device__ __forceinline__ void bar_chain() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_prod() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_arrive_issuer(int id) { asm volatile("bar.arrive %0, 160;" ::"r"(id) : "memory"); }
__device__ __forceinline__ void bar_wait_chain(int id) { asm volatile("bar.sync %0, 160;" ::"r"(id) : "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(b)) : "memory");
}

// The chain with a one-chunk lookahead.  With c_{n+1} = rowdot(V_{n+1}, S_n K~_{n+1}^T),
// K~_{n+1} = K+_{n+1} diag(gamma_C of chunk n), and the cross-chunk matrix
// H_{n+1} = (V_{n+1} V_n^T) o (K+_{n+1} K^e_n^T) (fwd_cross_tc):
//   b0_{n+1} = rowdot(V_{n+1}, S_{n+1} K+_{n+1}^T) = c_{n+1} + H_{n+1} u_n,
// so c_{n+1} (an MMA on the state, a column dot and the cluster all-reduce)
// is formed while u_n and the update of chunk n proceed; only two 64 x 64
// matrix-vector products separate u_n from u_{n+1}.
//
// Warp roles (288 threads):
//   warps 0-3  chain: u, the update operand, the column dots, the cluster
//              all-reduce, the state update; thread r owns tensor-memory lane r.
//   warps 4-7  producer: TMA / bulk loads of each chunk's operands (built by
//              fwd_cross_tc) into a ring of three slots, A and H into a ring
//              of two, and the save of each chunk-start state slice.
//   warp 8     issuer: one thread issues every tcgen05 MMA.
// Hand-offs: mbarriers raw_full (a slot's loads landed), slot_free (chain done
// with a slot), aux_full / aux_free (A, H), s_ready (state of chunk n in
// tensor memory), s_saved (producer has read it), mma1 / mma2 (MMA done);
// named barriers 3 and 4 (chain -> issuer).
template <int R>
__global__ void __launch_bounds__(288, 1) fwd_chain_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_ke, const float* __restrict__ beta, const float* __restrict__ S0,
    float* __restrict__ ST, int H, int T, int NC, const float* __restrict__ wy, const float* __restrict__ wA,
    const float* __restrict__ wHx, const float* __restrict__ wGC, const __nv_bfloat16* __restrict__ wVt,
    float* __restrict__ wS0blob,
    float* __restrict__ wu, float* __restrict__ wb0, __nv_bfloat16* __restrict__ wS0b, int* __restrict__ err) {
  using Cf = ChainCfg<R>;
  constexpr int NJ = Cf::NJ;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t raw_full[3], slot_free[3], aux_full[2], aux_free[2], s_ready, s_saved, x_bar[2], mma1_bar,
      mma2_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_rank();
  const int unit = blockIdx.x / R;  // (b, h)
  const int b = unit / H, h = unit % H;
  const int j0 = static_cast<int>(rank) * NJ;
  const int jb = j0 & ~31;  // first channel of the 32-channel K~ block

  float* bs = reinterpret_cast<float*>(sm + Cf::SM_BS);
  float* ws = reinterpret_cast<float*>(sm + Cf::SM_W);
  float* us = reinterpret_cast<float*>(sm + Cf::SM_U);
  float* up = reinterpret_cast<float*>(sm + Cf::SM_UP);
  float* mine = reinterpret_cast<float*>(sm + Cf::SM_MINE);
  float* xred = reinterpret_cast<float*>(sm + Cf::SM_XRED);
  float* recv = reinterpret_cast<float*>(sm + Cf::SM_RECV);
  auto slot = [&](int m) { return sm + (m % 3) * Cf::SL_SZ; };

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) {
      tc::mbar_init(&raw_full[i], 1);
      tc::mbar_init(&slot_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux_full[i], 1);
      tc::mbar_init(&aux_free[i], 1);
      tc::mbar_init(&x_bar[i], 1);
    }
    tc::mbar_init(&s_ready, 1);
    tc::mbar_init(&s_saved, 1);
    tc::mbar_init(&mma1_bar, 1);
    tc::mbar_init(&mma2_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, Cf::TMEM_COLS);
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();  // peers' barriers are initialised before any remote arrive
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t my_lanes = tc::tmem_lane_addr(tmem, warp, 0);  // lanes 32*(warp%4) ..

  if (warp == 8) {
    // ============================== issuer warp ==============================
    const uint32_t ID1 = tc::idesc(128, 64, 2);
    const uint32_t ID2 = tc::idesc(128, NJ, 1);  // bf16, both K-major
    // X' = S K~_m^T  (M = 128 rows r, N = 64 positions, K = NJ; A = the state in tensor memory)
    auto issue_x = [&](int m) {
      tc::mbar_wait<false>(&raw_full[m % 3], (uint32_t)((m / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* st = slot(m);
#pragma unroll
        for (int ks = 0; ks < NJ / 8; ++ks) {
          const uint64_t bd = tc::desc_sw128(tc::smem_u32(st + Cf::SL_B1 + (Cf::KBJ * (rank & 1) + ks) * 32));
          tc::mma_tf32_ts(tmem + Cf::D1_COL, tmem + Cf::S_COL + ks * 8, bd, ID1, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mma1_bar);
      }
      __syncwarp();
    };
    bar_wait_chain(4);  // S_0 in tensor memory
    tc::tc_after_sync();
    issue_x(0);
    for (int n = 0; n < NC; ++n) {
      if (n + 1 < NC) {
        if (n >= 1) {
          bar_wait_chain(4);  // S_n in tensor memory (update of chunk n-1 done)
          tc::tc_after_sync();
        }
        issue_x(n + 1);
      }
      bar_wait_chain(3);  // update operand of chunk n built
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* st = slot(n);
        // dS = V_n^T (B2hi + B2lo)^T  (M = 128 rows r, N = NJ, K = 64 positions)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128(tc::smem_u32(st + Cf::SL_V + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::D2_COL, ad, tc::desc_sw128(tc::smem_u32(sm + Cf::B2 + ks * 32)), ID2,
                          ks > 0 ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::D2_COL, ad, tc::desc_sw128(tc::smem_u32(sm + Cf::B2 + NJ * 128 + ks * 32)),
                          ID2, 1u);
        }
        tc::mma_commit(&mma2_bar);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // =========================== producer warps ===========================
    const int p = tid - 128;
    // the operands of chunk m into its slot (chunk m - 3 must be done)
    auto prepare = [&](int m) {
      unsigned char* st = slot(m);
      const int si = m % 3;
      if (m >= 3)
        tc::mbar_wait<false>(&slot_free[si], (uint32_t)((m / 3 - 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      if (p == 0) {
        uint64_t* bar = &raw_full[si];
        const size_t ch = (size_t)unit * NC + m;
        tc::fence_proxy_async();
        tc::mbar_expect_tx(bar, Cf::LOAD_BYTES);
        tc::bulk_g2s(st + Cf::SL_V, wVt + ch * (D * C), 16384u, bar);
        tc::tma_load_4d(st + Cf::SL_B1, &tm_kt, jb, h, m * C, b, bar);
        tc::tma_load_4d(st + Cf::SL_KE, &tm_ke, j0, h, m * C, b, bar);
        tc::bulk_g2s(st + Cf::SL_GC, wGC + ch * D + j0, NJ * 4u, bar);
        tc::bulk_g2s(st + Cf::SL_Y, wy + ch * C, 256u, bar);
      }
      if (p < C) bs[si * 64 + p] = (m * C + p < T) ? beta[((size_t)b * T + m * C + p) * H + h] : 0.f;
    };
    // A and H of chunk m (chunk m - 2 must have consumed its buffer)
    auto aux = [&](int m) {
      if (p != 0) return;
      const int ai = m & 1;
      if (m >= 2)
        tc::mbar_wait<false>(&aux_free[ai], (uint32_t)(((m - 2) >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      unsigned char* ax = sm + Cf::AUX + ai * Cf::AUX_SZ;
      const size_t ch = (size_t)unit * NC + m;
      tc::fence_proxy_async();
      tc::mbar_expect_tx(&aux_full[ai], m >= 1 ? 32768u : 16384u);
      tc::bulk_g2s(ax, wA + ch * C * C, 16384u, &aux_full[ai]);
      if (m >= 1) tc::bulk_g2s(ax + 16384, wHx + ch * C * C, 16384u, &aux_full[ai]);
    };
    prepare(0);
    aux(0);
    if (NC > 1) prepare(1);
    for (int m = 0; m < NC; ++m) {
      if (m + 2 < NC) prepare(m + 2);
      if (m + 1 < NC) aux(m + 1);
      // save the chunk-start state slice of chunk m once the chain has it in tensor memory
      tc::mbar_wait<false>(&s_ready, (uint32_t)(m & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        float* blob = wS0blob + ((size_t)unit * NC + m) * D * D;
        const int r = p;
#pragma unroll
        for (int jj = 0; jj < NJ; jj += 16) {
          float x[16];
          tc::tmem_ld16(my_lanes + Cf::S_COL + jj, x);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int jg = j0 + jj + 4 * q4;
            *reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(blob) + tc::sw128_off(r, jg, 128, 4)) =
                make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
          }
          if (wS0b) save_bf16_tile(wS0b, (size_t)unit * NC + m, r, j0 + jj, x);
        }
      }
      tc::tc_before_sync();
      bar_prod();
      if (p == 0) mbar_arrive(&s_saved);
    }
  } else {
    // ============================= chain warps ============================
    const int r = tid;  // tensor-memory lane = state row
    {
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = S0 ? S0[(size_t)unit * D * D + (size_t)r * D + j0 + jj + i] : 0.f;
        tc::tmem_st16(my_lanes + Cf::S_COL + jj, x);
      }
      tc::tmem_st_wait();
      tc::tc_before_sync();
      bar_chain();
      if (tid == 0) mbar_arrive(&s_ready);
      bar_arrive_issuer(4);
    }
    int mma1_par = 0, mma2_par = 0;
    // c_m partial: sum_r V_m[t,r] X'[r,t] over this CTA's rows, then all-reduce over the cluster
    auto column_dot_send = [&](int m) {
      tc::mbar_wait<false>(&mma1_bar, (uint32_t)mma1_par, err, tc::kErrTimeoutMma, &abort_flag);
      mma1_par ^= 1;
      tc::tc_after_sync();
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
        const unsigned char* vt = slot(m) + Cf::SL_V;  // row r of V^T: V[t, r] for t = 0..63
        float lo[32], hi[32];
#pragma unroll
        for (int g8 = 0; g8 < 8; ++g8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(vt + tc::sw128_off(r, 8 * g8, 128, 2));
          const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            if (t < 32) lo[t] = x[t] * __bfloat162float(e[i]);
            else hi[t - 32] = x[t] * __bfloat162float(e[i]);
          }
        }
        warp_transpose_reduce<32>(lo, lane);
        warp_transpose_reduce<32>(hi, lane);
        xred[warp * 64 + lane] = lo[0];
        xred[warp * 64 + 32 + lane] = hi[0];
      }
      tc::tc_before_sync();
      bar_chain();
      if (tid < C) mine[tid] = xred[tid] + xred[64 + tid] + xred[128 + tid] + xred[192 + tid];
      bar_chain();
      const int xb = m & 1;
      float* rv = recv + xb * R * 64;
      if (tid == 0) tc::mbar_expect_tx(&x_bar[xb], R * 64u * 4u);
      if (tid < 16 * R) {
        const int peer = tid / 16, q4 = tid % 16;
        const float4 val = *reinterpret_cast<const float4*>(mine + 4 * q4);
        const uint32_t raddr = tc::mapa(tc::smem_u32(rv + rank * 64 + 4 * q4), (uint32_t)peer);
        const uint32_t rbar = tc::mapa(tc::smem_u32(&x_bar[xb]), (uint32_t)peer);
        tc::st_async_v4(raddr, val, rbar);
      }
    };
    column_dot_send(0);
    for (int n = 0; n < NC; ++n) {
      const unsigned char* st = slot(n);
      const size_t ch = (size_t)unit * NC + n;
      // ---- b0_n = c_n + H_n u_{n-1};  u_n = y_n - A_n (beta o b0_n)
      tc::mbar_wait<true>(&x_bar[n & 1], (uint32_t)((n >> 1) & 1), err, tc::kErrTimeoutCluster, &abort_flag);
      tc::mbar_wait<false>(&aux_full[n & 1], (uint32_t)((n >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      const float* Am = reinterpret_cast<const float*>(sm + Cf::AUX + (n & 1) * Cf::AUX_SZ);
      const float* Hm = Am + C * C;
      // two threads per position t (lanes 2t', 2t'+1 of a warp), halves of i, rotated reads
      const int t = tid >> 1, half = tid & 1;
      const int rot = t + 16 * half;
      float s = 0.f;
      {
        const float* rv = recv + (n & 1) * R * 64;
#pragma unroll
        for (int c2 = 0; c2 < R; ++c2) s += rv[c2 * 64 + t];
      }
      if (n > 0) {
        const float* Hrow = Hm + t * 64 + 32 * half;
        const float* uh = us + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int i0 = (i + rot) & 31, i1 = (i + 1 + rot) & 31, i2 = (i + 2 + rot) & 31, i3 = (i + 3 + rot) & 31;
          a0 = fmaf(Hrow[i0], uh[i0], a0);
          a1 = fmaf(Hrow[i1], uh[i1], a1);
          a2 = fmaf(Hrow[i2], uh[i2], a2);
          a3 = fmaf(Hrow[i3], uh[i3], a3);
        }
        float hu = (a0 + a1) + (a2 + a3);
        hu += __shfl_xor_sync(0xffffffffu, hu, 1);
        s += hu;
      }
      // s = b0_n[t] in both threads of the pair
      if (half == 0) {
        ws[t] = bs[(n % 3) * 64 + t] * s;
        if (rank == 0 && wb0) wb0[ch * C + t] = s;
      }
      bar_chain();
      float uval;
      {
        const float* Arow = Am + t * 64 + 32 * half;
        const float* wh = ws + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int i0 = (i + rot) & 31, i1 = (i + 1 + rot) & 31, i2 = (i + 2 + rot) & 31, i3 = (i + 3 + rot) & 31;
          a0 = fmaf(Arow[i0], wh[i0], a0);
          a1 = fmaf(Arow[i1], wh[i1], a1);
          a2 = fmaf(Arow[i2], wh[i2], a2);
          a3 = fmaf(Arow[i3], wh[i3], a3);
        }
        float aw = (a0 + a1) + (a2 + a3);
        aw += __shfl_xor_sync(0xffffffffu, aw, 1);
        uval = reinterpret_cast<const float*>(st + Cf::SL_Y)[t] - aw;
      }
      bar_chain();  // every thread has read u_{n-1} (us) and w
      if (half == 0) {
        us[t] = uval;
        if (rank == 0 && wu) wu[ch * C + t] = uval;
      }
      bar_chain();
      if (tid == 0) mbar_arrive(&aux_free[n & 1]);
      // ---- B2 = diag(u_n) K^e_n slice as bf16 hi + lo (N = NJ rows j, K = 64 positions):
      //      thread (channel jl, 64/TQ consecutive positions) writes 16-byte pieces of row jl
      {
        constexpr int TQ = 128 / NJ, TPT = C / TQ;  // position groups, positions per thread
        const int jl = tid % NJ, tq = tid / NJ;
        const float* KE = reinterpret_cast<const float*>(st + Cf::SL_KE);
#pragma unroll
        for (int g8 = 0; g8 < TPT; g8 += 8) {
          __align__(16) __nv_bfloat16 hi8[8], lo8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int tt = tq * TPT + g8 + i;
            const float x = us[tt] * KE[tt * NJ + jl];
            hi8[i] = __float2bfloat16_rn(x);
            lo8[i] = __float2bfloat16_rn(x - __bfloat162float(hi8[i]));
          }
          const uint32_t off = tc::sw128_off(jl, tq * TPT + g8, NJ, 2);
          *reinterpret_cast<uint4*>(sm + Cf::B2 + off) = *reinterpret_cast<const uint4*>(hi8);
          *reinterpret_cast<uint4*>(sm + Cf::B2 + NJ * 128 + off) = *reinterpret_cast<const uint4*>(lo8);
        }
      }
      tc::fence_proxy_async();
      tc::tc_before_sync();
      bar_arrive_issuer(3);
      // ---- c_{n+1} from X' (its all-reduce overlaps the update)
      if (n + 1 < NC) column_dot_send(n + 1);
      tc::mbar_wait<false>(&mma2_bar, (uint32_t)mma2_par, err, tc::kErrTimeoutMma, &abort_flag);
      mma2_par ^= 1;
      // the producer must have saved this chunk's start state before it changes
      tc::mbar_wait<false>(&s_saved, (uint32_t)(n & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      // ---- S <- S diag(gamma_C) + dS
      {
        const float* gC = reinterpret_cast<const float*>(st + Cf::SL_GC);
#pragma unroll
        for (int jj = 0; jj < NJ; jj += 16) {
          float s[16], d2[16];
          tc::tmem_ld16(my_lanes + Cf::S_COL + jj, s);
          tc::tmem_ld16(my_lanes + Cf::D2_COL + jj, d2);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) s[i] = fmaf(s[i], gC[jj + i], d2[i]);
          tc::tmem_st16(my_lanes + Cf::S_COL + jj, s);
        }
        tc::tmem_st_wait();
      }
      tc::tc_before_sync();
      bar_chain();
      if (tid == 0) {
        mbar_arrive(&slot_free[n % 3]);
        mbar_arrive(&s_ready);
      }
      if (n + 2 < NC) bar_arrive_issuer(4);
    }
    if (ST) {
      tc::tc_after_sync();
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float x[16];
        tc::tmem_ld16(my_lanes + Cf::S_COL + jj, x);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) ST[(size_t)unit * D * D + (size_t)r * D + j0 + jj + i] = x[i];
      }
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();  // no peer may still write into this CTA's shared memory
  if (warp == 0) tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// output kernel, one CTA per chunk:
//   O^T[r,t] = sum_j S0[r,j] Q+[t,j] + sum_i V[i,r] u_i P[t,i],  P = tril(Q+ K-^T)
// The state product and P run in tf32 (the state and the decays are fp32);
// the intra-chunk product V^T (diag(u) P^T) in bf16 (V is bf16 already).
// ---------------------------------------------------------------------------
struct OutCfg {
  static constexpr uint32_t S0 = 0;           // S0 blob, tf32 SW128 [4 kb][128][128 B]
  static constexpr uint32_t QK = 65536;       // tf32 [Q+; K-]: per 32-channel K block rows 0-63 Q+, 64-127 K-
  static constexpr uint32_t VB = 131072;      // V bf16 [i][r], 2 K blocks x 64 rows (TMA, 128-byte swizzle)
  static constexpr uint32_t B3 = 147456;      // diag(u) P^T as bf16 [t][i], 64 rows x 64
  static constexpr uint32_t QR = 155648;      // q bf16 [64][128] (TMA)
  static constexpr uint32_t KR = 172032;      // k bf16 [64][128] (TMA)
  static constexpr uint32_t LG = 188416;      // logf fp32 [64][128] (TMA)
  static constexpr uint32_t U = 221184;       // u [64]
  static constexpr uint32_t XCH = U + 256;    // prefix exchange [128]
  static constexpr uint32_t BYTES = XCH + 512 + 1024;
  static constexpr uint32_t LOAD_BYTES = 65536 + 16384 + 2 * 16384 + 32768 + 256;
  static constexpr uint32_t OO = QK;          // output staging O bf16 [t][r] (after the MMAs)
};

__global__ void __launch_bounds__(256, 1) fwd_out_tc(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_logf,
    const __grid_constant__ CUtensorMap tm_out, int H, int NC, const float* __restrict__ wS0blob,
    const float* __restrict__ wu, int* __restrict__ unsafe_flags, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C;
  const size_t ch = (size_t)unit * NC + n;

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, OutCfg::LOAD_BYTES);
#pragma unroll
    for (int part = 0; part < 4; ++part)
      tc::bulk_g2s(sm + OutCfg::S0 + part * 16384, wS0blob + ch * D * D + part * 4096, 16384u, &ld_bar);
    tc::tma_load_4d(sm + OutCfg::VB, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + OutCfg::VB + 8192, &tm_v, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + OutCfg::QR, &tm_q, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + OutCfg::KR, &tm_k, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + OutCfg::LG, &tm_logf, 0, h, t0, b, &ld_bar);
    tc::bulk_g2s(sm + OutCfg::U, wu + ch * C, 256u, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 128);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);

  // Q+ = q o gamma, K- = k / gamma (tf32); thread (j, half) covers 32 positions
  const int j = tid & 127, half = tid >> 7;
  float mx = 0.f;
  {
    float Lr[32];
    const float* lg = reinterpret_cast<const float*>(sm + OutCfg::LG);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      acc += lg[(32 * half + i) * D + j];
      Lr[i] = acc;
    }
    float* xch = reinterpret_cast<float*>(sm + OutCfg::XCH);
    if (half == 0) xch[j] = acc;
    __syncthreads();
    const float off = half ? xch[j] : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * half + i;
      const float L = Lr[i] + off;
      mx = fmaxf(mx, fabsf(L));
      const float qq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OutCfg::QR + (t * D + j) * 2));
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OutCfg::KR + (t * D + j) * 2));
      *reinterpret_cast<float*>(sm + OutCfg::QK + tc::sw128_off(t, j, 128, 4)) = qq * expf(L);
      *reinterpret_cast<float*>(sm + OutCfg::QK + tc::sw128_off(64 + t, j, 128, 4)) = kk * expf(-L);
    }
  }
  const bool is_unsafe = __syncthreads_or(!(mx < kSafeLogRange)) != 0;
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  // MMA: D_P[t,i] (cols 0..63, lanes 0..63) = [Q+; K-] K-^T ; D_O[r,t] (cols 64..127) = S0 Q+^T
  if (tid == 0) {
    const uint32_t IDT = tc::idesc(128, 64, 2);
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
      const uint64_t qa = tc::desc_sw128(tc::smem_u32(sm + OutCfg::QK + o));
      const uint64_t kmb = tc::desc_sw128(tc::smem_u32(sm + OutCfg::QK + o + 8192));
      const uint64_t sa = tc::desc_sw128(tc::smem_u32(sm + OutCfg::S0 + o));
      tc::mma_tf32_ss(tmem + 0, qa, kmb, IDT, ks > 0 ? 1u : 0u);
      tc::mma_tf32_ss(tmem + 64, sa, qa, IDT, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  // B3[t][i] = u_i P[t,i] for i <= t (bf16; rows t: warps 0-1 own TMEM lanes 0..63)
  if (warp < 2) {
    const int t = tid;
    const float* us = reinterpret_cast<const float*>(sm + OutCfg::U);
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float x[16];
      tc::tmem_ld16(tc::tmem_lane_addr(tmem, warp, 16 * c16), x);
      tc::tmem_ld_wait();
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) {
        const int i = 16 * c16 + i2;
        x[i2] = (i <= t && !is_unsafe) ? x[i2] * us[i] : 0.f;
      }
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[i] = __float2bfloat16_rn(x[8 * h8 + i]);
        *reinterpret_cast<uint4*>(sm + OutCfg::B3 + tc::sw128_off(t, 16 * c16 + 8 * h8, 64, 2)) =
            *reinterpret_cast<const uint4*>(v8);
      }
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    // D_O += V^T (diag(u) P^T): A = V as an MN-major operand (M = r, K = i)
    const uint32_t IDO = tc::idesc(128, 64, 1) | (1u << 15);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      tc::mma_bf16_ss(tmem + 64, tc::desc_sw128_mn(tc::smem_u32(sm + OutCfg::VB + ks * 2048), 8192u),
                      tc::desc_sw128(tc::smem_u32(sm + OutCfg::B3 + ks * 32)), IDO, 1u);
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 1, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  if (!is_unsafe) {
    // O[t, r] from D_O lane r (positions 32*half .. +31), staged as the bf16 tile of the TMA store
    unsigned char* oo = sm + OutCfg::OO;
#pragma unroll
    for (int c16 = 0; c16 < 2; ++c16) {
      float x[16];
      const int tb = 32 * half + 16 * c16;
      tc::tmem_ld16(tc::tmem_lane_addr(tmem, warp, 64 + tb), x);
      tc::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i)
        *reinterpret_cast<__nv_bfloat16*>(oo + tc::sw128_off(tb + i, j, 64, 2)) = __float2bfloat16_rn(x[i]);
    }
    tc::fence_proxy_async();
  }
  __syncthreads();
  if (tid == 0) {
    if (!is_unsafe) {
      tc::tma_store_4d(&tm_out, sm + OutCfg::OO, 0, h, t0, b);
      tc::tma_store_4d(&tm_out, sm + OutCfg::OO + 8192, 64, h, t0, b);
      tc::bulk_commit();
      tc::bulk_wait_read();
    }
    if (unsafe_flags) unsafe_flags[ch] = is_unsafe ? 1 : 0;
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
  (void)lane;
}

// Exact recomputation of O for chunks whose decay range is outside the
// factorised form's fp32 range (flagged by fwd_out_tc): per-element decays.
__global__ void __launch_bounds__(128) fwd_out_fixup(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ logf, int H, int T, int NC,
    const float* __restrict__ wS0blob, const float* __restrict__ wu, const int* __restrict__ unsafe_flags,
    __nv_bfloat16* __restrict__ out) {
  const size_t ch = blockIdx.x;
  if (unsafe_flags[ch] == 0) return;
  extern __shared__ float fx[];
  float (*Ls)[D + 1] = reinterpret_cast<float (*)[D + 1]>(fx);
  float (*qs)[D + 1] = reinterpret_cast<float (*)[D + 1]>(fx + C * (D + 1));
  float (*ks)[D + 1] = reinterpret_cast<float (*)[D + 1]>(fx + 2 * C * (D + 1));
  float* us = fx + 3 * C * (D + 1);
  const int tid = threadIdx.x;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  for (int e = tid; e < C * D; e += 128) {
    const int t = e / D, j = e % D;
    const bool ok = t < nv;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * D + j;
    Ls[t][j] = ok ? logf[g] : 0.f;
    qs[t][j] = ok ? __bfloat162float(q[g]) : 0.f;
    ks[t][j] = ok ? __bfloat162float(k[g]) : 0.f;
  }
  if (tid < C) us[tid] = wu[ch * C + tid];
  __syncthreads();
  {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t][tid];
      Ls[t][tid] = acc;
    }
  }
  __syncthreads();
  const unsigned char* blob = reinterpret_cast<const unsigned char*>(wS0blob + ch * D * D);
  const int r = tid;
  for (int t = 0; t < nv; ++t) {
    float o = 0.f;
    for (int j = 0; j < D; ++j)
      o = fmaf(*reinterpret_cast<const float*>(blob + tc::sw128_off(r, j, 128, 4)), qs[t][j] * expf(Ls[t][j]), o);
    for (int i = 0; i <= t; ++i) {
      float p = 0.f;
      for (int j = 0; j < D; ++j) p = fmaf(qs[t][j] * ks[i][j], expf(Ls[t][j] - Ls[i][j]), p);
      o = fmaf(p * us[i], __bfloat162float(v[(((size_t)b * T + t0 + i) * H + h) * D + r]), o);
    }
    out[(((size_t)b * T + t0 + t) * H + h) * D + r] = __float2bfloat16_rn(o);
  }
}

// ---------------------------------------------------------------------------
// Chunk preparation on tensor cores, one CTA per chunk, all chunks in parallel:
//   [K+; Q+] K-^T (tf32)  -> rows 0-63: decayed key Gram, rows 64-127: P
//   V V^T (bf16, exact)   -> value Gram
//   M = tril(G_K o G_V, -1); A = (I + diag(beta) M)^{-1}; y = A c
// The inverse is blocked by 16: the four diagonal blocks by forward
// substitution in parallel, then the off-diagonal blocks block-row by
// block-row, X_ab = -X_aa sum_{c=b}^{a-1} N_ac X_cb, all in fp32.
// Chunks outside the factorised decay range take exact per-element Grams.
// ---------------------------------------------------------------------------
struct PrepCfg {
  static constexpr uint32_t AKQ = 0;        // [K+; Q+] tf32, 4 K blocks x 128 rows x 128 B
  static constexpr uint32_t BKM = 65536;    // K- tf32, 4 K blocks x 64 rows x 128 B
  static constexpr uint32_t VT = 98304;     // V bf16 [t][r], 2 K blocks x 64 rows (TMA, 128-byte swizzle);
                                            // the Gram's M = 128 rows read 8 KB past a block (unused lanes)
  static constexpr uint32_t QR = 114688;    // q bf16 [64][128] (TMA)
  static constexpr uint32_t KR = 131072;    // k bf16 [64][128] (TMA)
  static constexpr uint32_t LS = 147456;    // logf fp32 [64][128] (TMA), then L in place
  static constexpr uint32_t NS = 180224;    // N = diag(beta) M, fp32 [64][65]
  static constexpr uint32_t XS = NS + 64 * 65 * 4;    // A, fp32 [64][65]
  static constexpr uint32_t TS = XS + 64 * 65 * 4;    // block temporaries [3][16][17]
  static constexpr uint32_t SMALL = TS + 3 * 16 * 17 * 4;  // beta, c [64] each; prefix exchange [128]
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
  static constexpr uint32_t LOAD_BYTES = 16384 + 2 * 16384 + 32768;
};

__global__ void __launch_bounds__(256, 1) fwd_prep_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_logf,
    const float* __restrict__ beta, const float* __restrict__ c, int H, int T, int NC, float* __restrict__ wy,
    float* __restrict__ wA, float* __restrict__ wP, int* __restrict__ err) {
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
  float* Ls = reinterpret_cast<float*>(sm + PrepCfg::LS);
  float* Ns = reinterpret_cast<float*>(sm + PrepCfg::NS);
  float* Xs = reinterpret_cast<float*>(sm + PrepCfg::XS);
  float* Ts = reinterpret_cast<float*>(sm + PrepCfg::TS);
  float* bs = reinterpret_cast<float*>(sm + PrepCfg::SMALL);
  float* cs = bs + 64;
  float* xch = cs + 64;

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, PrepCfg::LOAD_BYTES);
    tc::tma_load_4d(sm + PrepCfg::VT, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PrepCfg::VT + 8192, &tm_v, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PrepCfg::QR, &tm_q, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PrepCfg::KR, &tm_k, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + PrepCfg::LS, &tm_logf, 0, h, t0, b, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 128);
  if (tid < C) {
    const bool ok = tid < nv;
    const size_t g = ((size_t)b * T + t0 + tid) * H + h;
    bs[tid] = ok ? beta[g] : 0.f;
    cs[tid] = ok ? c[g] : 0.f;
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  // decay prefix (thread (j, half) covers 32 positions; L is written back for
  // the exact path) and the tf32 operands K+, Q+, K-
  float mx = 0.f;
  {
    const int j = tid & 127, half = tid >> 7;
    float Lr[32];
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      acc += Ls[(32 * half + i) * D + j];
      Lr[i] = acc;
    }
    if (half == 0) xch[j] = acc;
    __syncthreads();
    const float off = half ? xch[j] : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * half + i;
      const float L = Lr[i] + off;
      mx = fmaxf(mx, fabsf(L));
      Ls[t * D + j] = L;
      const float qq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::QR + (t * D + j) * 2));
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::KR + (t * D + j) * 2));
      const float gm = expf(L), ig = expf(-L);
      *reinterpret_cast<float*>(sm + PrepCfg::AKQ + tc::sw128_off(t, j, 128, 4)) = kk * gm;
      *reinterpret_cast<float*>(sm + PrepCfg::AKQ + tc::sw128_off(64 + t, j, 128, 4)) = qq * gm;
      *reinterpret_cast<float*>(sm + PrepCfg::BKM + tc::sw128_off(t, j, 64, 4)) = kk * ig;
    }
  }
  const bool is_unsafe = __syncthreads_or(!(mx < kSafeLogRange)) != 0;
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    const uint32_t IDT = tc::idesc(128, 64, 2), IDB = tc::idesc(128, 64, 1);
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      const uint32_t kb = ks / 4, w = (ks % 4) * 32;
      tc::mma_tf32_ss(tmem + 0, tc::desc_sw128(tc::smem_u32(sm + PrepCfg::AKQ + kb * 16384 + w)),
                      tc::desc_sw128(tc::smem_u32(sm + PrepCfg::BKM + kb * 8192 + w)), IDT, ks > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t vd = tc::desc_sw128(tc::smem_u32(sm + PrepCfg::VT + (ks / 4) * 8192 + (ks % 4) * 32));
      tc::mma_bf16_ss(tmem + 64, vd, vd, IDB, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  // rows t (TMEM lanes 0..63): N[t][i] = beta_t G_K G_V (i < t); lanes 64+t: P row t
  if (warp < 4) {
    const int row = warp * 32 + lane;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
    if (row < 64) {
      const int t = row;
      const float bt = bs[t];
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float gk[16], gv[16];
        tc::tmem_ld16(lanes + 16 * c16, gk);
        tc::tmem_ld16(lanes + 64 + 16 * c16, gv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int i = 16 * c16 + ii;
          Ns[t * 65 + i] = i < t ? bt * gk[ii] * gv[ii] : 0.f;
        }
      }
    } else if (wP && !is_unsafe) {
      const int t = row - 64;
      float* prow = wP + ch * C * C + t * C;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float pv[16];
        tc::tmem_ld16(lanes + 16 * c16, pv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          float4 o;
          const int i = 16 * c16 + 4 * i4;
          o.x = i <= t ? pv[4 * i4] : 0.f;
          o.y = i + 1 <= t ? pv[4 * i4 + 1] : 0.f;
          o.z = i + 2 <= t ? pv[4 * i4 + 2] : 0.f;
          o.w = i + 3 <= t ? pv[4 * i4 + 3] : 0.f;
          *reinterpret_cast<float4*>(prow + i) = o;
        }
      }
    }
  }
  __syncthreads();
  if (is_unsafe) {
    // exact decay weights e^{L_t - L_i} <= 1 per element (rare: extreme decays)
    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::QR);
    const __nv_bfloat16* ks = reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::KR);
    for (int e = tid; e < C * C; e += 256) {
      const int t = e / C, i = e % C;
      float gk = 0.f, gv = 0.f, pq = 0.f;
      if (i <= t) {
        for (int j = 0; j < D; ++j) {
          const float w = expf(Ls[t * D + j] - Ls[i * D + j]);
          const float ki = __bfloat162float(ks[i * D + j]);
          gk = fmaf(__bfloat162float(ks[t * D + j]) * ki, w, gk);
          pq = fmaf(__bfloat162float(qs[t * D + j]) * ki, w, pq);
        }
        for (int r = 0; r < D; ++r)
          gv = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::VT + tc::sw128_off(t, r, 64, 2))),
                    __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + PrepCfg::VT + tc::sw128_off(i, r, 64, 2))), gv);
      }
      Ns[t * 65 + i] = i < t ? bs[t] * gk * gv : 0.f;
      if (wP) wP[ch * C * C + e] = i <= t ? pq : 0.f;
    }
    __syncthreads();
  }
  // ---- X = (I + N)^{-1}, blocked by 16
  {
    // diagonal blocks: thread (blk, m) solves column m of block blk
    if (tid < 64) {
      const int blk = tid >> 4, m = tid & 15, o = 16 * blk;
      float col[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float s = t == m ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2)
          if (s2 >= m && s2 < t) s = fmaf(-Ns[(o + t) * 65 + o + s2], col[s2], s);
        col[t] = t < m ? 0.f : s;
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) Xs[(o + t) * 65 + o + m] = col[t];
    }
    // zero the strictly upper blocks
    for (int e = tid; e < C * C; e += 256) {
      const int t = e / C, i = e % C;
      if ((i >> 4) > (t >> 4)) Xs[t * 65 + i] = 0.f;
    }
    __syncthreads();
    for (int a = 1; a < 4; ++a) {
      // T_ab = sum_{cb=b}^{a-1} N_{a,cb} X_{cb,b} for b < a (16 x 16 each)
      for (int e = tid; e < a * 256; e += 256) {
        const int bb = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        float s = 0.f;
        for (int kk = 16 * bb; kk < 16 * a; ++kk) s = fmaf(Ns[(16 * a + rr) * 65 + kk], Xs[kk * 65 + 16 * bb + cc], s);
        Ts[bb * 272 + rr * 17 + cc] = s;
      }
      __syncthreads();
      // X_ab = -X_aa T_ab
      for (int e = tid; e < a * 256; e += 256) {
        const int bb = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        float s = 0.f;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) s = fmaf(Xs[(16 * a + rr) * 65 + 16 * a + kk], Ts[bb * 272 + kk * 17 + cc], s);
        Xs[(16 * a + rr) * 65 + 16 * bb + cc] = -s;
      }
      __syncthreads();
    }
  }
  if (tid < C) {
    float s = 0.f;
    for (int m = 0; m <= tid; ++m) s = fmaf(Xs[tid * 65 + m], cs[m], s);
    wy[ch * C + tid] = s;
  }
  for (int e = tid; e < C * C; e += 256) wA[ch * C * C + e] = Xs[(e / C) * 65 + (e % C)];
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// Per-chunk operands of the chain, one CTA per chunk n, all chunks in parallel:
//   K~_n  = k_n o e^{L_n + Lambda_{n-1}}   (B of the chain's lookahead MMA)
//   K^e_n = k_n o e^{Lambda_n - L_n}       (update operand),  gamma_C,n = e^{Lambda_n}
// and, for n >= 1, the cross-chunk matrix of the lookahead
//   H_n = (V_n V_{n-1}^T) o (K+_n K^e_{n-1}^T),   K+_n = k_n o e^{L_n}.
// Every factor is bounded by |k| (the exponents are <= 0), so all chunks take
// this path.  The key Gram runs in tf32, the value Gram in bf16 (exact
// products, fp32 sums).
// ---------------------------------------------------------------------------
struct CrossCfg {
  static constexpr uint32_t KK = 0;        // tf32 per 32-channel K block (16 KB): rows 0-63 K+_n, 64-127 K^e_{n-1}
  static constexpr uint32_t VV = 65536;    // bf16, 2 K blocks x 128 rows: rows 0-63 V_n, 64-127 V_{n-1} (TMA)
  static constexpr uint32_t KR = 98304;    // k_n, k_{n-1} bf16 [64][128] each (TMA)
  static constexpr uint32_t LG = 131072;   // logf_n, then K~_n staged in place; logf_{n-1}, then K^e_n (fp32 [64][128])
  static constexpr uint32_t XCH = 196608;  // Lambda_{n-1} [128]
  static constexpr uint32_t VT = 197632;   // V_n^T bf16 [r][t], 128 rows x 128 B, 128-byte swizzle (staging)
  static constexpr uint32_t BYTES = VT + 16384 + 1024;
  static constexpr uint32_t LOAD_CUR = 16384 + 16384 + 32768, LOAD_PREV = LOAD_CUR;
};

__global__ void __launch_bounds__(256, 1) fwd_cross_tc(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_logf, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_ke, int H, int NC, float* __restrict__ wGC, float* __restrict__ wHx,
    __nv_bfloat16* __restrict__ wVt, int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, tp = t0 - C;
  const bool has_prev = n > 0;
  const size_t ch = blockIdx.x;
  float* xch = reinterpret_cast<float*>(sm + CrossCfg::XCH);
  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, CrossCfg::LOAD_CUR + (has_prev ? CrossCfg::LOAD_PREV : 0u));
    tc::tma_load_4d(sm + CrossCfg::VV, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CrossCfg::VV + 16384, &tm_v, 64, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CrossCfg::KR, &tm_k, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + CrossCfg::LG, &tm_logf, 0, h, t0, b, &ld_bar);
    if (has_prev) {
      tc::tma_load_4d(sm + CrossCfg::VV + 8192, &tm_v, 0, h, tp, b, &ld_bar);
      tc::tma_load_4d(sm + CrossCfg::VV + 24576, &tm_v, 64, h, tp, b, &ld_bar);
      tc::tma_load_4d(sm + CrossCfg::KR + 16384, &tm_k, 0, h, tp, b, &ld_bar);
      tc::tma_load_4d(sm + CrossCfg::LG + 32768, &tm_logf, 0, h, tp, b, &ld_bar);
    }
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 128);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  // half 0: chunk n (channel j); half 1: chunk n-1 (channel j)
  const int j = tid & 127, half = tid >> 7;
  float* lg = reinterpret_cast<float*>(sm + CrossCfg::LG + half * 32768);
  const unsigned char* kr = sm + CrossCfg::KR + half * 16384;
  float tot = 0.f;
  if (half == 0 || has_prev) {
#pragma unroll 8
    for (int t = 0; t < C; ++t) tot += lg[t * D + j];
  }
  if (half) xch[j] = has_prev ? tot : 0.f;
  __syncthreads();
  float Lr[C];
  if (half == 0) {
    // K+_n (Gram operand, tf32) and K~_n (staged in place of logf_n)
    const float lam_prev = xch[j];
    float L = 0.f;
#pragma unroll
    for (int t = 0; t < C; ++t) {
      L += lg[t * D + j];
      Lr[t] = L;
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(kr + (t * D + j) * 2));
      const float kp = kk * expf(L);
      *reinterpret_cast<float*>(sm + CrossCfg::KK + tc::sw128_off(t, j, 128, 4)) = kp;
      lg[t * D + j] = kk * expf(L + lam_prev);
    }
    wGC[ch * D + j] = expf(tot);
  } else if (has_prev) {
    // K^e_{n-1} (Gram operand, tf32)
    float L = 0.f;
#pragma unroll 8
    for (int t = 0; t < C; ++t) {
      L += lg[t * D + j];
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(kr + (t * D + j) * 2));
      *reinterpret_cast<float*>(sm + CrossCfg::KK + tc::sw128_off(64 + t, j, 128, 4)) = kk * expf(tot - L);
    }
  }
  // V_n^T as the K-major tile [r][t] the chain's column dot and update MMA read
  {
    const int r = tid & 127, tb = 32 * (tid >> 7);
#pragma unroll
    for (int g8 = 0; g8 < 32; g8 += 8) {
      __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        v8[i] = *reinterpret_cast<const __nv_bfloat16*>(sm + CrossCfg::VV + tc::sw128_off(tb + g8 + i, r, 128, 2));
      *reinterpret_cast<uint4*>(sm + CrossCfg::VT + tc::sw128_off(r, tb + g8, 128, 2)) =
          *reinterpret_cast<const uint4*>(v8);
    }
  }
  __syncthreads();  // logf_{n-1} is dead: K^e_n goes there
  if (half == 0) {
    float* ke = reinterpret_cast<float*>(sm + CrossCfg::LG + 32768);
#pragma unroll
    for (int t = 0; t < C; ++t) {
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(kr + (t * D + j) * 2));
      ke[t * D + j] = kk * expf(tot - Lr[t]);
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    tc::tma_store_4d(&tm_kt, sm + CrossCfg::LG, 0, h, t0, b);
    tc::tma_store_4d(&tm_ke, sm + CrossCfg::LG + 32768, 0, h, t0, b);
    tc::bulk_s2g(wVt + ch * (D * C), sm + CrossCfg::VT, 16384u);
    tc::bulk_commit();
    if (has_prev) {
      const uint32_t IDT = tc::idesc(128, 64, 2), IDB = tc::idesc(128, 64, 1);
      // cols 0-63, lanes 0-63: K+_n K^e_{n-1}^T
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
        tc::mma_tf32_ss(tmem + 0, tc::desc_sw128(tc::smem_u32(sm + CrossCfg::KK + o)),
                        tc::desc_sw128(tc::smem_u32(sm + CrossCfg::KK + o + 8192)), IDT, ks > 0 ? 1u : 0u);
      }
      // cols 64-127, lanes 0-63: V_n V_{n-1}^T
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t o = (ks / 4) * 16384 + (ks % 4) * 32;
        tc::mma_bf16_ss(tmem + 64, tc::desc_sw128(tc::smem_u32(sm + CrossCfg::VV + o)),
                        tc::desc_sw128(tc::smem_u32(sm + CrossCfg::VV + o + 8192)), IDB, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(&mma_bar);
    }
  }
  if (has_prev) {
    tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
    tc::tc_after_sync();
    if (warp < 2) {
      const int t = warp * 32 + lane;
      const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
      float* hrow = wHx + ch * C * C + t * C;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float gk[16], gv[16];
        tc::tmem_ld16(lanes + 16 * c16, gk);
        tc::tmem_ld16(lanes + 64 + 16 * c16, gv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4)
          *reinterpret_cast<float4*>(hrow + 16 * c16 + 4 * i4) =
              make_float4(gk[4 * i4] * gv[4 * i4], gk[4 * i4 + 1] * gv[4 * i4 + 1], gk[4 * i4 + 2] * gv[4 * i4 + 2],
                          gk[4 * i4 + 3] * gv[4 * i4 + 3]);
      }
    }
  }
  if (tid == 0) tc::bulk_wait_read();
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

template <int R>
cudaError_t launch_chain(const FwdArgs& a, const float* wy, const float* wA, float* blob, float* wu,
                         float* wb0, int* err, cudaStream_t st) {
  const Layout& L = a.L;
  constexpr int NJ = ChainCfg<R>::NJ;
  CUtensorMap tm_v, tm_kt, tm_ke;
  if (!make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
      !make_tmap_bthd(&tm_kt, ws_ptr<float>(a.ws, L.Kt), 4, L.B, L.T, L.H, D, 32, true) ||
      !make_tmap_bthd(&tm_ke, ws_ptr<float>(a.ws, L.Ke), 4, L.B, L.T, L.H, D, NJ, false))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ChainCfg<R>::BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.B * L.H * R);
  cfg.blockDim = dim3(288);
  cfg.dynamicSmemBytes = ChainCfg<R>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(st, "fwd_chain_tc");
  __nv_bfloat16* s0b = a.save ? ws_ptr<__nv_bfloat16>(a.ws, L.S0b) : nullptr;
  e = cudaLaunchKernelEx(&cfg, fwd_chain_tc<R>, tm_v, tm_kt, tm_ke, a.beta, a.S0, a.ST, L.H, L.T, L.NC, wy, wA,
                         (const float*)ws_ptr<float>(a.ws, L.Hx), (const float*)ws_ptr<float>(a.ws, L.GC),
                         (const __nv_bfloat16*)ws_ptr<__nv_bfloat16>(a.ws, L.Vt), blob, wu, wb0, s0b, err);
  prof_end(st);
  return e;
}

}  // namespace

template <int R>
static int max_active_clusters() {
  if (cudaFuncSetAttribute(fwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ChainCfg<R>::BYTES) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(R * 1024);
  cfg.blockDim = dim3(288);
  cfg.dynamicSmemBytes = ChainCfg<R>::BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fwd_chain_tc<R>, &cfg) != cudaSuccess) return 0;
  return n;
}

// Largest cluster (8 or 4 CTAs per head) for which every head's cluster is
// resident at once; 4 when none is.
int choose_cluster(int units, int sms) {
  (void)sms;
  static int cap8 = -1, cap4 = -1;  // per process; the library targets one GPU model
  if (cap8 < 0) cap8 = max_active_clusters<8>();
  if (cap4 < 0) cap4 = max_active_clusters<4>();
  if (units <= cap8) return 8;
  return 4;
}

cudaError_t launch_fwd_tc(const FwdArgs& a, int* err, int sms, cudaStream_t st) {
  const Layout& L = a.L;
  cudaError_t e;
  if (a.phases & kPhaseLocal) {
    CUtensorMap tm_v, tm_q, tm_k, tm_logf;
    if (!make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
        !make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_logf, a.logf, 4, L.B, L.T, L.H, D, 128, false))
      return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(fwd_prep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)PrepCfg::BYTES)) != cudaSuccess)
      return e;
    prof_begin(st, "fwd_prep_tc");
    fwd_prep_tc<<<(unsigned)L.chunks, 256, PrepCfg::BYTES, st>>>(
        tm_v, tm_q, tm_k, tm_logf, a.beta, a.c, L.H, L.T, L.NC, ws_ptr<float>(a.ws, L.y), ws_ptr<float>(a.ws, L.A),
        a.save ? ws_ptr<float>(a.ws, L.P) : nullptr, err);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap tm_kt, tm_ke;
    if (!make_tmap_bthd(&tm_kt, ws_ptr<float>(a.ws, L.Kt), 4, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_ke, ws_ptr<float>(a.ws, L.Ke), 4, L.B, L.T, L.H, D, 128, false))
      return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(fwd_cross_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)CrossCfg::BYTES)) != cudaSuccess)
      return e;
    prof_begin(st, "fwd_cross_tc");
    fwd_cross_tc<<<(unsigned)L.chunks, 256, CrossCfg::BYTES, st>>>(
        tm_v, tm_k, tm_logf, tm_kt, tm_ke, L.H, L.NC, ws_ptr<float>(a.ws, L.GC), ws_ptr<float>(a.ws, L.Hx),
        ws_ptr<__nv_bfloat16>(a.ws, L.Vt), err);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!(a.phases & kPhaseCarry)) return cudaSuccess;
  const float* wy = ws_ptr<float>(a.ws, L.y);
  const float* wA = ws_ptr<float>(a.ws, L.A);
  float* blob = ws_ptr<float>(a.ws, L.S0);
  float* wu = ws_ptr<float>(a.ws, L.u);
  float* wb0 = ws_ptr<float>(a.ws, L.b0);
  int* flags = ws_ptr<int>(a.ws, L.flags);
  const int R = choose_cluster(L.B * L.H, sms);
  if (R == 8) e = launch_chain<8>(a, wy, wA, blob, wu, wb0, err, st);
  else e = launch_chain<4>(a, wy, wA, blob, wu, wb0, err, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(fwd_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)OutCfg::BYTES)) != cudaSuccess)
    return e;
  {
    CUtensorMap tm_q, tm_k, tm_v, tm_logf, tm_out;
    if (!make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 64, true) ||
        !make_tmap_bthd(&tm_logf, a.logf, 4, L.B, L.T, L.H, D, 128, false) ||
        !make_tmap_bthd(&tm_out, a.out, 2, L.B, L.T, L.H, D, 64, true))
      return cudaErrorInvalidValue;
    prof_begin(st, "fwd_out_tc");
    fwd_out_tc<<<(unsigned)L.chunks, 256, OutCfg::BYTES, st>>>(tm_q, tm_k, tm_v, tm_logf, tm_out, L.H, L.NC, blob,
                                                               wu, flags, err);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  constexpr int kFixSmem = (3 * C * (D + 1) + C) * 4;
  if ((e = cudaFuncSetAttribute(fwd_out_fixup, cudaFuncAttributeMaxDynamicSharedMemorySize, kFixSmem)) !=
      cudaSuccess)
    return e;
  prof_begin(st, "fwd_out_fixup");
  fwd_out_fixup<<<(unsigned)L.chunks, 128, kFixSmem, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.logf, L.H, L.T, L.NC, blob, wu, flags,
      static_cast<__nv_bfloat16*>(a.out));
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
