// kd_fchain_tc.cu -- the forward's sequential chunk chain on tensor cores
// (bf16 q, k, v and d_k = d_v = 128).
//
// Chunk form (KronLSTM digest, "무엇과 다른가": the DeltaNet chunk-parallel
// scheme applies; Gated DeltaNet-2 article, "기술 상세": C = 64, WY form).
// With S_n the state at the start of chunk n, K~_n = K+_n diag(gamma_C of
// chunk n-1) and the cross-chunk matrix H_n = (V_n V_{n-1}^T) o (K+_n K^e_{n-1}^T)
// (both built in parallel by fwd_cross_tc), the erase read of chunk n splits
// into a part that needs only the state one chunk earlier and a correction
// linear in the previous chunk's write coefficients:
//   c_n  = rowdot(V_n S_{n-1}, K~_n)             (one-chunk lookahead)
//   b0_n = c_n + H_n u_{n-1}
//   u_n  = y_n - A_n (beta_n o b0_n)
//   S_{n+1} = S_n diag(gamma_C,n) + V_n^T diag(u_n) K^e_n.
// Two loops run through the chain:
//   short: u_{n-1} -> u_n, two 64 x 64 matrix-vector products (CUDA cores);
//   long:  u_n -> update MMA -> S_{n+1} -> lookahead MMA U = V_{n+2} S_{n+1}
//          and the row dot with K~ -> cluster all-reduce -> c_{n+2} -> u_{n+2},
//          spanning two chunks.
// Each loop runs on its own warps, so the two overlap.  The lookahead MMA
// contracts over the state's rows (value channels), so each lane of its
// accumulator holds one position's partial sum over this CTA's key channels:
// the column dot is a per-lane dot product, with no reduction across lanes.
//
// One thread-block cluster of R CTAs per (b, h); CTA c owns the key-channel
// slice J_c (128 / R channels) of the state: row r of the slice lives in the
// registers of state thread r, in fp32.  Its bf16 high and low parts are also
// kept in shared memory as the lookahead MMA's B operand (MN-major: row r
// holds the slice's channels).
// Warp roles (320 threads):
//   warps 0-3  u warps: b0, u (every CTA computes the same u from the
//              all-reduced c), the update operand diag(u) K^e in bf16 hi + lo.
//   warps 4-7  state warps (thread r = state row r = tensor-memory lane r):
//              the state update S <- S diag(gamma) + dS, its bf16 operand
//              copy, the save of each chunk-start state (a bf16 tile for the
//              output kernel and the backward; an fp32 copy as well for chunks
//              bound for the exact paths); warps 4-5 (lanes = positions) the
//              row dot of the lookahead and the send of its partial sums to
//              every CTA of the cluster.
//   warp 8     issuer: one thread issues every tcgen05 MMA.
//   warp 9     producer: bulk / TMA loads of each chunk's operands (a ring of
//              three slots) and of the u recursion's matrices (a ring of two).
// Every wait is bounded; on expiry the kernel records a timeout in the
// library's error word, lets every loop run out without waiting, then drains
// its own copies and MMAs in flight before freeing tensor memory.
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;
// Chunks ahead of the shared-memory rings whose operands the producer pulls
// into L2, so that the ring's own copies are L2 hits.
constexpr int kL2Ahead = 3;

template <int R>
struct FcCfg {
  static constexpr int NJ = D / R;  // key channels per CTA
  // tensor memory: the lookahead accumulators U [2] and the update accumulators [2], NJ columns each
  static constexpr int U_COL = 0, D2_COL = 2 * NJ;
  static constexpr uint32_t TMEM_COLS = (4 * NJ) <= 64 ? 64u : 128u;
  static constexpr uint32_t up1k(uint32_t x) { return (x + 1023u) / 1024u * 1024u; }
  // chunk operand ring (3 slots), written by bulk copies / TMA
  static constexpr int NSLOT = 3;
  static constexpr uint32_t SL_V = 0;                     // V^T bf16 [r][t], 128-byte swizzle (16 KB)
  static constexpr uint32_t SL_KT = 16384;                // K~, the 32-channel block holding this CTA's
                                                          //   channels, fp32 [64][32], 128-byte swizzle (8 KB)
  static constexpr uint32_t SL_KE = SL_KT + 8192;         // K^e slice fp32 [64][NJ]
  static constexpr uint32_t SL_GC = SL_KE + 64 * NJ * 4;  // gamma_C slice [NJ]
  static constexpr uint32_t SL_SZ = up1k(SL_GC + NJ * 4);
  static constexpr uint32_t LOAD_BYTES = 16384 + 8192 + 64 * NJ * 4 + NJ * 4;
  // u-recursion ring (2 slots): A [64][64], H [64][64], y [64], beta [64]
  static constexpr uint32_t AUX = NSLOT * SL_SZ;
  static constexpr uint32_t AX_A = 0, AX_H = 16384, AX_Y = 32768, AX_B = 32768 + 256;
  static constexpr uint32_t AUX_SZ = up1k(AX_B + 256);
  // update operand diag(u) K^e slice [2 buffers][hi, lo][NJ rows x 128 B]
  static constexpr uint32_t B2 = AUX + 2 * AUX_SZ;
  static constexpr uint32_t B2_SZ = 2 * NJ * 128;
  // the state slice's bf16 high / low parts, MN-major B operand [r][j] (128 rows x 128 B each)
  static constexpr uint32_t SC = B2 + 2 * B2_SZ;
  static constexpr uint32_t SM = SC + 2 * 16384;
  static constexpr uint32_t SM_RECV = SM;                        // c partials [4][R][64]
  static constexpr uint32_t SM_US = SM_RECV + 4 * R * 64 * 4;    // u [2][64]
  static constexpr uint32_t SM_WS = SM_US + 2 * 64 * 4;          // beta o b0 [64]
  static constexpr uint32_t SM_END = SM_WS + 64 * 4;
  static constexpr uint32_t BYTES = SM_END + 1024;  // + alignment slack
};

// Writes 16 state values (row r, columns j..j+15) of one chunk into the bf16
// tile the output kernel and the backward read: [r][j] (rows r, K = j),
// 128-byte-swizzled K-major, 32 KB per chunk.
__device__ __forceinline__ void save_bf16_tile(__nv_bfloat16* rj, size_t ch, int r, int j, const float* x) {
  unsigned char* a = reinterpret_cast<unsigned char*>(rj + ch * D * D);
#pragma unroll
  for (int h8 = 0; h8 < 2; ++h8) {
    __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v8[i] = __float2bfloat16_rn(x[8 * h8 + i]);
    *reinterpret_cast<uint4*>(a + tc::sw128_off(r, j + 8 * h8, 128, 2)) = *reinterpret_cast<const uint4*>(v8);
  }
}
// The same 16 values into the fp32 copy the exact paths read (128-byte-swizzled
// K-major, [r][j], 64 KB per chunk).
__device__ __forceinline__ void save_f32_tile(float* blob, size_t ch, int r, int j, const float* x) {
  unsigned char* a = reinterpret_cast<unsigned char*>(blob + ch * D * D);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
    *reinterpret_cast<float4*>(a + tc::sw128_off(r, j + 4 * q4, 128, 4)) =
        make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
}

// named barriers: 1 = the u warps, 2 = the state warps (128 threads each)
__device__ __forceinline__ void bar_u() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void bar_s() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(b)) : "memory");
}
// Bounded wait that ignores the abort flag: used only to drain copies and
// MMAs this CTA issued itself before it frees tensor memory and exits.
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  int dummy_abort = 0;
  tc::mbar_wait<false>(b, parity, nullptr, 0, &dummy_abort);
}

template <int R>
__global__ void __launch_bounds__(320, 1) fwd_chain_tc(
    const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_ke,
    const float* __restrict__ beta, const float* __restrict__ S0, float* __restrict__ ST, int H, int T, int NC,
    const float* __restrict__ wy, const float* __restrict__ wA, const float* __restrict__ wHx,
    const float* __restrict__ wGC, const __nv_bfloat16* __restrict__ wVt, const int* __restrict__ wxflags,
    float* __restrict__ wS0blob, float* __restrict__ wu, float* __restrict__ wb0, __nv_bfloat16* __restrict__ wS0b,
    int* __restrict__ err) {
  using Cf = FcCfg<R>;
  constexpr int NJ = Cf::NJ;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t slot_full[3], slot_free[3], aux_full[2], aux_free[2], x_bar[4], b2_full[2], mma1_bar[2],
      mma2_bar[2], s_ready, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_rank();
  const int unit = blockIdx.x / R;  // (b, h)
  const int b = unit / H, h = unit % H;
  const int j0 = static_cast<int>(rank) * NJ;
  const int jb = j0 & ~31;  // first channel of the 32-channel K~ block

  float* recv = reinterpret_cast<float*>(sm + Cf::SM_RECV);
  float* us = reinterpret_cast<float*>(sm + Cf::SM_US);
  float* ws = reinterpret_cast<float*>(sm + Cf::SM_WS);
  auto slot = [&](int m) { return sm + (m % 3) * Cf::SL_SZ; };
  auto auxp = [&](int m) { return sm + Cf::AUX + (m & 1) * Cf::AUX_SZ; };

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) {
      tc::mbar_init(&slot_full[i], 1);
      tc::mbar_init(&slot_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux_full[i], 2);  // the copies' expect_tx arrival + the beta lanes' arrival
      tc::mbar_init(&aux_free[i], 1);
      tc::mbar_init(&b2_full[i], 128);
      tc::mbar_init(&mma1_bar[i], 1);
      tc::mbar_init(&mma2_bar[i], 1);
    }
    for (int i = 0; i < 4; ++i) tc::mbar_init(&x_bar[i], 1);
    tc::mbar_init(&s_ready, 1);
    tc::mbar_init(&drain_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, Cf::TMEM_COLS);
  tc::tc_before_sync();
  __syncthreads();
  // arm the all-reduce barriers of chunks 0..3 before any peer can send
  if (tid == 0)
    for (int i = 0; i < 4 && i < NC; ++i) tc::mbar_expect_tx(&x_bar[i], R * 64u * 4u);
  __syncthreads();
  tc::cluster_sync();  // peers' barriers are initialised and armed before any remote arrive
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp < 4) {
    // ================================ u warps ================================
    // two threads per position t, each half of the 64 columns; float4 reads
    // rotated by thread so the 8 threads of a quarter-warp hit distinct banks
    const int t = tid >> 1, half = tid & 1;
    // Waits that are normally complete long before they are reached are taken
    // one chunk early, off the u -> u step: chunk n's matrices and operand
    // slot, and the update operand buffer (read by the update MMA of chunk n-2).
    auto early_waits = [&](int n) {
      tc::mbar_wait<false>(&aux_full[n & 1], (uint32_t)((n >> 1) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::mbar_wait<false>(&slot_full[n % 3], (uint32_t)((n / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      if (n >= 2)
        tc::mbar_wait<false>(&mma2_bar[n & 1], (uint32_t)(((n - 2) >> 1) & 1), err, tc::kErrTimeoutMma,
                             &abort_flag);
    };
    early_waits(0);
    for (int n = 0; n < NC; ++n) {
      const size_t ch = (size_t)unit * NC + n;
      const int xs = n & 3;
      tc::mbar_wait<true>(&x_bar[xs], (uint32_t)((n >> 2) & 1), err, tc::kErrTimeoutCluster, &abort_flag);
      const unsigned char* ax = auxp(n);
      float s = 0.f;
      {
        const float* rv = recv + xs * R * 64;
#pragma unroll
        for (int c2 = 0; c2 < R; ++c2) s += rv[c2 * 64 + t];
      }
      if (n > 0) {
        const float* Hrow = reinterpret_cast<const float*>(ax + Cf::AX_H) + t * 64 + 32 * half;
        const float* uh = us + ((n - 1) & 1) * 64 + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int ci = (i + tid) & 7;
          const float4 hv = *reinterpret_cast<const float4*>(Hrow + 4 * ci);
          const float4 uv = *reinterpret_cast<const float4*>(uh + 4 * ci);
          a0 = fmaf(hv.x, uv.x, a0);
          a1 = fmaf(hv.y, uv.y, a1);
          a2 = fmaf(hv.z, uv.z, a2);
          a3 = fmaf(hv.w, uv.w, a3);
        }
        float hu = (a0 + a1) + (a2 + a3);
        hu += __shfl_xor_sync(0xffffffffu, hu, 1);
        s += hu;
      }
      // s = b0_n[t] in both threads of the pair
      if (half == 0) ws[t] = reinterpret_cast<const float*>(ax + Cf::AX_B)[t] * s;
      bar_u();  // every thread has read recv[xs]: arm it for chunk n + 4
      if (tid == 0 && n + 4 < NC) tc::mbar_expect_tx(&x_bar[xs], R * 64u * 4u);
      float uval;
      {
        const float* Arow = reinterpret_cast<const float*>(ax + Cf::AX_A) + t * 64 + 32 * half;
        const float* wh = ws + 32 * half;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int ci = (i + tid) & 7;
          const float4 av = *reinterpret_cast<const float4*>(Arow + 4 * ci);
          const float4 wv = *reinterpret_cast<const float4*>(wh + 4 * ci);
          a0 = fmaf(av.x, wv.x, a0);
          a1 = fmaf(av.y, wv.y, a1);
          a2 = fmaf(av.z, wv.z, a2);
          a3 = fmaf(av.w, wv.w, a3);
        }
        float aw = (a0 + a1) + (a2 + a3);
        aw += __shfl_xor_sync(0xffffffffu, aw, 1);
        uval = reinterpret_cast<const float*>(ax + Cf::AX_Y)[t] - aw;
      }
      float* un = us + (n & 1) * 64;
      if (half == 0) un[t] = uval;
      bar_u();
      if (tid == 0) mbar_arrive(&aux_free[n & 1]);
      // ---- B2 = diag(u_n) K^e_n slice as bf16 hi + lo (N = NJ rows j, K = 64 positions)
      {
        constexpr int TQ = 128 / NJ, TPT = C / TQ;  // position groups, positions per thread
        const int jl = tid % NJ, tq = tid / NJ;
        const float* KE = reinterpret_cast<const float*>(slot(n) + Cf::SL_KE);
        unsigned char* b2 = sm + Cf::B2 + (n & 1) * Cf::B2_SZ;
#pragma unroll
        for (int g8 = 0; g8 < TPT; g8 += 8) {
          __align__(16) __nv_bfloat16 hi8[8], lo8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int tt = tq * TPT + g8 + i;
            const float x = un[tt] * KE[tt * NJ + jl];
            hi8[i] = __float2bfloat16_rn(x);
            lo8[i] = __float2bfloat16_rn(x - __bfloat162float(hi8[i]));
          }
          const uint32_t off = tc::sw128_off(jl, tq * TPT + g8, NJ, 2);
          *reinterpret_cast<uint4*>(b2 + off) = *reinterpret_cast<const uint4*>(hi8);
          *reinterpret_cast<uint4*>(b2 + NJ * 128 + off) = *reinterpret_cast<const uint4*>(lo8);
        }
      }
      tc::fence_proxy_async();
      mbar_arrive(&b2_full[n & 1]);
      // the chain's outputs for the backward, off the step: u_n and b0_n
      if (rank == 0 && half == 0) {
        if (wu) wu[ch * C + t] = uval;
        if (wb0) wb0[ch * C + t] = s;
      }
      if (n + 1 < NC) early_waits(n + 1);
    }
    // drain: every peer sends all NC partial sums; wait for the last round of
    // each buffer so no peer still writes here once this CTA exits
    if (tid == 0)
      for (int m = NC - 1; m >= 0 && m >= NC - 4; --m) mbar_drain(&x_bar[m & 3], (uint32_t)((m >> 2) & 1));
  } else if (warp < 8) {
    // ============================== state warps ==============================
    const int r = tid - 128;  // state row = tensor-memory lane (lookahead rows: positions)
    const uint32_t my_lanes = tc::tmem_lane_addr(tmem, warp, 0);
    float sreg[NJ];           // row r of the state slice
    float kt[NJ];             // warps 4-5: row t = r of the next chunk's K~ slice
    // the state slice's bf16 parts into the lookahead MMA's operand, row r
    auto write_operand = [&]() {
      unsigned char* sc = sm + Cf::SC;
#pragma unroll
      for (int j8 = 0; j8 < NJ; j8 += 8) {
        __align__(16) __nv_bfloat16 hi8[8], lo8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hi8[i] = __float2bfloat16_rn(sreg[j8 + i]);
          lo8[i] = __float2bfloat16_rn(sreg[j8 + i] - __bfloat162float(hi8[i]));
        }
        const uint32_t off = tc::sw128_off(r, j8, 128, 2);
        *reinterpret_cast<uint4*>(sc + off) = *reinterpret_cast<const uint4*>(hi8);
        *reinterpret_cast<uint4*>(sc + 16384 + off) = *reinterpret_cast<const uint4*>(lo8);
      }
    };
    // warps 4-5: chunk m's K~ row into registers (overlapping the wait for its
    // MMA); the swizzled block spreads a quarter-warp's 16-byte reads over all banks
    auto load_kt = [&](int m) {
      tc::mbar_wait<false>(&slot_full[m % 3], (uint32_t)((m / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      const unsigned char* kb = slot(m) + Cf::SL_KT;
#pragma unroll
      for (int q = 0; q < NJ / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(kb + tc::sw128_off(r, j0 - jb + 4 * q, 64, 4));
        kt[4 * q] = v.x;
        kt[4 * q + 1] = v.y;
        kt[4 * q + 2] = v.z;
        kt[4 * q + 3] = v.w;
      }
    };
    // warps 4-5: c_m partial for position t = r: sum over this CTA's channels of
    // U[t, j] K~[t, j], sent to every CTA of the cluster
    auto row_dot_send = [&](int m) {
      load_kt(m);
      tc::mbar_wait<false>(&mma1_bar[m & 1], (uint32_t)((m >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      float c0 = 0.f, c1 = 0.f;
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float u16[16];
        tc::tmem_ld16(my_lanes + Cf::U_COL + (m & 1) * NJ + jj, u16);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          c0 = fmaf(u16[i], kt[jj + i], c0);
          c1 = fmaf(u16[i + 1], kt[jj + i + 1], c1);
        }
      }
      const float c = c0 + c1;
      float* rv = recv + (m & 3) * R * 64;
      const uint32_t la = tc::smem_u32(rv + rank * 64 + r), lb = tc::smem_u32(&x_bar[m & 3]);
#pragma unroll
      for (int peer = 0; peer < R; ++peer)
        tc::st_async_f32(tc::mapa(la, (uint32_t)peer), c, tc::mapa(lb, (uint32_t)peer));
    };
    const bool dots = warp < 6;  // lanes 0-63 of the lookahead accumulator are the positions
    // the initial state: registers and the operand copy (chunk 0's start state)
    {
#pragma unroll
      for (int j = 0; j < NJ; j += 4) {
        const float4 v = S0 ? *reinterpret_cast<const float4*>(S0 + (size_t)unit * D * D + (size_t)r * D + j0 + j)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x;
        sreg[j + 1] = v.y;
        sreg[j + 2] = v.z;
        sreg[j + 3] = v.w;
      }
      write_operand();
      tc::fence_proxy_async();
      bar_s();
      if (r == 0) mbar_arrive(&s_ready);
      const size_t ch0 = (size_t)unit * NC;
      const bool f32copy = wxflags[ch0] != 0;
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        save_bf16_tile(wS0b, ch0, r, j0 + jj, sreg + jj);
        if (f32copy) save_f32_tile(wS0blob, ch0, r, j0 + jj, sreg + jj);
      }
    }
    if (dots) {
      row_dot_send(0);
      if (NC > 1) row_dot_send(1);
    }
    for (int n = 0; n < NC; ++n) {
      const float* gC = reinterpret_cast<const float*>(slot(n) + Cf::SL_GC);
      tc::mbar_wait<false>(&mma2_bar[n & 1], (uint32_t)((n >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      // ---- S_{n+1} = S_n diag(gamma_C) + dS_n
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 16) {
        float d2[16];
        tc::tmem_ld16(my_lanes + Cf::D2_COL + (n & 1) * NJ + jj, d2);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) sreg[jj + i] = fmaf(sreg[jj + i], gC[jj + i], d2[i]);
      }
      if (n + 2 < NC) write_operand();  // read by the lookahead MMA of chunk n + 2
      tc::fence_proxy_async();
      tc::tc_before_sync();
      bar_s();
      if (r == 0) {
        mbar_arrive(&slot_free[n % 3]);
        mbar_arrive(&s_ready);
      }
      // ---- c_{n+2}
      if (dots && n + 2 < NC) row_dot_send(n + 2);
      // ---- saved as chunk n+1's start state (or S_T), off the step
      if (n + 1 < NC) {
        const size_t chn = (size_t)unit * NC + n + 1;
        const bool f32copy = wxflags[chn] != 0;
#pragma unroll
        for (int jj = 0; jj < NJ; jj += 16) {
          save_bf16_tile(wS0b, chn, r, j0 + jj, sreg + jj);
          if (f32copy) save_f32_tile(wS0blob, chn, r, j0 + jj, sreg + jj);
        }
      } else if (ST) {
#pragma unroll
        for (int j = 0; j < NJ; j += 4)
          *reinterpret_cast<float4*>(ST + (size_t)unit * D * D + (size_t)r * D + j0 + j) =
              make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
      }
    }
  } else if (warp == 8) {
    // ================================ issuer ================================
    // lookahead U_m = V_m S_{m-1}^T: A = V^T read MN-major (M = 128 positions,
    // rows 64-127 are unused), B = the state operand read MN-major (N = NJ
    // channels), K = 128 value channels, hi and lo parts
    const uint32_t IDU = tc::idesc(128, NJ, 1) | tc::kMajorA | tc::kMajorB;
    const uint32_t ID2 = tc::idesc(128, NJ, 1);  // bf16: M = 128 rows r, N = NJ channels, both K-major
    auto issue_u = [&](int m) {
      tc::mbar_wait<false>(&slot_full[m % 3], (uint32_t)((m / 3) & 1), err, tc::kErrTimeoutLoad, &abort_flag);
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* vt = slot(m) + Cf::SL_V;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // second 64-position block of A: the next 16 KB of the slot (in bounds, results unused)
          const uint64_t ad = tc::desc_sw128_mn(tc::smem_u32(vt + ks * 2048), 16384u);
          tc::mma_bf16_ss(tmem + Cf::U_COL + (m & 1) * NJ, ad,
                          tc::desc_sw128_mn(tc::smem_u32(sm + Cf::SC + ks * 2048), 16384u), IDU, ks > 0 ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::U_COL + (m & 1) * NJ, ad,
                          tc::desc_sw128_mn(tc::smem_u32(sm + Cf::SC + 16384 + ks * 2048), 16384u), IDU, 1u);
        }
        tc::mma_commit(&mma1_bar[m & 1]);
      }
      __syncwarp();
    };
    tc::mbar_wait<false>(&s_ready, 0u, err, tc::kErrTimeoutMma, &abort_flag);  // S_0's operand
    tc::tc_after_sync();
    issue_u(0);
    if (NC > 1) issue_u(1);
    for (int n = 0; n < NC; ++n) {
      if (n >= 1 && n + 1 < NC) {
        tc::mbar_wait<false>(&s_ready, (uint32_t)(n & 1), err, tc::kErrTimeoutMma, &abort_flag);  // S_n
        tc::tc_after_sync();
        issue_u(n + 1);
      }
      tc::mbar_wait<false>(&b2_full[n & 1], (uint32_t)((n >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      if (lane == 0) {
        const unsigned char* st = slot(n);
        const unsigned char* b2 = sm + Cf::B2 + (n & 1) * Cf::B2_SZ;
        // dS = V_n^T (B2hi + B2lo)^T  (M = 128 rows r, N = NJ, K = 64 positions)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::desc_sw128(tc::smem_u32(st + Cf::SL_V + ks * 32));
          tc::mma_bf16_ss(tmem + Cf::D2_COL + (n & 1) * NJ, ad, tc::desc_sw128(tc::smem_u32(b2 + ks * 32)), ID2,
                          ks > 0 ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::D2_COL + (n & 1) * NJ, ad,
                          tc::desc_sw128(tc::smem_u32(b2 + NJ * 128 + ks * 32)), ID2, 1u);
        }
        tc::mma_commit(&mma2_bar[n & 1]);
      }
      __syncwarp();
    }
    // drain: every MMA issued above has completed before tensor memory is freed
    if (lane == 0) tc::mma_commit(&drain_bar);
    __syncwarp();
    mbar_drain(&drain_bar, 0u);
  } else {
    // =============================== producer ===============================
    auto main_load = [&](int m) {
      unsigned char* st = slot(m);
      const int si = m % 3;
      if (m >= 3)
        tc::mbar_wait<false>(&slot_free[si], (uint32_t)((m / 3 - 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      if (lane == 0) {
        uint64_t* bar = &slot_full[si];
        const size_t ch = (size_t)unit * NC + m;
        tc::fence_proxy_async();
        tc::mbar_expect_tx(bar, Cf::LOAD_BYTES);
        tc::bulk_g2s(st + Cf::SL_V, wVt + ch * (D * C), 16384u, bar);
        tc::tma_load_4d(st + Cf::SL_KT, &tm_kt, jb, h, m * C, b, bar);
        tc::tma_load_4d(st + Cf::SL_KE, &tm_ke, j0, h, m * C, b, bar);
        tc::bulk_g2s(st + Cf::SL_GC, wGC + ch * D + j0, NJ * 4u, bar);
        const int mp = m + kL2Ahead;
        if (mp < NC) {
          tc::prefetch_l2(wVt + (ch + kL2Ahead) * (D * C), 16384u);
          tc::tma_prefetch_l2_4d(&tm_kt, jb, h, mp * C, b);
          tc::tma_prefetch_l2_4d(&tm_ke, j0, h, mp * C, b);
        }
      }
      __syncwarp();
    };
    auto aux_load = [&](int m) {
      const int ai = m & 1;
      if (m >= 2)
        tc::mbar_wait<false>(&aux_free[ai], (uint32_t)(((m - 2) >> 1) & 1), err, tc::kErrTimeoutMma, &abort_flag);
      unsigned char* ax = auxp(m);
      const size_t ch = (size_t)unit * NC + m;
      if (lane == 0) {
        tc::fence_proxy_async();
        tc::mbar_expect_tx(&aux_full[ai], m >= 1 ? 33024u : 16640u);
        tc::bulk_g2s(ax + Cf::AX_A, wA + ch * C * C, 16384u, &aux_full[ai]);
        if (m >= 1) tc::bulk_g2s(ax + Cf::AX_H, wHx + ch * C * C, 16384u, &aux_full[ai]);
        tc::bulk_g2s(ax + Cf::AX_Y, wy + ch * C, 256u, &aux_full[ai]);
        if (m + kL2Ahead < NC) {
          tc::prefetch_l2(wA + (ch + kL2Ahead) * C * C, 16384u);
          tc::prefetch_l2(wHx + (ch + kL2Ahead) * C * C, 16384u);
        }
      }
      float* bs = reinterpret_cast<float*>(ax + Cf::AX_B);
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int p = lane + 32 * k2;
        bs[p] = (m * C + p < T) ? beta[((size_t)b * T + m * C + p) * H + h] : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&aux_full[ai]);
      __syncwarp();
    };
    for (int m = 0; m < 3 && m < NC; ++m) main_load(m);
    for (int m = 0; m < 2 && m < NC; ++m) aux_load(m);
    for (int m = 0; m < NC; ++m) {
      if (m + 2 < NC) aux_load(m + 2);
      if (m + 3 < NC) main_load(m + 3);
    }
    // drain: the last load issued into every slot has landed
    if (lane == 0) {
      for (int m = NC - 1; m >= 0 && m >= NC - 3; --m) mbar_drain(&slot_full[m % 3], (uint32_t)((m / 3) & 1));
      for (int m = NC - 1; m >= 0 && m >= NC - 2; --m) mbar_drain(&aux_full[m & 1], (uint32_t)((m >> 1) & 1));
    }
    __syncwarp();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::cluster_sync();  // no peer still writes into this CTA's shared memory
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
}

template <int R>
cudaError_t launch_chain_r(const FwdArgs& a, int* err, cudaStream_t st) {
  const Layout& L = a.L;
  constexpr int NJ = FcCfg<R>::NJ;
  CUtensorMap tm_kt, tm_ke;
  if (!make_tmap_bthd(&tm_kt, ws_ptr<float>(a.ws, L.Kt), 4, L.B, L.T, L.H, D, 32, true) ||
      !make_tmap_bthd(&tm_ke, ws_ptr<float>(a.ws, L.Ke), 4, L.B, L.T, L.H, D, NJ, false))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)FcCfg<R>::BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.B * L.H * R);
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = FcCfg<R>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(st, "fwd_chain_tc");
  e = cudaLaunchKernelEx(&cfg, fwd_chain_tc<R>, tm_kt, tm_ke, a.beta, a.S0, a.ST, L.H, L.T, L.NC,
                         (const float*)ws_ptr<float>(a.ws, L.y), (const float*)ws_ptr<float>(a.ws, L.A),
                         (const float*)ws_ptr<float>(a.ws, L.Hx), (const float*)ws_ptr<float>(a.ws, L.GC),
                         (const __nv_bfloat16*)ws_ptr<__nv_bfloat16>(a.ws, L.Vt),
                         (const int*)ws_ptr<int>(a.ws, L.xflags), ws_ptr<float>(a.ws, L.S0),
                         ws_ptr<float>(a.ws, L.u), ws_ptr<float>(a.ws, L.b0), ws_ptr<__nv_bfloat16>(a.ws, L.S0b), err);
  prof_end(st);
  return e;
}

template <int R>
int max_active_clusters() {
  if (cudaFuncSetAttribute(fwd_chain_tc<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FcCfg<R>::BYTES) !=
      cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(R * 1024);
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = FcCfg<R>::BYTES;
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

}  // namespace

// Largest cluster (8 or 4 CTAs per head) for which every head's cluster is
// resident at once; 4 when none is.
int choose_cluster(int units, int sms) {
  (void)sms;
  static int cap8 = -1;  // per process; the library targets one GPU model
  if (cap8 < 0) cap8 = max_active_clusters<8>();
  return units <= cap8 ? 8 : 4;
}

cudaError_t launch_fwd_chain_tc(const FwdArgs& a, int R, int* err, cudaStream_t st) {
  return R == 8 ? launch_chain_r<8>(a, err, st) : launch_chain_r<4>(a, err, st);
}

}  // namespace kd
