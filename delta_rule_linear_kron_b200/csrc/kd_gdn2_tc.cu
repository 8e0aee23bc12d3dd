// kd_gdn2_tc.cu -- Gated DeltaNet-2's per-chunk preparation on tensor cores
// (bf16 q, k, v and d_k = d_v = 128).
//
// Gated DeltaNet-2 article (aitrends.kr), sections "방법론" and "기술 상세": the
// chunkwise WY form with the channel decay absorbed into the erase side.  In
// the library's state convention (S in R^{dv x dk}, decay from the right), per
// chunk of C = 64 positions with in-chunk cumulative log-decay L (per key
// channel), gamma = e^L and Lambda = L at the chunk end:
//   E+ = b o k o gamma,  K- = k / gamma,  Q+ = q o gamma,  Z = w o v
//   T = tril(E+ K-^T, -1),  P = tril(Q+ K-^T),  A = (I + T)^{-1}
//   W = A E+,  U' = A Z,  K^e = k o e^{Lambda - L},  gamma_C = e^Lambda
// One CTA per chunk, all chunks in parallel:
//   1. [E+; Q+] K-^T on tcgen05 (M = 128: rows 0-63 give T, rows 64-127 P),
//      with bf16 high and low parts of both operands as in step 3.
//   2. A by a blocked inverse on CUDA cores (16 x 16 diagonal blocks by
//      substitution, then block rows), in fp32.
//   3. W^T = E+^T A^T and U'^T = Z^T A^T on tcgen05 (bf16 high and low parts of
//      both operands: hi hi + hi lo + lo hi, so the products keep about 16
//      significant bits of each factor), M = 128 channels, N = 64 positions;
//      E+^T and Z^T are the MN-major views of E+ [i][j] and Z [i][r].
// Chunks whose in-chunk |L| reaches 60 (where k / gamma could overflow) take T
// and P with per-element weights e^{L_t - L_i} <= 1 on CUDA cores instead of
// step 1.  Its outputs: A, P, Q+, U' and e^Lambda in fp32 (the CUDA-core
// kernel's layouts), and W and K^e as bf16 hi, lo images [t][j] for the two
// chains (the operand tiles as the chains' shared memory holds them).
#include "kd_common.cuh"
#include "kd_kernels.h"
#include "kd_tc.cuh"
#include "kd_tmap.h"

namespace kd {
namespace {

constexpr int C = kChunk;
constexpr int D = 128;
// in-chunk |L| below which the weights factor (e^{+-60} stays well inside fp32)
constexpr float kGdnTcSafeLog = 60.f;
// chunks ahead of the chain's slots whose operands its producer pulls into L2
constexpr int kChainAhead = 3;

struct GPrepCfg {
  static constexpr uint32_t AKQ = 0;        // [E+; Q+] bf16 hi, lo (2 K blocks x 128 rows each, 32 KB); then
                                            // [E+; Z] for step 3 (Z = w o v over Q+)
  static constexpr uint32_t BKM = 65536;    // K- bf16 hi, lo (2 K blocks x 64 rows each, 16 KB); then A hi, lo
  static constexpr uint32_t QR = 98304;     // q bf16 [64][128] (TMA)
  static constexpr uint32_t KR = 114688;    // k bf16 [64][128] (TMA)
  static constexpr uint32_t VR = 131072;    // v bf16 [64][128] (TMA)
  static constexpr uint32_t LS = 147456;    // loga fp32 [64][128] (TMA), then L in place
  static constexpr uint32_t TS = 180224;    // T fp32 [64][65]
  static constexpr uint32_t XS = TS + 64 * 65 * 4;        // A fp32 [64][65]
  static constexpr uint32_t TB = XS + 64 * 65 * 4;        // block temporaries [3][16][17]
  static constexpr uint32_t SMALL = TB + 3 * 16 * 17 * 4;  // prefix exchange [128], Lambda [128]
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
  static constexpr uint32_t LOAD_BYTES = 3 * 16384 + 32768;
  // A (the B operand of step 3), hi and lo
  static constexpr uint32_t AH = 65536, AL = 73728;
  // the chains' operand images W [t][j] and K^e [t][j], staged once step 3 is done (32 KB each)
  static constexpr uint32_t IW = 0, IK = 32768;
};

__device__ __forceinline__ void put_hl(unsigned char* hi, unsigned char* lo, uint32_t off, float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  *reinterpret_cast<__nv_bfloat16*>(hi + off) = h;
  *reinterpret_cast<__nv_bfloat16*>(lo + off) = __float2bfloat16_rn(x - __bfloat162float(h));
}

__global__ void __launch_bounds__(256, 1) gdn2_prep_tc(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_loga,
    const float* __restrict__ bg, const float* __restrict__ wg, int H, int T, int NC, GdnWs p,
    int* __restrict__ err) {
  using Cf = GPrepCfg;
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
  float* Ls = reinterpret_cast<float*>(sm + Cf::LS);
  float* Ts = reinterpret_cast<float*>(sm + Cf::TS);
  float* Xs = reinterpret_cast<float*>(sm + Cf::XS);
  float* Tb = reinterpret_cast<float*>(sm + Cf::TB);
  float* xch = reinterpret_cast<float*>(sm + Cf::SMALL);
  float* lam = xch + 128;
  const auto row = [&](int t) { return (((size_t)b * T + t0 + t) * H + h) * D; };

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, Cf::LOAD_BYTES);
    tc::tma_load_4d(sm + Cf::QR, &tm_q, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + Cf::KR, &tm_k, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + Cf::VR, &tm_v, 0, h, t0, b, &ld_bar);
    tc::tma_load_4d(sm + Cf::LS, &tm_loga, 0, h, t0, b, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 128);
  // the erase and write gates' rows into L2 while the tiles land: their loads
  // (steps 1 and 3) then wait on L2, not on HBM
  if (tid < 2 * C && (tid & 63) < nv) tc::prefetch_l2((tid < C ? bg : wg) + row(tid & 63), 4u * D);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);

  // decay prefix of key channel j, split over two threads (half 0: positions
  // 0-31, half 1: 32-63), then the operands of step 1 and the per-token outputs
  const int j = tid & 127, half = tid >> 7;
  float mx = 0.f;
  {
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
    if (half) lam[j] = acc + off;  // padded positions carry loga = 0: L at 63 is Lambda
    __syncthreads();
    const float lj = lam[j];
    if (half == 0) p.gC[ch * D + j] = expf(lj);
    float bv[32];  // the erase gates of this thread's positions, all loads in flight together
#pragma unroll
    for (int i = 0; i < 32; ++i) bv[i] = 32 * half + i < nv ? bg[row(32 * half + i) + j] : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * half + i;
      const float L = Lr[i] + off;
      mx = fmaxf(mx, fabsf(L));
      Ls[t * D + j] = L;
      const float qq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Cf::QR + (t * D + j) * 2));
      const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Cf::KR + (t * D + j) * 2));
      const float bb = bv[i];
      const float gm = expf(L), ig = expf(-L);
      const float qp = qq * gm;
      put_hl(sm + Cf::AKQ, sm + Cf::AKQ + 32768, tc::sw128_off(t, j, 128, 2), bb * kk * gm);
      put_hl(sm + Cf::AKQ, sm + Cf::AKQ + 32768, tc::sw128_off(64 + t, j, 128, 2), qp);
      put_hl(sm + Cf::BKM, sm + Cf::BKM + 16384, tc::sw128_off(t, j, 64, 2), kk * ig);
      p.Qp[(ch * C + t) * D + j] = qp;
    }
  }
  const bool is_unsafe = __syncthreads_or(!(mx < kGdnTcSafeLog)) != 0;
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0 && !is_unsafe) {
    const uint32_t IDB = tc::idesc(128, 64, 1);
    const uint32_t ops[3][2] = {{0u, 0u}, {0u, 16384u}, {32768u, 0u}};  // hi hi, hi lo, lo hi
#pragma unroll
    for (int pr = 0; pr < 3; ++pr)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kb = ks / 4, w = (ks % 4) * 32;
        tc::mma_bf16_ss(tmem, tc::desc_sw128(tc::smem_u32(sm + Cf::AKQ + ops[pr][0] + kb * 16384 + w)),
                        tc::desc_sw128(tc::smem_u32(sm + Cf::BKM + ops[pr][1] + kb * 8192 + w)), IDB,
                        (pr | ks) ? 1u : 0u);
      }
    tc::mma_commit(&mma_bar);
  }
  if (!is_unsafe) {
    tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
    tc::tc_after_sync();
    // lanes 0-63: T row t (strictly lower); lanes 64-127: P row t (lower with the diagonal)
    if (warp < 4) {
      const int r = warp * 32 + lane;
      const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, 0);
      const int t = r & 63;
      float* prow = p.P + (ch * C + t) * C;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float v[16];
        tc::tmem_ld16(lanes + 16 * c16, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int i = 16 * c16 + ii;
          if (r < 64)
            Ts[t * 65 + i] = i < t ? v[ii] : 0.f;
          else
            prow[i] = i <= t ? v[ii] : 0.f;
        }
      }
    }
  } else {
    // exact decay weights e^{L_t - L_i} <= 1 per element (rare: extreme decays)
    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(sm + Cf::QR);
    const __nv_bfloat16* ks = reinterpret_cast<const __nv_bfloat16*>(sm + Cf::KR);
    for (int e = tid; e < C * C; e += 256) {
      const int t = e / C, i = e % C;
      float st = 0.f, sp = 0.f;
      if (i <= t && t < nv) {
        for (int jj = 0; jj < D; ++jj) {
          const float kw = __bfloat162float(ks[i * D + jj]) * expf(Ls[t * D + jj] - Ls[i * D + jj]);
          st = fmaf(bg[row(t) + jj] * __bfloat162float(ks[t * D + jj]), kw, st);
          sp = fmaf(__bfloat162float(qs[t * D + jj]), kw, sp);
        }
      }
      Ts[t * 65 + i] = i < t ? st : 0.f;
      p.P[(ch * C + t) * C + i] = i <= t ? sp : 0.f;
    }
  }
  __syncthreads();

  // ---- A = (I + T)^{-1}, blocked by 16
  if (tid < 64) {
    const int blk = tid >> 4, m = tid & 15, o = 16 * blk;
    float col[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float s = t == m ? 1.f : 0.f;
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2)
        if (s2 >= m && s2 < t) s = fmaf(-Ts[(o + t) * 65 + o + s2], col[s2], s);
      col[t] = t < m ? 0.f : s;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) Xs[(o + t) * 65 + o + m] = col[t];
  }
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    if ((i >> 4) > (t >> 4)) Xs[t * 65 + i] = 0.f;
  }
  __syncthreads();
  for (int a = 1; a < 4; ++a) {
    for (int e = tid; e < a * 256; e += 256) {
      const int bb = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
      for (int kk = 16 * bb; kk < 16 * a; ++kk) s = fmaf(Ts[(16 * a + rr) * 65 + kk], Xs[kk * 65 + 16 * bb + cc], s);
      Tb[bb * 272 + rr * 17 + cc] = s;
    }
    __syncthreads();
    for (int e = tid; e < a * 256; e += 256) {
      const int bb = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) s = fmaf(Xs[(16 * a + rr) * 65 + 16 * a + kk], Tb[bb * 272 + kk * 17 + cc], s);
      Xs[(16 * a + rr) * 65 + 16 * bb + cc] = -s;
    }
    __syncthreads();
  }
  for (int e = tid; e < C * C; e += 256) p.A[ch * C * C + e] = Xs[(e / C) * 65 + (e % C)];

  // ---- the bf16 operands of step 3: E+ stays where step 1 read it (rows
  // 0-63 of the [E+; Q+] tile, its MN-major view is E+^T); Z = w o v goes over
  // Q+ in rows 64-127, and A into the K- tile (that MMA has completed)
  float wv[32];  // the write gates of this thread's positions, loads in flight together
#pragma unroll
  for (int i = 0; i < 32; ++i) wv[i] = 32 * half + i < nv ? wg[row(32 * half + i) + j] : 0.f;
#pragma unroll
  for (int i0 = 0; i0 < 32; ++i0) {
    const int i = 32 * half + i0;
    const float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Cf::VR + (i * D + j) * 2));
    put_hl(sm + Cf::AKQ, sm + Cf::AKQ + 32768, tc::sw128_off(64 + i, j, 128, 2), wv[i0] * vv);  // Z [i][r = j]
  }
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    put_hl(sm + Cf::AH, sm + Cf::AL, tc::sw128_off(t, i, 64, 2), Xs[t * 65 + i]);
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    // TMEM columns 0-63: W^T = E+^T A^T; columns 64-127: U'^T = Z^T A^T (E+^T and
    // Z^T as the MN-major views of E+ [i][j] and Z [i][r])
    const uint32_t IDB = tc::idesc(128, 64, 1) | tc::kMajorA;
    const uint32_t ops[3][2] = {{0u, Cf::AH}, {0u, Cf::AL}, {32768u, Cf::AH}};  // hi hi, hi lo, lo hi
#pragma unroll
    for (int pr = 0; pr < 3; ++pr)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bd = tc::desc_sw128(tc::smem_u32(sm + ops[pr][1] + ks * 32));
        tc::mma_bf16_ss(tmem, tc::desc_sw128_mn(tc::smem_u32(sm + Cf::AKQ + ops[pr][0] + ks * 2048), 16384u), bd,
                        IDB, (pr | ks) ? 1u : 0u);
        tc::mma_bf16_ss(tmem + 64,
                        tc::desc_sw128_mn(tc::smem_u32(sm + Cf::AKQ + ops[pr][0] + 8192 + ks * 2048), 16384u), bd,
                        IDB, (pr | ks) ? 1u : 0u);
      }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, is_unsafe ? 0 : 1, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  {
    // warps 0-3: lane j of W^T -> the chains' image of W ([t][j], bf16 hi, lo);
    // warps 4-7: lane r of U'^T -> U'[t][r]; then each group half of the
    // chains' image of K^e ([t][j], bf16 hi, lo) for channel j = lane.  The
    // operand tiles of steps 1 and 3 are free (their MMAs have completed).
    const int lr = (warp & 3) * 32 + lane;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, warp < 4 ? 0 : 64);
    float* up = p.Up + ch * C * D + lr;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float v[16];
      tc::tmem_ld16(lanes + 16 * c16, v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int t = 16 * c16 + ii;
        if (warp < 4)
          put_hl(sm + Cf::IW, sm + Cf::IW + 16384, tc::sw128_off(t, lr, 64, 2), v[ii]);
        else
          up[t * D] = v[ii];
      }
    }
    {
      const float lj = lam[lr];
      const int tk = warp < 4 ? 0 : 32;
#pragma unroll 8
      for (int t = tk; t < tk + 32; ++t) {
        const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Cf::KR + (t * D + lr) * 2));
        put_hl(sm + Cf::IK, sm + Cf::IK + 16384, tc::sw128_off(t, lr, 64, 2), kk * expf(lj - Ls[t * D + lr]));
      }
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  if (tid == 0) {
    tc::bulk_s2g(p.Wimg + ch * (2 * C * D), sm + Cf::IW, 4u * C * D);
    tc::bulk_s2g(p.Kimg + ch * (2 * C * D), sm + Cf::IK, 4u * C * D);
    tc::bulk_commit();
    tc::bulk_wait_read();
  }
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// The chunk outputs O = Q+ S0^T + P U, one CTA per chunk, all chunks in
// parallel, computed transposed on tcgen05 (M = 128 value channels, N = 64
// positions): O^T = S0 Q+^T + U^T P^T.  S0 arrives as the chain's saved bf16
// image (one bulk copy) and meets Q+'s high and low parts; Q+, P (preparation
// kernel) and U (chain) arrive in fp32 and are split into bf16 high and low
// parts while they are staged (hi hi + hi lo + lo hi).
// ---------------------------------------------------------------------------
struct GOutCfg {
  static constexpr uint32_t SH = 0;                      // S0 [r][j] bf16, 2 K blocks x 128 rows (32 KB)
  static constexpr uint32_t QH = 65536, QL = 81920;      // Q+ [t][j], 2 K blocks x 64 rows
  static constexpr uint32_t UH = 98304, UL = 114688;     // U [i][r], 64 rows (read MN-major as U^T)
  static constexpr uint32_t PH = 131072, PL = 139264;    // P [t][i], 64 rows
  static constexpr uint32_t BYTES = 147456 + 1024;
};

// four consecutive K elements (a 16-byte-aligned quarter of a swizzle chunk) as hi and lo parts
__device__ __forceinline__ void put_hl4(unsigned char* hi, unsigned char* lo, uint32_t off, float4 x) {
  const __nv_bfloat162 h0 = __floats2bfloat162_rn(x.x, x.y), h1 = __floats2bfloat162_rn(x.z, x.w);
  const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
  uint2 hv, lv;
  hv.x = *reinterpret_cast<const uint32_t*>(&h0);
  hv.y = *reinterpret_cast<const uint32_t*>(&h1);
  const __nv_bfloat162 l0 = __floats2bfloat162_rn(x.x - f0.x, x.y - f0.y), l1 = __floats2bfloat162_rn(x.z - f1.x, x.w - f1.y);
  lv.x = *reinterpret_cast<const uint32_t*>(&l0);
  lv.y = *reinterpret_cast<const uint32_t*>(&l1);
  *reinterpret_cast<uint2*>(hi + off) = hv;
  *reinterpret_cast<uint2*>(lo + off) = lv;
}

__global__ void __launch_bounds__(256, 1) gdn2_out_tc(int H, int T, int NC, GdnWs p, __nv_bfloat16* __restrict__ out,
                                                      int* __restrict__ err) {
  using Cf = GOutCfg;
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
  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    // S0 arrives as the chain's saved bf16 image, as it is
    tc::mbar_expect_tx(&ld_bar, 2u * D * D);
    tc::bulk_g2s(sm + Cf::SH, p.S0img + ch * (D * D), 2u * D * D, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 64);
  // stage the operands: four consecutive elements per thread and step, read as
  // float4, every load of a group issued before its data is used
  {
    const float4* qp = reinterpret_cast<const float4*>(p.Qp + ch * C * D);
    const float4* pp = reinterpret_cast<const float4*>(p.P + ch * C * C);
    const float4* uu = reinterpret_cast<const float4*>(p.U + ch * C * D);
    float4 x[12], y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = qp[tid + 256 * i];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = uu[tid + 256 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[8 + i] = pp[tid + 256 * i];
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // Q+ [t][j]
      const int e = tid + 256 * i, t = e / (D / 4), j = 4 * (e % (D / 4));
      put_hl4(sm + Cf::QH, sm + Cf::QL, tc::sw128_off(t, j, 64, 2), y[i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // P [t][i]
      const int e = tid + 256 * i, t = e / (C / 4), ii = 4 * (e % (C / 4));
      put_hl4(sm + Cf::PH, sm + Cf::PL, tc::sw128_off(t, ii, 64, 2), x[8 + i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // U [i][r]
      const int e = tid + 256 * i, ii = e / (D / 4), r = 4 * (e % (D / 4));
      put_hl4(sm + Cf::UH, sm + Cf::UL, tc::sw128_off(ii, r, 64, 2), x[i]);
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  if (tid == 0) {
    const uint32_t IDB = tc::idesc(128, 64, 1), IDU = tc::idesc(128, 64, 1) | tc::kMajorA;
    const uint32_t sq[2] = {Cf::QH, Cf::QL};  // S0 (bf16) Q+^T: Q+ hi, then lo
    const uint32_t up[3][2] = {{Cf::UH, Cf::PH}, {Cf::UH, Cf::PL}, {Cf::UL, Cf::PH}};
#pragma unroll
    for (int pr = 0; pr < 3; ++pr) {
      if (pr < 2) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // S0 Q+^T: K = 128 channels, two swizzle blocks
          tc::mma_bf16_ss(tmem, tc::desc_sw128(tc::smem_u32(sm + Cf::SH + (ks / 4) * 16384 + (ks % 4) * 32)),
                          tc::desc_sw128(tc::smem_u32(sm + sq[pr] + (ks / 4) * 8192 + (ks % 4) * 32)), IDB,
                          (pr | ks) ? 1u : 0u);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)  // U^T P^T: K = 64 positions (U^T the MN-major view of U)
        tc::mma_bf16_ss(tmem, tc::desc_sw128_mn(tc::smem_u32(sm + up[pr][0] + ks * 2048), 8192u),
                        tc::desc_sw128(tc::smem_u32(sm + up[pr][1] + ks * 32)), IDU, 1u);
    }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  {
    // lane r of O^T; warps 0-3 take positions 0-31, warps 4-7 positions 32-63
    const int r = (warp & 3) * 32 + lane, tb = (warp >> 2) * 32;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, tb);
#pragma unroll
    for (int c16 = 0; c16 < 2; ++c16) {
      float v[16];
      tc::tmem_ld16(lanes + 16 * c16, v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int t = tb + 16 * c16 + ii;
        if (t < nv) out[(((size_t)b * T + t0 + t) * H + h) * D + r] = __float2bfloat16_rn(v[ii]);
      }
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------------------
// The forward chain on tcgen05, one CTA per (b, h), chunks in order:
//   U_n     = U'_n - W_n S_n^T                 (MMA 1: X^T = S W^T, M = 128 rows of S, N = 64)
//   S_{n+1} = S_n diag(gamma_C,n) + U_n^T K^e_n  (MMA 2: U^T K^e, M = 128, N = 128)
// Every value row of the state evolves on its own (the erase reads S e, one
// value per row), so one CTA holds the whole state, row r in TMEM lane r, and
// no exchange between CTAs is needed.  Both products take bf16 high and low
// parts of both operands (hi hi + hi lo + lo hi); the state itself stays fp32
// in registers.
// Warp roles (320 threads):
//   warps 0-7   state warps: thread (r, c) holds row r, key channels 64c..64c+63
//               of S, and positions 32c..32c+31 of U; U = U' - X, the operand
//               U^T, the state update and its operand copy (bf16 hi, lo), whose
//               hi part the issuer also copies out as the chunk's saved start
//               state (bf16).
//   warp 8      producer: one thread copies chunk n+1's operand images (bf16
//               hi, lo, written by the preparation kernel) and gamma_C into one
//               of two slots while chunk n runs, and pulls later chunks into L2.
//   warp 9      issuer: one thread issues every MMA.
// Every wait is bounded; on expiry the kernel records a timeout in the
// library's error word and each role runs its loop out without waiting.
// ---------------------------------------------------------------------------
struct GChainCfg {
  static constexpr uint32_t SH = 0, SL = 32768;        // S [r][j] hi, lo: 2 K blocks x 128 rows
  static constexpr uint32_t UH = 65536, UL = 81920;    // U^T [r][t] hi, lo: 128 rows
  static constexpr uint32_t SLOT = 98304;              // 2 slots of 64 KB:
  static constexpr uint32_t SLOT_SZ = 65536;
  static constexpr uint32_t WH = 0, WL = 16384;        //   MMA 1's B [t][j] hi, lo: 2 K blocks x 64 rows
  static constexpr uint32_t KH = 32768, KL = 49152;    //   MMA 2's B [t][j] hi, lo, read MN-major
  static constexpr uint32_t BYTES = SLOT + 2 * SLOT_SZ + 1024;
  static constexpr int THREADS = 320;
  static constexpr uint32_t X_COL = 0, D_COL = 64;     // TMEM: X^T (64 columns), S update (128 columns)
};

__device__ __forceinline__ void g_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(b)) : "memory");
}

// eight consecutive K elements (one 16-byte swizzle chunk) of an operand row as hi and lo parts
__device__ __forceinline__ void put_hl8(unsigned char* hi, unsigned char* lo, uint32_t off, const float* x) {
  uint4 hv, lv;
  uint32_t* hp = reinterpret_cast<uint32_t*>(&hv);
  uint32_t* lp = reinterpret_cast<uint32_t*>(&lv);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 f = __bfloat1622float2(hh);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * q] - f.x, x[2 * q + 1] - f.y);
    hp[q] = *reinterpret_cast<const uint32_t*>(&hh);
    lp[q] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  *reinterpret_cast<uint4*>(hi + off) = hv;
  *reinterpret_cast<uint4*>(lo + off) = lv;
}

// What the two directions of the chain read and write.
struct GChainIO {
  const float* init;   // S0 (forward) or dS_T (backward) [B][H][dv][dk]; nullptr: zero
  float* fin;          // S_T or dS0; nullptr: not written
  const __nv_bfloat16* b1;  // MMA 1's B operand image [ch] ([t][j] hi, lo): W (forward) or K^e (backward)
  const __nv_bfloat16* b2;  // MMA 2's B operand image [ch] ([t][j] hi, lo): K^e (forward) or W (backward)
  const float* gC;     // gamma_C [ch][j]
  const float* ul;     // [ch][t][r]: U' (forward) or P^T dO (backward)
  const float* l2t;    // backward: (dO^T Q+)^T [ch][j][r], added to the state update
  float* uout;         // U (forward) or dU (backward) [ch][t][r]
  __nv_bfloat16* img;  // the saved state images [ch] (bf16: the hi part of MMA 1's operand)
};

template <bool BWD>
__global__ void __launch_bounds__(GChainCfg::THREADS, 1) gdn2_chain_tc(GChainIO io, int NC, int* __restrict__ err) {
  using Cf = GChainCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  // full / empty: a slot's tiles staged / read by the MMAs; g_free: its gamma_C read by the state warps
  __shared__ uint64_t full[2], empty[2], g_free[2], s_ready, x_done, u_ready, d_done;
  __shared__ __align__(16) float gs[2][D];  // gamma_C per slot (a bulk-copy destination)
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t unit = blockIdx.x;  // b * H + h
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], 1);
      tc::mbar_init(&g_free[i], 256);
    }
    tc::mbar_init(&s_ready, 256);
    tc::mbar_init(&x_done, 1);
    tc::mbar_init(&u_ready, 256);
    tc::mbar_init(&d_done, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 256);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp < 8) {
    // ---- state warps
    const int r = (warp & 3) * 32 + lane, c = warp >> 2;
    float S[64];
    {
      const float* src = io.init ? io.init + (unit * D + r) * D + 64 * c : nullptr;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 v = src ? reinterpret_cast<const float4*>(src)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * q] = v.x;
        S[4 * q + 1] = v.y;
        S[4 * q + 2] = v.z;
        S[4 * q + 3] = v.w;
      }
    }
    for (int k = 0; k < NC; ++k) {
      const int n = BWD ? NC - 1 - k : k;  // the backward runs from the last chunk to the first
      const size_t ch = unit * NC + n;
      // this chunk's start state as MMA 1's operand; the issuer also copies
      // its hi part out as the chunk's saved start state (one bulk copy: the
      // rows of a thread-per-row state would scatter over 128 rows)
#pragma unroll
      for (int q = 0; q < 8; ++q)
        put_hl8(sm + Cf::SH, sm + Cf::SL, tc::sw128_off(r, 64 * c + 8 * q, 128, 2), S + 8 * q);
      tc::fence_proxy_async();
      g_arrive(&s_ready);
      // U' (forward) or P^T dO (backward) at this thread's positions, loaded
      // while MMA 1 runs
      float up[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) up[i] = io.ul[(ch * C + 32 * c + i) * D + r];
      tc::mbar_wait<false>(&x_done, k & 1, err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, Cf::X_COL + 32 * c);
        float u[32];
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          float x[16];
          tc::tmem_ld16(lanes + 16 * h16, x);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) u[16 * h16 + i] = BWD ? up[16 * h16 + i] + x[i] : up[16 * h16 + i] - x[i];
        }
        float ua[32];  // MMA 2's operand: U^T, or -dU^T (the backward subtracts dU^T W)
#pragma unroll
        for (int i = 0; i < 32; ++i) ua[i] = BWD ? -u[i] : u[i];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          put_hl8(sm + Cf::UH, sm + Cf::UL, tc::sw128_off(r, 32 * c + 8 * q, 128, 2), ua + 8 * q);
        tc::fence_proxy_async();
        tc::tc_before_sync();
        g_arrive(&u_ready);
        // U (dU) to the workspace while MMA 2 runs
#pragma unroll
        for (int i = 0; i < 32; ++i) io.uout[(ch * C + 32 * c + i) * D + r] = u[i];
      }
      // the backward's dO^T Q+ term of this thread's state row, loaded while MMA 2 runs
      float l2[BWD ? 64 : 1];
      if (BWD) {
#pragma unroll
        for (int i = 0; i < 64; ++i) l2[i] = io.l2t[(ch * D + 64 * c + i) * D + r];
      }
      tc::mbar_wait<false>(&d_done, k & 1, err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      {
        const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, Cf::D_COL + 64 * c);
        const float* g = gs[k & 1] + 64 * c;
#pragma unroll
        for (int h16 = 0; h16 < 4; ++h16) {
          float dd[16];
          tc::tmem_ld16(lanes + 16 * h16, dd);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            S[16 * h16 + i] = fmaf(S[16 * h16 + i], g[16 * h16 + i], BWD ? dd[i] + l2[16 * h16 + i] : dd[i]);
        }
      }
      g_arrive(&g_free[k & 1]);
      tc::tc_before_sync();
    }
    if (io.fin) {
      float4* dst = reinterpret_cast<float4*>(io.fin + (unit * D + r) * D + 64 * c);
#pragma unroll
      for (int q = 0; q < 16; ++q) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
    }
  } else if (warp == 8 && lane == 0) {
    // ---- producer: chunk k's operand images and gamma_C into slot k % 2
    for (int k = 0; k < NC; ++k) {
      const int slot = k & 1, n = BWD ? NC - 1 - k : k;
      if (k >= 2) {
        tc::mbar_wait<false>(&empty[slot], ((k >> 1) - 1) & 1, err, tc::kErrTimeoutMma, &abort_flag);
        tc::mbar_wait<false>(&g_free[slot], ((k >> 1) - 1) & 1, err, tc::kErrTimeoutMma, &abort_flag);
      }
      unsigned char* sl = sm + Cf::SLOT + slot * Cf::SLOT_SZ;
      const size_t ch = unit * NC + n;
      tc::mbar_expect_tx(&full[slot], 4u * (2 * C * D) + 4u * D);
      tc::bulk_g2s(sl + Cf::WH, io.b1 + ch * (2 * C * D), 4u * C * D, &full[slot]);
      tc::bulk_g2s(sl + Cf::KH, io.b2 + ch * (2 * C * D), 4u * C * D, &full[slot]);
      tc::bulk_g2s(gs[slot], io.gC + ch * D, 4u * D, &full[slot]);
      if (k + kChainAhead < NC) {
        // pull the operands kChainAhead chunks ahead into L2, so that the
        // copies above and the state warps' loads find them there
        const size_t ca = unit * NC + (BWD ? n - kChainAhead : n + kChainAhead);
        tc::prefetch_l2(io.b1 + ca * (2 * C * D), 4u * C * D);
        tc::prefetch_l2(io.b2 + ca * (2 * C * D), 4u * C * D);
        tc::prefetch_l2(io.ul + ca * C * D, 4u * C * D);
        if (BWD) tc::prefetch_l2(io.l2t + ca * D * D, 4u * D * D);
      }
    }
  } else if (warp == 9 && lane == 0) {
    // ---- issuer
    const uint32_t ID1 = tc::idesc(128, 64, 1), ID2 = tc::idesc(128, 128, 1) | tc::kMajorB;
    // descriptors of the operand bases; a byte offset o moves a descriptor by
    // o >> 4 in its start-address field (shared addresses stay below 2^18)
    const uint64_t dSH = tc::desc_sw128(tc::smem_u32(sm + Cf::SH)), dSL = tc::desc_sw128(tc::smem_u32(sm + Cf::SL));
    const uint64_t dUH = tc::desc_sw128(tc::smem_u32(sm + Cf::UH)), dUL = tc::desc_sw128(tc::smem_u32(sm + Cf::UL));
    const uint64_t dSlot = tc::desc_sw128(tc::smem_u32(sm + Cf::SLOT));
    const uint64_t dSlotMN = tc::desc_sw128_mn(tc::smem_u32(sm + Cf::SLOT), 8192u);
    for (int k = 0; k < NC; ++k) {
      const int slot = k & 1, n = BWD ? NC - 1 - k : k;
      const uint64_t ds = dSlot + ((slot * Cf::SLOT_SZ) >> 4);
      tc::mbar_wait<false>(&full[slot], (k >> 1) & 1, err, tc::kErrTimeoutLoad, &abort_flag);
      tc::mbar_wait<false>(&s_ready, k & 1, err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      const uint64_t a1[3] = {dSH, dSH, dSL};
      const uint64_t b1[3] = {ds + (Cf::WH >> 4), ds + (Cf::WL >> 4), ds + (Cf::WH >> 4)};
#pragma unroll
      for (int pr = 0; pr < 3; ++pr)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_bf16_ss(tmem + Cf::X_COL, a1[pr] + (((ks / 4) * 16384 + (ks % 4) * 32) >> 4),
                          b1[pr] + (((ks / 4) * 8192 + (ks % 4) * 32) >> 4), ID1, (pr | ks) ? 1u : 0u);
      tc::mma_commit(&x_done);
      {
        // the chunk's start state image out, while MMA 1 runs
        __nv_bfloat16* img = io.img + (unit * NC + n) * (D * D);
        tc::bulk_s2g(img, sm + Cf::SH, 2u * D * D);
        tc::bulk_commit();
      }
      tc::mbar_wait<false>(&u_ready, k & 1, err, tc::kErrTimeoutMma, &abort_flag);
      tc::tc_after_sync();
      // B [t][j] MN-major: a K step of 16 positions is 16 rows (2048 bytes)
      const uint64_t dm = dSlotMN + ((slot * Cf::SLOT_SZ) >> 4);
      const uint64_t a2[3] = {dUH, dUH, dUL};
      const uint64_t b2[3] = {dm + (Cf::KH >> 4), dm + (Cf::KL >> 4), dm + (Cf::KH >> 4)};
#pragma unroll
      for (int pr = 0; pr < 3; ++pr)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_bf16_ss(tmem + Cf::D_COL, a2[pr] + ((ks * 32) >> 4), b2[pr] + ((ks * 2048) >> 4), ID2,
                          (pr | ks) ? 1u : 0u);
      tc::bulk_wait_read();  // the state image is read out before the state warps write the next one
      tc::mma_commit(&d_done);
      tc::mma_commit(&empty[slot]);
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// The backward's chunk-local terms, one CTA per chunk, all chunks in parallel.
// Reverse mode of the chain (derivation in kd_gdn2.cu's header):
//   dU = P^T dO + K^e dS^T,   dS <- dS Gamma + dO^T Q+ - dU^T W
// P^T dO and dO^T Q+ need no state, so they are formed here, transposed on
// tcgen05 with M = 128 value rows r (dO is exact in bf16; P and Q+ as hi + lo),
// every operand read MN-major from its natural layout:
//   columns 0-63:   (P^T dO)^T [r][t]  -> dUi [t][r]
//   columns 64-191: dO^T Q+   [r][j]  -> L2t [j][r]
// (The reverse chain's operand images are the forward's: K^e and W [t][j].)
// ---------------------------------------------------------------------------
struct GBpreCfg {
  static constexpr uint32_t DO = 0;                      // dO [t][r] bf16, 64 rows (16 KB)
  static constexpr uint32_t PH = 16384, PL = 24576;      // P [i][t] hi, lo, 64 rows (8 KB each)
  static constexpr uint32_t QH = 32768, QL = 49152;      // Q+ [t][j] hi, lo, 64 rows (16 KB each)
  static constexpr uint32_t BYTES = 65536 + 1024;
};

__global__ void __launch_bounds__(256, 1) gdn2_bpre_tc(const __nv_bfloat16* __restrict__ dO, int H, int T, int NC,
                                                       GdnWs p, int* __restrict__ err) {
  using Cf = GBpreCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  if (tid == 0) {
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 256);
  {
    // loads first (every load of a group in flight together), then the hi, lo
    // splits into the operand tiles, all in their natural layouts
    const float4* pp = reinterpret_cast<const float4*>(p.P + ch * C * C);
    const float4* qp = reinterpret_cast<const float4*>(p.Qp + ch * C * D);
    float4 q4[8], p4[4];
    uint4 o8[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) q4[i] = qp[tid + 256 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) p4[i] = pp[tid + 256 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // dO rows: eight channels per step
      const int e = tid + 256 * i, t = e / (D / 8), r = 8 * (e % (D / 8));
      o8[i] = t < nv ? *reinterpret_cast<const uint4*>(dO + (((size_t)b * T + t0 + t) * H + h) * D + r)
                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i, t = e / (D / 8), r = 8 * (e % (D / 8));
      *reinterpret_cast<uint4*>(sm + Cf::DO + tc::sw128_off(t, r, 64, 2)) = o8[i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // P [i][t]
      const int e = tid + 256 * i, ii = e / (C / 4), t = 4 * (e % (C / 4));
      put_hl4(sm + Cf::PH, sm + Cf::PL, tc::sw128_off(ii, t, 64, 2), p4[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // Q+ [t][j]
      const int e = tid + 256 * i, t = e / (D / 4), j = 4 * (e % (D / 4));
      put_hl4(sm + Cf::QH, sm + Cf::QL, tc::sw128_off(t, j, 64, 2), q4[i]);
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  if (tid == 0) {
    // A = dO^T (MN-major view of dO [t][r]); B = P^T, Q+^T (MN-major views of P, Q+)
    const uint32_t ID1 = tc::idesc(128, 64, 1) | tc::kMajorA | tc::kMajorB;
    const uint32_t ID2 = tc::idesc(128, 128, 1) | tc::kMajorA | tc::kMajorB;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint32_t mn = ks * 2048;
        const uint64_t a = tc::desc_sw128_mn(tc::smem_u32(sm + Cf::DO + mn), 8192u);
        tc::mma_bf16_ss(tmem, a, tc::desc_sw128_mn(tc::smem_u32(sm + (pr ? Cf::PL : Cf::PH) + mn), 8192u), ID1,
                        (pr | ks) ? 1u : 0u);
        tc::mma_bf16_ss(tmem + 64, a, tc::desc_sw128_mn(tc::smem_u32(sm + (pr ? Cf::QL : Cf::QH) + mn), 8192u), ID2,
                        (pr | ks) ? 1u : 0u);
      }
    tc::mma_commit(&mma_bar);
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  {
    // lane r: warps 0-3 take columns 0-95 (the 64 of P^T dO, then j 0-31),
    // warps 4-7 columns 96-191 (j 32-127)
    const int r = (warp & 3) * 32 + lane, c0 = (warp >> 2) * 96;
    const uint32_t lanes = tc::tmem_lane_addr(tmem, warp, c0);
#pragma unroll
    for (int c16 = 0; c16 < 6; ++c16) {
      float v[16];
      tc::tmem_ld16(lanes + 16 * c16, v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int col = c0 + 16 * c16 + ii;
        if (col < 64)
          p.dUi[(ch * C + col) * D + r] = v[ii];
        else
          p.L2t[(ch * D + col - 64) * D + r] = v[ii];
      }
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// The backward's per-chunk gradients on tcgen05, one CTA per chunk, all chunks
// in parallel (reverse mode of the chunk form, derivation in kd_gdn2.cu's
// header).  With S0 and dS the chunk's start state and the gradient of its end
// state (the chains' saved images), U, dU from the chains and A, U', W from
// the forward's preparation:
//   1. dQ+ = dO S0,  dW = -dU S0,  dK^e = U dS,  dP = tril(dO U^T)
//   2. dZ = A^T dU (-> dv = dZ o w, dw = dZ o v),  dE = A^T dW
//   3. dT = -tril(dZ U'^T + dE W^T, -1)
// and, for chunks whose in-chunk |L| stays below kGdnSafeLog (the decay
// weights factor as gamma_t / gamma_i), the pair sums of dq, dk, db and dloga
// as three more products with K- = k / gamma, E+ = b o k o gamma, Q+ = q o gamma:
//   4. X1 = dT K-,  X2 = dP K-,  Y = dT^T E+ + dP^T Q+
//      de = gamma (dE + X1),  dq = gamma (dQ+ + X2),  dk~ = dK^e e^{Lambda-L} + Y / gamma
//      dk = de o b + dk~,  db = de o k,  dL = b k de + q dq - k dk~
//      dloga_t = sum_{t' >= t} dL_t' + sum_t dK^e o K^e + e^Lambda sum_r dS[r] o S0[r]
// Every product runs transposed, with M = 128 key or value channels in TMEM
// lanes; the two 64 x 64 results (dP^T, dT^T) take their 64-row operand
// stacked as [hi; lo] parts over the 128 lanes, and the two halves are summed.
// Operands are bf16 high and low parts (hi hi + hi lo + lo hi); dO is exact in
// bf16, and the saved states S0 and dS arrive as the chains' bf16 images.  A
// thread owns key (or value) channel j = lane of its warp's TMEM quarter and
// positions 16 * (warp / 4) .. + 15, so the dloga suffix sums run down its own
// registers (one exchange between the four position groups).  Chunks beyond the factorised range leave dQ+, dK^e,
// dE, dT, dP and S0, dS (fp32) in the workspace for the exact kernel.
// ---------------------------------------------------------------------------
struct GBpostCfg {
  // step 1
  static constexpr uint32_t SI = 0;                      // S0 image [r][j] bf16 (32 KB)
  static constexpr uint32_t DI = 65536;                  // dS image, the same
  static constexpr uint32_t BO = 131072;                 // [dO; dU hi] [t][r], 128 rows (32 KB)
  static constexpr uint32_t DUL = 163840;                // dU lo [t][r], 64 rows (16 KB)
  static constexpr uint32_t US = 180224;                 // [U hi; U lo] [t][r], 128 rows (32 KB)
  // from step 2 on, over U: the decay prefix L fp32 [t][j] (32 KB)
  static constexpr uint32_t LS = 180224;
  // step 2, over the state images
  static constexpr uint32_t AH = 0, AL = 8192;           // A [i][t], 64 rows (8 KB each)
  static constexpr uint32_t DWH = 16384, DWL = 32768;    // dW [i][j], 64 rows (16 KB each)
  static constexpr uint32_t UPS = 49152;                 // [U' hi; U' lo] [i][r], 128 rows
  static constexpr uint32_t WS = 81920;                  // [W hi; W lo] [i][j], 128 rows
  // step 3, over dO and dU
  static constexpr uint32_t ZH = 114688, ZL = 131072;    // dZ [t][r], 64 rows
  static constexpr uint32_t EH = 147456, EL = 163840;    // dE [t][j], 64 rows
  // step 4, over everything before it but L
  static constexpr uint32_t KMH = 0, KML = 16384;        // K- [i][j], 64 rows
  static constexpr uint32_t EPH = 32768, EPL = 49152;    // E+ [t][j]
  static constexpr uint32_t QPH = 65536, QPL = 81920;    // Q+ [t][j]
  static constexpr uint32_t TPH = 98304, TPL = 114688;   // [dT; dP] [t][i], 128 rows (16 KB each)
  static constexpr uint32_t SCT = 131072;                // fp32 [64][65]: the lo halves of dT^T, dP^T
  static constexpr uint32_t SCP = SCT + 64 * 65 * 4;
  static constexpr uint32_t DLS = 131072;                // fp32 [64][128]: dL, over the halves once read
  static constexpr uint32_t BYTES = 212992 + 1024;
  // TMEM columns: dQ+^T, dW^T (then Y^T), dK^e^T, dP^T, dZ^T, dE^T, dT^T (then X1^T, X2^T)
  static constexpr uint32_t C_DQ = 0, C_DW = 64, C_Y = 64, C_DK = 128, C_DP = 192, C_DZ = 256, C_DE = 320,
                            C_DT = 384, C_X = 384;
};

__device__ __forceinline__ float ld_bf(const unsigned char* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

constexpr int kBpostThreads = 512;

__global__ void __launch_bounds__(kBpostThreads, 1) gdn2_bpost_tc(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ bg, const float* __restrict__ wg, const float* __restrict__ loga,
    const __nv_bfloat16* __restrict__ dO, int H, int T, int NC, GdnWs p, __nv_bfloat16* __restrict__ dq,
    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, float* __restrict__ db,
    float* __restrict__ dw, float* __restrict__ dloga, int* __restrict__ err) {
  using Cf = GBpostCfg;
  constexpr int NT = kBpostThreads, NG = NT / 128;  // NG groups of 16 positions
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t ld_bar, w_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  // per key channel: the running prefix, Lambda, sum dS o S0 (per warp, then
  // total), and each position group's sum of dK^e o K^e and of dL
  __shared__ float xpre[D], xlam[D], xst[D], xred[NT / 32][D], xkk[NG][D], xdl[NG][D];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % NC, unit = blockIdx.x / NC;
  const int b = unit / H, h = unit % H;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = blockIdx.x;
  // this thread: channel j (the lane of its warp's TMEM quarter), positions tb .. tb + 15
  const int j = (warp & 3) * 32 + lane, grp = warp >> 2, tb = 16 * grp;
  const auto row = [&](int t) { return (((size_t)b * T + t0 + t) * H + h) * D; };

  if (tid == 0) {
    tc::mbar_init(&ld_bar, 1);
    tc::mbar_init(&w_bar, 1);
    tc::mbar_init(&mma_bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
    tc::mbar_expect_tx(&ld_bar, 4u * D * D);
    tc::bulk_g2s(sm + Cf::SI, p.S0img + ch * (D * D), 2u * D * D, &ld_bar);
    tc::bulk_g2s(sm + Cf::DI, p.dSimg + ch * (D * D), 2u * D * D, &ld_bar);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 512);

  float L[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) L[i] = tb + i < nv ? loga[row(tb + i) + j] : 0.f;
  // step 1's operands: dO exact, dU and U as hi, lo; A and U' held for step 2
  float4 a4[2], u4[4];
  {
    const float4* dup = reinterpret_cast<const float4*>(p.dU + ch * C * D);
    const float4* up = reinterpret_cast<const float4*>(p.U + ch * C * D);
    float4 x[4], y[4];
    uint4 o8[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = dup[tid + NT * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = up[tid + NT * i];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int e = tid + NT * i, t = e / (D / 8), r = 8 * (e % (D / 8));
      o8[i] = t < nv ? *reinterpret_cast<const uint4*>(dO + row(t) + r) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + NT * i, t = e / (D / 4), r = 4 * (e % (D / 4));
      const uint32_t o = tc::sw128_off(t, r, 128, 2);
      put_hl4(sm + Cf::BO + 8192 + o, sm + Cf::DUL + tc::sw128_off(t, r, 64, 2), 0u, x[i]);  // dU hi, lo
      put_hl4(sm + Cf::US, sm + Cf::US + 8192, o, y[i]);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int e = tid + NT * i, t = e / (D / 8), r = 8 * (e % (D / 8));
      *reinterpret_cast<uint4*>(sm + Cf::BO + tc::sw128_off(t, r, 128, 2)) = o8[i];
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) a4[i] = reinterpret_cast<const float4*>(p.A + ch * C * C)[tid + NT * i];
#pragma unroll
  for (int i = 0; i < 4; ++i) u4[i] = reinterpret_cast<const float4*>(p.Up + ch * C * D)[tid + NT * i];
  // the decay prefix of channel j, group after group, in the same sequential
  // order as the exact kernel's (so both take the same chunks)
#pragma unroll 1
  for (int g = 0; g < NG; ++g) {
    if (grp == g) {
      float acc = g ? xpre[j] : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) L[i] = acc = acc + L[i];
      xpre[j] = acc;
      if (g == NG - 1) xlam[j] = acc;  // padded positions carry loga = 0: L at 63 is Lambda
    }
    __syncthreads();
  }
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(L[i]));
  const bool exact = __syncthreads_or(!(mx < kGdnSafeLog)) != 0;
  if (tid == 0) p.xflag[ch] = exact ? 1 : 0;
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tmem = tmem_slot;
  tc::mbar_wait<false>(&ld_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
  const auto sd = [&](uint32_t o) { return tc::smem_u32(sm + o); };
  if (tid == 0) {
    tc::tc_after_sync();
    const uint32_t ID128 = tc::idesc(128, 128, 1) | tc::kMajorA, ID64 = tc::idesc(128, 64, 1) | tc::kMajorA;
    const uint32_t ID64K = tc::idesc(128, 64, 1);
#pragma unroll 1
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t kb = (ks / 4) * 16384 + (ks % 4) * 32, kb64 = (ks / 4) * 8192 + (ks % 4) * 32;
      const uint32_t mn = ks * 2048;
      // [dQ+^T | (dU S0)^T] = S0^T [dO; dU]^T (S0 in bf16), with dU's lo part on the dU half
      tc::mma_bf16_ss(tmem + Cf::C_DQ, tc::desc_sw128_mn(sd(Cf::SI + mn), 16384u), tc::desc_sw128(sd(Cf::BO + kb)),
                      ID128, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + Cf::C_DW, tc::desc_sw128_mn(sd(Cf::SI + mn), 16384u), tc::desc_sw128(sd(Cf::DUL + kb64)),
                      ID64, 1u);
      // dK^e^T = dS^T U^T (dS in bf16; U hi and lo)
      tc::mma_bf16_ss(tmem + Cf::C_DK, tc::desc_sw128_mn(sd(Cf::DI + mn), 16384u), tc::desc_sw128(sd(Cf::US + kb)),
                      ID64, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + Cf::C_DK, tc::desc_sw128_mn(sd(Cf::DI + mn), 16384u),
                      tc::desc_sw128(sd(Cf::US + 8192 + kb)), ID64, 1u);
      // [U hi; U lo] dO^T: lanes 0-63 and 64-127 are the two parts of dP^T
      tc::mma_bf16_ss(tmem + Cf::C_DP, tc::desc_sw128(sd(Cf::US + kb)), tc::desc_sw128(sd(Cf::BO + kb)), ID64K,
                      ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mma_bar);
  }
  {
    // sum_r dS[r][j] S0[r][j] while the MMAs run: a thread takes eight
    // channels (one 16-byte swizzle chunk of each part) of four rows; the two
    // row groups of a warp are added by a shuffle, the warps in order
    const int jg = lane & 15, rg = 2 * warp + (lane >> 4);
    float acc8[8] = {};
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const uint32_t o = tc::sw128_off(4 * rg + rr, 8 * jg, 128, 2);
      const uint4 sh = *reinterpret_cast<const uint4*>(sm + Cf::SI + o);
      const uint4 dh = *reinterpret_cast<const uint4*>(sm + Cf::DI + o);
      const __nv_bfloat162* a0 = reinterpret_cast<const __nv_bfloat162*>(&sh);
      const __nv_bfloat162* b0 = reinterpret_cast<const __nv_bfloat162*>(&dh);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float2 s2 = __bfloat1622float2(a0[c]), d2 = __bfloat1622float2(b0[c]);
        acc8[2 * c] = fmaf(d2.x, s2.x, acc8[2 * c]);
        acc8[2 * c + 1] = fmaf(d2.y, s2.y, acc8[2 * c + 1]);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) acc8[c] += __shfl_xor_sync(0xffffffffu, acc8[c], 16);
    if (lane < 16) {
#pragma unroll
      for (int c = 0; c < 8; ++c) xred[warp][8 * jg + c] = acc8[c];
    }
    if (exact) {
      // the exact kernel reads S0 and dS in fp32 [r][j]
      float* s0 = p.S0 + ch * D * D;
      float* ds = p.dS + ch * D * D;
      for (int e = tid; e < D * D; e += NT) {
        const int r = e / D, jj = e % D;
        const uint32_t o = tc::sw128_off(r, jj, 128, 2);
        s0[e] = ld_bf(sm + Cf::SI + o);
        ds[e] = ld_bf(sm + Cf::DI + o);
      }
    }
  }
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  __syncthreads();  // the state images and U are read: step 2's operands and L go over them
  if (tid == 0) {
    // W's image as [hi; lo] per K block
    const unsigned char* wi = reinterpret_cast<const unsigned char*>(p.Wimg + ch * (2 * C * D));
    tc::mbar_expect_tx(&w_bar, 4u * C * D);
    tc::bulk_g2s(sm + Cf::WS, wi, 8192u, &w_bar);
    tc::bulk_g2s(sm + Cf::WS + 8192, wi + 16384, 8192u, &w_bar);
    tc::bulk_g2s(sm + Cf::WS + 16384, wi + 8192, 8192u, &w_bar);
    tc::bulk_g2s(sm + Cf::WS + 24576, wi + 24576, 8192u, &w_bar);
  }
  if (tid < D) {
    float st = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) st += xred[w][tid];
    xst[tid] = st;
  }
  float* Ls = reinterpret_cast<float*>(sm + Cf::LS);  // [64][128]: L at (t, j)
#pragma unroll
  for (int i = 0; i < 16; ++i) Ls[(tb + i) * D + j] = L[i];
#pragma unroll
  for (int i = 0; i < 2; ++i) {  // A [i][t]
    const int e = tid + NT * i, r = e / (C / 4), c = 4 * (e % (C / 4));
    put_hl4(sm + Cf::AH, sm + Cf::AL, tc::sw128_off(r, c, 64, 2), a4[i]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // [U' hi; U' lo]
    const int e = tid + NT * i, t = e / (D / 4), r = 4 * (e % (D / 4));
    put_hl4(sm + Cf::UPS, sm + Cf::UPS + 8192, tc::sw128_off(t, r, 128, 2), u4[i]);
  }
  // dW = -(dU S0) from TMEM into dW [i][j] (MN-major operand of dE^T)
#pragma unroll 1
  for (int c8 = 0; c8 < 2; ++c8) {
    const int c0 = tb + 8 * c8;
    float x[8];
    tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DW + c0), x);
    tc::tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) put_hl(sm + Cf::DWH, sm + Cf::DWL, tc::sw128_off(c0 + i, j, 64, 2), -x[i]);
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    // dZ^T = dU^T A, dE^T = dW^T A (A as the MN-major B operand)
    const uint32_t ID = tc::idesc(128, 64, 1) | tc::kMajorA | tc::kMajorB;
#pragma unroll 1
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t mn = ks * 2048;
      const uint64_t ah = tc::desc_sw128_mn(sd(Cf::AH + mn), 8192u), al = tc::desc_sw128_mn(sd(Cf::AL + mn), 8192u);
      const uint64_t uh = tc::desc_sw128_mn(sd(Cf::BO + 8192 + mn), 16384u);
      const uint64_t ul = tc::desc_sw128_mn(sd(Cf::DUL + mn), 8192u);
      const uint64_t wh = tc::desc_sw128_mn(sd(Cf::DWH + mn), 8192u), wl = tc::desc_sw128_mn(sd(Cf::DWL + mn), 8192u);
      tc::mma_bf16_ss(tmem + Cf::C_DZ, uh, ah, ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + Cf::C_DZ, uh, al, ID, 1u);
      tc::mma_bf16_ss(tmem + Cf::C_DZ, ul, ah, ID, 1u);
      tc::mma_bf16_ss(tmem + Cf::C_DE, wh, ah, ID, ks > 0 ? 1u : 0u);
      tc::mma_bf16_ss(tmem + Cf::C_DE, wh, al, ID, 1u);
      tc::mma_bf16_ss(tmem + Cf::C_DE, wl, ah, ID, 1u);
    }
    tc::mma_commit(&mma_bar);
  }
  // the write gates and values at this thread's (t, channel r = j) for dv and
  // dw, eight positions per step, the next step's loads in flight meanwhile
  const auto ld_wv = [&](int c0, float (&w8)[8], float (&v8)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool ok = c0 + i < nv;
      w8[i] = ok ? wg[row(c0 + i) + j] : 0.f;
      v8[i] = ok ? __bfloat162float(v[row(c0 + i) + j]) : 0.f;
    }
  };
  float wn[8], vn[8];
  ld_wv(tb, wn, vn);
  tc::mbar_wait<false>(&mma_bar, 1, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  // dZ^T (lane r) -> dZ [t][r] operand, dv and dw; dE^T (lane j) -> dE [t][j] operand
#pragma unroll 1
  for (int c8 = 0; c8 < 2; ++c8) {
    const int c0 = tb + 8 * c8;
    float w8[8], v8[8], z[8], e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w8[i] = wn[i];
      v8[i] = vn[i];
    }
    if (c8 == 0) ld_wv(c0 + 8, wn, vn);
    tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DZ + c0), z);
    tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DE + c0), e);
    tc::tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = c0 + i;
      const uint32_t o = tc::sw128_off(t, j, 64, 2);
      put_hl(sm + Cf::ZH, sm + Cf::ZL, o, z[i]);
      put_hl(sm + Cf::EH, sm + Cf::EL, o, e[i]);
      if (t < nv) {
        dv[row(t) + j] = __float2bfloat16_rn(z[i] * w8[i]);
        dw[row(t) + j] = z[i] * v8[i];
      }
    }
  }
  tc::fence_proxy_async();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (tid == 0) {
    // [U' hi; U' lo] dZ^T + [W hi; W lo] dE^T, with dZ, dE hi and then lo
    tc::mbar_wait<false>(&w_bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
    const uint32_t ID = tc::idesc(128, 64, 1);
#pragma unroll 1
    for (int pr = 0; pr < 2; ++pr)
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kb = (ks / 4) * 16384 + (ks % 4) * 32, kb64 = (ks / 4) * 8192 + (ks % 4) * 32;
        tc::mma_bf16_ss(tmem + Cf::C_DT, tc::desc_sw128(sd(Cf::UPS + kb)),
                        tc::desc_sw128(sd((pr ? Cf::ZL : Cf::ZH) + kb64)), ID, (pr | ks) ? 1u : 0u);
        tc::mma_bf16_ss(tmem + Cf::C_DT, tc::desc_sw128(sd(Cf::WS + kb)),
                        tc::desc_sw128(sd((pr ? Cf::EL : Cf::EH) + kb64)), ID, 1u);
      }
    tc::mma_commit(&mma_bar);
  }
  // k, b, q at this thread's (t, j), eight positions per step
  const auto ld_kbq = [&](int c0, float (&k8)[8], float (&b8)[8], float (&q8)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool ok = c0 + i < nv;
      k8[i] = ok ? __bfloat162float(k[row(c0 + i) + j]) : 0.f;
      b8[i] = ok ? bg[row(c0 + i) + j] : 0.f;
      q8[i] = ok ? __bfloat162float(q[row(c0 + i) + j]) : 0.f;
    }
  };
  float kn[8], bn[8], qn[8];
  if (!exact) ld_kbq(tb, kn, bn, qn);
  tc::mbar_wait<false>(&mma_bar, 0, err, tc::kErrTimeoutMma, &abort_flag);
  tc::tc_after_sync();
  __syncthreads();  // every operand of steps 2 and 3 is read
  // dT^T and dP^T: lanes 64-127 (the lo parts) park their halves in shared
  // memory, lanes 0-63 add them and write the [dT; dP] operand
  float* sct = reinterpret_cast<float*>(sm + Cf::SCT);
  float* scp = reinterpret_cast<float*>(sm + Cf::SCP);
  if ((warp & 3) >= 2) {
    const int i = j - 64;
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      const int c0 = tb + 8 * c8;
      float x[8], y[8];
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DT + c0), x);
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DP + c0), y);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        sct[i * 65 + c0 + ii] = x[ii];
        scp[i * 65 + c0 + ii] = y[ii];
      }
    }
  }
  if (!exact) {
    // step 4's operands K-, E+, Q+ [t][j] at this thread's positions
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      const int c0 = tb + 8 * c8;
      float k8[8], b8[8], q8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        k8[i] = kn[i];
        b8[i] = bn[i];
        q8[i] = qn[i];
      }
      if (c8 == 0) ld_kbq(c0 + 8, kn, bn, qn);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t o = tc::sw128_off(c0 + i, j, 64, 2);
        const float Lt = Ls[(c0 + i) * D + j], gm = __expf(Lt), ig = __expf(-Lt);
        put_hl(sm + Cf::KMH, sm + Cf::KML, o, k8[i] * ig);
        put_hl(sm + Cf::EPH, sm + Cf::EPL, o, b8[i] * k8[i] * gm);
        put_hl(sm + Cf::QPH, sm + Cf::QPL, o, q8[i] * gm);
      }
    }
  }
  __syncthreads();
  if ((warp & 3) < 2) {
    const int i = j;
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      const int c0 = tb + 8 * c8;
      float x[8], y[8];
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DT + c0), x);
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DP + c0), y);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        const int t = c0 + ii;
        const float dtv = i < t ? -(x[ii] + sct[i * 65 + t]) : 0.f;
        const float dpv = i <= t ? y[ii] + scp[i * 65 + t] : 0.f;
        if (exact) {
          p.dT[(ch * C + t) * C + i] = dtv;
          p.dP[(ch * C + t) * C + i] = dpv;
        } else {
          put_hl(sm + Cf::TPH, sm + Cf::TPL, tc::sw128_off(t, i, 128, 2), dtv);
          put_hl(sm + Cf::TPH, sm + Cf::TPL, tc::sw128_off(64 + t, i, 128, 2), dpv);
        }
      }
    }
  }
  if (exact) {
    // dQ+, dK^e and dE [t][j] for the exact kernel
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      const int c0 = tb + 8 * c8;
      float x[8], y[8], z[8];
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DQ + c0), x);
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DK + c0), y);
      tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DE + c0), z);
      tc::tmem_ld_wait();
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        const size_t o = (ch * C + c0 + ii) * D + j;
        p.dQp[o] = x[ii];
        p.dKe[o] = y[ii];
        p.dE[o] = z[ii];
      }
    }
  } else {
    tc::fence_proxy_async();
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    if (tid == 0) {
      // [X1^T | X2^T] = K-^T [dT; dP]^T and Y^T = E+^T dT + Q+^T dP
      const uint32_t IDX = tc::idesc(128, 128, 1) | tc::kMajorA;
      const uint32_t IDY = tc::idesc(128, 64, 1) | tc::kMajorA | tc::kMajorB;
#pragma unroll 1
      for (int pr = 0; pr < 3; ++pr)
#pragma unroll 1
        for (int ks = 0; ks < 4; ++ks) {
          // (A, B) part offsets: hi hi, hi lo, lo hi
          const uint32_t mn = ks * 2048, a = pr == 2 ? 16384u : 0u, bo = pr == 1 ? 16384u : 0u;
          tc::mma_bf16_ss(tmem + Cf::C_X, tc::desc_sw128_mn(sd(Cf::KMH + a + mn), 8192u),
                          tc::desc_sw128(sd(Cf::TPH + bo + ks * 32)), IDX, (pr | ks) ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::C_Y, tc::desc_sw128_mn(sd(Cf::EPH + a + mn), 8192u),
                          tc::desc_sw128_mn(sd(Cf::TPH + bo + mn), 8192u), IDY, (pr | ks) ? 1u : 0u);
          tc::mma_bf16_ss(tmem + Cf::C_Y, tc::desc_sw128_mn(sd(Cf::QPH + a + mn), 8192u),
                          tc::desc_sw128_mn(sd(Cf::TPH + 8192 + bo + mn), 8192u), IDY, 1u);
        }
      tc::mma_commit(&mma_bar);
    }
    ld_kbq(tb, kn, bn, qn);
    tc::mbar_wait<false>(&mma_bar, 1, err, tc::kErrTimeoutMma, &abort_flag);
    tc::tc_after_sync();
    const float lam = xlam[j];
    float* dLs = reinterpret_cast<float*>(sm + Cf::DLS);  // [64][128]: dL at (t, j)
    float kpart = 0.f, tot = 0.f;
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      const int c0 = tb + 8 * c8;
      float k8[8], b8[8], q8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        k8[i] = kn[i];
        b8[i] = bn[i];
        q8[i] = qn[i];
      }
      if (c8 == 0) ld_kbq(c0 + 8, kn, bn, qn);
      float se[8], sq[8], xk[8], yy[8];
      {
        float a8[8], b8x[8];
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DE + c0), a8);
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_X + c0), b8x);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) se[i] = a8[i] + b8x[i];  // dE + X1
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DQ + c0), a8);
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_X + 64 + c0), b8x);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) sq[i] = a8[i] + b8x[i];  // dQ+ + X2
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_DK + c0), xk);
        tc::tmem_ld8(tc::tmem_lane_addr(tmem, warp, Cf::C_Y + c0), yy);
        tc::tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = c0 + i;
        const float Lt = Ls[t * D + j], gm = __expf(Lt), ke = __expf(lam - Lt), ig = __expf(-Lt);
        const float dee = gm * se[i];
        const float dqq = gm * sq[i];
        const float dkk = fmaf(xk[i], ke, yy[i] * ig);
        kpart = fmaf(xk[i], k8[i] * ke, kpart);
        const float dl = b8[i] * k8[i] * dee + q8[i] * dqq - k8[i] * dkk;
        dLs[t * D + j] = dl;
        tot += dl;
        if (t < nv) {
          const size_t g = row(t) + j;
          dq[g] = __float2bfloat16_rn(dqq);
          dk[g] = __float2bfloat16_rn(fmaf(dee, b8[i], dkk));
          db[g] = dee * k8[i];
        }
      }
    }
    xkk[grp][j] = kpart;
    xdl[grp][j] = tot;
    __syncthreads();
    float acc = xst[j] * __expf(lam);
#pragma unroll
    for (int g = 0; g < NG; ++g) acc += xkk[g][j] + (g > grp ? xdl[g][j] : 0.f);
#pragma unroll 4
    for (int i = 15; i >= 0; --i) {
      acc += dLs[(tb + i) * D + j];
      if (tb + i < nv) dloga[row(tb + i) + j] = acc;
    }
  }
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

bool gdn2_tc_supported(const GdnLayout& L) { return L.dtype == 1 && L.dk == D && L.dv == D; }

cudaError_t launch_gdn2_bchain_tc(const GdnArgs& a, const GdnWs& p, int* err, cudaStream_t st) {
  const GdnLayout& L = a.L;
  cudaError_t e = cudaFuncSetAttribute(gdn2_bpre_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GBpreCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "gdn2_bpre_tc");
  gdn2_bpre_tc<<<(unsigned)L.chunks, 256, GBpreCfg::BYTES, st>>>(static_cast<const __nv_bfloat16*>(a.dO), L.H,
                                                                 L.T, L.NC, p, err);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(gdn2_chain_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GChainCfg::BYTES)) != cudaSuccess)
    return e;
  const GChainIO io{a.dST, a.dS0, p.Kimg, p.Wimg, p.gC, p.dUi, p.L2t, p.dU, p.dSimg};
  prof_begin(st, "gdn2_bchain_tc");
  gdn2_chain_tc<true><<<(unsigned)(L.B * L.H), GChainCfg::THREADS, GChainCfg::BYTES, st>>>(io, L.NC, err);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gdn2_bpost_tc(const GdnArgs& a, const GdnWs& p, int* err, cudaStream_t st) {
  const GdnLayout& L = a.L;
  cudaError_t e = cudaFuncSetAttribute(gdn2_bpost_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GBpostCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "gdn2_bpost_tc");
  gdn2_bpost_tc<<<(unsigned)L.chunks, kBpostThreads, GBpostCfg::BYTES, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.b, a.w, a.loga, static_cast<const __nv_bfloat16*>(a.dO), L.H, L.T,
      L.NC, p, static_cast<__nv_bfloat16*>(a.dq), static_cast<__nv_bfloat16*>(a.dk), static_cast<__nv_bfloat16*>(a.dv),
      a.db, a.dw, a.dloga, err);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gdn2_chain_tc(const GdnArgs& a, int* err, cudaStream_t st) {
  const GdnLayout& L = a.L;
  const GdnWs p = gdn_ws(a.ws, L);
  cudaError_t e = cudaFuncSetAttribute(gdn2_chain_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GChainCfg::BYTES);
  if (e != cudaSuccess) return e;
  const GChainIO io{a.S0, a.ST, p.Wimg, p.Kimg, p.gC, p.Up, nullptr, p.U, p.S0img};
  prof_begin(st, "gdn2_chain_tc");
  gdn2_chain_tc<false><<<(unsigned)(L.B * L.H), GChainCfg::THREADS, GChainCfg::BYTES, st>>>(io, L.NC, err);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gdn2_out_tc(const GdnArgs& a, int* err, cudaStream_t st) {
  const GdnLayout& L = a.L;
  const GdnWs p = gdn_ws(a.ws, L);
  cudaError_t e = cudaFuncSetAttribute(gdn2_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GOutCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "gdn2_out_tc");
  gdn2_out_tc<<<(unsigned)L.chunks, 256, GOutCfg::BYTES, st>>>(L.H, L.T, L.NC, p,
                                                               static_cast<__nv_bfloat16*>(a.out), err);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gdn2_prep_tc(const GdnArgs& a, int* err, cudaStream_t st) {
  const GdnLayout& L = a.L;
  const GdnWs p = gdn_ws(a.ws, L);
  CUtensorMap tm_q, tm_k, tm_v, tm_loga;
  if (!make_tmap_bthd(&tm_q, a.q, 2, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_k, a.k, 2, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_v, a.v, 2, L.B, L.T, L.H, D, 128, false) ||
      !make_tmap_bthd(&tm_loga, a.loga, 4, L.B, L.T, L.H, D, 128, false))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gdn2_prep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GPrepCfg::BYTES);
  if (e != cudaSuccess) return e;
  prof_begin(st, "gdn2_prep_tc");
  gdn2_prep_tc<<<(unsigned)L.chunks, 256, GPrepCfg::BYTES, st>>>(tm_q, tm_k, tm_v, tm_loga, a.b, a.w, L.H, L.T,
                                                                 L.NC, p, err);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
