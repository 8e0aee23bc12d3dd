// kd_decode.cu -- one recurrent decode step of the Kronecker delta rule.
//
// Per (b,h): Sbar = S diag(exp(logf)); b = v^T Sbar k; u = c - beta b;
// S <- Sbar + u v k^T (in place); o = S q = Sbar q + u (k.q) v.
// (KronLSTM digest, "KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을
// 줄인다", sections "어떻게 동작하나" and "어떻게 쓰나".)
//
// The step is HBM-bound: each head's fp32 state (dv*dk*4 bytes) is read once
// and written once; everything else is a few hundred bytes.  One CTA of 8
// warps per head; warp w owns dv/8 consecutive state rows, lane l owns dk/32
// consecutive columns, so every row is one coalesced vector access per warp.
// All row loads are issued before any arithmetic.
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

template <int CPL> struct VecOf;
template <> struct VecOf<1> { using type = float; };
template <> struct VecOf<2> { using type = float2; };
template <> struct VecOf<4> { using type = float4; };

template <int CPL>
__device__ __forceinline__ void load_vec(const float* p, float (&x)[CPL]) {
  using V = typename VecOf<CPL>::type;
  V t = __ldcs(reinterpret_cast<const V*>(p));
  const float* f = reinterpret_cast<const float*>(&t);
#pragma unroll
  for (int i = 0; i < CPL; ++i) x[i] = f[i];
}

template <int CPL>
__device__ __forceinline__ void store_vec(float* p, const float (&x)[CPL]) {
  using V = typename VecOf<CPL>::type;
  V t;
  float* f = reinterpret_cast<float*>(&t);
#pragma unroll
  for (int i = 0; i < CPL; ++i) f[i] = x[i];
  __stcs(reinterpret_cast<V*>(p), t);
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) decode_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ c,
    const float* __restrict__ logf, float* __restrict__ S, Tin* __restrict__ out) {
  constexpr int RPW = DV / 8;   // rows per warp
  constexpr int CPL = DK / 32;  // columns per lane
  constexpr int NV = 2 * RPW;   // per-lane partials: (S k, S q) per row
  const int unit = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* Su = S + (size_t)unit * DV * DK;

  float s[RPW][CPL];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    load_vec<CPL>(Su + (size_t)(warp * RPW + rr) * DK + lane * CPL, s[rr]);

  float kk[CPL], qq[CPL], ff[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int j = lane * CPL + i;
    kk[i] = to_f(k[(size_t)unit * DK + j]);
    qq[i] = to_f(q[(size_t)unit * DK + j]);
    ff[i] = expf(logf[(size_t)unit * DK + j]);
  }
  float vr[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) vr[rr] = to_f(v[(size_t)unit * DV + warp * RPW + rr]);
  const float bt = beta[unit], ct = c[unit];

  // decay from the right, then per-row partial dot products with k and q
  float part[NV];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    float pk = 0.f, pq = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      s[rr][i] *= ff[i];
      pk = fmaf(s[rr][i], kk[i], pk);
      pq = fmaf(s[rr][i], qq[i], pq);
    }
    part[2 * rr] = pk;
    part[2 * rr + 1] = pq;
  }
  float kq = 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) kq = fmaf(kk[i], qq[i], kq);
  kq = warp_sum(kq);

  warp_transpose_reduce<NV>(part, lane);
  // lane l (< NV) now holds row (l/2) of this warp: (Sbar k)_r if l even, (Sbar q)_r if odd
  const int my_rr = (lane % NV) >> 1;
  const bool is_k = (lane & 1) == 0;
  float vmine = 0.f;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    if (rr == my_rr) vmine = vr[rr];
  float bpart = (lane < NV && is_k) ? vmine * part[0] : 0.f;
  bpart = warp_sum(bpart);

  __shared__ float red[8];
  if (lane == 0) red[warp] = bpart;
  __syncthreads();
  float b = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) b += red[w];
  const float u = ct - bt * b;

  if (lane < NV && !is_k)
    out[(size_t)unit * DV + warp * RPW + my_rr] = from_f<Tin>(part[0] + u * kq * vmine);

#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const float uv = u * vr[rr];
#pragma unroll
    for (int i = 0; i < CPL; ++i) s[rr][i] = fmaf(uv, kk[i], s[rr][i]);
    store_vec<CPL>(Su + (size_t)(warp * RPW + rr) * DK + lane * CPL, s[rr]);
  }
}

template <typename Tin>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(256);
  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  Tin* o = static_cast<Tin*>(a.out);
#define KD_DEC(DK_, DV_)                                                                     \
  if (a.dk == DK_ && a.dv == DV_) {                                                          \
    prof_begin(st, "decode_kernel");                                                         \
    decode_kernel<DK_, DV_, Tin><<<grid, block, 0, st>>>(q, k, v, a.beta, a.c, a.logf, a.S, o); \
    prof_end(st);                                                                            \
    return cudaGetLastError();                                                               \
  }
  KD_DEC(32, 32) KD_DEC(32, 64) KD_DEC(32, 128)
  KD_DEC(64, 32) KD_DEC(64, 64) KD_DEC(64, 128)
  KD_DEC(128, 32) KD_DEC(128, 64) KD_DEC(128, 128)
#undef KD_DEC
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  return a.dtype == 0 ? launch_decode_t<float>(a, st) : launch_decode_t<__nv_bfloat16>(a, st);
}

}  // namespace kd
