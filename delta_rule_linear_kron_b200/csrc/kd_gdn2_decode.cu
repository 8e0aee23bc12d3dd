// kd_gdn2_decode.cu -- one recurrent decode step of the Gated DeltaNet-2 rule.
//
// Per (b,h), in the library's state convention (S in R^{dv x dk}): with
// e = b o k and z = w o v (Gated DeltaNet-2 article, sections "핵심 기여" and
// "방법론"),
//   Sbar = S diag(exp(loga)),  u = z - Sbar e,  S <- Sbar + u k^T,  o = S q.
// Every value row of the state updates on its own (u_r reads only row r), so
// unlike the Kronecker rule's decode there is no reduction across warps.
// HBM-bound: the fp32 state (dv*dk*4 bytes) is read once and written once.
// One CTA of 8 warps per head; warp w owns dv/8 consecutive rows, lane l owns
// dk/32 consecutive columns, so every row is one coalesced vector access.
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

namespace {

template <int CPL> struct Vec;
template <> struct Vec<1> { using type = float; };
template <> struct Vec<2> { using type = float2; };
template <> struct Vec<4> { using type = float4; };

template <int CPL>
__device__ __forceinline__ void ld_row(const float* p, float (&x)[CPL]) {
  using V = typename Vec<CPL>::type;
  const V t = __ldcs(reinterpret_cast<const V*>(p));
  const float* f = reinterpret_cast<const float*>(&t);
#pragma unroll
  for (int i = 0; i < CPL; ++i) x[i] = f[i];
}

template <int CPL>
__device__ __forceinline__ void st_row(float* p, const float (&x)[CPL]) {
  using V = typename Vec<CPL>::type;
  V t;
  float* f = reinterpret_cast<float*>(&t);
#pragma unroll
  for (int i = 0; i < CPL; ++i) f[i] = x[i];
  __stcs(reinterpret_cast<V*>(p), t);
}

}  // namespace

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_decode_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ bg, const float* __restrict__ wg, const float* __restrict__ loga,
    float* __restrict__ S, Tin* __restrict__ out) {
  constexpr int RPW = DV / 8;   // rows per warp
  constexpr int CPL = DK / 32;  // columns per lane
  const int unit = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* Su = S + (size_t)unit * DV * DK;

  float s[RPW][CPL];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) ld_row<CPL>(Su + (size_t)(warp * RPW + rr) * DK + lane * CPL, s[rr]);
  float kk[CPL], qq[CPL], ee[CPL], ff[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const size_t g = (size_t)unit * DK + lane * CPL + i;
    kk[i] = to_f(k[g]);
    qq[i] = to_f(q[g]);
    ee[i] = bg[g] * kk[i];
    ff[i] = expf(loga[g]);
  }
  // decay, then this lane's part of (Sbar e)_r for each of the warp's rows
  float part[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    float pe = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      s[rr][i] *= ff[i];
      pe = fmaf(s[rr][i], ee[i], pe);
    }
    part[rr] = pe;
  }
  warp_transpose_reduce<RPW>(part, lane);  // lane l: (Sbar e) of row l % RPW
  float pq[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = warp * RPW + rr;
    const size_t gv = (size_t)unit * DV + r;
    const float u = wg[gv] * to_f(v[gv]) - __shfl_sync(0xffffffffu, part[0], rr);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      s[rr][i] = fmaf(u, kk[i], s[rr][i]);
      acc = fmaf(s[rr][i], qq[i], acc);
    }
    pq[rr] = acc;
    st_row<CPL>(Su + (size_t)r * DK + lane * CPL, s[rr]);
  }
  warp_transpose_reduce<RPW>(pq, lane);
  if (lane < RPW) out[(size_t)unit * DV + warp * RPW + lane] = from_f<Tin>(pq[0]);
}

template <typename Tin>
static cudaError_t launch_gdn2_decode_t(const GdnDecodeArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(256);
  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  Tin* o = static_cast<Tin*>(a.out);
#define KD_GDEC(DK_, DV_)                                                                               \
  if (a.dk == DK_ && a.dv == DV_) {                                                                     \
    prof_begin(st, "gdn2_decode_kernel");                                                               \
    gdn2_decode_kernel<DK_, DV_, Tin><<<grid, block, 0, st>>>(q, k, v, a.b, a.w, a.loga, a.S, o);      \
    prof_end(st);                                                                                       \
    return cudaGetLastError();                                                                          \
  }
  KD_GDEC(32, 32) KD_GDEC(32, 64) KD_GDEC(32, 128)
  KD_GDEC(64, 32) KD_GDEC(64, 64) KD_GDEC(64, 128)
  KD_GDEC(128, 32) KD_GDEC(128, 64) KD_GDEC(128, 128)
#undef KD_GDEC
  return cudaErrorInvalidValue;
}

cudaError_t launch_gdn2_decode(const GdnDecodeArgs& a, cudaStream_t st) {
  return a.dtype == 0 ? launch_gdn2_decode_t<float>(a, st) : launch_gdn2_decode_t<__nv_bfloat16>(a, st);
}

}  // namespace kd
