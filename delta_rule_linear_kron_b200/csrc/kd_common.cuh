// kd_common.cuh -- small device helpers shared by the CUDA kernels of the
// Kronecker delta rule library (element conversion, warp reductions, the
// chunk size).  Nothing here is used by the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kd_kernels.h"

namespace kd {

// Largest |cumulative log decay| inside one chunk for which the factorised
// decay exp(L_t - L_i) = exp(L_t) * exp(-L_i) stays inside fp32/bf16 normal
// range (e^80 ~ 5.5e34, e^-80 ~ 1.8e-35).  Chunks beyond it take the exact
// per-element path.
constexpr float kSafeLogRange = 80.0f;

// |L| bound of the backward's factorised post-chain products: e^{-40} keeps
// dS' = dS e^Lambda well inside bf16's normal range for any |dS| above 1e-20.
// Chunks at or beyond it take the exact per-element backward path.
constexpr float kPostSafe = 40.0f;

// Chunks whose in-chunk |L| reaches this bound (below both bounds above, so
// that float rounding of L cannot leave a chunk on an exact path without it)
// also keep their chunk-start state in fp32 for the exact paths.
constexpr float kExactStateRange = 36.0f;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---- gated inputs: the forget gate formed from its pre-activation ----------
// KronLSTM digest, "어떻게 쓰나": f = sigma(f~)^a with a = e^{a_log} per head, so
// the log-decay is logf = a log sigma(f~), and log sigma(x) = -softplus(-x) =
// min(x, 0) - log(1 + e^{-|x|}).  These run once per element of every tile a
// chunk kernel loads, so they use the hardware exp2/log2 approximations with
// short Taylor series where those would cancel.

// log(1 + e) for e in [0, 1]: the series e - e^2/2 + e^3/3 - e^4/4 while
// e < 1/32 (truncation below e^5/5, relative 2e-7), else log of 1 + e, which
// is at least 0.03 there (relative error about 5e-6).
__device__ __forceinline__ float log1p_unit(float e) {
  return e < 0.03125f ? e * (1.f - e * (0.5f - e * (0.33333334f - 0.25f * e))) : __logf(1.f + e);
}
__device__ __forceinline__ float log_sigmoid(float x) { return fminf(x, 0.f) - log1p_unit(__expf(-fabsf(x))); }
// e^s - 1 for s <= 0: the series s + s^2/2 + s^3/6 + s^4/24 while s > -1/16
// (relative truncation below s^4/120 = 1.3e-7), else e^s - 1, at most -0.06 there.
__device__ __forceinline__ float expm1_nonpos(float s) {
  return s > -0.0625f ? s * (1.f + s * (0.5f + s * (0.16666667f + s * 0.041666668f))) : __expf(s) - 1.f;
}
// d logf / d f~ = a sigma(-f~); with ls = log sigma(f~) = logf / a, sigma(-f~) =
// 1 - e^{ls} = -(e^{ls} - 1), accurate when sigma(f~) is close to 1.
__device__ __forceinline__ float dlogf_dfpre(float logf, float a, float inv_a) {
  return -a * expm1_nonpos(fminf(logf * inv_a, 0.f));
}

// A chunk's bf16 forget pre-activation tile [64][128] (16 KB, landed at `src`,
// which may be the upper half of `dst`) becomes its fp32 log-decay tile at
// `dst` (32 KB): logf = a log sigma(f~), and 0 on positions t >= nv beyond the
// sequence (the zero-padded tail).  Thread tid takes the 4-element groups
// tid, tid + 256, ..., tid + 1792, so a warp's 8-byte loads and 16-byte stores
// are contiguous (no shared-memory bank conflicts).  All 256 threads of the
// CTA take part; the call ends with a CTA barrier.
__device__ __forceinline__ void gate_logf_tile(float* dst, const unsigned char* src, float a, int nv) {
  const int tid = threadIdx.x;
  uint2 raw[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) raw[r] = reinterpret_cast<const uint2*>(src)[r * 256 + tid];
  __syncthreads();  // every thread has read its source before any destination is written
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int grp = r * 256 + tid;  // elements 4 grp .. 4 grp + 3, all in row grp / 32
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw[r]);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grp / 32 < nv)
      o = make_float4(a * log_sigmoid(__bfloat162float(e[0])), a * log_sigmoid(__bfloat162float(e[1])),
                      a * log_sigmoid(__bfloat162float(e[2])), a * log_sigmoid(__bfloat162float(e[3])));
    reinterpret_cast<float4*>(dst)[grp] = o;
  }
  __syncthreads();
}

// ---- the rest of the fused input prologue (struct Pro in kd_kernels.h) ----
// The L2 normalisation's epsilon: x / sqrt(|x|^2 + kNormEps).
constexpr float kNormEps = 1e-6f;

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float gate_beta(float x, Pro p) { return p.bscale > 0.f ? p.bscale * sigmoid_f(x) : x; }
__device__ __forceinline__ float gate_c(float x, Pro p) { return p.bscale > 0.f ? sigmoid_f(x) : x; }
// d sigma(x) / dx = sigma(x) sigma(-x), each factor formed directly (no 1 - sigma cancellation)
__device__ __forceinline__ float dsigmoid_f(float x) { return sigmoid_f(x) * sigmoid_f(-x); }

// Normalises the rows of a [64][128] bf16 tile in shared memory in place.  Row
// t is two 128-byte halves, at seg0 + t * pitch and seg1 + t * pitch, each
// holding 64 channels in any order of its 16-byte chunks (a 128-byte swizzle
// permutes chunks only within a row, so the row's norm and scaling do not
// depend on it).  Four threads take a row, two chunks of each half apiece;
// each rewrites only what it read, so there is no barrier inside; the caller
// places one before any other thread reads the tile.  Zero rows (the padded
// tail) stay zero.  All 256 threads of the CTA call it.
__device__ __forceinline__ void l2norm_tile(unsigned char* seg0, unsigned char* seg1, int pitch) {
  const int t = threadIdx.x >> 2, q = threadIdx.x & 3;
  uint4* p[4] = {reinterpret_cast<uint4*>(seg0 + t * pitch + q * 16),
                 reinterpret_cast<uint4*>(seg0 + t * pitch + (q + 4) * 16),
                 reinterpret_cast<uint4*>(seg1 + t * pitch + q * 16),
                 reinterpret_cast<uint4*>(seg1 + t * pitch + (q + 4) * 16)};
  uint4 x[4];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    x[c] = *p[c];
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&x[c]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(e[i]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  const float r = rsqrtf(ss + kNormEps);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&x[c]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(e[i]);
      e[i] = __floats2bfloat162_rn(f.x * r, f.y * r);
    }
    *p[c] = x[c];
  }
}


__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Sum over groups of G consecutive lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = G / 2; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Warp "transpose-reduce": each lane holds N partial values (N a power of two
// <= 32).  On return lane l holds, in v[0], the sum over the warp of value
// index (l % N).  Uses N-1 + log2(32/N) shuffles instead of N*5.
template <int N>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[N], int lane) {
#pragma unroll
  for (int s = N / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      float send = upper ? v[i] : v[i + s];
      float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
#pragma unroll
  for (int o = N; o < 32; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
}

}  // namespace kd
