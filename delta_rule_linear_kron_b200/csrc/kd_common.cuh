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
