// kd_rows.cuh -- helpers of the row-wise gate and normalisation kernels (the
// input prologue and the output epilogue): one token-head row per warp, each
// lane E consecutive channels moved as one vector access, and the gate
// functions.
#pragma once

#include "kd_common.cuh"

namespace kd {

template <typename T, int E>
struct alignas(sizeof(T) * E) Pack {
  T x[E];
};

// __ldcs has no overload for the packed structs; go through their raw bits.
template <int BYTES> struct RawOf;
template <> struct RawOf<2> { using type = unsigned short; };
template <> struct RawOf<4> { using type = unsigned int; };
template <> struct RawOf<8> { using type = uint2; };
template <> struct RawOf<16> { using type = uint4; };

// Streaming (evict-first) load of E consecutive elements, widened to fp32.
template <typename T, int E>
__device__ __forceinline__ void load_stream(const T* p, float (&out)[E]) {
  using R = typename RawOf<sizeof(Pack<T, E>)>::type;
  const R r = __ldcs(reinterpret_cast<const R*>(p));
  Pack<T, E> t;
  memcpy(&t, &r, sizeof(t));
#pragma unroll
  for (int i = 0; i < E; ++i) out[i] = to_f(t.x[i]);
}

// Store of E consecutive elements, rounded to T (round to nearest even).
template <typename T, int E>
__device__ __forceinline__ void store_row(T* p, const float (&in)[E]) {
  Pack<T, E> t;
#pragma unroll
  for (int i = 0; i < E; ++i) t.x[i] = from_f<T>(in[i]);
  *reinterpret_cast<Pack<T, E>*>(p) = t;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }

// log sigmoid(x) = -(max(-x, 0) + log1p(exp(-|x|))), finite for every finite x.
__device__ __forceinline__ float log_sigmoidf_(float x) {
  return -(fmaxf(-x, 0.f) + log1pf(expf(-fabsf(x))));
}

}  // namespace kd
