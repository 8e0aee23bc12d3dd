// kd_gate.cu -- gated inputs and the fused prologue: the forget gate formed
// from its pre-activation, and the backward through the normalisation and the
// erase/write gate sigmoids.
//
// KronLSTM digest, "어떻게 쓰나": the forget gate is f = sigma(f~)^a with
// a = e^{a_log} per head, so logf = a log sigma(f~).  Its backward:
//   df~    = dlogf a sigma(-f~)
//   da_log = sum over tokens and key channels of dlogf logf   (d logf / d a_log = logf)
// The tensor-core kernels form logf from f~ inside their own loads (and df~
// in their epilogues); these kernels serve the CUDA-core path, which converts
// f~ into a logf buffer before its forward and dlogf into df~ after its
// backward, and both paths' fixed-order reduction of da_log.
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {
namespace {

template <typename Tf>
__global__ void __launch_bounds__(256) gate_logf_kernel(const Tf* __restrict__ fpre, const float* __restrict__ a_log,
                                                        float* __restrict__ logf, size_t n, int H, int dk) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const int h = static_cast<int>((e / dk) % H);
    logf[e] = expf(a_log[h]) * log_sigmoid(to_f(fpre[e]));
  }
}

// one CTA per chunk (b, h, n): df~ for its positions and channels, and the
// chunk's part of da_log reduced in a fixed order
__global__ void __launch_bounds__(256) gate_dlogf_kernel(const float* __restrict__ dlogf,
                                                         const float* __restrict__ logf,
                                                         const float* __restrict__ a_log, float* __restrict__ dfpre,
                                                         float* __restrict__ dapart, int T, int H, int dk, int NC) {
  __shared__ float red[8];
  const int n = blockIdx.x % NC, u = blockIdx.x / NC, h = u % H, b = u / H;
  const int t0 = n * kChunk, nv = min(kChunk, T - t0);
  const float a = expf(a_log[h]), inv_a = expf(-a_log[h]);
  float part = 0.f;
  for (int e = threadIdx.x; e < nv * dk; e += blockDim.x) {
    const int t = e / dk, j = e % dk;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * dk + j;
    const float lf = logf[g], dl = dlogf[g];
    part = fmaf(dl, lf, part);
    dfpre[g] = dl * dlogf_dfpre(lf, a, inv_a);
  }
  part = warp_sum(part);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) s += red[w];
    dapart[blockIdx.x] = s;
  }
}

// one warp per head: lane l sums the chunks l, l + 32, ... of every sequence
// in order, then a fixed butterfly adds the lanes (the same order every call)
__global__ void __launch_bounds__(32) reduce_dalog_kernel(const float* __restrict__ dapart, int B, int H, int NC,
                                                          float* __restrict__ da_log) {
  const int h = blockIdx.x, lane = threadIdx.x;
  float s = 0.f;
  for (int b = 0; b < B; ++b)
    for (int n = lane; n < NC; n += 32) s += dapart[((size_t)b * H + h) * NC + n];
  s = warp_sum(s);
  if (lane == 0) da_log[h] = s;
}

// The fused prologue's backward through the normalisation and the gate
// sigmoids (tensor-core path: bf16, d = 128), in place on the gradients the
// chunk kernels wrote for the normalised q, k, v and the gated beta, c.  With
// y = x r, r = (|x|^2 + eps)^(-1/2), the gradient of x is r (dy - y (y . dy));
// beta = s sigma(x) gives dx = dbeta s sigma(x) sigma(-x), and c likewise with
// s = 1.  One warp per token and head, each lane four channels.
__global__ void __launch_bounds__(256) prologue_tail_bwd(const __nv_bfloat16* __restrict__ q_raw,
                                                         const __nv_bfloat16* __restrict__ k_raw,
                                                         const __nv_bfloat16* __restrict__ v_raw,
                                                         const float* __restrict__ beta_pre,
                                                         const float* __restrict__ c_pre, float bscale,
                                                         __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                                                         __nv_bfloat16* __restrict__ dv, float* __restrict__ dbeta,
                                                         float* __restrict__ dc, size_t rows) {
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* xs[3] = {q_raw, k_raw, v_raw};
  __nv_bfloat16* ds[3] = {dq, dk, dv};
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const size_t o = row * 128 + 4 * lane;
    const uint2 xr = *reinterpret_cast<const uint2*>(xs[m] + o);
    const uint2 dr = *reinterpret_cast<const uint2*>(ds[m] + o);
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xr);
    const __nv_bfloat162* dp = reinterpret_cast<const __nv_bfloat162*>(&dr);
    const float2 x0 = __bfloat1622float2(xp[0]), x1 = __bfloat1622float2(xp[1]);
    const float2 d0 = __bfloat1622float2(dp[0]), d1 = __bfloat1622float2(dp[1]);
    const float ss = warp_sum(fmaf(x0.x, x0.x, fmaf(x0.y, x0.y, fmaf(x1.x, x1.x, x1.y * x1.y))));
    const float r = rsqrtf(ss + kNormEps);
    const float dot = warp_sum(fmaf(x0.x, d0.x, fmaf(x0.y, d0.y, fmaf(x1.x, d1.x, x1.y * d1.y)))) * r;  // y . dy
    uint2 out;
    __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(&out);
    const float rd = r * dot * r;  // r (y . dy) r: y = x r
    op[0] = __floats2bfloat162_rn(fmaf(-x0.x, rd, r * d0.x), fmaf(-x0.y, rd, r * d0.y));
    op[1] = __floats2bfloat162_rn(fmaf(-x1.x, rd, r * d1.x), fmaf(-x1.y, rd, r * d1.y));
    *reinterpret_cast<uint2*>(ds[m] + o) = out;
  }
  if (lane == 0) {
    dbeta[row] *= bscale * dsigmoid_f(beta_pre[row]);
    dc[row] *= dsigmoid_f(c_pre[row]);
  }
}

}  // namespace

cudaError_t launch_prologue_tail_bwd(const void* q_raw, const void* k_raw, const void* v_raw, const float* beta_pre,
                                     const float* c_pre, float bscale, void* dq, void* dk, void* dv, float* dbeta,
                                     float* dc, size_t rows, cudaStream_t st) {
  prof_begin(st, "prologue_tail_bwd");
  prologue_tail_bwd<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
      static_cast<const __nv_bfloat16*>(v_raw), beta_pre, c_pre, bscale, static_cast<__nv_bfloat16*>(dq),
      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), dbeta, dc, rows);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gate_logf(const void* fpre, int dtype, const float* a_log, float* logf, int B, int T, int H,
                             int dk, cudaStream_t st) {
  const size_t n = (size_t)B * T * H * dk;
  const unsigned blocks = static_cast<unsigned>(n / 256 + 1 < 148u * 16u ? n / 256 + 1 : 148u * 16u);
  prof_begin(st, "gate_logf_kernel");
  if (dtype == 0)
    gate_logf_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(fpre), a_log, logf, n, H, dk);
  else
    gate_logf_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(fpre), a_log, logf,
                                                            n, H, dk);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_gate_dlogf(const float* dlogf, const float* logf, const float* a_log, float* dfpre,
                              float* dapart, int B, int T, int H, int dk, int NC, cudaStream_t st) {
  prof_begin(st, "gate_dlogf_kernel");
  gate_dlogf_kernel<<<(unsigned)((size_t)B * H * NC), 256, 0, st>>>(dlogf, logf, a_log, dfpre, dapart, T, H, dk, NC);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_reduce_dalog(const float* dapart, int B, int H, int NC, float* da_log, cudaStream_t st) {
  prof_begin(st, "reduce_dalog_kernel");
  reduce_dalog_kernel<<<(unsigned)H, 32, 0, st>>>(dapart, B, H, NC, da_log);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
