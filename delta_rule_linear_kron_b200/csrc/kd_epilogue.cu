// kd_epilogue.cu -- the mixer's output epilogue and its backward, one fused
// pass each.
//
// KronLSTM digest ("KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을
// 줄인다", section "어떻게 쓰나"): the read-out o_t goes through a sigmoid
// output gate and a per-head RMSNorm before the output projection.  Reading:
// norm first, then the gate, eps = 1e-6, weight w [dv] shared by the heads:
//
//   y  = w * o * r * s,   r = (mean_j o_j^2 + eps)^(-1/2),   s = sigmoid(g)
//
// Backward for the loss <dy, y>, with n = o r:
//   dn = dy w s;   do = r (dn - n mean_j(n_j dn_j))
//   dg = dy w n s sigmoid(-g)
//   dw = sum over tokens and heads of dy n s
//
// HBM-bound like the prologue.  Rows (token, head) of dv channels, one row per
// warp, each lane dv/32 consecutive channels.  Grid: nb blocks of 8 warps;
// warp w of block x takes rows x*8 + w + i*8*nb.  dw is reduced
// deterministically: each lane keeps its channels' running sums, a block adds
// its 8 warps in a fixed order into one partial row [dv], and a second kernel
// adds the nb partial rows of each channel in a fixed order.
#include "kd_kernels.h"
#include "kd_rows.cuh"

namespace kd {

namespace {
constexpr float kRmsEps = 1e-6f;
constexpr long long kEpiMaxBlocks = 4096;
}  // namespace

template <typename Tin, int DV>
__global__ void __launch_bounds__(256) epilogue_fwd_kernel(const Tin* __restrict__ o, const Tin* __restrict__ g,
                                                           const float* __restrict__ w, long long rows,
                                                           Tin* __restrict__ y) {
  constexpr int EV = DV / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float wl[EV];
#pragma unroll
  for (int i = 0; i < EV; ++i) wl[i] = w[lane * EV + i];
  const long long stride = (long long)gridDim.x * 8;
  for (long long r = (long long)blockIdx.x * 8 + warp; r < rows; r += stride) {
    const size_t off = (size_t)r * DV + lane * EV;
    float xo[EV], xg[EV];
    load_stream<Tin, EV>(o + off, xo);
    load_stream<Tin, EV>(g + off, xg);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < EV; ++i) ss = fmaf(xo[i], xo[i], ss);
    ss = warp_sum(ss);
    const float rr = rsqrtf(ss * (1.f / DV) + kRmsEps);
#pragma unroll
    for (int i = 0; i < EV; ++i) xo[i] = wl[i] * (xo[i] * rr) * sigmoidf_(xg[i]);
    store_row<Tin, EV>(y + off, xo);
  }
}

template <typename Tin, int DV>
__global__ void __launch_bounds__(256) epilogue_bwd_kernel(const Tin* __restrict__ o, const Tin* __restrict__ g,
                                                           const float* __restrict__ w,
                                                           const Tin* __restrict__ dy, long long rows,
                                                           Tin* __restrict__ dO, Tin* __restrict__ dg,
                                                           float* __restrict__ part) {
  constexpr int EV = DV / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float wl[EV], acc[EV];
#pragma unroll
  for (int i = 0; i < EV; ++i) {
    wl[i] = w[lane * EV + i];
    acc[i] = 0.f;
  }
  const long long stride = (long long)gridDim.x * 8;
  for (long long r = (long long)blockIdx.x * 8 + warp; r < rows; r += stride) {
    const size_t off = (size_t)r * DV + lane * EV;
    float xo[EV], xg[EV], gy[EV];
    load_stream<Tin, EV>(o + off, xo);
    load_stream<Tin, EV>(g + off, xg);
    load_stream<Tin, EV>(dy + off, gy);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < EV; ++i) ss = fmaf(xo[i], xo[i], ss);
    ss = warp_sum(ss);
    const float rr = rsqrtf(ss * (1.f / DV) + kRmsEps);
    float dn[EV], gg[EV], p = 0.f;
#pragma unroll
    for (int i = 0; i < EV; ++i) {
      const float n = xo[i] * rr, s = sigmoidf_(xg[i]);
      xo[i] = n;
      const float dys = gy[i] * s;
      dn[i] = dys * wl[i];
      gg[i] = gy[i] * wl[i] * n * (s * sigmoidf_(-xg[i]));
      acc[i] = fmaf(dys, n, acc[i]);
      p = fmaf(n, dn[i], p);
    }
    p = warp_sum(p) * (1.f / DV);
#pragma unroll
    for (int i = 0; i < EV; ++i) dn[i] = rr * fmaf(-xo[i], p, dn[i]);
    store_row<Tin, EV>(dO + off, dn);
    store_row<Tin, EV>(dg + off, gg);
  }
  __shared__ float red[8][DV];
#pragma unroll
  for (int i = 0; i < EV; ++i) red[warp][lane * EV + i] = acc[i];
  __syncthreads();
  for (int j = threadIdx.x; j < DV; j += 256) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][j];
    part[(size_t)blockIdx.x * DV + j] = t;
  }
}

// dw[j] = sum of the nb partial rows' channel j, in a fixed order.
__global__ void __launch_bounds__(256) epilogue_dw_kernel(const float* __restrict__ part, int nb, int dv,
                                                          float* __restrict__ dw) {
  const int j = blockIdx.x;
  float t = 0.f;
  for (int i = threadIdx.x; i < nb; i += 256) t += part[(size_t)i * dv + j];
  __shared__ float ws[8];
  t = warp_sum(t);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += ws[q];
    dw[j] = s;
  }
}

int epilogue_blocks(long long rows) {
  long long nb = (rows + 63) / 64;  // eight rows per warp on average
  if (nb > kEpiMaxBlocks) nb = kEpiMaxBlocks;
  return (int)(nb < 1 ? 1 : nb);
}

namespace {

template <typename Tin, int DV>
cudaError_t epi_t(const EpilogueArgs& a, bool bwd, int nb, cudaStream_t st) {
  if (!bwd) {
    epilogue_fwd_kernel<Tin, DV><<<nb, 256, 0, st>>>(static_cast<const Tin*>(a.o), static_cast<const Tin*>(a.g),
                                                      a.w, a.rows, static_cast<Tin*>(a.y));
  } else {
    epilogue_bwd_kernel<Tin, DV><<<nb, 256, 0, st>>>(static_cast<const Tin*>(a.o), static_cast<const Tin*>(a.g),
                                                      a.w, static_cast<const Tin*>(a.dy), a.rows,
                                                      static_cast<Tin*>(a.dO), static_cast<Tin*>(a.dg), a.part);
  }
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t epi_dv(const EpilogueArgs& a, bool bwd, int nb, cudaStream_t st) {
  switch (a.dv) {
    case 32: return epi_t<Tin, 32>(a, bwd, nb, st);
    case 64: return epi_t<Tin, 64>(a, bwd, nb, st);
    default: return epi_t<Tin, 128>(a, bwd, nb, st);
  }
}

}  // namespace

cudaError_t launch_epilogue_fwd(const EpilogueArgs& a, cudaStream_t st) {
  const int nb = epilogue_blocks(a.rows);
  prof_begin(st, "epilogue_fwd");
  cudaError_t e = a.dtype == 1 ? epi_dv<__nv_bfloat16>(a, false, nb, st) : epi_dv<float>(a, false, nb, st);
  prof_end(st);
  return e;
}

cudaError_t launch_epilogue_bwd(const EpilogueArgs& a, cudaStream_t st) {
  const int nb = epilogue_blocks(a.rows);
  prof_begin(st, "epilogue_bwd");
  cudaError_t e = a.dtype == 1 ? epi_dv<__nv_bfloat16>(a, true, nb, st) : epi_dv<float>(a, true, nb, st);
  prof_end(st);
  if (e != cudaSuccess) return e;
  prof_begin(st, "epilogue_dw");
  epilogue_dw_kernel<<<a.dv, 256, 0, st>>>(a.part, nb, a.dv, a.dw);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
