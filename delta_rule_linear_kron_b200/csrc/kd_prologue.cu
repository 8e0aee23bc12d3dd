// kd_prologue.cu -- the mixer's input prologue and its backward, fused into
// one pass each.
//
// KronLSTM digest ("KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을
// 줄인다", section "어떻게 쓰나"): q, k, v are L2-normalised; the erase and
// write gates are per-head scalars, sigmoids of their projections (the erase
// gate doubled for state tracking, same page, experiments paragraph); the
// forget gate is the sigmoid raised to the head's learned exponent
// a = exp(a_log), so log f = a * log sigmoid(x).  Normalisation reading:
// y = x / sqrt(|x|^2 + 1e-6).
//
// Forward, per (token n, head h):
//   q, k, v   = L2-normalised q~, k~, v~            (dtype)
//   beta      = beta_scale * sigmoid(beta_pre)      (fp32)
//   c         = sigmoid(c_pre)                      (fp32)
//   logf_j    = exp(a_log[h]) * log sigmoid(f_j)    (fp32, per key channel)
// Backward, given the gradients of those outputs:
//   dx~       = r (dy - x r^2 (x . dy)),  r = (|x|^2 + eps)^(-1/2)
//   dbeta_pre = dbeta * beta_scale * s (1 - s),  s = sigmoid(beta_pre)
//   dc_pre    = dc * s (1 - s),                   s = sigmoid(c_pre)
//   df_j      = dlogf_j * a * (1 - sigmoid(f_j))
// (1 - sigmoid(x) is evaluated as sigmoid(-x), exact in relative terms in
// both tails, where 1 - sigmoid(x) in fp32 would cancel to zero.)
//   da_log[h] = sum over (n, j) of dlogf_j * logf_j
//
// Both passes are HBM-bound (about 2 flops per byte).  Layout of the work:
// grid (nb, H), 8 warps per block; warp w of block x handles the tokens
// n = x*8 + w + i*8*nb of head h, one token-head row per step, each lane
// dk/32 (dv/32) consecutive channels -- so every row is one coalesced vector
// access per warp and a block's rows all belong to one head.  da_log is
// reduced deterministically: each block writes one partial per head in a fixed
// warp order, and a second small kernel adds the nb partials of a head in a
// fixed order.
#include "kd_kernels.h"
#include "kd_rows.cuh"

namespace kd {

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(256) prologue_fwd_kernel(
    const Tin* __restrict__ qr, const Tin* __restrict__ kr, const Tin* __restrict__ vr,
    const float* __restrict__ beta_pre, const float* __restrict__ c_pre, const Tin* __restrict__ fr,
    const float* __restrict__ a_log, float beta_scale, long long N, int H, Tin* __restrict__ q,
    Tin* __restrict__ k, Tin* __restrict__ v, float* __restrict__ beta, float* __restrict__ c,
    float* __restrict__ logf) {
  constexpr int EK = DK / 32, EV = DV / 32;
  const int h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float a = expf(a_log[h]);
  const long long stride = (long long)gridDim.x * 8;
  for (long long n = (long long)blockIdx.x * 8 + warp; n < N; n += stride) {
    const size_t row = (size_t)n * H + h;
    const size_t ok = row * DK + lane * EK, ov = row * DV + lane * EV;
    float xq[EK], xk[EK], xf[EK], xv[EV];
    load_stream<Tin, EK>(qr + ok, xq);
    load_stream<Tin, EK>(kr + ok, xk);
    load_stream<Tin, EV>(vr + ov, xv);
    load_stream<Tin, EK>(fr + ok, xf);
    float sq = 0.f, sk = 0.f, sv = 0.f;
#pragma unroll
    for (int i = 0; i < EK; ++i) {
      sq = fmaf(xq[i], xq[i], sq);
      sk = fmaf(xk[i], xk[i], sk);
    }
#pragma unroll
    for (int i = 0; i < EV; ++i) sv = fmaf(xv[i], xv[i], sv);
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    sv = warp_sum(sv);
    const float rq = rsqrtf(sq + kNormEps), rk = rsqrtf(sk + kNormEps), rv = rsqrtf(sv + kNormEps);
    float lf[EK];
#pragma unroll
    for (int i = 0; i < EK; ++i) {
      xq[i] *= rq;
      xk[i] *= rk;
      lf[i] = a * log_sigmoidf_(xf[i]);
    }
#pragma unroll
    for (int i = 0; i < EV; ++i) xv[i] *= rv;
    store_row<Tin, EK>(q + ok, xq);
    store_row<Tin, EK>(k + ok, xk);
    store_row<Tin, EV>(v + ov, xv);
    store_row<float, EK>(logf + ok, lf);
    if (lane == 0) {
      beta[row] = beta_scale * sigmoidf_(beta_pre[row]);
      c[row] = sigmoidf_(c_pre[row]);
    }
  }
}

// dx = r (g - x r^2 (x . g)) for one row held E values per lane.
template <int E>
__device__ __forceinline__ void l2norm_bwd(float (&x)[E], const float (&g)[E]) {
  float s = 0.f, p = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    s = fmaf(x[i], x[i], s);
    p = fmaf(x[i], g[i], p);
  }
  s = warp_sum(s);
  p = warp_sum(p);
  const float r = rsqrtf(s + kNormEps);
  const float w = r * r * p;
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = r * fmaf(-x[i], w, g[i]);
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(256, 4) prologue_bwd_kernel(
    const Tin* __restrict__ qr, const Tin* __restrict__ kr, const Tin* __restrict__ vr,
    const float* __restrict__ beta_pre, const float* __restrict__ c_pre, const Tin* __restrict__ fr,
    const float* __restrict__ a_log, float beta_scale, const Tin* __restrict__ dq,
    const Tin* __restrict__ dk, const Tin* __restrict__ dv, const float* __restrict__ dbeta,
    const float* __restrict__ dc, const float* __restrict__ dlogf, long long N, int H,
    Tin* __restrict__ dqr, Tin* __restrict__ dkr, Tin* __restrict__ dvr, float* __restrict__ dbeta_pre,
    float* __restrict__ dc_pre, Tin* __restrict__ dfr, float* __restrict__ part) {
  constexpr int EK = DK / 32, EV = DV / 32;
  const int h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float a = expf(a_log[h]);
  const long long stride = (long long)gridDim.x * 8;
  float acc = 0.f;  // this lane's share of sum dlogf * logf
  for (long long n = (long long)blockIdx.x * 8 + warp; n < N; n += stride) {
    const size_t row = (size_t)n * H + h;
    const size_t ok = row * DK + lane * EK, ov = row * DV + lane * EV;
    float xq[EK], xk[EK], xv[EV], gq[EK], gk[EK], gv[EV], xf[EK], gl[EK];
    load_stream<Tin, EK>(qr + ok, xq);
    load_stream<Tin, EK>(kr + ok, xk);
    load_stream<Tin, EV>(vr + ov, xv);
    load_stream<Tin, EK>(dq + ok, gq);
    load_stream<Tin, EK>(dk + ok, gk);
    load_stream<Tin, EV>(dv + ov, gv);
    load_stream<Tin, EK>(fr + ok, xf);
    load_stream<float, EK>(dlogf + ok, gl);
    l2norm_bwd<EK>(xq, gq);
    l2norm_bwd<EK>(xk, gk);
    l2norm_bwd<EV>(xv, gv);
    float df[EK];
#pragma unroll
    for (int i = 0; i < EK; ++i) {
      // 1 - sigmoid(x) taken as sigmoid(-x): no cancellation for large x
      df[i] = gl[i] * a * sigmoidf_(-xf[i]);
      acc = fmaf(gl[i], a * log_sigmoidf_(xf[i]), acc);
    }
    store_row<Tin, EK>(dqr + ok, xq);
    store_row<Tin, EK>(dkr + ok, xk);
    store_row<Tin, EV>(dvr + ov, xv);
    store_row<Tin, EK>(dfr + ok, df);
    if (lane == 0) {
      const float b = beta_pre[row], p = c_pre[row];
      dbeta_pre[row] = dbeta[row] * beta_scale * (sigmoidf_(b) * sigmoidf_(-b));
      dc_pre[row] = dc[row] * (sigmoidf_(p) * sigmoidf_(-p));
    }
  }
  __shared__ float ws[8];
  acc = warp_sum(acc);
  if (lane == 0) ws[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += ws[w];
    part[(size_t)h * gridDim.x + blockIdx.x] = t;
  }
}

// da_log[h] = sum of the nb partials of head h, added in a fixed order.
__global__ void __launch_bounds__(256) prologue_dalog_kernel(const float* __restrict__ part, int nb,
                                                             float* __restrict__ da_log) {
  const int h = blockIdx.x;
  float t = 0.f;
  for (int i = threadIdx.x; i < nb; i += 256) t += part[(size_t)h * nb + i];
  __shared__ float ws[8];
  t = warp_sum(t);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += ws[w];
    da_log[h] = s;
  }
}

int prologue_blocks(long long N) {
  // eight tokens per warp (64 per block) on average
  long long nb = (N + 63) / 64;
  if (nb > 65535) nb = 65535;
  return (int)(nb < 1 ? 1 : nb);
}

namespace {

template <typename Tin, int DK, int DV>
cudaError_t pro_fwd_t(const PrologueArgs& a, int nb, cudaStream_t st) {
  prologue_fwd_kernel<Tin, DK, DV><<<dim3(nb, a.H), 256, 0, st>>>(
      static_cast<const Tin*>(a.q_raw), static_cast<const Tin*>(a.k_raw), static_cast<const Tin*>(a.v_raw),
      a.beta_pre, a.c_pre, static_cast<const Tin*>(a.f_pre), a.a_log, a.beta_scale, a.N, a.H,
      static_cast<Tin*>(a.q), static_cast<Tin*>(a.k), static_cast<Tin*>(a.v), a.beta, a.c, a.logf);
  return cudaGetLastError();
}

template <typename Tin, int DK, int DV>
cudaError_t pro_bwd_t(const PrologueArgs& a, int nb, cudaStream_t st) {
  prologue_bwd_kernel<Tin, DK, DV><<<dim3(nb, a.H), 256, 0, st>>>(
      static_cast<const Tin*>(a.q_raw), static_cast<const Tin*>(a.k_raw), static_cast<const Tin*>(a.v_raw),
      a.beta_pre, a.c_pre, static_cast<const Tin*>(a.f_pre), a.a_log, a.beta_scale,
      static_cast<const Tin*>(a.gq), static_cast<const Tin*>(a.gk), static_cast<const Tin*>(a.gv), a.dbeta,
      a.dc, a.dlogf, a.N, a.H, static_cast<Tin*>(a.dq_raw), static_cast<Tin*>(a.dk_raw),
      static_cast<Tin*>(a.dv_raw), a.dbeta_pre, a.dc_pre, static_cast<Tin*>(a.df_pre), a.part);
  return cudaGetLastError();
}

template <bool BWD, typename Tin, int DK>
cudaError_t pro_dv(const PrologueArgs& a, int nb, cudaStream_t st) {
  switch (a.dv) {
    case 32: return BWD ? pro_bwd_t<Tin, DK, 32>(a, nb, st) : pro_fwd_t<Tin, DK, 32>(a, nb, st);
    case 64: return BWD ? pro_bwd_t<Tin, DK, 64>(a, nb, st) : pro_fwd_t<Tin, DK, 64>(a, nb, st);
    default: return BWD ? pro_bwd_t<Tin, DK, 128>(a, nb, st) : pro_fwd_t<Tin, DK, 128>(a, nb, st);
  }
}

template <bool BWD, typename Tin>
cudaError_t pro_dk(const PrologueArgs& a, int nb, cudaStream_t st) {
  switch (a.dk) {
    case 32: return pro_dv<BWD, Tin, 32>(a, nb, st);
    case 64: return pro_dv<BWD, Tin, 64>(a, nb, st);
    default: return pro_dv<BWD, Tin, 128>(a, nb, st);
  }
}

}  // namespace

cudaError_t launch_prologue_fwd(const PrologueArgs& a, cudaStream_t st) {
  const int nb = prologue_blocks(a.N);
  prof_begin(st, "prologue_fwd");
  cudaError_t e = a.dtype == 1 ? pro_dk<false, __nv_bfloat16>(a, nb, st) : pro_dk<false, float>(a, nb, st);
  prof_end(st);
  return e;
}

cudaError_t launch_prologue_bwd(const PrologueArgs& a, cudaStream_t st) {
  const int nb = prologue_blocks(a.N);
  prof_begin(st, "prologue_bwd");
  cudaError_t e = a.dtype == 1 ? pro_dk<true, __nv_bfloat16>(a, nb, st) : pro_dk<true, float>(a, nb, st);
  prof_end(st);
  if (e != cudaSuccess) return e;
  prof_begin(st, "prologue_dalog");
  prologue_dalog_kernel<<<a.H, 256, 0, st>>>(a.part, nb, a.da_log);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace kd
