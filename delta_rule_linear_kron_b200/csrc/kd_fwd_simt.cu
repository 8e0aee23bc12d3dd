// kd_fwd_simt.cu -- chunk-parallel forward on CUDA cores (fp32 FFMA).
//
// This is the general forward: any supported dk/dv and both dtypes, exact
// fp32 arithmetic (the fp32 workload's 1e-4 tolerance needs it).  The bf16
// d=128 workloads run the tensor-core kernels instead.
//
// Chunk form (the KronLSTM digest, section "무엇과 다른가": the vectorised rule
// is a Widrow-Hoff rule on k (x) v with a generalised Householder transition,
// so DeltaNet's chunk-parallel scheme applies; the Gated DeltaNet-2 article,
// sections "방법론" and "기술 상세": WY form, C = 64, forward substitution).
// Inside a chunk with start state S0, L_t = sum_{s<=t} logf_s, gamma = e^L:
//   M[t,i] = (v_t.v_i) sum_j k_t[j] k_i[j] e^{L_t[j]-L_i[j]}   (i < t)
//   P[t,i] = sum_j q_t[j] k_i[j] e^{L_t[j]-L_i[j]}             (i <= t)
//   A = (I + diag(beta) M)^{-1},  y = A c
//   b0_t = v_t^T S0 (k_t o gamma_t),  u = y - A (beta o b0)
//   O_t = S0 (q_t o gamma_t) + sum_{i<=t} P[t,i] u_i v_i
//   S_C = S0 diag(gamma_C) + sum_i u_i v_i (k_i o e^{L_C - L_i})^T
//
// Kernel 1 (prep, one CTA per chunk, all chunks in parallel) builds M, P, A
// and y.  Kernel 2 (chain, one CTA per head) walks the chunks in order.
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

constexpr int C = kChunk;

template <int DK, int DV>
constexpr size_t prep_smem_floats() {
  return 4 * (size_t)C * (DK + 1) + (size_t)C * (DV + 1) + 3 * (size_t)C * (C + 1) + 2 * C;
}

// ---------------------------------------------------------------------------
// prep: decay prefix, Grams, triangular inverse, y
// ---------------------------------------------------------------------------
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) fwd_prep_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ c,
    const float* __restrict__ logf, int H, int T, int NC, float* __restrict__ wy,
    float* __restrict__ wA, float* __restrict__ wP) {
  constexpr int SK = DK + 1, SV = DV + 1, SC = C + 1;
  extern __shared__ float smem[];
  float* Kp = smem;              // k o gamma          [C][SK]
  float* Km = Kp + C * SK;       // raw k, then k / gamma
  float* Qp = Km + C * SK;       // raw q, then q o gamma
  float* Ls = Qp + C * SK;       // log decay prefix L
  float* Vs = Ls + C * SK;       // v                  [C][SV]
  float* Ms = Vs + C * SV;       // M                  [C][SC]
  float* Ps = Ms + C * SC;       // P
  float* As = Ps + C * SC;       // A
  float* bs = As + C * SC;       // beta [C]
  float* cs = bs + C;            // c    [C]
  __shared__ int unsafe;

  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = n * C;
  const int nv = min(C, T - t0);
  const size_t ch = ((size_t)b * H + h) * NC + n;
  const int tid = threadIdx.x;

  for (int e = tid; e < C * DK; e += blockDim.x) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
    Km[t * SK + j] = ok ? to_f(k[g]) : 0.f;
    Qp[t * SK + j] = ok ? to_f(q[g]) : 0.f;
    Ls[t * SK + j] = ok ? logf[g] : 0.f;
  }
  for (int e = tid; e < C * DV; e += blockDim.x) {
    const int t = e / DV, r = e % DV;
    Vs[t * SV + r] = t < nv ? to_f(v[(((size_t)b * T + t0 + t) * H + h) * DV + r]) : 0.f;
  }
  if (tid < C) {
    const bool ok = tid < nv;
    const size_t g = ((size_t)b * T + t0 + tid) * H + h;
    bs[tid] = ok ? beta[g] : 0.f;
    cs[tid] = ok ? c[g] : 0.f;
  }
  if (tid == 0) unsafe = 0;
  __syncthreads();

  // a1: within-chunk inclusive prefix of the log decay, per key channel
  if (tid < DK) {
    float acc = 0.f, mx = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * SK + tid];
      Ls[t * SK + tid] = acc;
      mx = fmaxf(mx, fabsf(acc));
    }
    if (!(mx < kSafeLogRange)) atomicOr(&unsafe, 1);
  }
  __syncthreads();
  const bool safe = unsafe == 0;
  if (safe) {
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int t = e / DK, j = e % DK;
      const float l = Ls[t * SK + j];
      const float kk = Km[t * SK + j];
      const float ep = expf(l), em = expf(-l);
      Kp[t * SK + j] = kk * ep;
      Km[t * SK + j] = kk * em;
      Qp[t * SK + j] *= ep;
    }
  }
  __syncthreads();

  // a2, a3: Hadamard Gram M and query-key decay matrix P
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < C; t += 8) {
    const int i0 = lane, i1 = lane + 32;
    float gk0 = 0.f, gk1 = 0.f, pq0 = 0.f, pq1 = 0.f, gv0 = 0.f, gv1 = 0.f;
    if (safe) {
      for (int j = 0; j < DK; ++j) {
        const float kp = Kp[t * SK + j], qp = Qp[t * SK + j];
        const float m0 = Km[i0 * SK + j], m1 = Km[i1 * SK + j];
        gk0 = fmaf(kp, m0, gk0);
        gk1 = fmaf(kp, m1, gk1);
        pq0 = fmaf(qp, m0, pq0);
        pq1 = fmaf(qp, m1, pq1);
      }
    } else {
      // exact decay weights exp(L_t - L_i) <= 1, one per element
      for (int j = 0; j < DK; ++j) {
        const float lt = Ls[t * SK + j], kt = Km[t * SK + j], qt = Qp[t * SK + j];
        if (i0 <= t) {
          const float w = Km[i0 * SK + j] * expf(lt - Ls[i0 * SK + j]);
          gk0 = fmaf(kt, w, gk0);
          pq0 = fmaf(qt, w, pq0);
        }
        if (i1 <= t) {
          const float w = Km[i1 * SK + j] * expf(lt - Ls[i1 * SK + j]);
          gk1 = fmaf(kt, w, gk1);
          pq1 = fmaf(qt, w, pq1);
        }
      }
    }
    for (int r = 0; r < DV; ++r) {
      const float vt = Vs[t * SV + r];
      gv0 = fmaf(vt, Vs[i0 * SV + r], gv0);
      gv1 = fmaf(vt, Vs[i1 * SV + r], gv1);
    }
    Ms[t * SC + i0] = i0 < t ? gk0 * gv0 : 0.f;
    Ms[t * SC + i1] = i1 < t ? gk1 * gv1 : 0.f;
    Ps[t * SC + i0] = i0 <= t ? pq0 : 0.f;
    Ps[t * SC + i1] = i1 <= t ? pq1 : 0.f;
  }
  __syncthreads();

  // a4: A = (I + diag(beta) M)^{-1} by forward substitution; column m of the
  // unit lower-triangular inverse depends only on earlier rows of column m.
  if (tid < C) {
    const int m = tid;
    for (int t = 0; t < C; ++t) {
      float a;
      if (t < m) {
        a = 0.f;
      } else if (t == m) {
        a = 1.f;
      } else {
        float s = 0.f;
        for (int i = m; i < t; ++i) s = fmaf(Ms[t * SC + i], As[i * SC + m], s);
        a = -bs[t] * s;
      }
      As[t * SC + m] = a;
    }
  }
  __syncthreads();
  if (tid < C) {
    float s = 0.f;
    for (int m = 0; m <= tid; ++m) s = fmaf(As[tid * SC + m], cs[m], s);
    wy[ch * C + tid] = s;
  }
  for (int e = tid; e < C * C; e += blockDim.x) {
    const int t = e / C, i = e % C;
    wA[ch * C * C + e] = As[t * SC + i];
    if (wP) wP[ch * C * C + e] = Ps[t * SC + i];
  }
}

template <int DK, int DV>
constexpr size_t chain_smem_floats() {
  return 3 * (size_t)C * DK + (size_t)C * DV + 2 * (size_t)C * (C + 1) +
         (size_t)C * ((DK > DV ? DK : DV) + 1) + DK + 5 * C + (DV / 16) * C;
}

// ---------------------------------------------------------------------------
// chain: sequential over chunks, one CTA (2*dv threads) per (b,h).
// Thread (r, hh) keeps state row r, columns j = 2m + hh, in registers.
// ---------------------------------------------------------------------------
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(2 * DV) fwd_chain_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ logf,
    const float* __restrict__ S0, Tin* __restrict__ out, float* __restrict__ ST, int H, int T,
    int NC, const float* __restrict__ wy, const float* __restrict__ wA,
    const float* __restrict__ wP, int save, float* __restrict__ wS0, float* __restrict__ wu,
    float* __restrict__ wb0) {
  constexpr int HK = DK / 2, SC = C + 1, SR = (DK > DV ? DK : DV) + 1;
  extern __shared__ float smem[];
  float* Kp = smem;            // [C][DK]
  float* Qp = Kp + C * DK;     // [C][DK]
  float* Ke = Qp + C * DK;     // [C][DK]
  float* Vs = Ke + C * DK;     // [C][DV]
  float* As = Vs + C * DV;     // [C][SC]
  float* Ps = As + C * SC;     // [C][SC]
  float* Rb = Ps + C * SC;     // L prefix, then O_inter [C][SR]
  float* gC = Rb + C * SR;     // [DK]
  float* ys = gC + DK;         // [C]
  float* bs = ys + C;          // beta
  float* b0s = bs + C;         // b0
  float* us = b0s + C;         // u
  float* ws_ = us + C;         // beta o b0
  float* wpart = ws_ + C;      // per-warp partial sums of b0 [DV/16][C]
  constexpr int NW = DV / 16;

  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int r = tid >> 1, hh = tid & 1;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t unit = (size_t)b * H + h;

  float S[HK];
#pragma unroll
  for (int m = 0; m < HK; ++m) S[m] = S0 ? S0[unit * DV * DK + (size_t)r * DK + 2 * m + hh] : 0.f;

  for (int n = 0; n < NC; ++n) {
    const int t0 = n * C;
    const int nv = min(C, T - t0);
    const size_t ch = unit * NC + n;
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int t = e / DK, j = e % DK;
      const bool ok = t < nv;
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
      Kp[e] = ok ? to_f(k[g]) : 0.f;
      Qp[e] = ok ? to_f(q[g]) : 0.f;
      Rb[t * SR + j] = ok ? logf[g] : 0.f;
    }
    for (int e = tid; e < C * DV; e += blockDim.x) {
      const int t = e / DV, rr = e % DV;
      Vs[e] = t < nv ? to_f(v[(((size_t)b * T + t0 + t) * H + h) * DV + rr]) : 0.f;
    }
    for (int e = tid; e < C * C; e += blockDim.x) {
      As[(e / C) * SC + (e % C)] = wA[ch * C * C + e];
      Ps[(e / C) * SC + (e % C)] = wP[ch * C * C + e];
    }
    if (tid < C) {
      ys[tid] = wy[ch * C + tid];
      bs[tid] = tid < nv ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
    }
    __syncthreads();
    for (int j = tid; j < DK; j += blockDim.x) {
      float acc = 0.f;
      for (int t = 0; t < C; ++t) {
        acc += Rb[t * SR + j];
        Rb[t * SR + j] = acc;
      }
    }
    __syncthreads();
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int t = e / DK, j = e % DK;
      const float l = Rb[t * SR + j], lC = Rb[(C - 1) * SR + j];
      const float ep = expf(l);
      const float kk = Kp[e];
      Kp[e] = kk * ep;
      Ke[e] = kk * expf(lC - l);
      Qp[e] *= ep;
      if (t == 0) gC[j] = expf(lC);
    }
    __syncthreads();

    // a5 + inter-chunk part of a8: X = S K+^T -> b0; O_inter = S Q+^T
    for (int t = 0; t < C; ++t) {
      float xk = 0.f, xq = 0.f;
#pragma unroll
      for (int m = 0; m < HK; ++m) {
        xk = fmaf(S[m], Kp[t * DK + 2 * m + hh], xk);
        xq = fmaf(S[m], Qp[t * DK + 2 * m + hh], xq);
      }
      xk += __shfl_xor_sync(0xffffffffu, xk, 1);
      xq += __shfl_xor_sync(0xffffffffu, xq, 1);
      float p = hh == 0 ? Vs[t * DV + r] * xk : 0.f;
      p = warp_sum(p);
      if (lane == 0) wpart[warp * C + t] = p;
      if (hh == 0) Rb[t * SR + r] = xq;
    }
    __syncthreads();
    if (tid < C) {
      float s = 0.f;
      for (int w = 0; w < NW; ++w) s += wpart[w * C + tid];  // fixed order: deterministic
      b0s[tid] = s;
      ws_[tid] = bs[tid] * s;
    }
    __syncthreads();
    // a6: u = y - A (beta o b0)
    if (tid < C) {
      float s = ys[tid];
      for (int i = 0; i <= tid; ++i) s = fmaf(-As[tid * SC + i], ws_[i], s);
      us[tid] = s;
      if (save) {
        wu[ch * C + tid] = s;
        wb0[ch * C + tid] = b0s[tid];
      }
    }
    __syncthreads();

    // a8: O_t = O_inter + sum_{i<=t} P[t,i] u_i v_i ; thread (r,hh) takes t = 2tt + hh
    for (int tt = 0; tt < C / 2; ++tt) {
      const int t = 2 * tt + hh;
      float o = Rb[t * SR + r];
      for (int i = 0; i <= t; ++i) o = fmaf(Ps[t * SC + i], us[i] * Vs[i * DV + r], o);
      if (t < nv) out[(((size_t)b * T + t0 + t) * H + h) * DV + r] = from_f<Tin>(o);
    }

    // a7: S <- S diag(gamma_C) + V^T diag(u) K^e
    if (save) {
#pragma unroll
      for (int m = 0; m < HK; ++m) wS0[ch * DV * DK + (size_t)r * DK + 2 * m + hh] = S[m];
    }
#pragma unroll
    for (int m = 0; m < HK; ++m) S[m] *= gC[2 * m + hh];
    for (int t = 0; t < C; ++t) {
      const float w = us[t] * Vs[t * DV + r];
#pragma unroll
      for (int m = 0; m < HK; ++m) S[m] = fmaf(w, Ke[t * DK + 2 * m + hh], S[m]);
    }
    __syncthreads();
  }
  if (ST) {
#pragma unroll
    for (int m = 0; m < HK; ++m) ST[unit * DV * DK + (size_t)r * DK + 2 * m + hh] = S[m];
  }
}

template <int DK, int DV, typename Tin>
static cudaError_t run_fwd(const FwdArgs& a, cudaStream_t st) {
  const Layout& L = a.L;
  const size_t sp = prep_smem_floats<DK, DV>() * sizeof(float);
  const size_t sc = chain_smem_floats<DK, DV>() * sizeof(float);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(fwd_prep_simt<DK, DV, Tin>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fwd_chain_simt<DK, DV, Tin>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc)) != cudaSuccess)
    return e;
  float* wy = ws_ptr<float>(a.ws, L.y);
  float* wA = ws_ptr<float>(a.ws, L.A);
  float* wP = ws_ptr<float>(a.ws, L.P);
  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  if (a.phases & kPhaseLocal) {
    prof_begin(st, "fwd_prep_simt");
    fwd_prep_simt<DK, DV, Tin><<<dim3(L.NC, L.H, L.B), 256, sp, st>>>(
        q, k, v, a.beta, a.c, a.logf, L.H, L.T, L.NC, wy, wA, wP);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!(a.phases & kPhaseCarry)) return cudaSuccess;
  prof_begin(st, "fwd_chain_simt");
  fwd_chain_simt<DK, DV, Tin><<<dim3(L.H, L.B), 2 * DV, sc, st>>>(
      q, k, v, a.beta, a.logf, a.S0, static_cast<Tin*>(a.out), a.ST, L.H, L.T, L.NC, wy, wA, wP,
      a.save, a.save ? ws_ptr<float>(a.ws, L.S0) : nullptr,
      a.save ? ws_ptr<float>(a.ws, L.u) : nullptr, a.save ? ws_ptr<float>(a.ws, L.b0) : nullptr);
  prof_end(st);
  return cudaGetLastError();
}

template <int DK, int DV, typename Tin>
static cudaError_t run_prep(const FwdArgs& a, bool with_P, cudaStream_t st) {
  const Layout& L = a.L;
  const size_t sp = prep_smem_floats<DK, DV>() * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(fwd_prep_simt<DK, DV, Tin>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp);
  if (e != cudaSuccess) return e;
  prof_begin(st, "fwd_prep_simt");
  fwd_prep_simt<DK, DV, Tin><<<dim3(L.NC, L.H, L.B), 256, sp, st>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v), a.beta,
      a.c, a.logf, L.H, L.T, L.NC, ws_ptr<float>(a.ws, L.y), ws_ptr<float>(a.ws, L.A),
      with_P ? ws_ptr<float>(a.ws, L.P) : nullptr);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t launch_fwd_prep(const FwdArgs& a, bool with_P, cudaStream_t st) {
#define KD_P(DK_, DV_)                                                            \
  if (a.L.dk == DK_ && a.L.dv == DV_)                                             \
    return a.L.dtype == 0 ? run_prep<DK_, DV_, float>(a, with_P, st)              \
                          : run_prep<DK_, DV_, __nv_bfloat16>(a, with_P, st);
  KD_P(32, 32) KD_P(32, 64) KD_P(32, 128)
  KD_P(64, 32) KD_P(64, 64) KD_P(64, 128)
  KD_P(128, 32) KD_P(128, 64) KD_P(128, 128)
#undef KD_P
  return cudaErrorInvalidValue;
}

template <typename Tin>
static cudaError_t run_fwd_t(const FwdArgs& a, cudaStream_t st) {
#define KD_F(DK_, DV_) \
  if (a.L.dk == DK_ && a.L.dv == DV_) return run_fwd<DK_, DV_, Tin>(a, st);
  KD_F(32, 32) KD_F(32, 64) KD_F(32, 128)
  KD_F(64, 32) KD_F(64, 64) KD_F(64, 128)
  KD_F(128, 32) KD_F(128, 64) KD_F(128, 128)
#undef KD_F
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t st) {
  return a.L.dtype == 0 ? run_fwd_t<float>(a, st) : run_fwd_t<__nv_bfloat16>(a, st);
}

}  // namespace kd
