// kd_gdn2.cu -- the Gated DeltaNet-2 rule (decoupled channel-wise erase and
// write) on the chunk machinery: forward and backward, CUDA cores, every
// d_k, d_v in {32, 64, 128}, fp32 or bf16 activations.
//
// Gated DeltaNet-2 article (aitrends.kr), sections "핵심 기여" and "방법론": per
// token, e = b o k and z = w o v, the decay applied first; in the library's
// state convention (S in R^{dv x dk}, decay from the right, o = S q):
//   Sbar = S diag(exp(loga)),  u = z - Sbar e,  S = Sbar + u k^T,  o = S q.
// Chunk form (C = 64, the article's "기술 상세"; L = in-chunk cumulative loga,
// gamma = e^L, Lambda = L at the chunk end):
//   T[t,i] = sum_j e_t[j] k_i[j] e^{L_t[j]-L_i[j]} (i < t)   A = (I + T)^{-1}
//   P[t,i] = sum_j q_t[j] k_i[j] e^{L_t[j]-L_i[j]} (i <= t)
//   W = A (e o gamma),  U' = A (w o v)                       (per chunk, parallel)
//   U = U' - W S0^T,  S_C = S0 diag(e^Lambda) + U^T K^e      (chain over chunks)
//   O = Q+ S0^T + P U,  Q+ = q o gamma,  K^e = k o e^{Lambda-L}
// The decay weights inside T and P are taken per element, so no factor ever
// exceeds 1 and no chunk needs a separate exact path.
//
// Unlike the Kronecker rule, whose erase reads one scalar of the whole state,
// every value row of the state evolves on its own here: row r of U and of the
// next state depend only on row r of the current one.  So the chain kernels
// split each head's state by value rows over several CTAs with no exchange.
//
// Backward (reverse-mode of the chunk form; derivation checked in fp64 against
// the token recurrence by the tests):
//   dU  = P^T dO + K^e dS^T,  dS_prev = dO^T Q+ + dS Gamma - dU^T W   (chain)
//   dP = tril(dO U^T), dQ+ = dO S0, dK^e = U dS, dW = -dU S0,
//   dZ = A^T dU, dE = A^T dW, dT = -tril(dZ U'^T + dE W^T, -1),
//   and through the gates and exact weights to dq, dk, db, dv, dw, dloga.
//
// Kernels: gdn2_prep (A, P, W, U', Q+, K^e, e^Lambda per chunk), gdn2_chain,
// gdn2_out; gdn2_bchain, gdn2_bpost_a (dP, dZ -> dv, dw, dE, dT),
// gdn2_bpost_b (dq, dk, db, dloga).
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

namespace {

constexpr int C = kChunk;
constexpr int kRows = 8;  // value rows of the state per chain CTA

template <int DK, int DV>
struct GP {
  static constexpr int PK = DK + 1, PV = DV + 1, PZ = (DK > DV ? DK : DV) + 1, PC = C + 1;
};

__device__ __forceinline__ size_t row_bthd(int b, int T, int t, int H, int h, int D) {
  return (((size_t)b * T + t) * H + h) * D;
}

}  // namespace

// ---------------------------------------------------------------------------
// Per chunk, all chunks in parallel.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_prep(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                 const Tin* __restrict__ v, const float* __restrict__ bg,
                                                 const float* __restrict__ wg, const float* __restrict__ loga, int H,
                                                 int T, int NC, GdnWs p) {
  using G = GP<DK, DV>;
  extern __shared__ float gsm[];
  float* Ls = gsm;                   // [C][PK]  L
  float* Ks = Ls + C * G::PK;        // [C][PK]  k
  float* Es = Ks + C * G::PK;        // [C][PK]  e, then E+, then W
  float* Qs = Es + C * G::PK;        // [C][PZ]  q, then Z, then U'
  float* Ts = Qs + C * G::PZ;        // [C][PC]  T
  float* As = Ts + C * G::PC;        // [C][PC]  A
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;

  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
    const float kk = ok ? to_f(k[g]) : 0.f;
    Ks[t * G::PK + j] = kk;
    Qs[t * G::PZ + j] = ok ? to_f(q[g]) : 0.f;
    Es[t * G::PK + j] = ok ? bg[g] * kk : 0.f;
    Ls[t * G::PK + j] = ok ? loga[g] : 0.f;
  }
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * G::PK + tid];
      Ls[t * G::PK + tid] = acc;
    }
  }
  __syncthreads();
  // T and P with per-element decay weights e^{L_t - L_i} <= 1
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    float sT = 0.f, sP = 0.f;
    if (i <= t) {
      for (int j = 0; j < DK; ++j) {
        const float kw = Ks[i * G::PK + j] * expf(Ls[t * G::PK + j] - Ls[i * G::PK + j]);
        sT = fmaf(Es[t * G::PK + j], kw, sT);
        sP = fmaf(Qs[t * G::PZ + j], kw, sP);
      }
    }
    Ts[t * G::PC + i] = i < t ? sT : 0.f;
    p.P[ch * C * C + e] = i <= t ? sP : 0.f;
  }
  __syncthreads();
  const float* Llast = Ls + (C - 1) * G::PK;  // padded rows carry loga = 0: L at row C-1 is Lambda
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    const float L = Ls[t * G::PK + j], gm = expf(L);
    p.Qp[ch * C * DK + e] = Qs[t * G::PZ + j] * gm;
    p.Ke[ch * C * DK + e] = Ks[t * G::PK + j] * expf(Llast[j] - L);
    Es[t * G::PK + j] *= gm;
  }
  if (tid < DK) p.gC[ch * DK + tid] = expf(Llast[tid]);
  __syncthreads();
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DV) + r;
    Qs[t * G::PZ + r] = ok ? wg[g] * to_f(v[g]) : 0.f;
  }
  for (int e = tid; e < C * C; e += 256) As[(e / C) * G::PC + e % C] = (e / C == e % C) ? 1.f : 0.f;
  __syncthreads();
  // forward substitution (I + T) X = R, in place, for X = W (R = E+), U' (R = Z), A (R = I)
  constexpr int NCOL = DK + DV + C;
  for (int t = 1; t < C; ++t) {
    for (int c = tid; c < NCOL; c += 256) {
      float* X;
      int pitch, col;
      if (c < DK) { X = Es; pitch = G::PK; col = c; }
      else if (c < DK + DV) { X = Qs; pitch = G::PZ; col = c - DK; }
      else { X = As; pitch = G::PC; col = c - DK - DV; }
      float s = X[t * pitch + col];
      for (int i = 0; i < t; ++i) s = fmaf(-Ts[t * G::PC + i], X[i * pitch + col], s);
      X[t * pitch + col] = s;
    }
    __syncthreads();
  }
  for (int e = tid; e < C * DK; e += 256) p.W[ch * C * DK + e] = Es[(e / DK) * G::PK + e % DK];
  for (int e = tid; e < C * DV; e += 256) p.Up[ch * C * DV + e] = Qs[(e / DV) * G::PZ + e % DV];
  for (int e = tid; e < C * C; e += 256) p.A[ch * C * C + e] = As[(e / C) * G::PC + e % C];
}

// ---------------------------------------------------------------------------
// The chain: one CTA per (kRows value rows, head); chunks in order.
template <int DK, int DV>
__global__ void __launch_bounds__(256) gdn2_chain(const float* __restrict__ S0, float* __restrict__ ST, int H,
                                                  int NC, GdnWs p) {
  using G = GP<DK, DV>;
  constexpr int RS = kRows, PR = RS + 1;
  extern __shared__ float gsm[];
  float* Ws = gsm;                  // [C][PK]
  float* Kes = Ws + C * G::PK;      // [C][PK]
  float* Ss = Kes + C * G::PK;      // [RS][PK] state rows
  float* Us = Ss + RS * G::PK;      // [C][PR]
  float* gcs = Us + C * PR;         // [DK]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * RS, h = blockIdx.y, bb = blockIdx.z;
  const size_t unit = (size_t)bb * H + h;
  for (int e = tid; e < RS * DK; e += 256) {
    const int r = e / DK, j = e % DK;
    Ss[r * G::PK + j] = S0 ? S0[(unit * DV + r0 + r) * DK + j] : 0.f;
  }
  for (int n = 0; n < NC; ++n) {
    const size_t ch = unit * NC + n;
    for (int e = tid; e < C * DK; e += 256) {
      const int t = e / DK, j = e % DK;
      Ws[t * G::PK + j] = p.W[ch * C * DK + e];
      Kes[t * G::PK + j] = p.Ke[ch * C * DK + e];
    }
    for (int e = tid; e < C * RS; e += 256) {
      const int t = e / RS, r = e % RS;
      Us[t * PR + r] = p.Up[ch * C * DV + t * DV + r0 + r];
    }
    if (tid < DK) gcs[tid] = p.gC[ch * DK + tid];
    __syncthreads();
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      p.S0[ch * DV * DK + (size_t)(r0 + r) * DK + j] = Ss[r * G::PK + j];
    }
    for (int e = tid; e < C * RS; e += 256) {
      const int t = e / RS, r = e % RS;
      float s = Us[t * PR + r];
      for (int j = 0; j < DK; ++j) s = fmaf(-Ws[t * G::PK + j], Ss[r * G::PK + j], s);
      Us[t * PR + r] = s;
      p.U[ch * C * DV + t * DV + r0 + r] = s;
    }
    __syncthreads();
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      float s = Ss[r * G::PK + j] * gcs[j];
      for (int t = 0; t < C; ++t) s = fmaf(Us[t * PR + r], Kes[t * G::PK + j], s);
      Ss[r * G::PK + j] = s;
    }
    __syncthreads();
  }
  if (ST)
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      ST[(unit * DV + r0 + r) * DK + j] = Ss[r * G::PK + j];
    }
}

// ---------------------------------------------------------------------------
// O = Q+ S0^T + P U per chunk, all chunks in parallel.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_out(int H, int T, int NC, GdnWs p, Tin* __restrict__ out) {
  using G = GP<DK, DV>;
  extern __shared__ float gsm[];
  float* Qps = gsm;                 // [C][PK]
  float* S0s = Qps + C * G::PK;     // [DV][PK]
  float* Ps = S0s + DV * G::PK;     // [C][PC]
  float* Uss = Ps + C * G::PC;      // [C][PV]
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;
  for (int e = tid; e < C * DK; e += 256) Qps[(e / DK) * G::PK + e % DK] = p.Qp[ch * C * DK + e];
  for (int e = tid; e < DV * DK; e += 256) S0s[(e / DK) * G::PK + e % DK] = p.S0[ch * DV * DK + e];
  for (int e = tid; e < C * C; e += 256) Ps[(e / C) * G::PC + e % C] = p.P[ch * C * C + e];
  for (int e = tid; e < C * DV; e += 256) Uss[(e / DV) * G::PV + e % DV] = p.U[ch * C * DV + e];
  __syncthreads();
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    if (t >= nv) continue;
    float s = 0.f;
    for (int j = 0; j < DK; ++j) s = fmaf(Qps[t * G::PK + j], S0s[r * G::PK + j], s);
    for (int i = 0; i <= t; ++i) s = fmaf(Ps[t * G::PC + i], Uss[i * G::PV + r], s);
    out[row_bthd(bb, T, t0 + t, H, h, DV) + r] = from_f<Tin>(s);
  }
}

// ---------------------------------------------------------------------------
// Reverse chain: one CTA per (kRows value rows, head); chunks last to first.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_bchain(const Tin* __restrict__ dO, const float* __restrict__ dST,
                                                   float* __restrict__ dS0, int H, int T, int NC, GdnWs p) {
  using G = GP<DK, DV>;
  constexpr int RS = kRows, PR = RS + 1;
  extern __shared__ float gsm[];
  float* Ps = gsm;                  // [C][PC]
  float* Kes = Ps + C * G::PC;      // [C][PK]
  float* Qps = Kes + C * G::PK;     // [C][PK]
  float* Ws = Qps + C * G::PK;      // [C][PK]
  float* dOs = Ws + C * G::PK;      // [C][PR]
  float* dUs = dOs + C * PR;        // [C][PR]
  float* dSs = dUs + C * PR;        // [RS][PK]
  float* gcs = dSs + RS * G::PK;    // [DK]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * RS, h = blockIdx.y, bb = blockIdx.z;
  const size_t unit = (size_t)bb * H + h;
  for (int e = tid; e < RS * DK; e += 256) {
    const int r = e / DK, j = e % DK;
    dSs[r * G::PK + j] = dST ? dST[(unit * DV + r0 + r) * DK + j] : 0.f;
  }
  for (int n = NC - 1; n >= 0; --n) {
    const size_t ch = unit * NC + n;
    const int t0 = n * C, nv = min(C, T - t0);
    for (int e = tid; e < C * C; e += 256) Ps[(e / C) * G::PC + e % C] = p.P[ch * C * C + e];
    for (int e = tid; e < C * DK; e += 256) {
      const int t = e / DK, j = e % DK;
      Kes[t * G::PK + j] = p.Ke[ch * C * DK + e];
      Qps[t * G::PK + j] = p.Qp[ch * C * DK + e];
      Ws[t * G::PK + j] = p.W[ch * C * DK + e];
    }
    for (int e = tid; e < C * RS; e += 256) {
      const int t = e / RS, r = e % RS;
      dOs[t * PR + r] = t < nv ? to_f(dO[row_bthd(bb, T, t0 + t, H, h, DV) + r0 + r]) : 0.f;
    }
    if (tid < DK) gcs[tid] = p.gC[ch * DK + tid];
    __syncthreads();
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      p.dS[ch * DV * DK + (size_t)(r0 + r) * DK + j] = dSs[r * G::PK + j];
    }
    for (int e = tid; e < C * RS; e += 256) {
      const int t = e / RS, r = e % RS;
      float s = 0.f;
      for (int tp = t; tp < C; ++tp) s = fmaf(Ps[tp * G::PC + t], dOs[tp * PR + r], s);
      for (int j = 0; j < DK; ++j) s = fmaf(Kes[t * G::PK + j], dSs[r * G::PK + j], s);
      dUs[t * PR + r] = s;
      p.dU[ch * C * DV + t * DV + r0 + r] = s;
    }
    __syncthreads();
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      float s = dSs[r * G::PK + j] * gcs[j];
      for (int t = 0; t < C; ++t)
        s = fmaf(dOs[t * PR + r], Qps[t * G::PK + j], fmaf(-dUs[t * PR + r], Ws[t * G::PK + j], s));
      dSs[r * G::PK + j] = s;
    }
    __syncthreads();
  }
  if (dS0)
    for (int e = tid; e < RS * DK; e += 256) {
      const int r = e / DK, j = e % DK;
      dS0[(unit * DV + r0 + r) * DK + j] = dSs[r * G::PK + j];
    }
}

// ---------------------------------------------------------------------------
// Per chunk: dP, dZ (-> dv, dw), dW, dE, dT.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_bpost_a(const Tin* __restrict__ v, const float* __restrict__ wg,
                                                    const Tin* __restrict__ dO, int H, int T, int NC, GdnWs p,
                                                    Tin* __restrict__ dv, float* __restrict__ dw) {
  using G = GP<DK, DV>;
  extern __shared__ float gsm[];
  float* R1 = gsm;                  // [C][PZ] dO, then dE
  float* R2 = R1 + C * G::PZ;       // [C][PZ] U, then dZ
  float* R3 = R2 + C * G::PZ;       // [C][PZ] dU, then U'
  float* R4 = R3 + C * G::PZ;       // [C][PK] dW, then W
  float* As = R4 + C * G::PK;       // [C][PC]
  float* dPs = As + C * G::PC;      // [C][PC]
  float* dTs = dPs + C * G::PC;     // [C][PC]
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    R1[t * G::PZ + r] = t < nv ? to_f(dO[row_bthd(bb, T, t0 + t, H, h, DV) + r]) : 0.f;
    R2[t * G::PZ + r] = p.U[ch * C * DV + e];
    R3[t * G::PZ + r] = p.dU[ch * C * DV + e];
  }
  for (int e = tid; e < C * C; e += 256) As[(e / C) * G::PC + e % C] = p.A[ch * C * C + e];
  __syncthreads();
  // dP = tril(dO U^T)
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    float s = 0.f;
    if (i <= t)
      for (int r = 0; r < DV; ++r) s = fmaf(R1[t * G::PZ + r], R2[i * G::PZ + r], s);
    dPs[t * G::PC + i] = s;
  }
  __syncthreads();
  // dZ = A^T dU (A lower triangular) -> dv = dZ w, dw = dZ v;  dW = -dU S0
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    float s = 0.f;
    for (int i = t; i < C; ++i) s = fmaf(As[i * G::PC + t], R3[i * G::PZ + r], s);
    R2[t * G::PZ + r] = s;
    if (t < nv) {
      const size_t g = row_bthd(bb, T, t0 + t, H, h, DV) + r;
      dv[g] = from_f<Tin>(s * wg[g]);
      dw[g] = s * to_f(v[g]);
    }
  }
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    float s = 0.f;
    for (int r = 0; r < DV; ++r) s = fmaf(R3[t * G::PZ + r], p.S0[ch * DV * DK + (size_t)r * DK + j], s);
    R4[t * G::PK + j] = -s;
  }
  __syncthreads();
  // dE = A^T dW
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    float s = 0.f;
    for (int i = t; i < C; ++i) s = fmaf(As[i * G::PC + t], R4[i * G::PK + j], s);
    R1[t * G::PZ + j] = s;
    p.dE[ch * C * DK + e] = s;
  }
  __syncthreads();
  for (int e = tid; e < C * DV; e += 256) R3[(e / DV) * G::PZ + e % DV] = p.Up[ch * C * DV + e];
  for (int e = tid; e < C * DK; e += 256) R4[(e / DK) * G::PK + e % DK] = p.W[ch * C * DK + e];
  __syncthreads();
  // dT = -tril(dZ U'^T + dE W^T, -1)
  for (int e = tid; e < C * C; e += 256) {
    const int t = e / C, i = e % C;
    float s = 0.f;
    if (i < t) {
      for (int r = 0; r < DV; ++r) s = fmaf(R2[t * G::PZ + r], R3[i * G::PZ + r], s);
      for (int j = 0; j < DK; ++j) s = fmaf(R1[t * G::PZ + j], R4[i * G::PK + j], s);
    }
    dTs[t * G::PC + i] = -s;
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += 256) {
    p.dT[ch * C * C + e] = dTs[(e / C) * G::PC + e % C];
    p.dP[ch * C * C + e] = dPs[(e / C) * G::PC + e % C];
  }
}

// ---------------------------------------------------------------------------
// Per chunk: dq, dk, db, dloga.  Thread e handles (t, j) with j = e % DK fixed
// per thread (256 is a multiple of DK).
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) gdn2_bpost_b(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                    const float* __restrict__ bg, const float* __restrict__ loga,
                                                    const Tin* __restrict__ dO, int H, int T, int NC, GdnWs p,
                                                    Tin* __restrict__ dq, Tin* __restrict__ dk,
                                                    float* __restrict__ db, float* __restrict__ dloga) {
  using G = GP<DK, DV>;
  constexpr int TPJ = 256 / DK;     // threads sharing one key channel
  extern __shared__ float gsm[];
  float* Ls = gsm;                  // [C][PK]
  float* Ks = Ls + C * G::PK;       // [C][PK]
  float* Qs = Ks + C * G::PK;       // [C][PK]
  float* Es = Qs + C * G::PK;       // [C][PK]  e = b o k
  float* dLs = Es + C * G::PK;      // [C][PK]
  float* dPs = dLs + C * G::PK;     // [C][PC]
  float* dTs = dPs + C * G::PC;     // [C][PC]
  float* red = dTs + C * G::PC;     // [TPJ][DK]
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
    const float kk = ok ? to_f(k[g]) : 0.f;
    Ks[t * G::PK + j] = kk;
    Qs[t * G::PK + j] = ok ? to_f(q[g]) : 0.f;
    Es[t * G::PK + j] = ok ? bg[g] * kk : 0.f;
    Ls[t * G::PK + j] = ok ? loga[g] : 0.f;
  }
  for (int e = tid; e < C * C; e += 256) {
    dPs[(e / C) * G::PC + e % C] = p.dP[ch * C * C + e];
    dTs[(e / C) * G::PC + e % C] = p.dT[ch * C * C + e];
  }
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * G::PK + tid];
      Ls[t * G::PK + tid] = acc;
    }
  }
  __syncthreads();
  const int j = tid % DK;
  const float Lam = Ls[(C - 1) * G::PK + j];
  float lam_part = 0.f;  // sum over this thread's t of dK^e o K^e
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK;
    const float L = Ls[t * G::PK + j], gm = expf(L), ke = expf(Lam - L);
    const float kk = Ks[t * G::PK + j], qq = Qs[t * G::PK + j], ee = Es[t * G::PK + j];
    float dQp = 0.f, dKe = 0.f;
    const size_t orow = row_bthd(bb, T, t0 + t, H, h, DV);
    for (int r = 0; r < DV; ++r) {
      const float go = t < nv ? to_f(dO[orow + r]) : 0.f;
      dQp = fmaf(go, p.S0[ch * DV * DK + (size_t)r * DK + j], dQp);
      dKe = fmaf(p.U[ch * C * DV + t * DV + r], p.dS[ch * DV * DK + (size_t)r * DK + j], dKe);
    }
    const float dEv = p.dE[ch * C * DK + e];
    float dee = dEv * gm, dqq = dQp * gm, dkk = dKe * ke;
    float dL = dEv * ee * gm + dQp * qq * gm - dKe * kk * ke;
    lam_part = fmaf(dKe, kk * ke, lam_part);
    // this position as the later token t of a pair (i <= t)
    for (int i = 0; i <= t; ++i) {
      const float ki = Ks[i * G::PK + j] * expf(L - Ls[i * G::PK + j]);
      const float dTti = dTs[t * G::PC + i], dPti = dPs[t * G::PC + i];
      dee = fmaf(dTti, ki, dee);
      dqq = fmaf(dPti, ki, dqq);
      dL = fmaf(dTti * ee + dPti * qq, ki, dL);
    }
    // this position as the earlier token i of a pair (t' >= i)
    for (int tp = t; tp < C; ++tp) {
      const float wgt = expf(Ls[tp * G::PK + j] - L);
      const float side = dTs[tp * G::PC + t] * Es[tp * G::PK + j] + dPs[tp * G::PC + t] * Qs[tp * G::PK + j];
      dkk = fmaf(side, wgt, dkk);
      dL = fmaf(-side * kk, wgt, dL);
    }
    dLs[t * G::PK + j] = dL;
    if (t < nv) {
      const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
      dq[g] = from_f<Tin>(dqq);
      dk[g] = from_f<Tin>(fmaf(dee, bg[g], dkk));
      db[g] = dee * kk;
    }
  }
  red[(tid / DK) * DK + j] = lam_part;
  __syncthreads();
  if (tid < DK) {
    float lam = 0.f;
    for (int s = 0; s < TPJ; ++s) lam += red[s * DK + tid];
    float st = 0.f;
    for (int r = 0; r < DV; ++r)
      st = fmaf(p.dS[ch * DV * DK + (size_t)r * DK + tid], p.S0[ch * DV * DK + (size_t)r * DK + tid], st);
    lam = fmaf(st, expf(Lam), lam);
    float acc = lam;
    for (int t = C - 1; t >= 0; --t) {
      acc += dLs[t * G::PK + tid];
      if (t < nv) dloga[row_bthd(bb, T, t0 + t, H, h, DK) + tid] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
namespace {

template <int DK, int DV>
struct GSmem {
  using G = GP<DK, DV>;
  static constexpr size_t prep = (size_t)(3 * C * G::PK + C * G::PZ + 2 * C * G::PC) * 4;
  static constexpr size_t chain = (size_t)(2 * C * G::PK + kRows * G::PK + C * (kRows + 1) + DK) * 4;
  static constexpr size_t out = (size_t)(C * G::PK + DV * G::PK + C * G::PC + C * G::PV) * 4;
  static constexpr size_t bchain =
      (size_t)(C * G::PC + 3 * C * G::PK + 2 * C * (kRows + 1) + kRows * G::PK + DK) * 4;
  static constexpr size_t bpa = (size_t)(3 * C * G::PZ + C * G::PK + 3 * C * G::PC) * 4;
  static constexpr size_t bpb = (size_t)(5 * C * G::PK + 2 * C * G::PC + 256) * 4;
};

template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define KD_TRYC(x)                              \
  do {                                          \
    cudaError_t e_ = (x);                       \
    if (e_ != cudaSuccess) return e_;           \
  } while (0)

template <int DK, int DV, typename Tin>
cudaError_t gdn2_fwd_t(const GdnArgs& a, cudaStream_t st) {
  using S = GSmem<DK, DV>;
  const GdnLayout& L = a.L;
  const GdnWs p = gdn_ws(a.ws, L);
  const dim3 gc(L.NC, L.H, L.B), gr(DV / kRows, L.H, L.B);
  KD_TRYC(set_smem(gdn2_prep<DK, DV, Tin>, S::prep));
  KD_TRYC(set_smem(gdn2_chain<DK, DV>, S::chain));
  KD_TRYC(set_smem(gdn2_out<DK, DV, Tin>, S::out));
  prof_begin(st, "gdn2_prep");
  gdn2_prep<DK, DV, Tin><<<gc, 256, S::prep, st>>>(static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
                                                   static_cast<const Tin*>(a.v), a.b, a.w, a.loga, L.H, L.T, L.NC, p);
  prof_end(st);
  KD_TRYC(cudaGetLastError());
  prof_begin(st, "gdn2_chain");
  gdn2_chain<DK, DV><<<gr, 256, S::chain, st>>>(a.S0, a.ST, L.H, L.NC, p);
  prof_end(st);
  KD_TRYC(cudaGetLastError());
  prof_begin(st, "gdn2_out");
  gdn2_out<DK, DV, Tin><<<gc, 256, S::out, st>>>(L.H, L.T, L.NC, p, static_cast<Tin*>(a.out));
  prof_end(st);
  return cudaGetLastError();
}

template <int DK, int DV, typename Tin>
cudaError_t gdn2_bwd_t(const GdnArgs& a, cudaStream_t st) {
  using S = GSmem<DK, DV>;
  const GdnLayout& L = a.L;
  GdnWs p = gdn_ws(const_cast<char*>(a.fws), L);
  gdn_bwd_ws(a.ws, L, &p);
  const dim3 gc(L.NC, L.H, L.B), gr(DV / kRows, L.H, L.B);
  KD_TRYC(set_smem(gdn2_bchain<DK, DV, Tin>, S::bchain));
  KD_TRYC(set_smem(gdn2_bpost_a<DK, DV, Tin>, S::bpa));
  KD_TRYC(set_smem(gdn2_bpost_b<DK, DV, Tin>, S::bpb));
  const Tin* dO = static_cast<const Tin*>(a.dO);
  prof_begin(st, "gdn2_bchain");
  gdn2_bchain<DK, DV, Tin><<<gr, 256, S::bchain, st>>>(dO, a.dST, a.dS0, L.H, L.T, L.NC, p);
  prof_end(st);
  KD_TRYC(cudaGetLastError());
  prof_begin(st, "gdn2_bpost_a");
  gdn2_bpost_a<DK, DV, Tin><<<gc, 256, S::bpa, st>>>(static_cast<const Tin*>(a.v), a.w, dO, L.H, L.T, L.NC, p,
                                                     static_cast<Tin*>(a.dv), a.dw);
  prof_end(st);
  KD_TRYC(cudaGetLastError());
  prof_begin(st, "gdn2_bpost_b");
  gdn2_bpost_b<DK, DV, Tin><<<gc, 256, S::bpb, st>>>(static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
                                                     a.b, a.loga, dO, L.H, L.T, L.NC, p, static_cast<Tin*>(a.dq),
                                                     static_cast<Tin*>(a.dk), a.db, a.dloga);
  prof_end(st);
  return cudaGetLastError();
}

template <bool BWD, typename Tin>
cudaError_t gdn2_dispatch(const GdnArgs& a, cudaStream_t st) {
#define KD_G(DK_, DV_)                                                                          \
  if (a.L.dk == DK_ && a.L.dv == DV_) return BWD ? gdn2_bwd_t<DK_, DV_, Tin>(a, st) : gdn2_fwd_t<DK_, DV_, Tin>(a, st);
  KD_G(32, 32) KD_G(32, 64) KD_G(32, 128)
  KD_G(64, 32) KD_G(64, 64) KD_G(64, 128)
  KD_G(128, 32) KD_G(128, 64) KD_G(128, 128)
#undef KD_G
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gdn2_fwd(const GdnArgs& a, cudaStream_t st) {
  return a.L.dtype == 0 ? gdn2_dispatch<false, float>(a, st) : gdn2_dispatch<false, __nv_bfloat16>(a, st);
}

cudaError_t launch_gdn2_bwd(const GdnArgs& a, cudaStream_t st) {
  return a.L.dtype == 0 ? gdn2_dispatch<true, float>(a, st) : gdn2_dispatch<true, __nv_bfloat16>(a, st);
}

}  // namespace kd
