// kd_bwd_simt.cu -- chunk-parallel backward on CUDA cores (fp32 FFMA).
//
// Reverse-mode of the chunk equations of the forward (see kd_fwd_simt.cu).
// The pages only say the backward must route the gradient through every gate
// product (Gated DeltaNet-2 article, "핵심 기여": gate-aware backward); the
// equations below are derived here.  Per chunk, with dS the gradient of the
// chunk-end state, g = A^T du, db0 = -beta o g:
//   du_i  = sum_{t>=i} P[t,i] (dO_t.v_i) + v_i^T dS K^e_i
//   dS0   = dS diag(gamma_C) + dO^T Q+ + V^T diag(db0) K+        (next dS)
//   dP[t,i] = u_i (dO_t.v_i) (i<=t);  dM[t,i] = -beta_t g_t u_i (i<t)
//   dG_K = dM o G_V;  dG_V = dM o G_K;  dbeta = -g o (b0 + M u);  dc = g
//   dq = (dO S0) o gamma + gamma o (dP K-)
//   dk = db0 o (V S0) o gamma + u o (V dS) o e^{L_C-L} + (dP^T Q+)/gamma
//        + gamma o (dG_K K-) + (dG_K^T K+)/gamma
//   dv = db0 o (K+ S0^T) + u o (K^e dS^T) + u o (P^T dO) + (dG_V + dG_V^T) V
//   dL = the matching decay terms; dlogf = reverse cumulative sum of dL.
// (K- = k / gamma.)
//
// Kernels: (1) reverse chain over chunks, one CTA per head: per-chunk dS and
// g; (2) C x C adjoints per chunk; (3) state products per chunk; (4) the
// intra-chunk products and the final gradients per chunk.
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

constexpr int C = kChunk;

// ---------------------------------------------------------------------------
// (1) reverse chain
// ---------------------------------------------------------------------------
template <int DK, int DV>
constexpr size_t bchain_smem_floats() {
  return 3 * (size_t)C * DK + 2 * (size_t)C * DV + 2 * (size_t)C * (C + 1) + 2 * DK + 4 * C +
         (DV / 16) * C;
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(2 * DV) bwd_chain_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ logf, const Tin* __restrict__ dO,
    const float* __restrict__ dST, int H, int T, int NC, const float* __restrict__ wA,
    const float* __restrict__ wP, float* __restrict__ dS0out, float* __restrict__ wdSC,
    float* __restrict__ wg) {
  constexpr int HK = DK / 2, SC = C + 1;
  extern __shared__ float smem[];
  float* Kp = smem;            // [C][DK]
  float* Qp = Kp + C * DK;     // [C][DK]
  float* Ke = Qp + C * DK;     // log decay prefix L, then K^e  [C][DK]
  float* Vs = Ke + C * DK;     // [C][DV]
  float* Ds = Vs + C * DV;     // dO [C][DV]
  float* As = Ds + C * DV;     // [C][SC]
  float* Ps = As + C * SC;     // [C][SC]
  float* lCs = Ps + C * SC;    // L at the chunk end [DK]
  float* gC = lCs + DK;        // exp of it [DK]
  float* bs = gC + DK;
  float* dus = bs + C;
  float* db0s = dus + C;
  float* wpart = db0s + C;     // per-warp partial sums of du [DV/16][C]
  constexpr int NW = DV / 16;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int r = tid >> 1, hh = tid & 1, lane = tid & 31, warp = tid >> 5;
  const size_t unit = (size_t)b * H + h;

  float dS[HK];
#pragma unroll
  for (int m = 0; m < HK; ++m) dS[m] = dST ? dST[unit * DV * DK + (size_t)r * DK + 2 * m + hh] : 0.f;

  for (int n = NC - 1; n >= 0; --n) {
    const int t0 = n * C;
    const int nv = min(C, T - t0);
    const size_t ch = unit * NC + n;
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int t = e / DK, j = e % DK;
      const bool ok = t < nv;
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
      Kp[e] = ok ? to_f(k[g]) : 0.f;
      Qp[e] = ok ? to_f(q[g]) : 0.f;
      Ke[e] = ok ? logf[g] : 0.f;
    }
    for (int e = tid; e < C * DV; e += blockDim.x) {
      const int t = e / DV, rr = e % DV;
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * DV + rr;
      Vs[e] = t < nv ? to_f(v[g]) : 0.f;
      Ds[e] = t < nv ? to_f(dO[g]) : 0.f;
    }
    for (int e = tid; e < C * C; e += blockDim.x) {
      As[(e / C) * SC + (e % C)] = wA[ch * C * C + e];
      Ps[(e / C) * SC + (e % C)] = wP[ch * C * C + e];
    }
    if (tid < C) {
      bs[tid] = tid < nv ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
    }
    __syncthreads();
    for (int j = tid; j < DK; j += blockDim.x) {
      float acc = 0.f;
      for (int t = 0; t < C; ++t) {
        acc += Ke[t * DK + j];
        Ke[t * DK + j] = acc;
      }
      lCs[j] = acc;
      gC[j] = expf(acc);
    }
    __syncthreads();
    // each element is read (as L) and rewritten (as K^e) by the same thread
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int j = e % DK;
      const float l = Ke[e], lC = lCs[j];
      const float ep = expf(l), kk = Kp[e];
      Kp[e] = kk * ep;
      Ke[e] = kk * expf(lC - l);
      Qp[e] *= ep;
    }
    __syncthreads();

    // du_i = sum_r V[i,r] ( (dS K^e^T)[r,i] + (P^T dO)[i,r] )
    for (int i = 0; i < C; ++i) {
      float z = 0.f;
#pragma unroll
      for (int m = 0; m < HK; ++m) z = fmaf(dS[m], Ke[i * DK + 2 * m + hh], z);
      float w = 0.f;
      for (int t = i + hh; t < C; t += 2) w = fmaf(Ps[t * SC + i], Ds[t * DV + r], w);
      z += __shfl_xor_sync(0xffffffffu, z, 1);
      w += __shfl_xor_sync(0xffffffffu, w, 1);
      float p = hh == 0 ? Vs[i * DV + r] * (z + w) : 0.f;
      p = warp_sum(p);
      if (lane == 0) wpart[warp * C + i] = p;
    }
    __syncthreads();
    if (tid < C) {
      float s = 0.f;
      for (int w = 0; w < NW; ++w) s += wpart[w * C + tid];  // fixed order: deterministic
      dus[tid] = s;
    }
    __syncthreads();
    if (tid < C) {
      float gsum = 0.f;
      for (int t = tid; t < C; ++t) gsum = fmaf(As[t * SC + tid], dus[t], gsum);
      db0s[tid] = -bs[tid] * gsum;
      wg[ch * C + tid] = gsum;
    }
#pragma unroll
    for (int m = 0; m < HK; ++m) wdSC[ch * DV * DK + (size_t)r * DK + 2 * m + hh] = dS[m];
    __syncthreads();
    // dS <- dS diag(gamma_C) + dO^T Q+ + V^T diag(db0) K+
#pragma unroll
    for (int m = 0; m < HK; ++m) dS[m] *= gC[2 * m + hh];
    for (int t = 0; t < C; ++t) {
      const float a1 = Ds[t * DV + r], a2 = db0s[t] * Vs[t * DV + r];
#pragma unroll
      for (int m = 0; m < HK; ++m)
        dS[m] = fmaf(a1, Qp[t * DK + 2 * m + hh], fmaf(a2, Kp[t * DK + 2 * m + hh], dS[m]));
    }
    __syncthreads();
  }
  if (dS0out) {
#pragma unroll
    for (int m = 0; m < HK; ++m) dS0out[unit * DV * DK + (size_t)r * DK + 2 * m + hh] = dS[m];
  }
}

// ---------------------------------------------------------------------------
// (2) C x C adjoints: dP, dG_K, dG_V + dG_V^T; dbeta, dc
// ---------------------------------------------------------------------------
template <int DK, int DV>
constexpr size_t bcc_smem_floats() {
  return 3 * (size_t)C * (DK + 1) + 2 * (size_t)C * (DV + 1) + (size_t)C * (C + 1) + 4 * C;
}

// Stage bodies take the chunk (n, h, b) and the scratch slot their dP, dG_K,
// dG_V' and accumulator tiles use: the chunk index on the CUDA-core path,
// a per-CTA slot in the tensor-core path's exact kernel.
template <int DK, int DV, typename Tin>
__device__ __forceinline__ void bwd_cc_body(
    int n, int h, int b, size_t slot,
    const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ beta,
    const float* __restrict__ logf, const Tin* __restrict__ dO,
    int H, int T, int NC, const float* __restrict__ wu, const float* __restrict__ wb0, const float* __restrict__ wg,
    float* __restrict__ dbeta, float* __restrict__ dc, float* __restrict__ wdP,
    float* __restrict__ wdGK, float* __restrict__ wdGVs) {
  constexpr int SK = DK + 1, SV = DV + 1, SC = C + 1;
  extern __shared__ float smem[];
  float* Kp = smem;            // [C][SK]
  float* Km = Kp + C * SK;     // raw k, then k / gamma
  float* Ls = Km + C * SK;
  float* Vs = Ls + C * SK;     // [C][SV]
  float* Ds = Vs + C * SV;     // dO
  float* dGV = Ds + C * SV;    // [C][SC]
  float* us = dGV + C * SC;
  float* gs = us + C;
  float* bs = gs + C;
  float* b0s = bs + C;
  __shared__ int unsafe;
  const int tid = threadIdx.x;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)b * H + h) * NC + n;

  for (int e = tid; e < C * DK; e += blockDim.x) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
    Km[t * SK + j] = ok ? to_f(k[g]) : 0.f;
    Ls[t * SK + j] = ok ? logf[g] : 0.f;
  }
  for (int e = tid; e < C * DV; e += blockDim.x) {
    const int t = e / DV, rr = e % DV;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DV + rr;
    Vs[t * SV + rr] = t < nv ? to_f(v[g]) : 0.f;
    Ds[t * SV + rr] = t < nv ? to_f(dO[g]) : 0.f;
  }
  if (tid < C) {
    us[tid] = wu[ch * C + tid];
    gs[tid] = wg[ch * C + tid];
    b0s[tid] = wb0[ch * C + tid];
    bs[tid] = tid < nv ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
  }
  if (tid == 0) unsafe = 0;
  __syncthreads();
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
      const float l = Ls[t * SK + j], kk = Km[t * SK + j];
      Kp[t * SK + j] = kk * expf(l);
      Km[t * SK + j] = kk * expf(-l);
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < C; t += 8) {
    float brow = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int i = lane + 32 * half;
      float gk = 0.f, gv = 0.f, dov = 0.f;
      if (i < t) {
        if (safe) {
          for (int j = 0; j < DK; ++j) gk = fmaf(Kp[t * SK + j], Km[i * SK + j], gk);
        } else {
          for (int j = 0; j < DK; ++j)
            gk = fmaf(Km[t * SK + j] * Km[i * SK + j], expf(Ls[t * SK + j] - Ls[i * SK + j]), gk);
        }
      }
      for (int rr = 0; rr < DV; ++rr) {
        gv = fmaf(Vs[t * SV + rr], Vs[i * SV + rr], gv);
        dov = fmaf(Ds[t * SV + rr], Vs[i * SV + rr], dov);
      }
      const float mm = i < t ? gk * gv : 0.f;
      brow = fmaf(mm, us[i], brow);
      const float dM = i < t ? -bs[t] * gs[t] * us[i] : 0.f;
      wdP[slot * C * C + t * C + i] = i <= t ? us[i] * dov : 0.f;
      wdGK[slot * C * C + t * C + i] = dM * gv;
      dGV[t * SC + i] = dM * gk;
    }
    brow = warp_sum(brow);
    if (lane == 0 && t < nv) {
      const size_t g = ((size_t)b * T + t0 + t) * H + h;
      dc[g] = gs[t];
      dbeta[g] = -gs[t] * (b0s[t] + brow);
    }
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += blockDim.x) {
    const int t = e / C, i = e % C;
    wdGVs[slot * C * C + e] = dGV[t * SC + i] + dGV[i * SC + t];
  }
}

// ---------------------------------------------------------------------------
// (3) state products: dO S0, V S0, V dS (C x dk) and K+ S0^T, K^e dS^T (C x dv)
// ---------------------------------------------------------------------------
constexpr int SLAB = 16;

// float index of (r, j) in a 128x128 tf32 tile stored K-major with 128-byte
// swizzle: 4 blocks of 32 columns, 1024-byte atoms of 8 rows, 16-byte chunks
// permuted by XOR with (row % 8)
__device__ __forceinline__ size_t sw128_index(int r, int j) {
  const int kb = j >> 5, chunk = (j & 31) >> 2;
  return (size_t)kb * 128 * 32 + (size_t)(r >> 3) * 256 + (size_t)(r & 7) * 32 +
         (size_t)(((chunk ^ (r & 7)) & 7) * 4) + (j & 3);
}

// byte offset of (r, j) in a 128x128 bf16 tile stored K-major with 128-byte
// swizzle: 2 blocks of 64 columns, 1024-byte atoms of 8 rows
__device__ __forceinline__ size_t sw128_bf16_off(int r, int j) {
  const int kb = j >> 6, chunk = (j & 63) >> 3;
  return (size_t)kb * 128 * 128 + (size_t)(r >> 3) * 1024 + (size_t)(r & 7) * 128 +
         (size_t)(((chunk ^ (r & 7)) & 7) * 16) + (size_t)(j & 7) * 2;
}

template <int DK, int DV>
constexpr size_t bstate_smem_floats() {
  return 3 * (size_t)C * (DK + 1) + 2 * (size_t)C * (DV + 1) + 2 * (size_t)SLAB * (DK + 1) + 2 * C +
         3 * DK + (256 / DK) * DK;
}

template <int DK, int DV, typename Tin>
__device__ __forceinline__ void bwd_state_body(
    int n, int h, int b, size_t slot,
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ logf, const Tin* __restrict__ dO, int H, int T, int NC, const float* __restrict__ wu, const float* __restrict__ wg,
    const float* __restrict__ wS0, const float* __restrict__ wdSC, float* __restrict__ waccq,
    float* __restrict__ wacck, float* __restrict__ waccL, float* __restrict__ waccv, int s0_swizzled,
    const __nv_bfloat16* __restrict__ wdSb) {
  constexpr int SK = DK + 1, SV = DV + 1;
  constexpr int TPJ = 256 / DK;   // thread groups over j
  constexpr int TPG = C / TPJ;    // rows per group
  extern __shared__ float smem[];
  float* Kp = smem;               // [C][SK]
  float* Ke = Kp + C * SK;
  float* Ls = Ke + C * SK;
  float* Ds = Ls + C * SK;        // [C][SV]
  float* Vs = Ds + C * SV;
  float* S0s = Vs + C * SV;       // [SLAB][SK]
  float* dSs = S0s + SLAB * SK;
  float* us = dSs + SLAB * SK;    // [C]
  float* db0s = us + C;
  float* csum = db0s + C;         // [DK]
  float* gC = csum + DK;          // [DK]
  float* lastL = gC + DK;         // [DK]
  float* ekL = lastL + DK;        // per-group partials [256/DK][DK]
  const int tid = threadIdx.x;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)b * H + h) * NC + n;

  for (int e = tid; e < C * DK; e += blockDim.x) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
    Kp[t * SK + j] = ok ? to_f(k[g]) : 0.f;
    Ls[t * SK + j] = ok ? logf[g] : 0.f;
  }
  for (int e = tid; e < C * DV; e += blockDim.x) {
    const int t = e / DV, rr = e % DV;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DV + rr;
    Vs[t * SV + rr] = t < nv ? to_f(v[g]) : 0.f;
    Ds[t * SV + rr] = t < nv ? to_f(dO[g]) : 0.f;
  }
  if (tid < C) {
    us[tid] = wu[ch * C + tid];
    const float bt = tid < nv ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
    db0s[tid] = -bt * wg[ch * C + tid];
  }
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * SK + tid];
      Ls[t * SK + tid] = acc;
    }
    gC[tid] = expf(acc);
  }
  __syncthreads();
  for (int e = tid; e < C * DK; e += blockDim.x) {
    const int t = e / DK, j = e % DK;
    const float l = Ls[t * SK + j], lC = Ls[(C - 1) * SK + j], kk = Kp[t * SK + j];
    Kp[t * SK + j] = kk * expf(l);
    Ke[t * SK + j] = kk * expf(lC - l);
  }
  __syncthreads();

  const int j = tid % DK, tq = tid / DK;
  float aQ[TPG], aVS[TPG], aVD[TPG];
#pragma unroll
  for (int i = 0; i < TPG; ++i) aQ[i] = aVS[i] = aVD[i] = 0.f;
  float cs_local = 0.f;
  const float* S0c = wS0 + ch * DV * DK;
  const float* dSc = wdSb ? nullptr : wdSC + ch * DV * DK;
  // the tensor-core path keeps dS as a bf16 tile [r][j], 128-byte-swizzled K-major
  const unsigned char* dSt = wdSb ? reinterpret_cast<const unsigned char*>(wdSb + ch * DV * DK) : nullptr;
  for (int r0 = 0; r0 < DV; r0 += SLAB) {
    for (int e = tid; e < SLAB * DK; e += blockDim.x) {
      const int rr = e / DK, jj = e % DK;
      // the tensor-core forward stores each chunk-start state as a 128x128
      // tf32 tile in the 128-byte-swizzled K-major layout of its MMAs
      S0s[rr * SK + jj] = s0_swizzled ? S0c[sw128_index(r0 + rr, jj)] : S0c[(size_t)(r0 + rr) * DK + jj];
      dSs[rr * SK + jj] = dSt ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                     dSt + sw128_bf16_off(r0 + rr, jj)))
                              : dSc[(size_t)(r0 + rr) * DK + jj];
    }
    __syncthreads();
    // C x dk products, accumulated over all slabs
    for (int rr = 0; rr < SLAB; ++rr) {
      const float s0 = S0s[rr * SK + j], ds = dSs[rr * SK + j];
      cs_local = fmaf(s0, ds, cs_local);
#pragma unroll
      for (int i = 0; i < TPG; ++i) {
        const int t = tq * TPG + i;
        const float vt = Vs[t * SV + r0 + rr];
        aQ[i] = fmaf(Ds[t * SV + r0 + rr], s0, aQ[i]);
        aVS[i] = fmaf(vt, s0, aVS[i]);
        aVD[i] = fmaf(vt, ds, aVD[i]);
      }
    }
    // C x dv products for this slab's rows
    {
      const int rr = tid & 15, tg = tid >> 4;
      for (int t = tg; t < C; t += 16) {
        float kps = 0.f, keds = 0.f;
        for (int jj = 0; jj < DK; ++jj) {
          kps = fmaf(Kp[t * SK + jj], S0s[rr * SK + jj], kps);
          keds = fmaf(Ke[t * SK + jj], dSs[rr * SK + jj], keds);
        }
        waccv[slot * C * DV + (size_t)t * DV + r0 + rr] = db0s[t] * kps + us[t] * keds;
      }
    }
    __syncthreads();
  }
  if (tq == 0) csum[j] = cs_local;
  float ek = 0.f;
#pragma unroll
  for (int i = 0; i < TPG; ++i) {
    const int t = tq * TPG + i;
    const float l = Ls[t * SK + j];
    const float gam = expf(l), eC = expf(Ls[(C - 1) * SK + j] - l);
    const float qv = t < nv ? to_f(q[(((size_t)b * T + t0 + t) * H + h) * DK + j]) : 0.f;
    const float dKp = db0s[t] * aVS[i], dKe = us[t] * aVD[i];
    const size_t o = slot * C * DK + (size_t)t * DK + j;
    waccq[o] = aQ[i] * gam;
    wacck[o] = dKp * gam + dKe * eC;
    const float keT = Ke[t * SK + j];
    const float dl = aQ[i] * qv * gam + dKp * Kp[t * SK + j] - dKe * keT;
    ek = fmaf(dKe, keT, ek);
    if (t == C - 1) lastL[j] = dl;
    else waccL[o] = dl;
  }
  ekL[tq * DK + j] = ek;
  __syncthreads();
  if (tid < DK) {
    float e = 0.f;
    for (int g2 = 0; g2 < TPJ; ++g2) e += ekL[g2 * DK + tid];  // fixed order: deterministic
    waccL[slot * C * DK + (size_t)(C - 1) * DK + tid] = lastL[tid] + e + gC[tid] * csum[tid];
  }
}

// ---------------------------------------------------------------------------
// (4) intra-chunk products and final gradients
// ---------------------------------------------------------------------------
template <int DK, int DV>
constexpr size_t bintra_smem_floats() {
  const size_t a = 2 * (size_t)C * (C + 1) + 2 * (size_t)C * (DV + 1);
  const size_t b = 4 * (size_t)C * (DK + 1) + 2 * (size_t)C * (C + 1);
  return (a > b ? a : b) + C;
}

template <int DK, int DV, typename Tin>
__device__ __forceinline__ void bwd_intra_body(
    int n, int h, int b, size_t slot,
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ logf, float ga, const Tin* __restrict__ dO,
    int H, int T, int NC,
    const float* __restrict__ wP, const float* __restrict__ wu, const float* __restrict__ wdP,
    const float* __restrict__ wdGK, const float* __restrict__ wdGVs,
    const float* __restrict__ waccq, const float* __restrict__ wacck,
    const float* __restrict__ waccL, const float* __restrict__ waccv, Tin* __restrict__ dq,
    Tin* __restrict__ dk, Tin* __restrict__ dv, float* __restrict__ dlogf, float* __restrict__ dapart) {
  constexpr int SK = DK + 1, SV = DV + 1, SC = C + 1;
  extern __shared__ float smem[];
  float* us = smem;            // [C]
  float* base = smem + C;
  __shared__ int unsafe;
  const int tid = threadIdx.x;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)b * H + h) * NC + n;

  // ---- phase A: dv = accv + u o (P^T dO) + (dG_V + dG_V^T) V
  {
    float* Ps = base;              // [C][SC]
    float* Gs = Ps + C * SC;       // dG_V + dG_V^T
    float* Vs = Gs + C * SC;       // [C][SV]
    float* Ds = Vs + C * SV;
    for (int e = tid; e < C * C; e += blockDim.x) {
      Ps[(e / C) * SC + e % C] = wP[ch * C * C + e];
      Gs[(e / C) * SC + e % C] = wdGVs[slot * C * C + e];
    }
    for (int e = tid; e < C * DV; e += blockDim.x) {
      const int t = e / DV, rr = e % DV;
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * DV + rr;
      Vs[t * SV + rr] = t < nv ? to_f(v[g]) : 0.f;
      Ds[t * SV + rr] = t < nv ? to_f(dO[g]) : 0.f;
    }
    if (tid < C) us[tid] = wu[ch * C + tid];
    if (tid == 0) unsafe = 0;
    __syncthreads();
    constexpr int NG = 256 / DV, IPG = C / NG;
    const int rr = tid % DV, gi = tid / DV;
    for (int ii = 0; ii < IPG; ++ii) {
      const int i = gi * IPG + ii;
      float a = 0.f, s = 0.f;
      for (int t = i; t < C; ++t) a = fmaf(Ps[t * SC + i], Ds[t * SV + rr], a);
      for (int t = 0; t < C; ++t) s = fmaf(Gs[i * SC + t], Vs[t * SV + rr], s);
      if (i < nv) {
        const size_t o = (((size_t)b * T + t0 + i) * H + h) * DV + rr;
        dv[o] = from_f<Tin>(waccv[slot * C * DV + (size_t)i * DV + rr] + us[i] * a + s);
      }
    }
    __syncthreads();
  }
  // ---- phase B: dq, dk, dlogf
  float* Km = base;             // raw k, then k / gamma   [C][SK]
  float* Kp = Km + C * SK;      // k o gamma
  float* Qp = Kp + C * SK;      // raw q, then q o gamma
  float* Ls = Qp + C * SK;      // L, later dL
  float* dPs = Ls + C * SK;     // [C][SC]
  float* dGs = dPs + C * SC;    // dG_K
  for (int e = tid; e < C * DK; e += blockDim.x) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
    Km[t * SK + j] = ok ? to_f(k[g]) : 0.f;
    Qp[t * SK + j] = ok ? to_f(q[g]) : 0.f;
    Ls[t * SK + j] = ok ? logf[g] : 0.f;
  }
  for (int e = tid; e < C * C; e += blockDim.x) {
    dPs[(e / C) * SC + e % C] = wdP[slot * C * C + e];
    dGs[(e / C) * SC + e % C] = wdGK[slot * C * C + e];
  }
  __syncthreads();
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
  // raw values of this thread's rows are needed for dL: keep them
  constexpr int TPJ = 256 / DK, TPG = C / TPJ;
  const int j = tid % DK, tq = tid / DK;
  float qraw[TPG], kraw[TPG], lrow[TPG];
#pragma unroll
  for (int i = 0; i < TPG; ++i) {
    const int t = tq * TPG + i;
    qraw[i] = Qp[t * SK + j];
    kraw[i] = Km[t * SK + j];
    lrow[i] = Ls[t * SK + j];
  }
  __syncthreads();
  if (safe) {
    for (int e = tid; e < C * DK; e += blockDim.x) {
      const int t = e / DK, jj = e % DK;
      const float l = Ls[t * SK + jj], ep = expf(l), kk = Km[t * SK + jj];
      Kp[t * SK + jj] = kk * ep;
      Km[t * SK + jj] = kk * expf(-l);
      Qp[t * SK + jj] *= ep;
    }
  }
  __syncthreads();
  float dLv[TPG];
#pragma unroll
  for (int i = 0; i < TPG; ++i) {
    const int t = tq * TPG + i;
    float dqP = 0.f, dkG1 = 0.f, dkP = 0.f, dkG2 = 0.f;
    if (safe) {
      for (int s = 0; s < C; ++s) {
        const float km = Km[s * SK + j];
        dqP = fmaf(dPs[t * SC + s], km, dqP);     // dP[t,s], s <= t (masked)
        dkG1 = fmaf(dGs[t * SC + s], km, dkG1);   // dG_K[t,s], s < t
        dkP = fmaf(dPs[s * SC + t], Qp[s * SK + j], dkP);   // dP[s,t], s >= t
        dkG2 = fmaf(dGs[s * SC + t], Kp[s * SK + j], dkG2); // dG_K[s,t], s > t
      }
      const float gam = expf(lrow[i]), igam = expf(-lrow[i]);
      dqP *= gam;
      dkG1 *= gam;
      dkP *= igam;
      dkG2 *= igam;
    } else {
      for (int s = 0; s < C; ++s) {
        const float ls = Ls[s * SK + j], ks = Km[s * SK + j];
        if (s <= t) {
          const float w = ks * expf(lrow[i] - ls);
          dqP = fmaf(dPs[t * SC + s], w, dqP);
          dkG1 = fmaf(dGs[t * SC + s], w, dkG1);
        }
        if (s >= t) {
          const float e2 = expf(ls - lrow[i]);
          dkP = fmaf(dPs[s * SC + t], Qp[s * SK + j] * e2, dkP);
          dkG2 = fmaf(dGs[s * SC + t], ks * e2, dkG2);
        }
      }
    }
    const size_t o = slot * C * DK + (size_t)t * DK + j;
    const float dqv = waccq[o] + dqP;
    const float dkv = wacck[o] + dkP + dkG1 + dkG2;
    dLv[i] = waccL[o] + qraw[i] * dqP - kraw[i] * dkP + kraw[i] * dkG1 - kraw[i] * dkG2;
    if (t < nv) {
      const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + j;
      dq[g] = from_f<Tin>(dqv);
      dk[g] = from_f<Tin>(dkv);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < TPG; ++i) Ls[(tq * TPG + i) * SK + j] = dLv[i];
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f, dap = 0.f;
    for (int t = C - 1; t >= 0; --t) {
      acc += Ls[t * SK + tid];
      if (t < nv) {
        const size_t g = (((size_t)b * T + t0 + t) * H + h) * DK + tid;
        if (ga > 0.f) {
          // gated inputs: df~ = dlogf a sigma(-f~); this chunk's part of da_log = sum dlogf logf
          const float lf = logf[g];
          dap = fmaf(acc, lf, dap);
          dlogf[g] = acc * dlogf_dfpre(lf, ga, 1.f / ga);
        } else {
          dlogf[g] = acc;
        }
      }
    }
    if (ga > 0.f) Ls[tid] = dap;  // the tile's row 0 is free again
  }
  if (ga > 0.f) {
    __syncthreads();
    if (tid == 0) {
      float s2 = 0.f;
      for (int j2 = 0; j2 < DK; ++j2) s2 += Ls[j2];  // fixed order
      dapart[((size_t)b * H + h) * NC + n] = s2;
    }
  }
}

// The CUDA-core path: one CTA per chunk for each stage, scratch indexed by chunk.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) bwd_cc_simt(
    const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ beta,
    const float* __restrict__ logf, const Tin* __restrict__ dO, int H, int T, int NC,
    const float* __restrict__ wu, const float* __restrict__ wb0, const float* __restrict__ wg,
    float* __restrict__ dbeta, float* __restrict__ dc, float* __restrict__ wdP,
    float* __restrict__ wdGK, float* __restrict__ wdGVs) {
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  bwd_cc_body<DK, DV, Tin>(n, h, b, ((size_t)b * H + h) * NC + n, k, v, beta, logf, dO, H, T, NC, wu, wb0, wg,
                           dbeta, dc, wdP, wdGK, wdGVs);
}
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) bwd_state_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ logf, const Tin* __restrict__ dO,
    int H, int T, int NC, const float* __restrict__ wu, const float* __restrict__ wg,
    const float* __restrict__ wS0, const float* __restrict__ wdSC, float* __restrict__ waccq,
    float* __restrict__ wacck, float* __restrict__ waccL, float* __restrict__ waccv) {
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  bwd_state_body<DK, DV, Tin>(n, h, b, ((size_t)b * H + h) * NC + n, q, k, v, beta, logf, dO, H, T, NC, wu, wg,
                              wS0, wdSC, waccq, wacck, waccL, waccv, 0, nullptr);
}
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) bwd_intra_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ logf, const Tin* __restrict__ dO, int H, int T, int NC,
    const float* __restrict__ wP, const float* __restrict__ wu, const float* __restrict__ wdP,
    const float* __restrict__ wdGK, const float* __restrict__ wdGVs,
    const float* __restrict__ waccq, const float* __restrict__ wacck,
    const float* __restrict__ waccL, const float* __restrict__ waccv, Tin* __restrict__ dq,
    Tin* __restrict__ dk, Tin* __restrict__ dv, float* __restrict__ dlogf) {
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  bwd_intra_body<DK, DV, Tin>(n, h, b, ((size_t)b * H + h) * NC + n, q, k, v, logf, 0.f, dO, H, T, NC, wP, wu,
                              wdP, wdGK, wdGVs, waccq, wacck, waccL, waccv, dq, dk, dv, dlogf, nullptr);
}

// The tensor-core path's exact recomputation of the chunks the per-chunk
// kernels flagged (in-chunk |L| beyond their factorised range): the three
// stages in one CTA, chunk after chunk, each CTA with its own scratch slot.
// Unflagged chunks are skipped, so the kernel is nearly free when none is
// flagged, and the scratch is sized by the number of CTAs, not of chunks.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256) bwd_exact_simt(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ beta, const float* __restrict__ logf, const float* __restrict__ a_log,
    const Tin* __restrict__ dO, int H, int T,
    int NC, size_t chunks, const float* __restrict__ wP, const float* __restrict__ wu,
    const float* __restrict__ wb0, const float* __restrict__ wg, const float* __restrict__ wS0,
    const __nv_bfloat16* __restrict__ wdSb, float* __restrict__ dbeta, float* __restrict__ dc,
    float* __restrict__ wdP, float* __restrict__ wdGK, float* __restrict__ wdGVs, float* __restrict__ waccq,
    float* __restrict__ wacck, float* __restrict__ waccL, float* __restrict__ waccv, Tin* __restrict__ dq,
    Tin* __restrict__ dk, Tin* __restrict__ dv, float* __restrict__ dlogf, float* __restrict__ dapart,
    const int* __restrict__ only) {
  const size_t slot = blockIdx.x;
  for (size_t ch = blockIdx.x; ch < chunks; ch += gridDim.x) {
    if (only[ch] == 0) continue;  // uniform across the CTA
    const int n = static_cast<int>(ch % NC), u = static_cast<int>(ch / NC);
    const int h = u % H, b = u / H;
    const float ga = a_log ? expf(a_log[h]) : 0.f;  // gated inputs: df~ and da_log parts in place of dlogf
    bwd_cc_body<DK, DV, Tin>(n, h, b, slot, k, v, beta, logf, dO, H, T, NC, wu, wb0, wg, dbeta, dc, wdP, wdGK,
                             wdGVs);
    __syncthreads();
    bwd_state_body<DK, DV, Tin>(n, h, b, slot, q, k, v, beta, logf, dO, H, T, NC, wu, wg, wS0, nullptr,
                                waccq, wacck, waccL, waccv, 1, wdSb);
    __syncthreads();
    bwd_intra_body<DK, DV, Tin>(n, h, b, slot, q, k, v, logf, ga, dO, H, T, NC, wP, wu, wdP, wdGK, wdGVs,
                                waccq, wacck, waccL, waccv, dq, dk, dv, dlogf, dapart);
    __syncthreads();
  }
}

template <int DK, int DV, typename Tin>
static cudaError_t run_bwd(const BwdArgs& a, int stages, const int* only, cudaStream_t st) {
  const Layout& L = a.L;
  const size_t s1 = bchain_smem_floats<DK, DV>() * 4, s2 = bcc_smem_floats<DK, DV>() * 4;
  const size_t s3 = bstate_smem_floats<DK, DV>() * 4, s4 = bintra_smem_floats<DK, DV>() * 4;
  cudaError_t e;
#define KD_ATTR(fn, sz)                                                                   \
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(sz))) != \
      cudaSuccess)                                                                        \
    return e;
  KD_ATTR((bwd_chain_simt<DK, DV, Tin>), s1)
  KD_ATTR((bwd_cc_simt<DK, DV, Tin>), s2)
  KD_ATTR((bwd_state_simt<DK, DV, Tin>), s3)
  KD_ATTR((bwd_intra_simt<DK, DV, Tin>), s4)
  const size_t s5 = s2 > s3 ? (s2 > s4 ? s2 : s4) : (s3 > s4 ? s3 : s4);
  KD_ATTR((bwd_exact_simt<DK, DV, Tin>), s5)
#undef KD_ATTR
  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  const Tin* dO = static_cast<const Tin*>(a.dO);
  const float* wA = ws_ptr<float>(a.fws, L.A);
  const float* wP = ws_ptr<float>(a.fws, L.P);
  const float* wu = ws_ptr<float>(a.fws, L.u);
  const float* wb0 = ws_ptr<float>(a.fws, L.b0);
  const float* wS0 = ws_ptr<float>(a.fws, L.S0);
  float* wdSC = L.tc ? nullptr : ws_ptr<float>(a.ws, L.dSC);
  float* wg = ws_ptr<float>(a.ws, L.g);
  float* wdP = ws_ptr<float>(a.ws, L.dP);
  float* wdGK = ws_ptr<float>(a.ws, L.dGK);
  float* wdGVs = ws_ptr<float>(a.ws, L.dGVs);
  float* waccq = ws_ptr<float>(a.ws, L.accq);
  float* wacck = ws_ptr<float>(a.ws, L.acck);
  float* waccL = ws_ptr<float>(a.ws, L.accL);
  float* waccv = ws_ptr<float>(a.ws, L.accv);
  const dim3 gridc(L.NC, L.H, L.B);
  if (stages & kStageChain) {
    prof_begin(st, "bwd_chain_simt");
    bwd_chain_simt<DK, DV, Tin><<<dim3(L.H, L.B), 2 * DV, s1, st>>>(
        q, k, v, a.beta, a.logf, dO, a.dST, L.H, L.T, L.NC, wA, wP, a.dS0, wdSC, wg);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (only) {
    // tensor-core path: the flagged chunks only, all stages in one kernel
    if (stages != (kStageCC | kStageState | kStageIntra)) return cudaErrorInvalidValue;
    prof_begin(st, "bwd_exact_simt");
    bwd_exact_simt<DK, DV, Tin><<<(unsigned)(L.chunks < (size_t)kExactSlots ? L.chunks : kExactSlots), 256, s5,
                                  st>>>(
        q, k, v, a.beta, a.logf, a.a_log, dO, L.H, L.T, L.NC, L.chunks,
        wP, wu, wb0, wg, wS0, ws_ptr<__nv_bfloat16>(a.ws, L.dSCb), a.dbeta, a.dc, wdP, wdGK, wdGVs, waccq, wacck,
        waccL, waccv, static_cast<Tin*>(a.dq), static_cast<Tin*>(a.dk), static_cast<Tin*>(a.dv), a.dlogf,
        ws_ptr<float>(a.ws, L.dapart), only);
    prof_end(st);
    return cudaGetLastError();
  }
  if (stages & kStageCC) {
    prof_begin(st, "bwd_cc_simt");
    bwd_cc_simt<DK, DV, Tin><<<gridc, 256, s2, st>>>(k, v, a.beta, a.logf, dO, L.H, L.T, L.NC, wu,
                                                     wb0, wg, a.dbeta, a.dc, wdP, wdGK, wdGVs);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (stages & kStageState) {
    prof_begin(st, "bwd_state_simt");
    bwd_state_simt<DK, DV, Tin><<<gridc, 256, s3, st>>>(q, k, v, a.beta, a.logf, dO, L.H, L.T, L.NC, wu, wg,
                                                        wS0, wdSC, waccq, wacck, waccL, waccv);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!(stages & kStageIntra)) return cudaSuccess;
  prof_begin(st, "bwd_intra_simt");
  bwd_intra_simt<DK, DV, Tin><<<gridc, 256, s4, st>>>(
      q, k, v, a.logf, dO, L.H, L.T, L.NC, wP, wu, wdP, wdGK, wdGVs, waccq, wacck, waccL, waccv,
      static_cast<Tin*>(a.dq), static_cast<Tin*>(a.dk), static_cast<Tin*>(a.dv), a.dlogf);
  prof_end(st);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t run_bwd_t(const BwdArgs& a, int stages, const int* only, cudaStream_t st) {
#define KD_B(DK_, DV_) \
  if (a.L.dk == DK_ && a.L.dv == DV_) return run_bwd<DK_, DV_, Tin>(a, stages, only, st);
  KD_B(32, 32) KD_B(32, 64) KD_B(32, 128)
  KD_B(64, 32) KD_B(64, 64) KD_B(64, 128)
  KD_B(128, 32) KD_B(128, 64) KD_B(128, 128)
#undef KD_B
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t st) {
  // the reverse chain comes first and needs dST: no state-independent phase
  if (!(a.phases & kPhaseCarry)) return cudaSuccess;
  return launch_bwd_simt_stages(a, kStageAll, nullptr, st);
}

cudaError_t launch_bwd_simt_stages(const BwdArgs& a, int stages, const int* only, cudaStream_t st) {
  return a.L.dtype == 0 ? run_bwd_t<float>(a, stages, only, st) : run_bwd_t<__nv_bfloat16>(a, stages, only, st);
}

}  // namespace kd
