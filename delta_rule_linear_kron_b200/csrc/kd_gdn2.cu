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
// Kernels: gdn2_prep (A by a blocked inverse, P, W, U', Q+, K^e, e^Lambda per chunk), gdn2_chain,
// gdn2_out; gdn2_bchain, gdn2_bpost_a (dP, dQ+, dK^e, dZ -> dv, dw, dE, dT),
// gdn2_bpost_b (dq, dk, db, dloga; chunks inside the safe decay range, by
// factorised products) and gdn2_bpost_exact (the other chunks, per-element
// weights).
#include "kd_common.cuh"
#include "kd_kernels.h"

namespace kd {

namespace {

constexpr int C = kChunk;
// Value rows of the state per chain CTA: d_v / 16 CTAs per head, so the
// chains of 16 heads at d_v = 128 fit in one wave on 148 SMs.
constexpr int kRows = 16;
constexpr int kChainThreads = 512;  // threads of a chain CTA
constexpr int kPostThreads = 512;   // threads of the factorised backward kernel

template <int DK, int DV>
struct GP {
  static constexpr int PK = DK + 1, PV = DV + 1, PZ = (DK > DV ? DK : DV) + 1, PC = C + 1;
};

__device__ __forceinline__ size_t row_bthd(int b, int T, int t, int H, int h, int D) {
  return (((size_t)b * T + t) * H + h) * D;
}

// A [N / D][D] fp32 tile held as float4s across the 256 threads of a CTA, so
// that all of a thread's loads are in flight before any is used.  N is a
// multiple of 1024 and D of 4; the source is 16-byte aligned.
template <int N, int NT = 256>
struct Frag {
  static constexpr int V = N / (4 * NT);
  static_assert(V >= 1 && V * 4 * NT == N, "tile size must be a multiple of 4 x threads");
  float4 x[V];
};

template <int N, int NT>
__device__ __forceinline__ void frag_load(Frag<N, NT>& f, const float* __restrict__ src) {
#pragma unroll
  for (int i = 0; i < Frag<N, NT>::V; ++i) f.x[i] = __ldg(reinterpret_cast<const float4*>(src) + threadIdx.x + NT * i);
}

// Stores the tile into shared memory rows of pitch P.
template <int N, int D, int P, int NT>
__device__ __forceinline__ void frag_store(float* dst, const Frag<N, NT>& f) {
#pragma unroll
  for (int i = 0; i < Frag<N, NT>::V; ++i) {
    const int e = 4 * (threadIdx.x + NT * i), t = e / D, j = e % D;
    float* d = dst + t * P + j;
    d[0] = f.x[i].x;
    d[1] = f.x[i].y;
    d[2] = f.x[i].z;
    d[3] = f.x[i].w;
  }
}

// acc[u][v] += sum over k in [k0, k1) of A[u * ar + k * ak] * B[k * bk + v * bc]
// (a 4 x 4 output tile per thread; A and B already point at the tile's first
// row and column, in shared memory).
__device__ __forceinline__ void mm4x4(float (&acc)[4][4], const float* A, int ar, int ak, const float* B, int bk,
                                      int bc, int k0, int k1) {
  for (int k = k0; k < k1; ++k) {
    float a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = A[u * ar + k * ak];
#pragma unroll
    for (int v = 0; v < 4; ++v) b[v] = B[k * bk + v * bc];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
  }
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
  float* Tb = As + C * G::PC;        // [3][16][17] block temporaries of the inverse
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;

#pragma unroll 8
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
  float mx = 0.f;  // largest in-chunk |L| of this thread's channel
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * G::PK + tid];
      Ls[t * G::PK + tid] = acc;
      mx = fmaxf(mx, fabsf(acc));
    }
  }
  const float* Llast = Ls + (C - 1) * G::PK;  // padded rows carry loga = 0: L at row C-1 is Lambda
  if (__syncthreads_or(!(mx < kGdnSafeLog))) {
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
    for (int e = tid; e < C * DK; e += 256) {
      const int t = e / DK, j = e % DK;
      const float L = Ls[t * G::PK + j], gm = expf(L);
      p.Qp[ch * C * DK + e] = Qs[t * G::PZ + j] * gm;
      p.Ke[ch * C * DK + e] = Ks[t * G::PK + j] * expf(Llast[j] - L);
      Es[t * G::PK + j] *= gm;
    }
  } else {
    // inside the safe range the weights factor: T = tril(E+ K-^T, -1), P = tril(Q+ K-^T)
    for (int e = tid; e < C * DK; e += 256) {
      const int t = e / DK, j = e % DK;
      const float L = Ls[t * G::PK + j], gm = expf(L);
      const float qp = Qs[t * G::PZ + j] * gm, kk = Ks[t * G::PK + j];
      p.Qp[ch * C * DK + e] = qp;
      p.Ke[ch * C * DK + e] = kk * expf(Llast[j] - L);
      Qs[t * G::PZ + j] = qp;
      Ks[t * G::PK + j] = kk * expf(-L);
      Es[t * G::PK + j] *= gm;
    }
    __syncthreads();
    const int ti = (tid >> 4) * 4, ii = (tid & 15) * 4;  // a 4 x 4 tile of T and P per thread
    float aT[4][4] = {}, aP[4][4] = {};
    if (ii <= ti + 3) {
      mm4x4(aT, Es + ti * G::PK, G::PK, 1, Ks + ii * G::PK, 1, G::PK, 0, DK);
      mm4x4(aP, Qs + ti * G::PZ, G::PZ, 1, Ks + ii * G::PK, 1, G::PK, 0, DK);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int t = ti + u, i = ii + v;
        Ts[t * G::PC + i] = i < t ? aT[u][v] : 0.f;
        p.P[ch * C * C + t * C + i] = i <= t ? aP[u][v] : 0.f;
      }
  }
  if (tid < DK) p.gC[ch * DK + tid] = expf(Llast[tid]);
  __syncthreads();
#pragma unroll 8
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DV) + r;
    Qs[t * G::PZ + r] = ok ? wg[g] * to_f(v[g]) : 0.f;
  }
  __syncthreads();
  // A = (I + T)^{-1} blocked by 16: the four diagonal blocks by substitution,
  // then A_ab = -A_aa sum_{c=b}^{a-1} T_ac A_cb below the diagonal
  {
    if (tid < C) {
      const int blk = tid >> 4, m = tid & 15, o = 16 * blk;
      float col[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float sacc = t == m ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2)
          if (s2 >= m && s2 < t) sacc = fmaf(-Ts[(o + t) * G::PC + o + s2], col[s2], sacc);
        col[t] = t < m ? 0.f : sacc;
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) As[(o + t) * G::PC + o + m] = col[t];
    }
    for (int e = tid; e < C * C; e += 256) {
      const int t = e / C, i = e % C;
      if ((i >> 4) > (t >> 4)) As[t * G::PC + i] = 0.f;
    }
    __syncthreads();
    for (int a = 1; a < 4; ++a) {
      for (int e = tid; e < a * 256; e += 256) {
        const int bb2 = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        float sacc = 0.f;
        for (int kk = 16 * bb2; kk < 16 * a; ++kk)
          sacc = fmaf(Ts[(16 * a + rr) * G::PC + kk], As[kk * G::PC + 16 * bb2 + cc], sacc);
        Tb[bb2 * 272 + rr * 17 + cc] = sacc;
      }
      __syncthreads();
      for (int e = tid; e < a * 256; e += 256) {
        const int bb2 = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        float sacc = 0.f;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          sacc = fmaf(As[(16 * a + rr) * G::PC + 16 * a + kk], Tb[bb2 * 272 + kk * 17 + cc], sacc);
        As[(16 * a + rr) * G::PC + 16 * bb2 + cc] = -sacc;
      }
      __syncthreads();
    }
  }
  // W = A E+ and U' = A Z (A lower triangular), 4 x 4 tiles straight to the workspace
  for (int tile = tid; tile < 16 * (DK / 4); tile += 256) {
    const int t4 = (tile / (DK / 4)) * 4, j4 = (tile % (DK / 4)) * 4;
    float acc[4][4] = {};
    mm4x4(acc, As + t4 * G::PC, G::PC, 1, Es + j4, G::PK, 1, 0, t4 + 4);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<float4*>(p.W + ch * C * DK + (t4 + u) * DK + j4) =
          make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
  }
  for (int tile = tid; tile < 16 * (DV / 4); tile += 256) {
    const int t4 = (tile / (DV / 4)) * 4, r4 = (tile % (DV / 4)) * 4;
    float acc[4][4] = {};
    mm4x4(acc, As + t4 * G::PC, G::PC, 1, Qs + r4, G::PZ, 1, 0, t4 + 4);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<float4*>(p.Up + ch * C * DV + (t4 + u) * DV + r4) =
          make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
  }
  for (int e = tid; e < C * C; e += 256) p.A[ch * C * C + e] = As[(e / C) * G::PC + e % C];
}

// ---------------------------------------------------------------------------
// The chain kernels and the output kernel keep their tiles in rows whose pitch
// is a multiple of 4 floats and form every dot product with 16-byte shared
// memory loads (four channels per load), so shared-memory bandwidth no longer
// bounds them.
__device__ __forceinline__ float dot4(float4 a, float4 b, float s) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, s))));
}

// sum over k < n (n a multiple of 4) of a[k] b[k], both 16-byte aligned
__device__ __forceinline__ float dotv(const float* a, const float* b, int n, float s) {
#pragma unroll 4
  for (int k = 0; k < n; k += 4)
    s = dot4(*reinterpret_cast<const float4*>(a + k), *reinterpret_cast<const float4*>(b + k), s);
  return s;
}

// The chain: one CTA per (kRows value rows, head); chunks in order.
template <int DK, int DV>
__global__ void __launch_bounds__(kChainThreads) gdn2_chain(const float* __restrict__ S0, float* __restrict__ ST,
                                                            int H, int NC, GdnWs p) {
  constexpr int RS = kRows, NT = kChainThreads, P4 = DK + 4, NJ = DK / 4;
  static_assert(RS * NJ <= NT && (C * RS) % NT == 0, "thread mapping");
  extern __shared__ __align__(16) float gsm[];
  float* Ws = gsm;                  // [C][P4]
  float* Kes = Ws + C * P4;         // [C][P4]
  float* Ss = Kes + C * P4;         // [RS][P4] state rows
  float* Us = Ss + RS * P4;         // [C][RS]
  float* gcs = Us + C * RS;         // [DK]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * RS, h = blockIdx.y, bb = blockIdx.z;
  const size_t unit = (size_t)bb * H + h;
  for (int e = tid; e < RS * DK; e += NT) {
    const int r = e / DK, j = e % DK;
    Ss[r * P4 + j] = S0 ? S0[(unit * DV + r0 + r) * DK + j] : 0.f;
  }
  // chunk n+1's W and K^e are loaded into registers while chunk n computes
  constexpr int UPT = C * RS / NT;  // U' values per thread
  Frag<C * DK, NT> fw, fk;
  float up[UPT], gc = 0.f;
  auto fetch = [&](int n) {
    const size_t ch = unit * NC + n;
    frag_load(fw, p.W + ch * C * DK);
    frag_load(fk, p.Ke + ch * C * DK);
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
      const int e = tid + NT * i;
      up[i] = p.Up[ch * C * DV + (e / RS) * DV + r0 + e % RS];
    }
    if (tid < DK) gc = p.gC[ch * DK + tid];
  };
  fetch(0);
  for (int n = 0; n < NC; ++n) {
    const size_t ch = unit * NC + n;
    frag_store<C * DK, DK, P4>(Ws, fw);
    frag_store<C * DK, DK, P4>(Kes, fk);
#pragma unroll
    for (int i = 0; i < UPT; ++i) Us[tid + NT * i] = up[i];
    if (tid < DK) gcs[tid] = gc;
    __syncthreads();
    if (n + 1 < NC) fetch(n + 1);
    for (int e = tid; e < RS * DK; e += NT) {
      const int r = e / DK, j = e % DK;
      p.S0[ch * DV * DK + (size_t)(r0 + r) * DK + j] = Ss[r * P4 + j];
    }
    // U[t][r] = U'[t][r] - W[t] . S[r]: 4 positions x 4 rows per thread, so each
    // 16-byte shared load feeds four dot products
    if (tid < (C / 4) * (RS / 4)) {
      const int t4 = (tid / (RS / 4)) * 4, r4 = (tid % (RS / 4)) * 4;
      float acc[4][4] = {};
#pragma unroll 2
      for (int k = 0; k < DK; k += 4) {
        float4 a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = *reinterpret_cast<const float4*>(Ws + (t4 + u) * P4 + k);
          b[u] = *reinterpret_cast<const float4*>(Ss + (r4 + u) * P4 + k);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = dot4(a[u], b[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int t = t4 + u, r = r4 + v;
          const float uu = Us[t * RS + r] - acc[u][v];
          Us[t * RS + r] = uu;
          p.U[ch * C * DV + t * DV + r0 + r] = uu;
        }
    }
    __syncthreads();
    // S[r][j..j+3] = S gamma_C + sum_t U[t][r] K^e[t][j..j+3]: 4 rows x 4 channels
    // per thread
    if (tid < (RS / 4) * NJ) {
      const int r4 = (tid / NJ) * 4, j = 4 * (tid % NJ);
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 sv = *reinterpret_cast<const float4*>(Ss + (r4 + u) * P4 + j);
        acc[u][0] = sv.x * gcs[j];
        acc[u][1] = sv.y * gcs[j + 1];
        acc[u][2] = sv.z * gcs[j + 2];
        acc[u][3] = sv.w * gcs[j + 3];
      }
#pragma unroll 4
      for (int t = 0; t < C; ++t) {
        const float4 uv = *reinterpret_cast<const float4*>(Us + t * RS + r4);
        const float4 kv = *reinterpret_cast<const float4*>(Kes + t * P4 + j);
        const float ua[4] = {uv.x, uv.y, uv.z, uv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[u][c] = fmaf(ua[u], ka[c], acc[u][c]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(Ss + (r4 + u) * P4 + j) = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
  }
  if (ST)
    for (int e = tid; e < RS * DK; e += NT) {
      const int r = e / DK, j = e % DK;
      ST[(unit * DV + r0 + r) * DK + j] = Ss[r * P4 + j];
    }
}

// ---------------------------------------------------------------------------
// O = Q+ S0^T + P U per chunk, all chunks in parallel.  Each thread owns one
// value row r and C / (256 / DV) positions; S0 passes through shared memory in
// 32-channel slabs, which keeps the CTA at about 100 KB so two fit on an SM.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256, 2) gdn2_out(int H, int T, int NC, GdnWs p, Tin* __restrict__ out) {
  constexpr int P4 = DK + 4, PC4 = C + 4, SL = 32, PS = SL + 4;
  constexpr int NTG = 256 / DV, TPT = C / NTG;  // position groups, positions per thread
  extern __shared__ __align__(16) float gsm[];
  float* Qps = gsm;                 // [C][P4]
  float* Ps = Qps + C * P4;         // [C][PC4]
  float* Ut = Ps + C * PC4;         // [DV][PC4]  U transposed
  float* S0s = Ut + DV * PC4;       // [DV][PS]   one 32-channel slab of S0
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;
  {
    Frag<C * DK> fq;
    Frag<C * C> fp;
    frag_load(fq, p.Qp + ch * C * DK);
    frag_load(fp, p.P + ch * C * C);
    frag_store<C * DK, DK, P4>(Qps, fq);
    frag_store<C * C, C, PC4>(Ps, fp);
  }
#pragma unroll 8
  for (int e = tid; e < C * DV; e += 256) Ut[(e % DV) * PC4 + e / DV] = p.U[ch * C * DV + e];
  const int r = tid % DV, tg = (tid / DV) * TPT;
  float acc[TPT];
#pragma unroll
  for (int i = 0; i < TPT; ++i) acc[i] = 0.f;
  const float* s0 = p.S0 + ch * DV * DK;
  for (int j0 = 0; j0 < DK; j0 += SL) {
    __syncthreads();  // the previous slab has been read (and, the first time, the tiles above are in)
#pragma unroll
    for (int e = tid; e < DV * SL / 4; e += 256) {
      const int rr = e / (SL / 4), c4 = 4 * (e % (SL / 4));
      *reinterpret_cast<float4*>(S0s + rr * PS + c4) = __ldg(reinterpret_cast<const float4*>(s0 + rr * DK + j0 + c4));
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < SL; j += 4) {
      const float4 sv = *reinterpret_cast<const float4*>(S0s + r * PS + j);
#pragma unroll
      for (int i = 0; i < TPT; ++i)
        acc[i] = dot4(*reinterpret_cast<const float4*>(Qps + (tg + i) * P4 + j0 + j), sv, acc[i]);
    }
  }
#pragma unroll 4
  for (int k = 0; k < C; k += 4) {
    const float4 uv = *reinterpret_cast<const float4*>(Ut + r * PC4 + k);
#pragma unroll
    for (int i = 0; i < TPT; ++i)
      acc[i] = dot4(*reinterpret_cast<const float4*>(Ps + (tg + i) * PC4 + k), uv, acc[i]);
  }
#pragma unroll
  for (int i = 0; i < TPT; ++i)
    if (tg + i < nv) out[row_bthd(bb, T, t0 + tg + i, H, h, DV) + r] = from_f<Tin>(acc[i]);
}

// ---------------------------------------------------------------------------
// Reverse chain: one CTA per (kRows value rows, head); chunks last to first.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kChainThreads) gdn2_bchain(const Tin* __restrict__ dO,
                                                             const float* __restrict__ dST, float* __restrict__ dS0,
                                                             int H, int T, int NC, GdnWs p) {
  constexpr int RS = kRows, NT = kChainThreads, P4 = DK + 4, PC4 = C + 4, NJ = DK / 4;
  static_assert(RS * NJ <= NT, "thread mapping");
  extern __shared__ __align__(16) float gsm[];
  float* Pt = gsm;                  // [C][PC4]  P transposed
  float* Kes = Pt + C * PC4;        // [C][P4]
  float* Qps = Kes + C * P4;        // [C][P4]
  float* Ws = Qps + C * P4;         // [C][P4]
  float* dOt = Ws + C * P4;         // [RS][PC4] dO transposed
  float* dOs = dOt + RS * PC4;      // [C][RS]
  float* dUs = dOs + C * RS;        // [C][RS]
  float* dSs = dUs + C * RS;        // [RS][P4]
  float* gcs = dSs + RS * P4;       // [DK]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * RS, h = blockIdx.y, bb = blockIdx.z;
  const size_t unit = (size_t)bb * H + h;
  for (int e = tid; e < RS * DK; e += NT) {
    const int r = e / DK, j = e % DK;
    dSs[r * P4 + j] = dST ? dST[(unit * DV + r0 + r) * DK + j] : 0.f;
  }
  // chunk n-1's tiles and dO slice are loaded into registers while chunk n computes
  constexpr int OPT = C * RS / NT;  // dO values per thread
  Frag<C * C, NT> fp;
  Frag<C * DK, NT> fk, fq, fw;
  float go[OPT], gc = 0.f;
  auto fetch = [&](int n) {
    const size_t ch = unit * NC + n;
    const int t0 = n * C, nv = min(C, T - t0);
    frag_load(fp, p.P + ch * C * C);
    frag_load(fk, p.Ke + ch * C * DK);
    frag_load(fq, p.Qp + ch * C * DK);
    frag_load(fw, p.W + ch * C * DK);
#pragma unroll
    for (int i = 0; i < OPT; ++i) {
      const int e = tid + NT * i, t = e / RS, r = e % RS;
      go[i] = t < nv ? to_f(dO[row_bthd(bb, T, t0 + t, H, h, DV) + r0 + r]) : 0.f;
    }
    if (tid < DK) gc = p.gC[ch * DK + tid];
  };
  fetch(NC - 1);
  for (int n = NC - 1; n >= 0; --n) {
    const size_t ch = unit * NC + n;
#pragma unroll
    for (int i = 0; i < Frag<C * C, NT>::V; ++i) {
      const int e = 4 * (tid + NT * i), t = e / C, c = e % C;
      Pt[c * PC4 + t] = fp.x[i].x;
      Pt[(c + 1) * PC4 + t] = fp.x[i].y;
      Pt[(c + 2) * PC4 + t] = fp.x[i].z;
      Pt[(c + 3) * PC4 + t] = fp.x[i].w;
    }
    frag_store<C * DK, DK, P4>(Kes, fk);
    frag_store<C * DK, DK, P4>(Qps, fq);
    frag_store<C * DK, DK, P4>(Ws, fw);
#pragma unroll
    for (int i = 0; i < OPT; ++i) {
      const int e = tid + NT * i, t = e / RS, r = e % RS;
      dOs[e] = go[i];
      dOt[r * PC4 + t] = go[i];
    }
    if (tid < DK) gcs[tid] = gc;
    __syncthreads();
    if (n > 0) fetch(n - 1);
    for (int e = tid; e < RS * DK; e += NT) {
      const int r = e / DK, j = e % DK;
      p.dS[ch * DV * DK + (size_t)(r0 + r) * DK + j] = dSs[r * P4 + j];
    }
    // dU[t][r] = sum_t' P[t'][t] dO[t'][r] + K^e[t] . dS[r]: 4 positions x 4 rows
    // per thread
    if (tid < (C / 4) * (RS / 4)) {
      const int t4 = (tid / (RS / 4)) * 4, r4 = (tid % (RS / 4)) * 4;
      float acc[4][4] = {};
#pragma unroll 2
      for (int k = 0; k < C; k += 4) {
        float4 a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = *reinterpret_cast<const float4*>(Pt + (t4 + u) * PC4 + k);
          b[u] = *reinterpret_cast<const float4*>(dOt + (r4 + u) * PC4 + k);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = dot4(a[u], b[v], acc[u][v]);
      }
#pragma unroll 2
      for (int k = 0; k < DK; k += 4) {
        float4 a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = *reinterpret_cast<const float4*>(Kes + (t4 + u) * P4 + k);
          b[u] = *reinterpret_cast<const float4*>(dSs + (r4 + u) * P4 + k);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = dot4(a[u], b[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int t = t4 + u, r = r4 + v;
          dUs[t * RS + r] = acc[u][v];
          p.dU[ch * C * DV + t * DV + r0 + r] = acc[u][v];
        }
    }
    __syncthreads();
    // dS[r][j..j+3] = dS gamma_C + sum_t dO[t][r] Q+[t] - dU[t][r] W[t]: 4 rows x
    // 4 channels per thread
    if (tid < (RS / 4) * NJ) {
      const int r4 = (tid / NJ) * 4, j = 4 * (tid % NJ);
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 sv = *reinterpret_cast<const float4*>(dSs + (r4 + u) * P4 + j);
        acc[u][0] = sv.x * gcs[j];
        acc[u][1] = sv.y * gcs[j + 1];
        acc[u][2] = sv.z * gcs[j + 2];
        acc[u][3] = sv.w * gcs[j + 3];
      }
#pragma unroll 4
      for (int t = 0; t < C; ++t) {
        const float4 gv = *reinterpret_cast<const float4*>(dOs + t * RS + r4);
        const float4 dv4 = *reinterpret_cast<const float4*>(dUs + t * RS + r4);
        const float4 qv = *reinterpret_cast<const float4*>(Qps + t * P4 + j);
        const float4 wv = *reinterpret_cast<const float4*>(Ws + t * P4 + j);
        const float ga[4] = {gv.x, gv.y, gv.z, gv.w}, da[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[u][c] = fmaf(ga[u], qa[c], fmaf(-da[u], wa[c], acc[u][c]));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(dSs + (r4 + u) * P4 + j) = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
  }
  if (dS0)
    for (int e = tid; e < RS * DK; e += NT) {
      const int r = e / DK, j = e % DK;
      dS0[(unit * DV + r0 + r) * DK + j] = dSs[r * P4 + j];
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
#pragma unroll 8
  for (int e = tid; e < C * DV; e += 256) {
    const int t = e / DV, r = e % DV;
    R1[t * G::PZ + r] = t < nv ? to_f(dO[row_bthd(bb, T, t0 + t, H, h, DV) + r]) : 0.f;
    R2[t * G::PZ + r] = p.U[ch * C * DV + e];
    R3[t * G::PZ + r] = p.dU[ch * C * DV + e];
  }
#pragma unroll 8
  for (int e = tid; e < C * C; e += 256) As[(e / C) * G::PC + e % C] = p.A[ch * C * C + e];
  __syncthreads();
  // dQ+ = dO S0 and dW = -dU S0 in one pass over the rows of S0, dK^e = U dS in
  // a second over dS (to the workspace): each thread an 8-position x 4-channel
  // tile, the state rows streamed as float4 four rows ahead
  {
    constexpr int NJG = DK / 4, AHEAD = 4;
    static_assert(DV % AHEAD == 0, "row groups");
    if (tid < NJG * 8) {
      const int jg = tid % NJG, t8 = (tid / NJG) * 8;
      {
        float aq[8][4] = {}, aw[8][4] = {};
        const float4* s0 = reinterpret_cast<const float4*>(p.S0 + ch * DV * DK) + jg;
        float4 ring[AHEAD];
#pragma unroll
        for (int i = 0; i < AHEAD; ++i) ring[i] = __ldg(s0 + i * NJG);
        for (int r0 = 0; r0 < DV; r0 += AHEAD) {
#pragma unroll
          for (int i = 0; i < AHEAD; ++i) {
            const int r = r0 + i;
            const float4 a = ring[i];
            if (r + AHEAD < DV) ring[i] = __ldg(s0 + (r + AHEAD) * NJG);
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float o = R1[(t8 + u) * G::PZ + r], du = R3[(t8 + u) * G::PZ + r];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                aq[u][c] = fmaf(o, av[c], aq[u][c]);
                aw[u][c] = fmaf(du, av[c], aw[u][c]);
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = t8 + u;
          *reinterpret_cast<float4*>(p.dQp + ch * C * DK + t * DK + 4 * jg) =
              make_float4(aq[u][0], aq[u][1], aq[u][2], aq[u][3]);
#pragma unroll
          for (int c = 0; c < 4; ++c) R4[t * G::PK + 4 * jg + c] = -aw[u][c];
        }
      }
      {
        float ak[8][4] = {};
        const float4* ds = reinterpret_cast<const float4*>(p.dS + ch * DV * DK) + jg;
        float4 ring[AHEAD];
#pragma unroll
        for (int i = 0; i < AHEAD; ++i) ring[i] = __ldg(ds + i * NJG);
        for (int r0 = 0; r0 < DV; r0 += AHEAD) {
#pragma unroll
          for (int i = 0; i < AHEAD; ++i) {
            const int r = r0 + i;
            const float4 d = ring[i];
            if (r + AHEAD < DV) ring[i] = __ldg(ds + (r + AHEAD) * NJG);
            const float dv4[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float uu = R2[(t8 + u) * G::PZ + r];
#pragma unroll
              for (int c = 0; c < 4; ++c) ak[u][c] = fmaf(uu, dv4[c], ak[u][c]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<float4*>(p.dKe + ch * C * DK + (t8 + u) * DK + 4 * jg) =
              make_float4(ak[u][0], ak[u][1], ak[u][2], ak[u][3]);
      }
    }
  }
  const int ti = (tid >> 4) * 4, ii = (tid & 15) * 4;  // this thread's 4 x 4 tile of a C x C result
  // dP = tril(dO U^T)
  {
    float acc[4][4] = {};
    if (ii <= ti + 3) mm4x4(acc, R1 + ti * G::PZ, G::PZ, 1, R2 + ii * G::PZ, 1, G::PZ, 0, DV);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) dPs[(ti + u) * G::PC + ii + v] = ii + v <= ti + u ? acc[u][v] : 0.f;
  }
  __syncthreads();
  // dZ = A^T dU (A lower triangular) -> dv = dZ w, dw = dZ v;  dE = A^T dW
  for (int tile = tid; tile < 16 * (DV / 4); tile += 256) {
    const int t4 = (tile / (DV / 4)) * 4, r4 = (tile % (DV / 4)) * 4;
    float acc[4][4] = {};
    mm4x4(acc, As + t4, 1, G::PC, R3 + r4, G::PZ, 1, t4, C);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int t = t4 + u, r = r4 + c;
        R2[t * G::PZ + r] = acc[u][c];
        if (t < nv) {
          const size_t g = row_bthd(bb, T, t0 + t, H, h, DV) + r;
          dv[g] = from_f<Tin>(acc[u][c] * wg[g]);
          dw[g] = acc[u][c] * to_f(v[g]);
        }
      }
  }
  for (int tile = tid; tile < 16 * (DK / 4); tile += 256) {
    const int t4 = (tile / (DK / 4)) * 4, j4 = (tile % (DK / 4)) * 4;
    float acc[4][4] = {};
    mm4x4(acc, As + t4, 1, G::PC, R4 + j4, G::PK, 1, t4, C);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        R1[(t4 + u) * G::PZ + j4 + c] = acc[u][c];
        p.dE[ch * C * DK + (t4 + u) * DK + j4 + c] = acc[u][c];
      }
  }
  __syncthreads();
#pragma unroll 8
  for (int e = tid; e < C * DV; e += 256) R3[(e / DV) * G::PZ + e % DV] = p.Up[ch * C * DV + e];
#pragma unroll 8
  for (int e = tid; e < C * DK; e += 256) R4[(e / DK) * G::PK + e % DK] = p.W[ch * C * DK + e];
  __syncthreads();
  // dT = -tril(dZ U'^T + dE W^T, -1)
  {
    float acc[4][4] = {};
    if (ii <= ti + 3) {
      mm4x4(acc, R2 + ti * G::PZ, G::PZ, 1, R3 + ii * G::PZ, 1, G::PZ, 0, DV);
      mm4x4(acc, R1 + ti * G::PZ, G::PZ, 1, R4 + ii * G::PK, 1, G::PK, 0, DK);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) dTs[(ti + u) * G::PC + ii + v] = ii + v < ti + u ? -acc[u][v] : 0.f;
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
__global__ void __launch_bounds__(256) gdn2_bpost_exact(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                    const float* __restrict__ bg, const float* __restrict__ loga,
                                                    int H, int T, int NC, GdnWs p,
                                                    Tin* __restrict__ dq, Tin* __restrict__ dk,
                                                    float* __restrict__ db, float* __restrict__ dloga,
                                                    const unsigned char* __restrict__ xflag) {
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
  // the tensor-core gradient kernel flags the chunks it leaves to this one
  if (xflag && !xflag[ch]) return;
  // the decay prefix first: chunks inside the safe range leave at once
  float mx = 0.f;
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += t < nv ? loga[row_bthd(bb, T, t0 + t, H, h, DK) + tid] : 0.f;
      Ls[t * G::PK + tid] = acc;
      mx = fmaxf(mx, fabsf(acc));
    }
  }
  if (!__syncthreads_or(!(mx < kGdnSafeLog)) && !xflag) return;  // the factorised kernel took this chunk
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
    const float kk = ok ? to_f(k[g]) : 0.f;
    Ks[t * G::PK + j] = kk;
    Qs[t * G::PK + j] = ok ? to_f(q[g]) : 0.f;
    Es[t * G::PK + j] = ok ? bg[g] * kk : 0.f;
  }
  for (int e = tid; e < C * C; e += 256) {
    dPs[(e / C) * G::PC + e % C] = p.dP[ch * C * C + e];
    dTs[(e / C) * G::PC + e % C] = p.dT[ch * C * C + e];
  }
  __syncthreads();
  const int j = tid % DK;
  const float Lam = Ls[(C - 1) * G::PK + j];
  float lam_part = 0.f;  // sum over this thread's t of dK^e o K^e
  for (int e = tid; e < C * DK; e += 256) {
    const int t = e / DK;
    const float L = Ls[t * G::PK + j], gm = expf(L), ke = expf(Lam - L);
    const float kk = Ks[t * G::PK + j], qq = Qs[t * G::PK + j], ee = Es[t * G::PK + j];
    const float dQp = p.dQp[ch * C * DK + e], dKe = p.dKe[ch * C * DK + e];
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
// Per chunk, chunks whose in-chunk |L| stays below kGdnSafeLog: the exact
// weights factor as e^{L_t - L_i} = gamma_t / gamma_i, and the pair sums become
// three products with K- = k / gamma, E+ = e o gamma, Q+ = q o gamma:
//   X1 = dT K-,  X2 = dP K-,  Y = dT^T E+ + dP^T Q+                 ([C][DK])
//   de = gamma (dE + X1),  dq = gamma (dQ+ + X2),  dk = dK^e e^{Lambda-L} + Y / gamma
//   dL = dE E+ + dQ+ Q+ - dK^e K^e + E+ X1 + Q+ X2 - K- Y
// Each thread owns a 4-position x 4-channel tile of all three products.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kPostThreads) gdn2_bpost_b(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                    const float* __restrict__ bg, const float* __restrict__ loga,
                                                    int H, int T, int NC, GdnWs p, Tin* __restrict__ dq,
                                                    Tin* __restrict__ dk, float* __restrict__ db,
                                                    float* __restrict__ dloga) {
  constexpr int P4 = DK + 4, PT = C + 4, NJG = DK / 4, NT = kPostThreads, NTG = C / 4;
  extern __shared__ __align__(16) float gsm[];
  float* Ls = gsm;                  // [C][P4]  L
  float* Km = Ls + C * P4;          // [C][P4]  K-
  float* Ep = Km + C * P4;          // [C][P4]  E+
  float* Qp = Ep + C * P4;          // [C][P4]  Q+
  float* dTr = Qp + C * P4;         // [C][PT]  dT, rows t
  float* dPr = dTr + C * PT;        // [C][PT]  dP, rows t
  float* dTc = dPr + C * PT;        // [C][PT]  dT^T, then dL
  float* dPc = dTc + C * PT;        // [C][PT]  dP^T
  float* red = dPc + C * PT;        // [NTG][DK]
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int t0 = n * C, nv = min(C, T - t0);
  const size_t ch = ((size_t)bb * H + h) * NC + n;
#pragma unroll 8
  for (int e = tid; e < C * DK; e += NT) {
    const int t = e / DK, j = e % DK;
    Ls[t * P4 + j] = t < nv ? loga[row_bthd(bb, T, t0 + t, H, h, DK) + j] : 0.f;
  }
#pragma unroll 8
  for (int e = tid; e < C * C; e += NT) {
    const int t = e / C, i = e % C;
    const float a = p.dT[ch * C * C + e], c = p.dP[ch * C * C + e];
    dTr[t * PT + i] = a;
    dPr[t * PT + i] = c;
    dTc[i * PT + t] = a;
    dPc[i * PT + t] = c;
  }
  __syncthreads();
  float mx = 0.f;
  if (tid < DK) {
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += Ls[t * P4 + tid];
      Ls[t * P4 + tid] = acc;
      mx = fmaxf(mx, fabsf(acc));
    }
  }
  if (__syncthreads_or(!(mx < kGdnSafeLog))) return;  // the exact kernel takes this chunk
#pragma unroll 8
  for (int e = tid; e < C * DK; e += NT) {
    const int t = e / DK, j = e % DK;
    const bool ok = t < nv;
    const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
    const float L = Ls[t * P4 + j], gm = expf(L), ig = expf(-L);
    const float kk = ok ? to_f(k[g]) : 0.f;
    Km[t * P4 + j] = kk * ig;
    Ep[t * P4 + j] = ok ? bg[g] * kk * gm : 0.f;
    Qp[t * P4 + j] = p.Qp[ch * C * DK + e];
  }
  __syncthreads();
  const bool act = tid < NJG * NTG;
  const int jg = tid % NJG, t4 = (tid / NJG) * 4;
  float x1[4][4] = {}, x2[4][4] = {}, y[4][4] = {};
  if (act) {
#pragma unroll 4
    for (int i = 0; i < C; ++i) {
      const float4 km = *reinterpret_cast<const float4*>(Km + i * P4 + 4 * jg);
      const float4 ta = *reinterpret_cast<const float4*>(dTc + i * PT + t4);
      const float4 pa = *reinterpret_cast<const float4*>(dPc + i * PT + t4);
      const float kv[4] = {km.x, km.y, km.z, km.w};
      const float tv[4] = {ta.x, ta.y, ta.z, ta.w};
      const float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          x1[u][c] = fmaf(tv[u], kv[c], x1[u][c]);
          x2[u][c] = fmaf(pv[u], kv[c], x2[u][c]);
        }
    }
#pragma unroll 4
    for (int tp = 0; tp < C; ++tp) {
      const float4 ea = *reinterpret_cast<const float4*>(Ep + tp * P4 + 4 * jg);
      const float4 qa = *reinterpret_cast<const float4*>(Qp + tp * P4 + 4 * jg);
      const float4 ta = *reinterpret_cast<const float4*>(dTr + tp * PT + t4);
      const float4 pa = *reinterpret_cast<const float4*>(dPr + tp * PT + t4);
      const float ev[4] = {ea.x, ea.y, ea.z, ea.w}, qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float tv[4] = {ta.x, ta.y, ta.z, ta.w};
      const float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int c = 0; c < 4; ++c) y[u][c] = fmaf(tv[u], ev[c], fmaf(pv[u], qv[c], y[u][c]));
    }
  }
  __syncthreads();  // dT^T is dead: dL goes there
  float* dLs = dTc;   // [C][P4] fits in two [C][PT] regions
  float lam[4] = {};
  if (act) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t4 + u;
      const bool ok = t < nv;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = 4 * jg + c;
        const size_t e = (size_t)t * DK + j;
        const float L = Ls[t * P4 + j], gm = expf(L), ke = expf(Ls[(C - 1) * P4 + j] - L);
        const float dQv = p.dQp[ch * C * DK + e], dKv = p.dKe[ch * C * DK + e], dEv = p.dE[ch * C * DK + e];
        const float ep = Ep[t * P4 + j], qp = Qp[t * P4 + j], km = Km[t * P4 + j];
        const size_t g = row_bthd(bb, T, t0 + t, H, h, DK) + j;
        const float kk = ok ? to_f(k[g]) : 0.f;
        const float dee = gm * (dEv + x1[u][c]);
        const float dqq = gm * (dQv + x2[u][c]);
        const float dkk = fmaf(dKv, ke, y[u][c] * expf(-L));
        lam[c] = fmaf(dKv, kk * ke, lam[c]);
        dLs[t * P4 + j] = dEv * ep + dQv * qp - dKv * kk * ke + ep * x1[u][c] + qp * x2[u][c] - km * y[u][c];
        if (ok) {
          dq[g] = from_f<Tin>(dqq);
          dk[g] = from_f<Tin>(fmaf(dee, bg[g], dkk));
          db[g] = dee * kk;
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) red[(tid / NJG) * DK + 4 * jg + c] = lam[c];
  }
  __syncthreads();
  if (tid < DK) {
    float lm = 0.f;
#pragma unroll
    for (int s8 = 0; s8 < NTG; ++s8) lm += red[s8 * DK + tid];
    float st = 0.f;
    for (int r = 0; r < DV; ++r)
      st = fmaf(p.dS[ch * DV * DK + (size_t)r * DK + tid], p.S0[ch * DV * DK + (size_t)r * DK + tid], st);
    const float Lam = Ls[(C - 1) * P4 + tid];
    float acc = fmaf(st, expf(Lam), lm);
    for (int t = C - 1; t >= 0; --t) {
      acc += dLs[t * P4 + tid];
      if (t < nv) dloga[row_bthd(bb, T, t0 + t, H, h, DK) + tid] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
namespace {

template <int DK, int DV>
struct GSmem {
  using G = GP<DK, DV>;
  static constexpr size_t prep = (size_t)(3 * C * G::PK + C * G::PZ + 2 * C * G::PC + 3 * 16 * 17) * 4;
  static constexpr int P4 = DK + 4, PC4 = C + 4;
  static constexpr size_t chain = (size_t)(2 * C * P4 + kRows * P4 + C * kRows + DK) * 4;
  static constexpr size_t out = (size_t)(C * P4 + C * PC4 + DV * PC4 + DV * 36) * 4;
  static constexpr size_t bchain =
      (size_t)(C * PC4 + 3 * C * P4 + kRows * PC4 + 2 * C * kRows + kRows * P4 + DK) * 4;
  static constexpr size_t bpa = (size_t)(3 * C * G::PZ + C * G::PK + 3 * C * G::PC) * 4;
  static constexpr size_t bpe = (size_t)(5 * C * G::PK + 2 * C * G::PC + 256) * 4;
  static constexpr size_t bpb = (size_t)(4 * C * (DK + 4) + 4 * C * (C + 4) + (C / 4) * DK) * 4;
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
  KD_TRYC(set_smem(gdn2_chain<DK, DV>, S::chain));
  if (!gdn2_tc_supported(L)) KD_TRYC(set_smem(gdn2_out<DK, DV, Tin>, S::out));
  if (gdn2_tc_supported(L)) {
    KD_TRYC(launch_gdn2_prep_tc(a, a.err, st));
  } else {
    KD_TRYC(set_smem(gdn2_prep<DK, DV, Tin>, S::prep));
    prof_begin(st, "gdn2_prep");
    gdn2_prep<DK, DV, Tin><<<gc, 256, S::prep, st>>>(static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
                                                     static_cast<const Tin*>(a.v), a.b, a.w, a.loga, L.H, L.T, L.NC,
                                                     p);
    prof_end(st);
    KD_TRYC(cudaGetLastError());
  }
  if (gdn2_tc_supported(L)) {
    KD_TRYC(launch_gdn2_chain_tc(a, a.err, st));
  } else {
    prof_begin(st, "gdn2_chain");
    gdn2_chain<DK, DV><<<gr, kChainThreads, S::chain, st>>>(a.S0, a.ST, L.H, L.NC, p);
    prof_end(st);
    KD_TRYC(cudaGetLastError());
  }
  if (gdn2_tc_supported(L)) return launch_gdn2_out_tc(a, a.err, st);
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
  if (!L.tc) KD_TRYC(set_smem(gdn2_bchain<DK, DV, Tin>, S::bchain));
  KD_TRYC(set_smem(gdn2_bpost_a<DK, DV, Tin>, S::bpa));
  KD_TRYC(set_smem(gdn2_bpost_b<DK, DV, Tin>, S::bpb));
  KD_TRYC(set_smem(gdn2_bpost_exact<DK, DV, Tin>, S::bpe));
  const Tin* dO = static_cast<const Tin*>(a.dO);
  if (L.tc) {
    KD_TRYC(launch_gdn2_bchain_tc(a, p, a.err, st));
  } else {
    prof_begin(st, "gdn2_bchain");
    gdn2_bchain<DK, DV, Tin><<<gr, kChainThreads, S::bchain, st>>>(dO, a.dST, a.dS0, L.H, L.T, L.NC, p);
    prof_end(st);
    KD_TRYC(cudaGetLastError());
  }
  if (L.tc) {
    // tensor cores: every gradient of the factorised chunks, and the exact
    // kernel's inputs for the others (read from the chains' state images)
    KD_TRYC(launch_gdn2_bpost_tc(a, p, a.err, st));
  } else {
    prof_begin(st, "gdn2_bpost_a");
    gdn2_bpost_a<DK, DV, Tin><<<gc, 256, S::bpa, st>>>(static_cast<const Tin*>(a.v), a.w, dO, L.H, L.T, L.NC, p,
                                                       static_cast<Tin*>(a.dv), a.dw);
    prof_end(st);
    KD_TRYC(cudaGetLastError());
    prof_begin(st, "gdn2_bpost_b");
    gdn2_bpost_b<DK, DV, Tin><<<gc, kPostThreads, S::bpb, st>>>(static_cast<const Tin*>(a.q),
                                                                static_cast<const Tin*>(a.k), a.b, a.loga, L.H, L.T,
                                                                L.NC, p, static_cast<Tin*>(a.dq),
                                                                static_cast<Tin*>(a.dk), a.db, a.dloga);
    prof_end(st);
    KD_TRYC(cudaGetLastError());
  }
  prof_begin(st, "gdn2_bpost_exact");
  gdn2_bpost_exact<DK, DV, Tin><<<gc, 256, S::bpe, st>>>(static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
                                                         a.b, a.loga, L.H, L.T, L.NC, p, static_cast<Tin*>(a.dq),
                                                         static_cast<Tin*>(a.dk), a.db, a.dloga, p.xflag);
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
