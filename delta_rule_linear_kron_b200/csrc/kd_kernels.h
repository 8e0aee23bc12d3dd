// kd_kernels.h -- internal launch interface between the chunk scheduler / C ABI
// and the CUDA kernels.  Not part of the public header.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kd {

// Chunk length of the chunk-parallel form (Gated DeltaNet-2 article, section
// "기술 상세": the chunk size is fixed at 64 and the chunk's triangular
// inverse is built by forward substitution).
constexpr int kChunk = 64;
// Gated DeltaNet-2 backward: in-chunk |L| below which the per-chunk gradient
// kernels factor e^{L_t - L_i} = gamma_t / gamma_i (e^{+-60} and their products
// stay well inside fp32's normal range); the chunks beyond it take the exact
// kernel.  Both sides decide from the same sequential prefix sum.
constexpr float kGdnSafeLog = 60.f;

// Scratch slots of the tensor-core backward's exact recomputation (the CTAs
// of bwd_exact_simt): its per-chunk scratch is sized by this, not by the
// number of chunks.
constexpr int kExactSlots = 128;

// The fused input prologue inside the chunk kernels (KronLSTM digest, "어떻게
// 쓰나"): the erase and write gates arrive as pre-activations (beta = s
// sigma(x), c = sigma(x)), and q, k, v as raw projections, L2-normalised per
// token and head, x / sqrt(|x|^2 + 1e-6), where a kernel loads them.  Both
// zero: the inputs are the recurrence's own.
struct Pro {
  float bscale = 0.f;  // > 0: beta and c are pre-activations, beta = bscale sigma(.), c = sigma(.)
  int norm = 0;        // 1: q, k, v are raw
};

// Workspace layout of one problem (B, H, T, dk, dv), decided by the chunk
// scheduler.  Offsets are in bytes from the workspace base, 256-byte aligned.
// "chunk" index ch = ((b * H) + h) * NC + n.
struct Layout {
  int B = 0, H = 0, T = 0, dk = 0, dv = 0, dtype = 0;
  // true: the tensor-core path (bf16, dk = dv = 128).  Its saved chunk-start
  // states are 128-byte-swizzled K-major tf32 tiles (see kd_fwd_tc.cu), and
  // its forward scratch always holds them.
  bool tc = false;
  int NC = 0;             // ceil(T / 64)
  size_t chunks = 0;      // B * H * NC
  // forward scratch (always): y [ch][64], A [ch][64][64], P [ch][64][64];
  // tensor-core path, operands of the chain: cross-chunk matrix Hx [ch][64][64],
  // K~ and K^e [B][T][H][dk] (fp32), gamma_C [ch][dk], V^T [ch][dv][64] (bf16 tile)
  size_t y = 0, A = 0, P = 0, Hx = 0, Kt = 0, Ke = 0, GC = 0, Vt = 0;
  // tensor-core path: one int per chunk, set by the preparation kernel when
  // the chunk's in-chunk |L| reaches kExactStateRange (the chain then also
  // keeps its chunk-start state in fp32 for the exact paths)
  size_t xflags = 0;
  size_t fwd_bytes = 0;
  // saved for the backward: S0 [ch][dv][dk], u [ch][64], b0 [ch][64]
  size_t S0 = 0, u = 0, b0 = 0, flags = 0;  // flags: one int per chunk (tensor-core path)
  // tensor-core path: chunk-start states as bf16 128-byte-swizzled K-major
  // tiles [r][j] (rows r, K = j), read by the output kernel and the backward
  size_t S0b = 0;
  size_t fwd_save_bytes = 0;
  // backward scratch: dSC [ch][dv][dk], g [ch][64], dP/dGK/dGVs [slot][64][64],
  // accq/acck/accL [slot][64][dk], accv [slot][64][dv] (slot = chunk on the
  // CUDA-core path; on the tensor-core path one of kExactSlots slots)
  size_t dSC = 0, g = 0, dP = 0, dGK = 0, dGVs = 0, accq = 0, acck = 0, accL = 0, accv = 0;
  size_t du = 0;  // per-chunk intra-chunk part of du (tensor-core path) [ch][64]
  size_t dSCb = 0;    // tensor-core path: dS per chunk as a bf16 tile (as S0b)
  size_t bflags = 0;  // tensor-core path: one int per chunk (exact-path fallback)
  // tensor-core path, chunk adjoints known before the reverse chain (bf16
  // 128-byte-swizzled tiles): [dP; E_V] (128 x 64), P diag(u) and E_K
  // (64 x 64 each); M u [ch][64]
  size_t T1 = 0, PU = 0, EK = 0, Mu = 0;
  // tensor-core path, written by the pre-chain kernel for the reverse chain:
  // K+ [B][T][H][dk] fp32, and Q+^T per chunk as a bf16 128-byte-swizzled
  // K-major tile [j][t] (128 rows x 64)
  size_t Kp = 0, QpT = 0;
  size_t dapart = 0;  // gated inputs: each chunk's part of da_log [ch]
  size_t bwd_bytes = 0;
  // Gated inputs (forget pre-activations in place of logf): logf is formed
  // once into the forward's workspace (glogf, [B][T][H][dk] fp32, after the
  // saved region; on the tensor-core path by the preparation kernel), and
  // every later kernel reads it there.  The CUDA-core path takes dlogf in the
  // backward's workspace (gdlogf) before forming df~.
  size_t glogf = 0, gdlogf = 0;
  size_t fwd_gated_bytes = 0, bwd_gated_bytes = 0;
  // Fused prologue (raw q, k, v and gate pre-activations).  Forward: the
  // gated beta and c [B][T][H] (fp32) and the normalised q, k, v [B][T][H][d]
  // (activation dtype) of every token, written by the preparation kernel on
  // the tensor-core path and by the prologue pass on the CUDA-core path, and
  // read by every later kernel.  Backward, CUDA-core path: the recurrence's
  // gradients and the prologue backward's scratch.
  size_t fbeta = 0, fc = 0, fq = 0, fk = 0, fv = 0;
  size_t gdq = 0, gdk = 0, gdv = 0, gdbeta = 0, gdc = 0, gdf = 0, gpro = 0;
  size_t fwd_fused_bytes = 0, bwd_fused_bytes = 0;
};

// Phases of a forward or backward call.  kPhaseLocal: the work that does not
// depend on the carried state (the initial state S0 in the forward, the
// final-state gradient dST in the backward); kPhaseCarry: the chain over
// chunks and everything after it.  A carry phase needs the local phase of the
// same call to have run before it on the same workspaces and inputs.
constexpr int kPhaseLocal = 1, kPhaseCarry = 2, kPhaseAll = 3;

struct DecodeArgs {
  const void *q, *k, *v;
  const float *beta, *c, *logf;
  float* S;
  void* out;
  int B, H, dk, dv, dtype;
};

struct FwdArgs {
  const void *q, *k, *v;
  const float *beta, *c, *logf, *S0;
  void* out;
  float* ST;
  int save;
  char* ws;  // workspace base
  Layout L;
  int phases = kPhaseAll;
  // gated inputs (tensor-core path): logf then points at the bf16 forget
  // pre-activations and a_log at the per-head exponents; nullptr otherwise
  const float* a_log = nullptr;
  Pro pro;  // fused prologue (tensor-core path)
  // false: stop after the chunk chain (the backward's recompute of the saved
  // quantities needs no output; tensor-core path)
  bool keep_out = true;
};

struct BwdArgs {
  const void *q, *k, *v;
  const float *beta, *c, *logf, *S0;
  const void* dO;
  const float* dST;
  void *dq, *dk, *dv;
  float *dbeta, *dc, *dlogf, *dS0;
  const char* fws;  // forward workspace (saved)
  char* ws;         // backward workspace
  Layout L;
  int phases = kPhaseAll;
  // gated inputs (tensor-core path): logf points at the bf16 forget
  // pre-activations, dlogf receives df~ (fp32) and a_log holds the per-head
  // exponents; nullptr otherwise
  const float* a_log = nullptr;
  Pro pro;  // fused prologue (tensor-core path): dbeta and dc then receive the pre-activations' gradients
};

// Sets the calling thread's kron_delta_last_error() string.
void set_error(const char* msg);

// Profiling brackets around each kernel launch (no-ops unless enabled).
void prof_begin(cudaStream_t st, const char* name);
void prof_end(cudaStream_t st);

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t st);
cudaError_t launch_fwd_prep(const FwdArgs& a, bool with_P, cudaStream_t st);
// err: the library's device error word; sms: multiprocessors of the device.
cudaError_t launch_fwd_tc(const FwdArgs& a, int* err, int sms, cudaStream_t st);
int choose_cluster(int units, int sms);
// the forward's sequential chunk chain on tensor cores, R CTAs per head (kd_fchain_tc.cu)
cudaError_t launch_fwd_chain_tc(const FwdArgs& a, int R, int* err, cudaStream_t st);
// the backward's reverse chunk chain on tensor cores (kd_bchain_tc.cu)
cudaError_t launch_bwd_chain_tc(const BwdArgs& a, int R, int* err, cudaStream_t st);
cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t st);
// CUDA-core backward kernels by stage; `only` (nullable) restricts the
// per-chunk stages (cc, state, intra) to chunks whose flag is set.
constexpr int kStageChain = 1, kStageCC = 2, kStageState = 4, kStageIntra = 8, kStageAll = 15;
cudaError_t launch_bwd_simt_stages(const BwdArgs& a, int stages, const int* only, cudaStream_t st);
cudaError_t launch_bwd_tc(const BwdArgs& a, int* err, int sms, cudaStream_t st);
// per-chunk tensor-core kernels before / after the reverse chain (kd_bwd_chunk_tc.cu)
cudaError_t launch_bwd_pre_tc(const BwdArgs& a, int* err, int sms, cudaStream_t st);
cudaError_t launch_bwd_post_tc(const BwdArgs& a, int* err, cudaStream_t st);

// Input prologue (kd_prologue.cu).  N = B*T tokens; rows are [N][H][d].
struct PrologueArgs {
  const void *q_raw, *k_raw, *v_raw;
  const float *beta_pre, *c_pre;
  const void* f_pre;
  const float* a_log;
  float beta_scale;
  // forward outputs
  void *q, *k, *v;
  float *beta, *c, *logf;
  // backward: upstream gradients in, input gradients out
  const void *gq, *gk, *gv;  // dq, dk, dv of the normalised q, k, v
  const float *dbeta, *dc, *dlogf;
  void *dq_raw, *dk_raw, *dv_raw;
  float *dbeta_pre, *dc_pre;
  void* df_pre;
  float* da_log;
  float* part;  // backward scratch: prologue_blocks(N) * H floats
  long long N;
  int H, dk, dv, dtype;
};
int prologue_blocks(long long N);
cudaError_t launch_prologue_fwd(const PrologueArgs& a, cudaStream_t st);
cudaError_t launch_prologue_bwd(const PrologueArgs& a, cudaStream_t st);

// Output epilogue (kd_epilogue.cu).  rows = B*T*H rows of dv channels.
struct EpilogueArgs {
  const void *o, *g;
  const float* w;
  void* y;                 // forward output
  const void* dy;          // backward: upstream gradient in
  void *dO, *dg;           // backward: gradients out
  float* dw;
  float* part;             // backward scratch: epilogue_blocks(rows) * dv floats
  long long rows;
  int dv, dtype;
};
int epilogue_blocks(long long rows);
cudaError_t launch_epilogue_fwd(const EpilogueArgs& a, cudaStream_t st);
cudaError_t launch_epilogue_bwd(const EpilogueArgs& a, cudaStream_t st);

// Gated DeltaNet-2 rule (kd_gdn2.cu).  Workspace per chunk ch (fp32):
// forward (read again by the backward): A, P [C][C]; W, Q+, K^e [C][dk];
// U', U [C][dv]; e^Lambda [dk]; chunk-start state S0 [dv][dk].  Backward:
// dU [C][dv], chunk-end state gradient dS [dv][dk], dE, dQ+, dK^e [C][dk],
// dT, dP [C][C].
struct GdnLayout {
  int B = 0, H = 0, T = 0, dk = 0, dv = 0, dtype = 0, NC = 0;
  size_t chunks = 0;
  size_t A = 0, P = 0, W = 0, Up = 0, Ke = 0, Qp = 0, gC = 0, S0 = 0, U = 0, fwd_bytes = 0;
  size_t dU = 0, dS = 0, dE = 0, dT = 0, dP = 0, dQp = 0, dKe = 0, bwd_bytes = 0;
  // tensor-core path (bf16, dk = dv = 128): the chunk-start states are kept in
  // bf16 (the high part of the chain's fp32 state) in the 128-byte-swizzled
  // K-major image the chain and the output kernel hold in shared memory ([ch]
  // 32 KB, in the forward's workspace, where S0 is not allocated), and so are
  // the backward's dS; its gradient kernel reads both images and writes fp32
  // S0 (S0b) and dS only for the chunks the exact kernel takes
  bool tc = false;
  size_t S0img = 0, S0b = 0;
  // tensor-core path: the chains' B operands as bf16 hi, lo images (32 KB per
  // chunk each), W [t][j] and K^e [t][j], written by the preparation kernel
  // and read by both chains; W and K^e are not kept in fp32 there
  size_t Wimg = 0, Kimg = 0;
  // tensor-core backward: the reverse chain's chunk-local terms P^T dO [ch][t][r]
  // and (dO^T Q+)^T [ch][j][r] (fp32), and its saved dS images (as S0img)
  size_t dUi = 0, L2t = 0, dSimg = 0;
  // tensor-core backward: one byte per chunk, set where the exact kernel takes the chunk
  size_t xflag = 0;
};
struct GdnWs {
  float *A, *P, *W, *Up, *Ke, *Qp, *gC, *S0, *U;
  float *dU, *dS, *dE, *dT, *dP, *dQp, *dKe;
  __nv_bfloat16* S0img;  // tensor-core path: the chunk-start state images
  __nv_bfloat16 *Wimg, *Kimg;                    // tensor-core path: the chains' operand images
  float *dUi, *L2t;                              // tensor-core backward: the chain's chunk-local terms
  __nv_bfloat16* dSimg;                          // tensor-core backward: the saved dS images
  unsigned char* xflag;                          // tensor-core backward: the exact kernel's chunks
};
inline GdnWs gdn_ws(char* base, const GdnLayout& L) {
  auto f = [&](size_t o) { return reinterpret_cast<float*>(base + o); };
  return GdnWs{f(L.A), f(L.P), L.tc ? nullptr : f(L.W), f(L.Up), L.tc ? nullptr : f(L.Ke), f(L.Qp), f(L.gC),
               L.tc ? nullptr : f(L.S0), f(L.U),
               nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
               L.tc ? reinterpret_cast<__nv_bfloat16*>(base + L.S0img) : nullptr,
               L.tc ? reinterpret_cast<__nv_bfloat16*>(base + L.Wimg) : nullptr,
               L.tc ? reinterpret_cast<__nv_bfloat16*>(base + L.Kimg) : nullptr,
               nullptr, nullptr, nullptr, nullptr};
}
inline void gdn_bwd_ws(char* base, const GdnLayout& L, GdnWs* p) {
  auto f = [&](size_t o) { return reinterpret_cast<float*>(base + o); };
  p->dU = f(L.dU); p->dS = f(L.dS); p->dE = f(L.dE); p->dT = f(L.dT); p->dP = f(L.dP);
  p->dQp = f(L.dQp); p->dKe = f(L.dKe);
  if (L.tc) {
    p->S0 = f(L.S0b);
    p->dUi = f(L.dUi);
    p->L2t = f(L.L2t);
    p->dSimg = reinterpret_cast<__nv_bfloat16*>(base + L.dSimg);
    p->xflag = reinterpret_cast<unsigned char*>(base + L.xflag);
  }
}
struct GdnArgs {
  const void *q, *k, *v;
  const float *b, *w, *loga, *S0;
  void* out;
  float* ST;
  const void* dO;
  const float* dST;
  void *dq, *dk, *dv;
  float *db, *dw, *dloga, *dS0;
  const char* fws;
  char* ws;
  GdnLayout L;
  int* err = nullptr;  // the library's device error word (tensor-core kernels' bounded waits)
};
struct GdnDecodeArgs {
  const void *q, *k, *v;
  const float *b, *w, *loga;
  float* S;
  void* out;
  int B, H, dk, dv, dtype;
};
cudaError_t launch_gdn2_decode(const GdnDecodeArgs& a, cudaStream_t st);
cudaError_t launch_gdn2_fwd(const GdnArgs& a, cudaStream_t st);
// bf16 with d_k = d_v = 128: the per-chunk preparation runs on tensor cores
bool gdn2_tc_supported(const GdnLayout& L);
cudaError_t launch_gdn2_prep_tc(const GdnArgs& a, int* err, cudaStream_t st);
cudaError_t launch_gdn2_out_tc(const GdnArgs& a, int* err, cudaStream_t st);
cudaError_t launch_gdn2_chain_tc(const GdnArgs& a, int* err, cudaStream_t st);
// the backward's pre-chain terms and operand images, and its reverse chain
cudaError_t launch_gdn2_bchain_tc(const GdnArgs& a, const GdnWs& p, int* err, cudaStream_t st);
// the backward's per-chunk gradients (every chunk's dv, dw; the factorised
// chunks' dq, dk, db, dloga; the exact kernel's inputs for the others)
cudaError_t launch_gdn2_bpost_tc(const GdnArgs& a, const GdnWs& p, int* err, cudaStream_t st);
cudaError_t launch_gdn2_bwd(const GdnArgs& a, cudaStream_t st);

// Gated inputs (kd_gate.cu): logf = e^{a_log} log sigma(f~) into a buffer
// (the CUDA-core path); df~ = dlogf a sigma(-f~) and each chunk's part of
// da_log from dlogf and logf (the CUDA-core path); da_log per head from the
// per-chunk parts, summed in a fixed order.
cudaError_t launch_gate_logf(const void* fpre, int dtype, const float* a_log, float* logf, int B, int T, int H,
                             int dk, cudaStream_t st);
cudaError_t launch_gate_dlogf(const float* dlogf, const float* logf, const float* a_log, float* dfpre,
                              float* dapart, int B, int T, int H, int dk, int NC, cudaStream_t st);
cudaError_t launch_prologue_tail_bwd(const void* q_raw, const void* k_raw, const void* v_raw, const float* beta_pre,
                                     const float* c_pre, float bscale, void* dq, void* dk, void* dv, float* dbeta,
                                     float* dc, size_t rows, cudaStream_t st);
cudaError_t launch_reduce_dalog(const float* dapart, int B, int H, int NC, float* da_log, cudaStream_t st);

// Failure-reporting self-test (kd_selftest.cu): a bounded wait that runs out.
cudaError_t launch_selftest_timeout(int* err, cudaStream_t st);

template <typename T>
inline T* ws_ptr(char* base, size_t off) { return reinterpret_cast<T*>(base + off); }
template <typename T>
inline const T* ws_ptr(const char* base, size_t off) { return reinterpret_cast<const T*>(base + off); }

}  // namespace kd
