// kd_api.cu -- C ABI and chunk scheduler of the Kronecker delta rule library.
//
// The scheduler validates a call, derives the chunk count NC = ceil(T/64)
// (Gated DeltaNet-2 article, "기술 상세": C = 64), lays out the workspace and
// enqueues the kernels of the call on the caller's stream, in order, without
// synchronising.  Declarations and argument contracts: include/kron_delta.h.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/kron_delta.h"
#include "kd_kernels.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int ok() {
  g_err.clear();
  return KD_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool dim_supported(int d) { return d == 32 || d == 64 || d == 128; }

// Validates sizes and fills the workspace layout.  Returns KD_OK or an error.
int plan(int B, int H, int T, int dk, int dv, int dtype, kd::Layout* L) {
  if (B <= 0 || H <= 0 || T <= 0) return fail(KD_ERR_INVALID_ARG, "B, H, T must be >= 1 (got %d, %d, %d)", B, H, T);
  if (!dim_supported(dk) || !dim_supported(dv))
    return fail(KD_ERR_UNSUPPORTED, "dk and dv must be 32, 64 or 128 (got %d, %d)", dk, dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  if (H > 65535 || B > 65535) return fail(KD_ERR_INVALID_ARG, "B and H must be <= 65535 (got %d, %d)", B, H);
  const int NC = (T + kd::kChunk - 1) / kd::kChunk;
  const size_t chunks = (size_t)B * H * NC;
  if (chunks > (size_t(1) << 31)) return fail(KD_ERR_INVALID_ARG, "problem too large (%zu chunks)", chunks);
  L->B = B; L->H = H; L->T = T; L->dk = dk; L->dv = dv; L->dtype = dtype;
  L->NC = NC;
  L->chunks = chunks;
  const size_t C = kd::kChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L->tc = dtype == KD_BF16 && dk == 128 && dv == 128;
  L->y = take(chunks * C * 4);
  L->A = take(chunks * C * C * 4);
  L->P = take(chunks * C * C * 4);  // tensor-core path: written only when saving for the backward
  if (L->tc) {
    L->Hx = take(chunks * C * C * 4);
    L->Kt = take((size_t)B * T * H * dk * 4);
    L->Ke = take((size_t)B * T * H * dk * 4);
    L->GC = take(chunks * (size_t)dk * 4);
    L->Vt = take(chunks * (size_t)dv * C * 2);
    L->xflags = take(chunks * 4);
  }
  L->fwd_bytes = off;
  L->S0 = take(chunks * (size_t)dv * dk * 4);  // tensor-core path: written only for chunks with xflags set
  L->u = take(chunks * C * 4);
  L->b0 = take(chunks * C * 4);
  L->flags = take(chunks * 4);
  if (L->tc) L->S0b = take(chunks * (size_t)dv * dk * 2);
  if (L->tc) L->fwd_bytes = off;  // the chain writes u, b0 and the chunk-start states on every call
  L->fwd_save_bytes = off;
  L->glogf = take((size_t)B * T * H * dk * 4);  // gated inputs: logf, formed once
  L->fwd_gated_bytes = off;
  // fused prologue: the gated beta and c of every token; q, k, v normalised
  // (tensor-core path: rows of chunks with xflags set, for the exact paths;
  // CUDA-core path: all, written by the prologue pass)
  const size_t act = dtype == KD_BF16 ? 2 : 4;
  L->fbeta = take((size_t)B * T * H * 4);
  L->fc = take((size_t)B * T * H * 4);
  L->fq = take((size_t)B * T * H * dk * act);
  L->fk = take((size_t)B * T * H * dk * act);
  L->fv = take((size_t)B * T * H * dv * act);
  L->fwd_fused_bytes = off;

  off = 0;
  L->dSC = L->tc ? 0 : take(chunks * (size_t)dv * dk * 4);  // the tensor-core path keeps bf16 tiles
  L->g = take(chunks * C * 4);
  // exact-path scratch: every chunk on the CUDA-core path; on the tensor-core
  // path only the flagged chunks use it, one kExactSlots slot per CTA
  const size_t slots = L->tc ? (chunks < (size_t)kd::kExactSlots ? chunks : (size_t)kd::kExactSlots) : chunks;
  L->dP = take(slots * C * C * 4);
  L->dGK = take(slots * C * C * 4);
  L->dGVs = take(slots * C * C * 4);
  L->accq = take(slots * C * dk * 4);
  L->acck = take(slots * C * dk * 4);
  L->accL = take(slots * C * dk * 4);
  L->accv = take(slots * C * dv * 4);
  L->du = take(chunks * C * 4);
  if (L->tc) {
    L->dSCb = take(chunks * (size_t)dv * dk * 2);
    L->bflags = take(chunks * 4);
    L->T1 = take(chunks * 2 * C * C * 2);
    L->PU = take(chunks * C * C * 2);
    L->EK = take(chunks * C * C * 2);
    L->Mu = take(chunks * C * 4);
    L->Kp = take((size_t)B * T * H * dk * 4);
    L->QpT = take(chunks * (size_t)dk * C * 2);
  }
  L->dapart = take(chunks * 4);
  L->bwd_bytes = off;
  if (!L->tc) L->gdlogf = take((size_t)B * T * H * dk * 4);  // gated inputs, CUDA-core path: dlogf
  L->bwd_gated_bytes = off;
  // fused prologue, CUDA-core path: the recurrence's gradients, then the
  // prologue backward's own scratch (the tensor-core path finishes in place)
  if (!L->tc) {
    L->gdq = take((size_t)B * T * H * dk * act);
    L->gdk = take((size_t)B * T * H * dk * act);
    L->gdv = take((size_t)B * T * H * dv * act);
    L->gdbeta = take((size_t)B * T * H * 4);
    L->gdc = take((size_t)B * T * H * 4);
    L->gdf = take((size_t)B * T * H * dk * act);  // the prologue backward's df~ (the fp32 one is formed apart)
    L->gpro = take((size_t)kd::prologue_blocks((long long)B * T) * H * sizeof(float));
  }
  L->bwd_fused_bytes = off;
  return KD_OK;
}

// Validates sizes and fills the Gated DeltaNet-2 workspace layout.
int gdn_plan(int B, int H, int T, int dk, int dv, int dtype, kd::GdnLayout* L) {
  if (B <= 0 || H <= 0 || T <= 0) return fail(KD_ERR_INVALID_ARG, "B, H, T must be >= 1 (got %d, %d, %d)", B, H, T);
  if (!dim_supported(dk) || !dim_supported(dv))
    return fail(KD_ERR_UNSUPPORTED, "dk and dv must be 32, 64 or 128 (got %d, %d)", dk, dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  if (H > 65535 || B > 65535) return fail(KD_ERR_INVALID_ARG, "B and H must be <= 65535 (got %d, %d)", B, H);
  const int NC = (T + kd::kChunk - 1) / kd::kChunk;
  const size_t chunks = (size_t)B * H * NC;
  if (chunks > (size_t(1) << 31)) return fail(KD_ERR_INVALID_ARG, "problem too large (%zu chunks)", chunks);
  L->B = B; L->H = H; L->T = T; L->dk = dk; L->dv = dv; L->dtype = dtype; L->NC = NC; L->chunks = chunks;
  const size_t C = kd::kChunk;
  size_t off = 0;
  auto take = [&](size_t floats) { size_t o = off; off = align256(off + floats * 4); return o; };
  L->tc = dtype == KD_BF16 && dk == 128 && dv == 128;
  L->A = take(chunks * C * C);
  L->P = take(chunks * C * C);
  L->Up = take(chunks * C * dv);
  L->Qp = take(chunks * C * dk);
  L->gC = take(chunks * dk);
  if (L->tc) {
    L->S0img = take(chunks * (size_t)dv * dk / 2);  // bf16
    L->Wimg = take(chunks * C * dk);
    L->Kimg = take(chunks * C * dk);
  } else {
    L->W = take(chunks * C * dk);
    L->Ke = take(chunks * C * dk);
    L->S0 = take(chunks * (size_t)dv * dk);
  }
  L->U = take(chunks * C * dv);
  L->fwd_bytes = off;
  off = 0;
  L->dU = take(chunks * C * dv);
  L->dS = take(chunks * (size_t)dv * dk);
  L->dE = take(chunks * C * dk);
  L->dT = take(chunks * C * C);
  L->dP = take(chunks * C * C);
  L->dQp = take(chunks * C * dk);
  L->dKe = take(chunks * C * dk);
  if (L->tc) {
    L->S0b = take(chunks * (size_t)dv * dk);
    L->dUi = take(chunks * C * dv);
    L->L2t = take(chunks * (size_t)dk * dv);
    L->dSimg = take(chunks * (size_t)dv * dk / 2);
    L->xflag = take((chunks + 3) / 4);
  }
  L->bwd_bytes = off;
  return KD_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_ptr(const void* p, const char* name, bool required) {
  if (!p) return required ? fail(KD_ERR_INVALID_ARG, "%s must not be NULL", name) : KD_OK;
  if (!aligned(p, 16)) return fail(KD_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  return KD_OK;
}

int check_stream(void* stream) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(KD_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
#if CUDART_VERSION >= 12080
  if (stream) {
    int sdev = -1;
    e = cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev);
    if (e != cudaSuccess) return fail(KD_ERR_INVALID_ARG, "invalid stream: %s", cudaGetErrorString(e));
    if (sdev != dev)
      return fail(KD_ERR_INVALID_ARG, "stream belongs to device %d but the current device is %d", sdev, dev);
  }
#endif
  return KD_OK;
}

int launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(KD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return ok();
}

// ---- device error word (bounded device-side waits report here) ------------
__device__ int g_kd_dev_err;

struct DeviceInfo {
  int* err = nullptr;
  int sms = 0;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

// Error-word address and SM count of the current device (queried once).
int device_info(DeviceInfo* out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(KD_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(KD_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> g(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.err) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kd_dev_err);
    if (e != cudaSuccess) return fail(KD_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(KD_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    d.sms = sms;
    d.err = static_cast<int*>(p);
  }
  *out = d;
  return KD_OK;
}

// ---- per-kernel timing (kron_delta_profile_*) ----------------------------
struct ProfState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  struct Pending { std::string name; cudaEvent_t a, b; };
  std::vector<Pending> pending;
  std::string open_name;
  cudaEvent_t open_a = nullptr;
  std::map<std::string, std::pair<long, double>> totals;  // launches, ms
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
ProfState& prof() {
  static ProfState* p = new ProfState();  // never destroyed: usable during exit
  return *p;
}

// The backward with recompute: its workspace holds a save-forward workspace,
// then (CUDA-core path only, whose forward always writes the output) a scratch
// output, then the backward's own scratch.
size_t recompute_out_bytes(const kd::Layout& L, int B, int H, int T, int dv, int dtype) {
  return L.tc ? 0 : align256((size_t)B * T * H * dv * (dtype == KD_BF16 ? 2 : 4));
}
size_t recompute_bytes(const kd::Layout& L, int B, int H, int T, int dv, int dtype) {
  return align256(L.fwd_save_bytes) + recompute_out_bytes(L, B, H, T, dv, dtype) + L.bwd_bytes;
}

}  // namespace

namespace kd {
void set_error(const char* msg) { g_err = msg ? msg : ""; }

void prof_begin(cudaStream_t st, const char* name) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on) return;
  p.open_a = p.get();
  p.open_name = name;
  if (p.open_a) cudaEventRecord(p.open_a, st);
}
void prof_end(cudaStream_t st) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on || !p.open_a) return;
  cudaEvent_t b = p.get();
  if (b) {
    cudaEventRecord(b, st);
    p.pending.push_back({p.open_name, p.open_a, b});
  } else {
    p.pool.push_back(p.open_a);
  }
  p.open_a = nullptr;
}
}  // namespace kd

#define KD_TRY(x)          \
  do {                     \
    int rc_ = (x);         \
    if (rc_ != KD_OK) return rc_; \
  } while (0)

extern "C" {

int kron_delta_version(void) { return 200; }

const char* kron_delta_last_error(void) { return g_err.c_str(); }

size_t kron_delta_workspace_size(int kind, int B, int H, int T, int dk, int dv, int dtype) {
  kd::Layout L;
  if (plan(B, H, T, dk, dv, dtype, &L) != KD_OK) return 0;
  switch (kind) {
    case KD_WS_FWD: ok(); return L.fwd_bytes;
    case KD_WS_FWD_SAVE: ok(); return L.fwd_save_bytes;
    case KD_WS_BWD: ok(); return L.bwd_bytes;
    case KD_WS_BWD_RECOMPUTE: ok(); return recompute_bytes(L, B, H, T, dv, dtype);
    case KD_WS_FWD_FUSED: ok(); return L.fwd_fused_bytes;
    case KD_WS_BWD_FUSED: ok(); return L.bwd_fused_bytes;
    case KD_WS_FWD_GATED: ok(); return L.fwd_gated_bytes;
    case KD_WS_BWD_GATED: ok(); return L.bwd_gated_bytes;
    case KD_WS_PROLOGUE_BWD:
      ok();
      return align256((size_t)kd::prologue_blocks((long long)B * T) * H * sizeof(float));
    case KD_WS_GDN2_FWD:
    case KD_WS_GDN2_BWD: {
      kd::GdnLayout G;
      if (gdn_plan(B, H, T, dk, dv, dtype, &G) != KD_OK) return 0;
      ok();
      return kind == KD_WS_GDN2_FWD ? G.fwd_bytes : G.bwd_bytes;
    }
    case KD_WS_EPILOGUE_BWD:
      ok();
      return align256((size_t)kd::epilogue_blocks((long long)B * T * H) * dv * sizeof(float));
    default: fail(KD_ERR_INVALID_ARG, "unknown workspace kind %d", kind); return 0;
  }
}

int kron_delta_fwd(const void* q, const void* k, const void* v, const float* beta,
                   const float* c, const float* logf, const float* S0, void* out, float* ST,
                   int B, int H, int T, int dk, int dv, int dtype, void* workspace,
                   size_t ws_bytes, int save, void* stream) {
  return kron_delta_fwd_phase(q, k, v, beta, c, logf, S0, out, ST, B, H, T, dk, dv, dtype, workspace,
                              ws_bytes, save, KD_PHASE_ALL, stream);
}

int kron_delta_fwd_phase(const void* q, const void* k, const void* v, const float* beta,
                         const float* c, const float* logf, const float* S0, void* out, float* ST,
                         int B, int H, int T, int dk, int dv, int dtype, void* workspace,
                         size_t ws_bytes, int save, int phase, void* stream) {
  if (phase != KD_PHASE_LOCAL && phase != KD_PHASE_CARRY && phase != KD_PHASE_ALL)
    return fail(KD_ERR_INVALID_ARG, "phase must be KD_PHASE_LOCAL, KD_PHASE_CARRY or KD_PHASE_ALL (got %d)", phase);
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk, dv, dtype, &L));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(beta, "beta", true));
  KD_TRY(check_ptr(c, "c", true));
  KD_TRY(check_ptr(logf, "logf", true));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(out, "out", true));
  KD_TRY(check_ptr(ST, "ST", false));
  if (save != 0 && save != 1) return fail(KD_ERR_INVALID_ARG, "save must be 0 or 1");
  const size_t need = save ? L.fwd_save_bytes : L.fwd_bytes;
  if (!workspace || ws_bytes < need)
    return fail(KD_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  kd::FwdArgs a{q, k, v, beta, c, logf, S0, out, ST, save, static_cast<char*>(workspace), L, phase};
  if (L.tc) {
    DeviceInfo di;
    KD_TRY(device_info(&di));
    return launched(kd::launch_fwd_tc(a, di.err, di.sms, static_cast<cudaStream_t>(stream)),
                    "forward launch");
  }
  return launched(kd::launch_fwd_simt(a, static_cast<cudaStream_t>(stream)), "forward launch");
}

int kron_delta_bwd(const void* q, const void* k, const void* v, const float* beta,
                   const float* c, const float* logf, const float* S0, const void* dO,
                   const float* dST, void* dq, void* dk, void* dv, float* dbeta, float* dc,
                   float* dlogf, float* dS0, int B, int H, int T, int dk_, int dv_, int dtype,
                   const void* fwd_ws, size_t fwd_ws_bytes, void* workspace, size_t ws_bytes,
                   void* stream) {
  return kron_delta_bwd_phase(q, k, v, beta, c, logf, S0, dO, dST, dq, dk, dv, dbeta, dc, dlogf, dS0, B, H,
                              T, dk_, dv_, dtype, fwd_ws, fwd_ws_bytes, workspace, ws_bytes, KD_PHASE_ALL,
                              stream);
}

int kron_delta_bwd_phase(const void* q, const void* k, const void* v, const float* beta,
                         const float* c, const float* logf, const float* S0, const void* dO,
                         const float* dST, void* dq, void* dk, void* dv, float* dbeta, float* dc,
                         float* dlogf, float* dS0, int B, int H, int T, int dk_, int dv_, int dtype,
                         const void* fwd_ws, size_t fwd_ws_bytes, void* workspace, size_t ws_bytes,
                         int phase, void* stream) {
  if (phase != KD_PHASE_LOCAL && phase != KD_PHASE_CARRY && phase != KD_PHASE_ALL)
    return fail(KD_ERR_INVALID_ARG, "phase must be KD_PHASE_LOCAL, KD_PHASE_CARRY or KD_PHASE_ALL (got %d)", phase);
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk_, dv_, dtype, &L));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(beta, "beta", true));
  KD_TRY(check_ptr(c, "c", true));
  KD_TRY(check_ptr(logf, "logf", true));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(dO, "dO", true));
  KD_TRY(check_ptr(dST, "dST", false));
  KD_TRY(check_ptr(dq, "dq", true));
  KD_TRY(check_ptr(dk, "dk", true));
  KD_TRY(check_ptr(dv, "dv", true));
  KD_TRY(check_ptr(dbeta, "dbeta", true));
  KD_TRY(check_ptr(dc, "dc", true));
  KD_TRY(check_ptr(dlogf, "dlogf", true));
  KD_TRY(check_ptr(dS0, "dS0", false));
  if (!fwd_ws || fwd_ws_bytes < L.fwd_save_bytes)
    return fail(KD_ERR_WORKSPACE, "forward workspace saved with save=1 of %zu bytes needed (got %zu)",
                L.fwd_save_bytes, fwd_ws ? fwd_ws_bytes : 0);
  if (!workspace || ws_bytes < L.bwd_bytes)
    return fail(KD_ERR_WORKSPACE, "backward workspace of %zu bytes needed (got %zu)", L.bwd_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256) || !aligned(fwd_ws, 256))
    return fail(KD_ERR_WORKSPACE, "workspaces must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  (void)S0;  // the forward state at every chunk start is read from fwd_ws
  kd::BwdArgs a{q, k, v, beta, c, logf, S0, dO, dST, dq, dk, dv, dbeta, dc, dlogf, dS0,
                static_cast<const char*>(fwd_ws), static_cast<char*>(workspace), L, phase};
  if (L.tc) {
    DeviceInfo di;
    KD_TRY(device_info(&di));
    return launched(kd::launch_bwd_tc(a, di.err, di.sms, static_cast<cudaStream_t>(stream)),
                    "backward launch");
  }
  return launched(kd::launch_bwd_simt(a, static_cast<cudaStream_t>(stream)), "backward launch");
}

int kron_delta_bwd_recompute(const void* q, const void* k, const void* v, const float* beta,
                             const float* c, const float* logf, const float* S0, const void* dO,
                             const float* dST, void* dq, void* dk, void* dv, float* dbeta, float* dc,
                             float* dlogf, float* dS0, int B, int H, int T, int dk_, int dv_, int dtype,
                             void* workspace, size_t ws_bytes, void* stream) {
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk_, dv_, dtype, &L));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(beta, "beta", true));
  KD_TRY(check_ptr(c, "c", true));
  KD_TRY(check_ptr(logf, "logf", true));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(dO, "dO", true));
  KD_TRY(check_ptr(dST, "dST", false));
  KD_TRY(check_ptr(dq, "dq", true));
  KD_TRY(check_ptr(dk, "dk", true));
  KD_TRY(check_ptr(dv, "dv", true));
  KD_TRY(check_ptr(dbeta, "dbeta", true));
  KD_TRY(check_ptr(dc, "dc", true));
  KD_TRY(check_ptr(dlogf, "dlogf", true));
  KD_TRY(check_ptr(dS0, "dS0", false));
  const size_t need = recompute_bytes(L, B, H, T, dv_, dtype);
  if (!workspace || ws_bytes < need)
    return fail(KD_ERR_WORKSPACE, "backward-with-recompute workspace of %zu bytes needed (got %zu)", need,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  char* ws = static_cast<char*>(workspace);
  const size_t fwd_part = align256(L.fwd_save_bytes), out_part = recompute_out_bytes(L, B, H, T, dv_, dtype);
  // the forward with save = 1 into the first part; its output is not kept
  if (L.tc) {
    kd::FwdArgs a{q, k, v, beta, c, logf, S0, nullptr, nullptr, 1, ws, L, KD_PHASE_ALL};
    a.keep_out = false;
    DeviceInfo di;
    KD_TRY(device_info(&di));
    KD_TRY(launched(kd::launch_fwd_tc(a, di.err, di.sms, static_cast<cudaStream_t>(stream)), "forward launch"));
  } else {
    KD_TRY(kron_delta_fwd(q, k, v, beta, c, logf, S0, ws + fwd_part, nullptr, B, H, T, dk_, dv_, dtype, ws,
                          fwd_part, 1, stream));
  }
  return kron_delta_bwd(q, k, v, beta, c, logf, S0, dO, dST, dq, dk, dv, dbeta, dc, dlogf, dS0, B, H, T, dk_, dv_,
                        dtype, ws, fwd_part, ws + fwd_part + out_part, ws_bytes - fwd_part - out_part, stream);
}

int kron_delta_fwd_gated(const void* q, const void* k, const void* v, const float* beta,
                         const float* c, const void* f_pre, const float* a_log, const float* S0, void* out,
                         float* ST, int B, int H, int T, int dk, int dv, int dtype, void* workspace,
                         size_t ws_bytes, int save, void* stream) {
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk, dv, dtype, &L));
  KD_TRY(check_ptr(f_pre, "f_pre", true));
  KD_TRY(check_ptr(a_log, "a_log", true));
  if (!workspace || ws_bytes < L.fwd_gated_bytes)
    return fail(KD_ERR_WORKSPACE, "gated forward workspace of %zu bytes needed (got %zu)", L.fwd_gated_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (save != 0 && save != 1) return fail(KD_ERR_INVALID_ARG, "save must be 0 or 1");
  KD_TRY(check_stream(stream));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (L.tc) {
    KD_TRY(check_ptr(q, "q", true));
    KD_TRY(check_ptr(k, "k", true));
    KD_TRY(check_ptr(v, "v", true));
    KD_TRY(check_ptr(beta, "beta", true));
    KD_TRY(check_ptr(c, "c", true));
    KD_TRY(check_ptr(S0, "S0", false));
    KD_TRY(check_ptr(out, "out", true));
    KD_TRY(check_ptr(ST, "ST", false));
    kd::FwdArgs a{q, k, v, beta, c, static_cast<const float*>(f_pre), S0, out, ST, save,
                  static_cast<char*>(workspace), L, KD_PHASE_ALL};
    a.a_log = a_log;
    DeviceInfo di;
    KD_TRY(device_info(&di));
    return launched(kd::launch_fwd_tc(a, di.err, di.sms, st), "gated forward launch");
  }
  // CUDA-core path: logf into the workspace, then the plain forward on it
  float* glogf = kd::ws_ptr<float>(static_cast<char*>(workspace), L.glogf);
  const cudaError_t e = kd::launch_gate_logf(f_pre, dtype, a_log, glogf, B, T, H, dk, st);
  if (e != cudaSuccess) return launched(e, "gated forward launch");
  return kron_delta_fwd(q, k, v, beta, c, glogf, S0, out, ST, B, H, T, dk, dv, dtype, workspace, ws_bytes, save,
                        stream);
}

int kron_delta_bwd_gated(const void* q, const void* k, const void* v, const float* beta,
                         const float* c, const void* f_pre, const float* a_log, const float* S0,
                         const void* dO, const float* dST, void* dq, void* dk, void* dv, float* dbeta,
                         float* dc, float* df_pre, float* da_log, float* dS0, int B, int H, int T,
                         int dk_, int dv_, int dtype, const void* fwd_ws, size_t fwd_ws_bytes,
                         void* workspace, size_t ws_bytes, void* stream) {
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk_, dv_, dtype, &L));
  KD_TRY(check_ptr(f_pre, "f_pre", true));
  KD_TRY(check_ptr(a_log, "a_log", true));
  KD_TRY(check_ptr(df_pre, "df_pre", true));
  KD_TRY(check_ptr(da_log, "da_log", true));
  if (!fwd_ws || fwd_ws_bytes < L.fwd_gated_bytes)
    return fail(KD_ERR_WORKSPACE, "the gated forward's workspace (save=1) of %zu bytes needed (got %zu)",
                L.fwd_gated_bytes, fwd_ws ? fwd_ws_bytes : 0);
  if (!workspace || ws_bytes < L.bwd_gated_bytes)
    return fail(KD_ERR_WORKSPACE, "gated backward workspace of %zu bytes needed (got %zu)", L.bwd_gated_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256) || !aligned(fwd_ws, 256))
    return fail(KD_ERR_WORKSPACE, "workspaces must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* dapart = kd::ws_ptr<float>(ws, L.dapart);
  if (L.tc) {
    KD_TRY(check_ptr(q, "q", true));
    KD_TRY(check_ptr(k, "k", true));
    KD_TRY(check_ptr(v, "v", true));
    KD_TRY(check_ptr(beta, "beta", true));
    KD_TRY(check_ptr(c, "c", true));
    KD_TRY(check_ptr(dO, "dO", true));
    KD_TRY(check_ptr(dST, "dST", false));
    KD_TRY(check_ptr(dq, "dq", true));
    KD_TRY(check_ptr(dk, "dk", true));
    KD_TRY(check_ptr(dv, "dv", true));
    KD_TRY(check_ptr(dbeta, "dbeta", true));
    KD_TRY(check_ptr(dc, "dc", true));
    KD_TRY(check_ptr(dS0, "dS0", false));
    kd::BwdArgs a{q, k, v, beta, c, static_cast<const float*>(f_pre), S0, dO, dST, dq, dk, dv, dbeta, dc, df_pre,
                  dS0, static_cast<const char*>(fwd_ws), ws, L, KD_PHASE_ALL};
    a.a_log = a_log;
    DeviceInfo di;
    KD_TRY(device_info(&di));
    cudaError_t e = kd::launch_bwd_tc(a, di.err, di.sms, st);
    if (e == cudaSuccess) e = kd::launch_reduce_dalog(dapart, B, H, L.NC, da_log, st);
    return launched(e, "gated backward launch");
  }
  // CUDA-core path: the plain backward on the forward's logf, then df~ and da_log from dlogf
  const float* glogf = kd::ws_ptr<float>(static_cast<const char*>(fwd_ws), L.glogf);
  float* gdlogf = kd::ws_ptr<float>(ws, L.gdlogf);
  KD_TRY(kron_delta_bwd(q, k, v, beta, c, glogf, S0, dO, dST, dq, dk, dv, dbeta, dc, gdlogf, dS0, B, H, T, dk_,
                        dv_, dtype, fwd_ws, fwd_ws_bytes, workspace, ws_bytes, stream));
  cudaError_t e = kd::launch_gate_dlogf(gdlogf, glogf, a_log, df_pre, dapart, B, T, H, dk_, L.NC, st);
  if (e == cudaSuccess) e = kd::launch_reduce_dalog(dapart, B, H, L.NC, da_log, st);
  return launched(e, "gated backward launch");
}

namespace {
int check_prologue(const void* q_raw, const void* k_raw, const void* v_raw, const float* beta_pre,
                   const float* c_pre, const void* f_pre, const float* a_log, float beta_scale, int B,
                   int H, int T, int dk, int dv, int dtype) {
  if (B <= 0 || H <= 0 || T <= 0) return fail(KD_ERR_INVALID_ARG, "B, H, T must be >= 1 (got %d, %d, %d)", B, H, T);
  if (H > 65535) return fail(KD_ERR_INVALID_ARG, "H must be <= 65535 (got %d)", H);
  if (!dim_supported(dk) || !dim_supported(dv))
    return fail(KD_ERR_UNSUPPORTED, "dk and dv must be 32, 64 or 128 (got %d, %d)", dk, dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  if (!(beta_scale > 0.f && beta_scale <= 2.f))
    return fail(KD_ERR_INVALID_ARG, "beta_scale must be in (0, 2] (got %g)", (double)beta_scale);
  KD_TRY(check_ptr(q_raw, "q_raw", true));
  KD_TRY(check_ptr(k_raw, "k_raw", true));
  KD_TRY(check_ptr(v_raw, "v_raw", true));
  KD_TRY(check_ptr(beta_pre, "beta_pre", true));
  KD_TRY(check_ptr(c_pre, "c_pre", true));
  KD_TRY(check_ptr(f_pre, "f_pre", true));
  return check_ptr(a_log, "a_log", true);
}
}  // namespace

int kron_delta_fwd_fused(const void* q_raw, const void* k_raw, const void* v_raw, const float* beta_pre,
                         const float* c_pre, const void* f_pre, const float* a_log, float beta_scale,
                         const float* S0, void* out, float* ST, int B, int H, int T, int dk, int dv, int dtype,
                         void* workspace, size_t ws_bytes, int save, void* stream) {
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk, dv, dtype, &L));
  KD_TRY(check_prologue(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, B, H, T, dk, dv, dtype));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(out, "out", true));
  KD_TRY(check_ptr(ST, "ST", false));
  if (!workspace || ws_bytes < L.fwd_fused_bytes)
    return fail(KD_ERR_WORKSPACE, "fused forward workspace of %zu bytes needed (got %zu)", L.fwd_fused_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (save != 0 && save != 1) return fail(KD_ERR_INVALID_ARG, "save must be 0 or 1");
  KD_TRY(check_stream(stream));
  char* ws = static_cast<char*>(workspace);
  if (L.tc) {
    kd::FwdArgs a{q_raw, k_raw, v_raw, beta_pre, c_pre, static_cast<const float*>(f_pre), S0, out, ST, save, ws, L,
                  KD_PHASE_ALL};
    a.a_log = a_log;
    a.pro.bscale = beta_scale;
    a.pro.norm = 1;
    DeviceInfo di;
    KD_TRY(device_info(&di));
    return launched(kd::launch_fwd_tc(a, di.err, di.sms, static_cast<cudaStream_t>(stream)), "fused forward launch");
  }
  // CUDA-core path: the prologue pass into the workspace, then the forward on its outputs
  float* logf = kd::ws_ptr<float>(ws, L.glogf);
  KD_TRY(kron_delta_prologue_fwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, ws + L.fq,
                                 ws + L.fk, ws + L.fv, kd::ws_ptr<float>(ws, L.fbeta), kd::ws_ptr<float>(ws, L.fc),
                                 logf, B, H, T, dk, dv, dtype, stream));
  return kron_delta_fwd(ws + L.fq, ws + L.fk, ws + L.fv, kd::ws_ptr<float>(ws, L.fbeta), kd::ws_ptr<float>(ws, L.fc),
                        logf, S0, out, ST, B, H, T, dk, dv, dtype, workspace, L.fwd_save_bytes, save, stream);
}

int kron_delta_bwd_fused(const void* q_raw, const void* k_raw, const void* v_raw, const float* beta_pre,
                         const float* c_pre, const void* f_pre, const float* a_log, float beta_scale,
                         const float* S0, const void* dO, const float* dST, void* dq_raw, void* dk_raw,
                         void* dv_raw, float* dbeta_pre, float* dc_pre, float* df_pre, float* da_log, float* dS0,
                         int B, int H, int T, int dk, int dv, int dtype, const void* fwd_ws, size_t fwd_ws_bytes,
                         void* workspace, size_t ws_bytes, void* stream) {
  kd::Layout L;
  KD_TRY(plan(B, H, T, dk, dv, dtype, &L));
  KD_TRY(check_prologue(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, B, H, T, dk, dv, dtype));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(dO, "dO", true));
  KD_TRY(check_ptr(dST, "dST", false));
  KD_TRY(check_ptr(dq_raw, "dq_raw", true));
  KD_TRY(check_ptr(dk_raw, "dk_raw", true));
  KD_TRY(check_ptr(dv_raw, "dv_raw", true));
  KD_TRY(check_ptr(dbeta_pre, "dbeta_pre", true));
  KD_TRY(check_ptr(dc_pre, "dc_pre", true));
  KD_TRY(check_ptr(df_pre, "df_pre", true));
  KD_TRY(check_ptr(da_log, "da_log", true));
  KD_TRY(check_ptr(dS0, "dS0", false));
  if (!fwd_ws || fwd_ws_bytes < L.fwd_fused_bytes)
    return fail(KD_ERR_WORKSPACE, "the fused forward's workspace (save=1) of %zu bytes needed (got %zu)",
                L.fwd_fused_bytes, fwd_ws ? fwd_ws_bytes : 0);
  if (!workspace || ws_bytes < L.bwd_fused_bytes)
    return fail(KD_ERR_WORKSPACE, "fused backward workspace of %zu bytes needed (got %zu)", L.bwd_fused_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256) || !aligned(fwd_ws, 256))
    return fail(KD_ERR_WORKSPACE, "workspaces must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const char* fws = static_cast<const char*>(fwd_ws);
  float* dapart = kd::ws_ptr<float>(ws, L.dapart);
  if (L.tc) {
    // the chunk kernels write the gradients of the normalised q, k, v and of
    // the gated beta, c into the outputs, and df~ with its da_log parts; the
    // tail pass then carries the first five through the prologue in place
    kd::BwdArgs a{q_raw, k_raw, v_raw, beta_pre, c_pre, static_cast<const float*>(f_pre), S0, dO, dST, dq_raw,
                  dk_raw, dv_raw, dbeta_pre, dc_pre, df_pre, dS0, fws, ws, L, KD_PHASE_ALL};
    a.a_log = a_log;
    a.pro.bscale = beta_scale;
    a.pro.norm = 1;
    DeviceInfo di;
    KD_TRY(device_info(&di));
    cudaError_t e = kd::launch_bwd_tc(a, di.err, di.sms, st);
    if (e == cudaSuccess) e = kd::launch_reduce_dalog(dapart, B, H, L.NC, da_log, st);
    if (e == cudaSuccess)
      e = kd::launch_prologue_tail_bwd(q_raw, k_raw, v_raw, beta_pre, c_pre, beta_scale, dq_raw, dk_raw, dv_raw,
                                       dbeta_pre, dc_pre, (size_t)B * T * H, st);
    return launched(e, "fused backward launch");
  }
  // CUDA-core path: the backward on the prologue's outputs, then the prologue's
  // backward; df~ (fp32) and da_log are formed from dlogf as on the gated path
  const float* logf = kd::ws_ptr<float>(fws, L.glogf);
  float* gdlogf = kd::ws_ptr<float>(ws, L.gdlogf);
  KD_TRY(kron_delta_bwd(fws + L.fq, fws + L.fk, fws + L.fv, kd::ws_ptr<float>(fws, L.fbeta),
                        kd::ws_ptr<float>(fws, L.fc), logf, S0, dO, dST, ws + L.gdq, ws + L.gdk, ws + L.gdv,
                        kd::ws_ptr<float>(ws, L.gdbeta), kd::ws_ptr<float>(ws, L.gdc), gdlogf, dS0, B, H, T, dk, dv,
                        dtype, fwd_ws, L.fwd_save_bytes, workspace, L.bwd_bytes, stream));
  KD_TRY(kron_delta_prologue_bwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, ws + L.gdq,
                                 ws + L.gdk, ws + L.gdv, kd::ws_ptr<float>(ws, L.gdbeta), kd::ws_ptr<float>(ws, L.gdc),
                                 gdlogf, dq_raw, dk_raw, dv_raw, dbeta_pre, dc_pre, ws + L.gdf, da_log, B, H, T, dk,
                                 dv, dtype, ws + L.gpro, ws_bytes - L.gpro, stream));
  cudaError_t e = kd::launch_gate_dlogf(gdlogf, logf, a_log, df_pre, dapart, B, T, H, dk, L.NC, st);
  if (e == cudaSuccess) e = kd::launch_reduce_dalog(dapart, B, H, L.NC, da_log, st);
  return launched(e, "fused backward launch");
}

int kron_delta_decode(const void* q, const void* k, const void* v, const float* beta,
                      const float* c, const float* logf, float* S, void* out, int B, int H,
                      int dk, int dv, int dtype, void* stream) {
  if (B <= 0 || H <= 0) return fail(KD_ERR_INVALID_ARG, "B, H must be >= 1 (got %d, %d)", B, H);
  if ((size_t)B * H > 0x7fffffffu) return fail(KD_ERR_INVALID_ARG, "B*H too large");
  if (!dim_supported(dk) || !dim_supported(dv))
    return fail(KD_ERR_UNSUPPORTED, "dk and dv must be 32, 64 or 128 (got %d, %d)", dk, dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(beta, "beta", true));
  KD_TRY(check_ptr(c, "c", true));
  KD_TRY(check_ptr(logf, "logf", true));
  KD_TRY(check_ptr(S, "S", true));
  KD_TRY(check_ptr(out, "out", true));
  KD_TRY(check_stream(stream));
  kd::DecodeArgs a{q, k, v, beta, c, logf, S, out, B, H, dk, dv, dtype};
  return launched(kd::launch_decode(a, static_cast<cudaStream_t>(stream)), "decode launch");
}


int kron_delta_prologue_fwd(const void* q_raw, const void* k_raw, const void* v_raw,
                            const float* beta_pre, const float* c_pre, const void* f_pre,
                            const float* a_log, float beta_scale, void* q, void* k, void* v,
                            float* beta, float* c, float* logf, int B, int H, int T, int dk, int dv,
                            int dtype, void* stream) {
  KD_TRY(check_prologue(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, B, H, T, dk, dv,
                        dtype));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(beta, "beta", true));
  KD_TRY(check_ptr(c, "c", true));
  KD_TRY(check_ptr(logf, "logf", true));
  KD_TRY(check_stream(stream));
  kd::PrologueArgs a{};
  a.q_raw = q_raw; a.k_raw = k_raw; a.v_raw = v_raw;
  a.beta_pre = beta_pre; a.c_pre = c_pre; a.f_pre = f_pre; a.a_log = a_log; a.beta_scale = beta_scale;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.c = c; a.logf = logf;
  a.N = (long long)B * T; a.H = H; a.dk = dk; a.dv = dv; a.dtype = dtype;
  return launched(kd::launch_prologue_fwd(a, static_cast<cudaStream_t>(stream)), "prologue launch");
}

int kron_delta_prologue_bwd(const void* q_raw, const void* k_raw, const void* v_raw,
                            const float* beta_pre, const float* c_pre, const void* f_pre,
                            const float* a_log, float beta_scale, const void* dq, const void* dk,
                            const void* dv, const float* dbeta, const float* dc, const float* dlogf,
                            void* dq_raw, void* dk_raw, void* dv_raw, float* dbeta_pre, float* dc_pre,
                            void* df_pre, float* da_log, int B, int H, int T, int dk_, int dv_,
                            int dtype, void* workspace, size_t ws_bytes, void* stream) {
  KD_TRY(check_prologue(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, B, H, T, dk_,
                        dv_, dtype));
  KD_TRY(check_ptr(dq, "dq", true));
  KD_TRY(check_ptr(dk, "dk", true));
  KD_TRY(check_ptr(dv, "dv", true));
  KD_TRY(check_ptr(dbeta, "dbeta", true));
  KD_TRY(check_ptr(dc, "dc", true));
  KD_TRY(check_ptr(dlogf, "dlogf", true));
  KD_TRY(check_ptr(dq_raw, "dq_raw", true));
  KD_TRY(check_ptr(dk_raw, "dk_raw", true));
  KD_TRY(check_ptr(dv_raw, "dv_raw", true));
  KD_TRY(check_ptr(dbeta_pre, "dbeta_pre", true));
  KD_TRY(check_ptr(dc_pre, "dc_pre", true));
  KD_TRY(check_ptr(df_pre, "df_pre", true));
  KD_TRY(check_ptr(da_log, "da_log", true));
  const long long N = (long long)B * T;
  const size_t need = (size_t)kd::prologue_blocks(N) * H * sizeof(float);
  if (!workspace || ws_bytes < need)
    return fail(KD_ERR_WORKSPACE, "prologue workspace of %zu bytes needed (got %zu)", need,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  kd::PrologueArgs a{};
  a.q_raw = q_raw; a.k_raw = k_raw; a.v_raw = v_raw;
  a.beta_pre = beta_pre; a.c_pre = c_pre; a.f_pre = f_pre; a.a_log = a_log; a.beta_scale = beta_scale;
  a.gq = dq; a.gk = dk; a.gv = dv; a.dbeta = dbeta; a.dc = dc; a.dlogf = dlogf;
  a.dq_raw = dq_raw; a.dk_raw = dk_raw; a.dv_raw = dv_raw;
  a.dbeta_pre = dbeta_pre; a.dc_pre = dc_pre; a.df_pre = df_pre; a.da_log = da_log;
  a.part = static_cast<float*>(workspace);
  a.N = N; a.H = H; a.dk = dk_; a.dv = dv_; a.dtype = dtype;
  return launched(kd::launch_prologue_bwd(a, static_cast<cudaStream_t>(stream)), "prologue backward launch");
}

namespace {
int check_epilogue(const void* o, const void* g, const float* w, int B, int H, int T, int dv, int dtype) {
  if (B <= 0 || H <= 0 || T <= 0) return fail(KD_ERR_INVALID_ARG, "B, H, T must be >= 1 (got %d, %d, %d)", B, H, T);
  if (!dim_supported(dv)) return fail(KD_ERR_UNSUPPORTED, "dv must be 32, 64 or 128 (got %d)", dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  KD_TRY(check_ptr(o, "o", true));
  KD_TRY(check_ptr(g, "g", true));
  return check_ptr(w, "w", true);
}
}  // namespace

int kron_delta_epilogue_fwd(const void* o, const void* g, const float* w, void* y, int B, int H, int T,
                            int dv, int dtype, void* stream) {
  KD_TRY(check_epilogue(o, g, w, B, H, T, dv, dtype));
  KD_TRY(check_ptr(y, "y", true));
  KD_TRY(check_stream(stream));
  kd::EpilogueArgs a{};
  a.o = o; a.g = g; a.w = w; a.y = y;
  a.rows = (long long)B * T * H; a.dv = dv; a.dtype = dtype;
  return launched(kd::launch_epilogue_fwd(a, static_cast<cudaStream_t>(stream)), "epilogue launch");
}

int kron_delta_epilogue_bwd(const void* o, const void* g, const float* w, const void* dy, void* dO,
                            void* dg, float* dw, int B, int H, int T, int dv, int dtype, void* workspace,
                            size_t ws_bytes, void* stream) {
  KD_TRY(check_epilogue(o, g, w, B, H, T, dv, dtype));
  KD_TRY(check_ptr(dy, "dy", true));
  KD_TRY(check_ptr(dO, "dO", true));
  KD_TRY(check_ptr(dg, "dg", true));
  KD_TRY(check_ptr(dw, "dw", true));
  const long long rows = (long long)B * T * H;
  const size_t need = (size_t)kd::epilogue_blocks(rows) * dv * sizeof(float);
  if (!workspace || ws_bytes < need)
    return fail(KD_ERR_WORKSPACE, "epilogue workspace of %zu bytes needed (got %zu)", need,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  kd::EpilogueArgs a{};
  a.o = o; a.g = g; a.w = w; a.dy = dy; a.dO = dO; a.dg = dg; a.dw = dw;
  a.part = static_cast<float*>(workspace);
  a.rows = rows; a.dv = dv; a.dtype = dtype;
  return launched(kd::launch_epilogue_bwd(a, static_cast<cudaStream_t>(stream)), "epilogue backward launch");
}

int kron_delta_gdn2_fwd(const void* q, const void* k, const void* v, const float* b, const float* w,
                        const float* loga, const float* S0, void* out, float* ST, int B, int H, int T, int dk,
                        int dv, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  kd::GdnLayout L;
  KD_TRY(gdn_plan(B, H, T, dk, dv, dtype, &L));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(b, "b", true));
  KD_TRY(check_ptr(w, "w", true));
  KD_TRY(check_ptr(loga, "loga", true));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(out, "out", true));
  KD_TRY(check_ptr(ST, "ST", false));
  if (!workspace || ws_bytes < L.fwd_bytes)
    return fail(KD_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", L.fwd_bytes, workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256)) return fail(KD_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  kd::GdnArgs a{};
  a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.loga = loga; a.S0 = S0; a.out = out; a.ST = ST;
  a.ws = static_cast<char*>(workspace);
  a.L = L;
  if (kd::gdn2_tc_supported(L)) {  // the tensor-core kernels report bounded-wait timeouts here
    DeviceInfo di;
    KD_TRY(device_info(&di));
    a.err = di.err;
  }
  return launched(kd::launch_gdn2_fwd(a, static_cast<cudaStream_t>(stream)), "gdn2 forward launch");
}

int kron_delta_gdn2_bwd(const void* q, const void* k, const void* v, const float* b, const float* w,
                        const float* loga, const float* S0, const void* dO, const float* dST, void* dq, void* dk,
                        void* dv, float* db, float* dw, float* dloga, float* dS0, int B, int H, int T, int dk_,
                        int dv_, int dtype, const void* fwd_ws, size_t fwd_ws_bytes, void* workspace,
                        size_t ws_bytes, void* stream) {
  kd::GdnLayout L;
  KD_TRY(gdn_plan(B, H, T, dk_, dv_, dtype, &L));
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(b, "b", true));
  KD_TRY(check_ptr(w, "w", true));
  KD_TRY(check_ptr(loga, "loga", true));
  KD_TRY(check_ptr(S0, "S0", false));
  KD_TRY(check_ptr(dO, "dO", true));
  KD_TRY(check_ptr(dST, "dST", false));
  KD_TRY(check_ptr(dq, "dq", true));
  KD_TRY(check_ptr(dk, "dk", true));
  KD_TRY(check_ptr(dv, "dv", true));
  KD_TRY(check_ptr(db, "db", true));
  KD_TRY(check_ptr(dw, "dw", true));
  KD_TRY(check_ptr(dloga, "dloga", true));
  KD_TRY(check_ptr(dS0, "dS0", false));
  if (!fwd_ws || fwd_ws_bytes < L.fwd_bytes)
    return fail(KD_ERR_WORKSPACE, "forward workspace of %zu bytes needed (got %zu)", L.fwd_bytes,
                fwd_ws ? fwd_ws_bytes : 0);
  if (!workspace || ws_bytes < L.bwd_bytes)
    return fail(KD_ERR_WORKSPACE, "backward workspace of %zu bytes needed (got %zu)", L.bwd_bytes,
                workspace ? ws_bytes : 0);
  if (!aligned(workspace, 256) || !aligned(fwd_ws, 256))
    return fail(KD_ERR_WORKSPACE, "workspaces must be 256-byte aligned");
  KD_TRY(check_stream(stream));
  (void)S0;  // the chunk-start states are read from fwd_ws
  kd::GdnArgs a{};
  a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.loga = loga; a.S0 = S0;
  a.dO = dO; a.dST = dST; a.dq = dq; a.dk = dk; a.dv = dv; a.db = db; a.dw = dw; a.dloga = dloga; a.dS0 = dS0;
  a.fws = static_cast<const char*>(fwd_ws);
  a.ws = static_cast<char*>(workspace);
  a.L = L;
  if (kd::gdn2_tc_supported(L)) {  // the tensor-core kernels report bounded-wait timeouts here
    DeviceInfo di;
    KD_TRY(device_info(&di));
    a.err = di.err;
  }
  return launched(kd::launch_gdn2_bwd(a, static_cast<cudaStream_t>(stream)), "gdn2 backward launch");
}

int kron_delta_gdn2_decode(const void* q, const void* k, const void* v, const float* b, const float* w,
                           const float* loga, float* S, void* out, int B, int H, int dk, int dv, int dtype,
                           void* stream) {
  if (B <= 0 || H <= 0) return fail(KD_ERR_INVALID_ARG, "B, H must be >= 1 (got %d, %d)", B, H);
  if ((size_t)B * H > 0x7fffffffu) return fail(KD_ERR_INVALID_ARG, "B*H too large");
  if (!dim_supported(dk) || !dim_supported(dv))
    return fail(KD_ERR_UNSUPPORTED, "dk and dv must be 32, 64 or 128 (got %d, %d)", dk, dv);
  if (dtype != KD_F32 && dtype != KD_BF16) return fail(KD_ERR_UNSUPPORTED, "dtype must be KD_F32 or KD_BF16 (got %d)", dtype);
  KD_TRY(check_ptr(q, "q", true));
  KD_TRY(check_ptr(k, "k", true));
  KD_TRY(check_ptr(v, "v", true));
  KD_TRY(check_ptr(b, "b", true));
  KD_TRY(check_ptr(w, "w", true));
  KD_TRY(check_ptr(loga, "loga", true));
  KD_TRY(check_ptr(S, "S", true));
  KD_TRY(check_ptr(out, "out", true));
  KD_TRY(check_stream(stream));
  kd::GdnDecodeArgs a{q, k, v, b, w, loga, S, out, B, H, dk, dv, dtype};
  return launched(kd::launch_gdn2_decode(a, static_cast<cudaStream_t>(stream)), "gdn2 decode launch");
}

int kron_delta_selftest_timeout(void* stream) {
  KD_TRY(check_stream(stream));
  DeviceInfo di;
  KD_TRY(device_info(&di));
  return launched(kd::launch_selftest_timeout(di.err, static_cast<cudaStream_t>(stream)), "self-test launch");
}

void kron_delta_profile_enable(int on) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = on != 0;
}

int kron_delta_profile_report(char* buf, size_t len, int reset) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    fail(KD_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
    return -KD_ERR_CUDA;
  }
  for (auto& r : p.pending) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      auto& t = p.totals[r.name];
      t.first += 1;
      t.second += ms;
    }
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.pending.clear();
  std::string out;
  char line[256];
  for (auto& kv : p.totals) {
    snprintf(line, sizeof(line), "%s %ld %.6f\n", kv.first.c_str(), kv.second.first, kv.second.second);
    out += line;
  }
  if (buf && len > 0) {
    size_t n = out.size() < len - 1 ? out.size() : len - 1;
    memcpy(buf, out.data(), n);
    buf[n] = 0;
  }
  const int count = (int)p.totals.size();
  if (reset) p.totals.clear();
  return count;
}

int kron_delta_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(KD_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  DeviceInfo di;
  KD_TRY(device_info(&di));
  int word = 0;
  e = cudaMemcpyAsync(&word, di.err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(KD_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  if (word != 0) {
    const int zero = 0;
    cudaMemcpyAsync(di.err, &zero, sizeof(int), cudaMemcpyHostToDevice, st);
    cudaStreamSynchronize(st);
    return fail(KD_ERR_TIMEOUT, "a bounded device-side wait gave up (code %d); outputs of that call are invalid",
                word);
  }
  return ok();
}

}  // extern "C"
