// kd_noalloc.cu -- forward entry point that needs no caller-provided workspace
// and allocates nothing.
//
// Who this is for: callers that cannot allocate device memory when they call
// the mixer -- for example a host process whose device memory is entirely
// reserved up front by another allocator (a serving runtime, or a plugin that
// has no handle to its host's allocator), or a loop with a no-allocation rule
// after start-up.  Such callers still own and pass their inputs and outputs;
// only the forward's scratch (the per-chunk y, A and P) comes from the fixed
// array below, which is part of the library image.
//
// Limits and behaviour:
//   * The scratch is a file-scope device array of kNoAllocScratchBytes
//     (32 MiB).  Every GPU that loads the library holds it until the process
//     exits.  A problem whose forward scratch (kron_delta_workspace_size with
//     KD_WS_FWD) exceeds it is rejected with KD_ERR_WORKSPACE before anything
//     is enqueued: beyond 145 chunk-heads (B * H * ceil(T/64)) on the
//     tensor-core path (bf16, dk = dv = 128, whose chain also keeps per-token
//     operands there), beyond 1016 on the others.
//   * All calls share the one array and it keeps the last call's contents.
//     The forward writes every scratch element it later reads, so nothing
//     has to start at zero.  Calls whose kernels overlap on the GPU (other
//     streams, other host threads) race on the array: the caller must order
//     them.
//   * The first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (with that device current) and caches it; make that
//     first call before any stream capture begins.  The cache is keyed on the
//     current context's unique ID: if the device's primary context was reset
//     (cudaDeviceReset) and recreated, the module is reloaded at a new
//     address, and the next call looks the address up again.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/kron_delta.h"
#include "kd_kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context ID the address belongs to

// Unique ID of the calling thread's current context (0 if it cannot be
// read), through the driver entry points, so no link-time libcuda.
unsigned long long current_context_id() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// The device address of the scratch array on the current device (the
// array's name is only a host-side stand-in).  Looked up once per device and
// context; looked up again when the context has changed.
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the primary context current
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

int kron_delta_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                           const float* c, const float* logf, const float* S0, void* out,
                           float* ST, int B, int H, int T, int dk, int dv, int dtype,
                           void* stream) {
  // Size the scratch with the library's own planner.  Invalid sizes: let the
  // regular entry point validate them (it rejects them before looking at the
  // workspace) so the error code and message are the usual ones.
  const size_t need = kron_delta_workspace_size(KD_WS_FWD, B, H, T, dk, dv, dtype);
  if (need == 0)
    return kron_delta_fwd(q, k, v, beta, c, logf, S0, out, ST, B, H, T, dk, dv, dtype, nullptr, 0,
                          0, stream);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kron_delta_fwd_noalloc: forward scratch of %zu bytes exceeds the fixed %zu-byte array; "
             "use kron_delta_fwd with a workspace",
             need, kNoAllocScratchBytes);
    kd::set_error(msg);
    return KD_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "kron_delta_fwd_noalloc: scratch address lookup failed: %s",
             cudaGetErrorString(e));
    kd::set_error(msg);
    return KD_ERR_CUDA;
  }
  return kron_delta_fwd(q, k, v, beta, c, logf, S0, out, ST, B, H, T, dk, dv, dtype, scratch,
                        kNoAllocScratchBytes, 0, stream);
}

}  // extern "C"
