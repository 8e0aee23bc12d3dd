/*
 * kron_delta.h -- C ABI of the B200 (sm_100a) Kronecker delta rule library.
 *
 * The operation is the KronLSTM token mixer.  Per (batch b, head h) there is
 * one fp32 state S in R^{dv x dk} (row r = value channel, column j = key
 * channel).  For each token t:
 *
 *     Sbar_t = S_{t-1} diag(f_t),  f_t = exp(logf_t)         (forget gate)
 *     b_t    = v_t^T Sbar_t k_t                              (association)
 *     u_t    = c_t - beta_t b_t                              (erase, write)
 *     S_t    = Sbar_t + u_t v_t k_t^T
 *     o_t    = S_t q_t
 *
 * Sources (web pages on the method, cited by title and section):
 *   KronLSTM digest, "KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억
 *     간섭을 줄인다": section "어떻게 동작하나" (the Kronecker delta rule:
 *     one scalar association v^T S k corrected along v k^T, erase amount beta,
 *     write amount c), section "어떻게 쓰나" (diagonal forget gate on the key
 *     dimension applied from the right; per-head scalar beta, c; L2-normalised
 *     q, k, v), section "무엇과 다른가" (DeltaNet-style chunk-parallel form).
 *   Gated DeltaNet-2 article (aitrends.kr), section "기술 상세": chunk size
 *     C = 64 and forward substitution for the chunk's triangular inverse.
 *
 * Entry points:
 *   Kronecker delta rule  kron_delta_fwd, kron_delta_bwd, kron_delta_decode,
 *                         kron_delta_bwd_recompute (no saved forward),
 *                         kron_delta_fwd_phase / _bwd_phase (split at the
 *                         carried state, for context parallelism),
 *                         kron_delta_fwd_noalloc,
 *                         kron_delta_fwd_gated / _bwd_gated (forget gate
 *                         from its pre-activation, formed inside the kernels),
 *                         kron_delta_fwd_fused / _bwd_fused (the whole input
 *                         prologue inside the kernels)
 *   around the mixer      kron_delta_prologue_fwd / _bwd (L2-norm, gates,
 *                         log-decay), kron_delta_epilogue_fwd / _bwd
 *                         (per-head RMSNorm and output gate)
 *   Gated DeltaNet-2      kron_delta_gdn2_fwd / _bwd / _decode
 *   support               kron_delta_workspace_size, kron_delta_device_status,
 *                         kron_delta_selftest_timeout, kron_delta_last_error,
 *                         kron_delta_version, kron_delta_profile_enable /
 *                         _report
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers on the current CUDA device unless
 *     stated otherwise.  The caller owns every buffer; the library allocates
 *     no device memory, keeps no state between calls except a thread-local
 *     error string and a cached device-property query, and never
 *     synchronises the stream (except kron_delta_device_status).
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work of a call is enqueued on it, in order.
 *   - Layouts (all contiguous, row-major):
 *       q, k            [B, T, H, dk]      dtype
 *       v, out, dO      [B, T, H, dv]      dtype
 *       beta, c         [B, T, H]          fp32
 *       logf            [B, T, H, dk]      fp32 (log of the forget gate, <= 0)
 *       S0, ST, dST,dS0 [B, H, dv, dk]     fp32
 *     dtype = KD_F32 (fp32) or KD_BF16 (bfloat16) for q, k, v, out, dO, dq,
 *     dk, dv; gates and states are fp32 in both cases.
 *   - Supported sizes: dk, dv in {32, 64, 128}; B, H >= 1; T >= 1 (a final
 *     partial chunk of fewer than 64 tokens is handled).  Pointers to fp32
 *     data must be 4-byte aligned, to bf16 data 2-byte aligned; 16-byte
 *     alignment of q, k, v, dO is required (checked).
 *   - Preconditions not checked on the device: q, k, v are L2-normalised by
 *     the caller (the library never renormalises); logf <= 0; beta in [0, 2);
 *     outputs do not alias inputs.
 *   - Return value: KD_OK, or an error code; on error nothing was enqueued
 *     and kron_delta_last_error() describes the first problem found.
 */
#ifndef KRON_DELTA_H
#define KRON_DELTA_H

#include <stddef.h>

#if defined(__GNUC__)
#define KD_API __attribute__((visibility("default")))
#else
#define KD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define KD_OK 0
#define KD_ERR_INVALID_ARG 1   /* null pointer, bad size, misalignment */
#define KD_ERR_UNSUPPORTED 2   /* dk/dv/dtype outside the supported set */
#define KD_ERR_WORKSPACE 3     /* workspace missing or too small */
#define KD_ERR_CUDA 4          /* a CUDA runtime call or launch failed */
#define KD_ERR_TIMEOUT 5       /* a bounded device-side wait gave up */

/* element types of q, k, v, out, dO, dq, dk, dv */
#define KD_F32 0
#define KD_BF16 1

/* workspace kinds for kron_delta_workspace_size */
#define KD_WS_FWD 0        /* forward only (prefill / inference) */
#define KD_WS_FWD_SAVE 1   /* forward that keeps what the backward needs */
#define KD_WS_BWD 2        /* backward scratch (besides the saved forward) */
#define KD_WS_PROLOGUE_BWD 3  /* scratch of kron_delta_prologue_bwd (dk, dv, dtype
                                 must be valid but do not change the size) */
#define KD_WS_EPILOGUE_BWD 4  /* scratch of kron_delta_epilogue_bwd (dk and dtype
                                 must be valid but do not change the size) */
#define KD_WS_GDN2_FWD 5      /* kron_delta_gdn2_fwd (kept for kron_delta_gdn2_bwd) */
#define KD_WS_GDN2_BWD 6      /* backward scratch of kron_delta_gdn2_bwd */
#define KD_WS_FWD_GATED 7     /* kron_delta_fwd_gated (kept for kron_delta_bwd_gated) */
#define KD_WS_BWD_GATED 8     /* backward scratch of kron_delta_bwd_gated */
#define KD_WS_BWD_RECOMPUTE 9 /* kron_delta_bwd_recompute (forward scratch included) */
#define KD_WS_FWD_FUSED 10    /* kron_delta_fwd_fused (kept for kron_delta_bwd_fused) */
#define KD_WS_BWD_FUSED 11    /* backward scratch of kron_delta_bwd_fused */

/* phases of kron_delta_fwd_phase / kron_delta_bwd_phase */
#define KD_PHASE_LOCAL 1   /* the work that does not depend on the carried state */
#define KD_PHASE_CARRY 2   /* the chunk chain and everything after it */
#define KD_PHASE_ALL 3     /* both, in order (what kron_delta_fwd / _bwd do) */

/* Library version, as 10000*major + 100*minor + patch. */
KD_API int kron_delta_version(void);

/* Description of the last error on the calling thread ("" if none).  The
 * string is owned by the library and valid until the next call on the same
 * thread. */
KD_API const char *kron_delta_last_error(void);

/* Bytes of device workspace the given call needs (0 for invalid sizes; the
 * reason is then in kron_delta_last_error).  The workspace must be 256-byte
 * aligned.  KD_WS_FWD_SAVE holds, per 64-token chunk and head, the chunk's
 * triangular inverse A = (I + diag(beta) M)^{-1}, the query-key decay matrix
 * P, the chunk-start state and the per-token b_t and u_t; kron_delta_bwd reads
 * them back. */
KD_API size_t kron_delta_workspace_size(int kind, int B, int H, int T, int dk, int dv,
                                 int dtype);

/*
 * Chunk-parallel forward (C = 64).
 *   q, k, v, beta, c, logf : inputs (layouts above).
 *   S0  : initial state [B,H,dv,dk] fp32, or NULL for zero.
 *   out : o_t for every token [B,T,H,dv] (dtype).
 *   ST  : final state [B,H,dv,dk] fp32, or NULL to skip.
 *   workspace, ws_bytes : device scratch of at least
 *         kron_delta_workspace_size(save ? KD_WS_FWD_SAVE : KD_WS_FWD, ...).
 *   save : 1 = keep the forward quantities the backward reads in the
 *         workspace (pass the same workspace to kron_delta_bwd); 0 = not.
 * Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_WORKSPACE,
 * KD_ERR_CUDA.  Asynchronous on `stream`.
 */
KD_API int kron_delta_fwd(const void *q, const void *k, const void *v,
                   const float *beta, const float *c, const float *logf,
                   const float *S0, void *out, float *ST, int B, int H, int T,
                   int dk, int dv, int dtype, void *workspace, size_t ws_bytes,
                   int save, void *stream);

/*
 * Backward of kron_delta_fwd for the loss l = <dO, out> + <dST, ST>.
 *   fwd_ws, fwd_ws_bytes : the workspace of a kron_delta_fwd call with save=1
 *         on exactly these inputs (read only).
 *   dO  : upstream gradient of out [B,T,H,dv] (dtype).
 *   dST : upstream gradient of ST [B,H,dv,dk] fp32, or NULL for zero.
 *   dq, dk, dv : [B,T,H,dk|dv] (dtype).  dbeta, dc : [B,T,H] fp32.
 *   dlogf : [B,T,H,dk] fp32.  dS0 : [B,H,dv,dk] fp32, or NULL to skip.
 *   workspace, ws_bytes : scratch of at least
 *         kron_delta_workspace_size(KD_WS_BWD, ...).
 * S0 is the same initial state given to the forward (NULL = zero).
 * kron_delta_bwd reads the forward's saved chunk quantities (fwd_ws) and
 * fails with KD_ERR_WORKSPACE without them; kron_delta_bwd_recompute (below)
 * is the backward for a caller that did not keep them.
 * Errors as for kron_delta_fwd.  Asynchronous on `stream`.
 */
KD_API int kron_delta_bwd(const void *q, const void *k, const void *v,
                   const float *beta, const float *c, const float *logf,
                   const float *S0, const void *dO, const float *dST,
                   void *dq, void *dk, void *dv, float *dbeta, float *dc,
                   float *dlogf, float *dS0, int B, int H, int T, int dk_,
                   int dv_, int dtype, const void *fwd_ws, size_t fwd_ws_bytes,
                   void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward of kron_delta_fwd that recomputes the forward's chunk quantities
 * instead of reading a saved forward workspace: it enqueues the forward's
 * chunk-local work and its chunk chain with save = 1 into the first part of
 * `workspace` (without writing an output), then kron_delta_bwd on it.  The
 * gradients are bitwise those of kron_delta_fwd(save = 1) + kron_delta_bwd on
 * the same inputs.  The cost is the forward's chain again, a sequential pass
 * over the chunks as long as the backward's own, and the workspace is the two
 * added together.
 *   workspace, ws_bytes : at least kron_delta_workspace_size(KD_WS_BWD_RECOMPUTE, ...).
 * The other arguments, layouts and errors are those of kron_delta_bwd.
 * Asynchronous on `stream`.
 */
KD_API int kron_delta_bwd_recompute(const void *q, const void *k, const void *v,
                             const float *beta, const float *c, const float *logf,
                             const float *S0, const void *dO, const float *dST,
                             void *dq, void *dk, void *dv, float *dbeta, float *dc,
                             float *dlogf, float *dS0, int B, int H, int T, int dk_,
                             int dv_, int dtype, void *workspace, size_t ws_bytes,
                             void *stream);

/*
 * Forward and backward with the forget gate taken as its pre-activation
 * (KronLSTM digest, "어떻게 쓰나": the forget gate is f = sigma(f~)^a with
 * a = e^{a_log} per head, so logf = a log sigma(f~)).  Identical to
 * kron_delta_fwd / kron_delta_bwd on logf = e^{a_log} log sigma(f_pre), but
 * on the tensor-core path (bf16, dk = dv = 128) every kernel reads the bf16
 * pre-activations and forms logf while loading them, so the fp32 logf tensor
 * (a third of the forward's input bytes) is never written or read.
 *   f_pre : forget pre-activations [B,T,H,dk] (dtype).
 *   a_log : per-head exponent [H] fp32.
 *   workspace (forward) : at least kron_delta_workspace_size(KD_WS_FWD_GATED, ...);
 *         pass it with save = 1 to kron_delta_bwd_gated as fwd_ws.
 *   df_pre : gradient of f_pre [B,T,H,dk] fp32 (dlogf a sigma(-f_pre)).
 *   da_log : gradient of a_log [H] fp32, the sum over the batch, the tokens
 *         and the key channels of dlogf logf, reduced in a fixed order
 *         (bitwise reproducible).
 *   workspace (backward) : at least kron_delta_workspace_size(KD_WS_BWD_GATED, ...).
 * The other arguments, layouts and errors are those of kron_delta_fwd and
 * kron_delta_bwd.  Asynchronous on `stream`.
 */
KD_API int kron_delta_fwd_gated(const void *q, const void *k, const void *v,
                         const float *beta, const float *c, const void *f_pre,
                         const float *a_log, const float *S0, void *out, float *ST,
                         int B, int H, int T, int dk, int dv, int dtype,
                         void *workspace, size_t ws_bytes, int save, void *stream);
KD_API int kron_delta_bwd_gated(const void *q, const void *k, const void *v,
                         const float *beta, const float *c, const void *f_pre,
                         const float *a_log, const float *S0, const void *dO,
                         const float *dST, void *dq, void *dk, void *dv, float *dbeta,
                         float *dc, float *df_pre, float *da_log, float *dS0, int B,
                         int H, int T, int dk_, int dv_, int dtype, const void *fwd_ws,
                         size_t fwd_ws_bytes, void *workspace, size_t ws_bytes,
                         void *stream);

/*
 * Forward and backward with the whole input prologue fused into the chunk
 * kernels (KronLSTM digest, section "어떻게 쓰나"): the inputs are the raw
 * projections and gate pre-activations of kron_delta_prologue_fwd, and the
 * result equals kron_delta_prologue_fwd followed by kron_delta_fwd (and, for
 * the backward, kron_delta_bwd followed by kron_delta_prologue_bwd) up to
 * rounding.  On the tensor-core path (bf16, dk = dv = 128) no normalised or
 * gated copy of the inputs is written: each chunk kernel normalises the q, k,
 * v rows it loads (x / sqrt(|x|^2 + 1e-6), rounded to bf16 as the prologue
 * would store them), the preparation kernel applies the gate sigmoids and
 * keeps the gated beta, c (8 bytes per token and head) for the chain, and
 * logf is formed from f_pre as in kron_delta_fwd_gated.  The backward's chunk
 * kernels form df_pre and da_log in their epilogue; one row-wise pass then
 * carries the gradients of the normalised q, k, v and of the gated beta, c
 * through the normalisation and the sigmoids, in place in the outputs.  Other
 * shapes run kron_delta_prologue_fwd / _bwd around the plain calls, inside the
 * workspace.
 *   q_raw, k_raw, f_pre [B,T,H,dk], v_raw [B,T,H,dv] (dtype); beta_pre, c_pre
 *   [B,T,H] fp32; a_log [H] fp32; beta_scale in (0, 2], as for
 *   kron_delta_prologue_fwd.
 *   workspace (forward) : at least kron_delta_workspace_size(KD_WS_FWD_FUSED, ...);
 *         pass it with save = 1 to kron_delta_bwd_fused as fwd_ws.
 *   dq_raw, dk_raw [B,T,H,dk], dv_raw [B,T,H,dv] (dtype); dbeta_pre, dc_pre
 *   [B,T,H] fp32; df_pre [B,T,H,dk] fp32; da_log [H] fp32 (fixed-order sum,
 *   bitwise reproducible).
 *   workspace (backward) : at least kron_delta_workspace_size(KD_WS_BWD_FUSED, ...).
 * S0, out, ST, dO, dST, dS0 and the errors are those of kron_delta_fwd and
 * kron_delta_bwd (beta_scale outside (0, 2] gives KD_ERR_INVALID_ARG).
 * Asynchronous on `stream`.
 */
KD_API int kron_delta_fwd_fused(const void *q_raw, const void *k_raw, const void *v_raw,
                                const float *beta_pre, const float *c_pre, const void *f_pre,
                                const float *a_log, float beta_scale, const float *S0, void *out,
                                float *ST, int B, int H, int T, int dk, int dv, int dtype,
                                void *workspace, size_t ws_bytes, int save, void *stream);
KD_API int kron_delta_bwd_fused(const void *q_raw, const void *k_raw, const void *v_raw,
                                const float *beta_pre, const float *c_pre, const void *f_pre,
                                const float *a_log, float beta_scale, const float *S0,
                                const void *dO, const float *dST, void *dq_raw, void *dk_raw,
                                void *dv_raw, float *dbeta_pre, float *dc_pre, float *df_pre,
                                float *da_log, float *dS0, int B, int H, int T, int dk, int dv,
                                int dtype, const void *fwd_ws, size_t fwd_ws_bytes,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * The forward and backward split at the carried state, for a caller that
 * holds one time segment of every sequence and receives the state at the
 * segment's start from elsewhere (e.g. a context-parallel relay, where the
 * previous segment lives on another GPU).  The chunk-local work (the
 * triangular inverses, the Grams and the cross-chunk operands in the forward;
 * the per-chunk adjoints in the backward) does not depend on S0 (forward) or
 * dST (backward), so it can run while that state is still on its way.
 *   phase = KD_PHASE_LOCAL : enqueue only the state-independent work.  S0,
 *           out, ST (forward) and dST, the gradients, dS0 (backward) are
 *           neither read nor written, but the argument checks are the same
 *           as for the carry call: pass the buffers it will use.
 *   phase = KD_PHASE_CARRY : enqueue the rest.  Must follow a LOCAL call with
 *           the same inputs, sizes, save flag and workspaces, on the same
 *           stream or after it completed; the workspace must not be reused in
 *           between.
 *   phase = KD_PHASE_ALL   : both; identical to kron_delta_fwd / _bwd.
 * The KronLSTM digest's chunk-parallel form ("무엇과 다른가") is what makes the
 * split possible: inside a chunk everything but the state terms is local.
 * Arguments and errors otherwise as kron_delta_fwd / kron_delta_bwd.
 */
KD_API int kron_delta_fwd_phase(const void *q, const void *k, const void *v,
                                const float *beta, const float *c, const float *logf,
                                const float *S0, void *out, float *ST, int B, int H, int T,
                                int dk, int dv, int dtype, void *workspace, size_t ws_bytes,
                                int save, int phase, void *stream);

KD_API int kron_delta_bwd_phase(const void *q, const void *k, const void *v,
                                const float *beta, const float *c, const float *logf,
                                const float *S0, const void *dO, const float *dST,
                                void *dq, void *dk, void *dv, float *dbeta, float *dc,
                                float *dlogf, float *dS0, int B, int H, int T, int dk_,
                                int dv_, int dtype, const void *fwd_ws, size_t fwd_ws_bytes,
                                void *workspace, size_t ws_bytes, int phase, void *stream);

/*
 * One recurrent decode step: one new token per (b, h).
 *   q, k : [B,H,dk] (dtype); v : [B,H,dv] (dtype).
 *   beta, c : [B,H] fp32; logf : [B,H,dk] fp32.
 *   S   : [B,H,dv,dk] fp32, read and overwritten in place with S_t.
 *   out : o_t = S_t q_t, [B,H,dv] (dtype).
 * No workspace.  Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_CUDA.
 * Asynchronous on `stream`.
 */
KD_API int kron_delta_decode(const void *q, const void *k, const void *v,
                      const float *beta, const float *c, const float *logf,
                      float *S, void *out, int B, int H, int dk, int dv,
                      int dtype, void *stream);

/*
 * Forward that allocates nothing and takes no workspace (no counterpart on the
 * method's pages; a library convenience).  For callers that cannot allocate
 * device memory at call time -- e.g. a process whose device memory is all
 * reserved up front by another allocator, or a plugin without access to its
 * host's allocator.  Same arguments and results as kron_delta_fwd with
 * save = 0, minus the workspace: the forward's scratch comes from one fixed
 * 32 MiB device array inside the library (held on every GPU that loads the
 * library until exit).
 *   - Problems whose forward scratch (kron_delta_workspace_size, KD_WS_FWD)
 *     exceeds that return KD_ERR_WORKSPACE (use kron_delta_fwd then): beyond
 *     145 chunk-heads B * H * ceil(T/64) for bf16 with dk = dv = 128, beyond
 *     1016 for the other shapes.
 *   - All calls share the array; concurrent calls that overlap on the GPU
 *     race on it, so the caller must serialise them (e.g. one stream).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make it before any stream capture.
 * Errors as for kron_delta_fwd.  Asynchronous on `stream`.
 */
KD_API int kron_delta_fwd_noalloc(const void *q, const void *k, const void *v,
                                  const float *beta, const float *c, const float *logf,
                                  const float *S0, void *out, float *ST, int B, int H,
                                  int T, int dk, int dv, int dtype, void *stream);

/*
 * Input prologue: from the raw projections to the recurrence's inputs, one
 * fused pass.  KronLSTM digest, section "어떻게 쓰나": q, k, v are
 * L2-normalised; the erase and write gates are sigmoids of per-head scalar
 * projections (the erase gate scaled by 2 for state tracking, experiments
 * paragraph of the same page); the forget gate is sigmoid(x) raised to the
 * head's learned exponent exp(a_log).  Per token t and head h:
 *     q = q_raw / sqrt(|q_raw|^2 + 1e-6)      (likewise k, v)
 *     beta = beta_scale * sigmoid(beta_pre)    c = sigmoid(c_pre)
 *     logf[j] = exp(a_log[h]) * log sigmoid(f_pre[j])
 *   q_raw, k_raw, f_pre : [B,T,H,dk] (dtype);  v_raw : [B,T,H,dv] (dtype).
 *   beta_pre, c_pre : [B,T,H] fp32;  a_log : [H] fp32.
 *   beta_scale : in (0, 2]; 1 gives beta in (0, 1), 2 gives beta in (0, 2).
 *   q, k, v, beta, c, logf : outputs in the layouts of kron_delta_fwd, ready
 *   to be passed to it.  All 16-byte aligned.  No workspace.
 * Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_CUDA.  Asynchronous
 * on `stream`.
 */
KD_API int kron_delta_prologue_fwd(const void *q_raw, const void *k_raw, const void *v_raw,
                                   const float *beta_pre, const float *c_pre, const void *f_pre,
                                   const float *a_log, float beta_scale, void *q, void *k, void *v,
                                   float *beta, float *c, float *logf, int B, int H, int T, int dk,
                                   int dv, int dtype, void *stream);

/*
 * Backward of kron_delta_prologue_fwd, for the loss
 * l = <dq,q> + <dk,k> + <dv,v> + <dbeta,beta> + <dc,c> + <dlogf,logf>
 * (dq, dk, dv, dbeta, dc, dlogf as kron_delta_bwd writes them).
 *   Inputs as for the forward, plus the upstream gradients dq, dk [B,T,H,dk],
 *   dv [B,T,H,dv] (dtype), dbeta, dc [B,T,H] fp32, dlogf [B,T,H,dk] fp32.
 *   Outputs: dq_raw, dk_raw, df_pre [B,T,H,dk] and dv_raw [B,T,H,dv] (dtype);
 *   dbeta_pre, dc_pre [B,T,H] fp32; da_log [H] fp32 (overwritten, not
 *   accumulated; the sum over tokens and channels runs in a fixed order, so
 *   the result is bitwise reproducible).
 *   workspace, ws_bytes : scratch of at least
 *     kron_delta_workspace_size(KD_WS_PROLOGUE_BWD, ...), 256-byte aligned.
 * Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_WORKSPACE,
 * KD_ERR_CUDA.  Asynchronous on `stream`.
 */
KD_API int kron_delta_prologue_bwd(const void *q_raw, const void *k_raw, const void *v_raw,
                                   const float *beta_pre, const float *c_pre, const void *f_pre,
                                   const float *a_log, float beta_scale, const void *dq,
                                   const void *dk, const void *dv, const float *dbeta,
                                   const float *dc, const float *dlogf, void *dq_raw, void *dk_raw,
                                   void *dv_raw, float *dbeta_pre, float *dc_pre, void *df_pre,
                                   float *da_log, int B, int H, int T, int dk_, int dv_, int dtype,
                                   void *workspace, size_t ws_bytes, void *stream);

/*
 * Output epilogue: per-head RMSNorm of the read-out followed by the sigmoid
 * output gate, one fused pass.  KronLSTM digest, section "어떻게 쓰나": the
 * read-out passes through a sigmoid output gate and a per-head RMSNorm
 * before the output projection (the projection is not part of this call).
 * Reading of the order and the constant: norm first, eps = 1e-6, a weight w
 * per channel shared by the heads.  Per token t, head h, channel j:
 *     y[j] = w[j] * o[j] / sqrt(mean_i o[i]^2 + 1e-6) * sigmoid(g[j])
 *   o : the read-out [B,T,H,dv] (dtype), e.g. kron_delta_fwd's out.
 *   g : the gate's pre-activation [B,T,H,dv] (dtype).   w : [dv] fp32.
 *   y : [B,T,H,dv] (dtype).  All 16-byte aligned.  No workspace.
 * Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_CUDA.  Asynchronous
 * on `stream`.
 */
KD_API int kron_delta_epilogue_fwd(const void *o, const void *g, const float *w, void *y, int B,
                                   int H, int T, int dv, int dtype, void *stream);

/*
 * Backward of kron_delta_epilogue_fwd for the loss l = <dy, y>.
 *   dy : [B,T,H,dv] (dtype).
 *   dO, dg : gradients of o and g, [B,T,H,dv] (dtype).  dO can be passed on
 *   to kron_delta_bwd as its dO.
 *   dw : [dv] fp32, overwritten (not accumulated); summed over tokens and
 *   heads in a fixed order, so bitwise reproducible.
 *   workspace, ws_bytes : scratch of at least
 *     kron_delta_workspace_size(KD_WS_EPILOGUE_BWD, ...), 256-byte aligned.
 * Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_WORKSPACE,
 * KD_ERR_CUDA.  Asynchronous on `stream`.
 */
KD_API int kron_delta_epilogue_bwd(const void *o, const void *g, const float *w, const void *dy,
                                   void *dO, void *dg, float *dw, int B, int H, int T, int dv,
                                   int dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * Gated DeltaNet-2 rule on the same chunk machinery (C = 64).  Gated
 * DeltaNet-2 article (aitrends.kr), sections "핵심 기여" and "방법론": the erase
 * gate b (per key channel) and the write gate w (per value channel) are
 * decoupled.  In this library's state convention (S in R^{dv x dk}, the
 * transpose of the article's), per token t:
 *     Sbar = S diag(exp(loga_t)),   u = w_t o v_t - Sbar (b_t o k_t),
 *     S = Sbar + u k_t^T,           o_t = S q_t
 * With b = w = beta 1 it is the gated delta rule (KDA); with a scalar decay,
 * Gated DeltaNet (same article, "핵심 기여").
 *   q, k : [B,T,H,dk] (dtype);  v : [B,T,H,dv] (dtype).
 *   b : erase gate [B,T,H,dk] fp32;  w : write gate [B,T,H,dv] fp32.
 *   loga : log of the channel decay [B,T,H,dk] fp32 (<= 0).
 *   S0 : [B,H,dv,dk] fp32 or NULL (zero);  out : [B,T,H,dv] (dtype);
 *   ST : [B,H,dv,dk] fp32 or NULL.
 *   workspace : at least kron_delta_workspace_size(KD_WS_GDN2_FWD, ...) bytes,
 *   256-byte aligned; it keeps what kron_delta_gdn2_bwd reads.
 * With dtype bf16 and dk = dv = 128 every chunk contraction runs on tensor
 * cores, on fp32 operands split into bf16 high and low parts; the chain's
 * state stays fp32, and the chunk-start states kept in the workspace for
 * the backward are bf16.  Other shapes run on CUDA cores in fp32.  Errors as
 * for kron_delta_fwd.  Asynchronous on `stream`.
 */
KD_API int kron_delta_gdn2_fwd(const void *q, const void *k, const void *v, const float *b,
                               const float *w, const float *loga, const float *S0, void *out,
                               float *ST, int B, int H, int T, int dk, int dv, int dtype,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward of kron_delta_gdn2_fwd for the loss <dO, out> + <dST, ST>.
 *   fwd_ws : the workspace of a kron_delta_gdn2_fwd call on exactly these
 *   inputs (read only).  dO [B,T,H,dv] (dtype); dST [B,H,dv,dk] fp32 or NULL.
 *   dq, dk [B,T,H,dk] and dv [B,T,H,dv] (dtype); db, dloga [B,T,H,dk] and
 *   dw [B,T,H,dv] fp32; dS0 [B,H,dv,dk] fp32 or NULL.
 *   workspace : at least kron_delta_workspace_size(KD_WS_GDN2_BWD, ...).
 * Same precision split as the forward (the per-chunk gradients read the
 * saved bf16 states); chunks whose in-chunk decay leaves the factorised range
 * (|cumulative loga| >= 60) take an exact CUDA-core kernel.  Deterministic.
 * Errors as for kron_delta_bwd.  Asynchronous on `stream`.
 */
KD_API int kron_delta_gdn2_bwd(const void *q, const void *k, const void *v, const float *b,
                               const float *w, const float *loga, const float *S0, const void *dO,
                               const float *dST, void *dq, void *dk, void *dv, float *db,
                               float *dw, float *dloga, float *dS0, int B, int H, int T, int dk_,
                               int dv_, int dtype, const void *fwd_ws, size_t fwd_ws_bytes,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * One recurrent decode step of the Gated DeltaNet-2 rule: one new token per
 * (b, h), the state updated in place (same rule and convention as
 * kron_delta_gdn2_fwd).
 *   q, k : [B,H,dk] (dtype); v : [B,H,dv] (dtype).
 *   b, loga : [B,H,dk] fp32; w : [B,H,dv] fp32.
 *   S : [B,H,dv,dk] fp32, read and overwritten with the new state.
 *   out : o = S q after the update, [B,H,dv] (dtype).
 * No workspace.  Errors: KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_CUDA.
 * Asynchronous on `stream`.
 */
KD_API int kron_delta_gdn2_decode(const void *q, const void *k, const void *v, const float *b,
                                  const float *w, const float *loga, float *S, void *out, int B,
                                  int H, int dk, int dv, int dtype, void *stream);

/*
 * Synchronises `stream` and reports device-side failures of earlier calls:
 * KD_OK, KD_ERR_TIMEOUT (a bounded inter-CTA wait gave up; the outputs of that
 * call are invalid) or KD_ERR_CUDA.  Clears the device error word.
 */
KD_API int kron_delta_device_status(void *stream);

/*
 * Self-test of the failure reporting: enqueues one small kernel whose bounded
 * device-side wait runs out on purpose (a barrier nothing arrives at).  It
 * faults, traps and hangs nothing; it records a timeout in the device error
 * word and returns, so the next kron_delta_device_status(stream) reports
 * KD_ERR_TIMEOUT (and clears it).  Other work in flight on the device at that
 * moment would see its status reported as failed too: call it on an idle
 * device.  Returns KD_OK or KD_ERR_CUDA.  Asynchronous on `stream`.
 */
KD_API int kron_delta_selftest_timeout(void *stream);

/*
 * Per-kernel device timing (tracing aid for tests and benchmarks; off by
 * default).  While enabled, every kernel the library launches is bracketed by
 * two CUDA events recorded on its stream; the events are pooled and reused.
 * Not thread-safe against concurrent calls from several host threads.
 */
KD_API void kron_delta_profile_enable(int on);

/*
 * Synchronises the current device, folds every finished bracket into
 * per-kernel totals and writes one line per kernel, "name launches total_ms\n",
 * into buf (host memory, at most len bytes including the terminating NUL;
 * buf may be NULL when len is 0).  reset = 1 clears the totals afterwards.
 * Returns the number of kernels listed, or -KD_ERR_CUDA on a CUDA failure.
 */
KD_API int kron_delta_profile_report(char *buf, size_t len, int reset);

#ifdef __cplusplus
}
#endif

#endif /* KRON_DELTA_H */
