/*
 * aurora_muon.h -- C ABI of libaurora_muon.so: the Muon / Aurora optimizer
 * step for the 2-D weight matrices of a transformer, on one B200 (sm_100a).
 *
 * The method is the one described in "modded-nanogpt Track 3 优化实录：Aurora
 * 行均衡 polar + Contra-Muon + u/w-floor 将 3.28 验证损失推进到 3175 步"
 * (sections "Aurora 的迭代伪代码", "源码实现", "组合优化栈", "u/w-floor",
 * "完整的超参配置表"), with the Newton-Schulz primitive and the quintic
 * coefficient set of the modded-nanogpt 2024-11-10 record write-up (section
 * "训练管线与系统实现 / 四路优化器分工").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - A matrix is m x n, row-major and contiguous (torch [out, in]); shapes
 *    are passed in a host array of muon_shape.  s = min(m,n), l = max(m,n).
 *  - Pointer arrays (params, grads, ...) are HOST arrays of DEVICE pointers.
 *    Every device pointer must be 16-byte aligned.
 *  - The caller owns every buffer.  The library allocates no device memory:
 *    all scratch lives in the caller's workspace, sized by
 *    muon_workspace_size().  The workspace may be reused freely between
 *    calls; no state is kept in it across calls.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Argument errors are detected on the
 *    host and returned before anything is launched.  A failed launch returns
 *    MUON_ERR_CUDA.  Kernels never trap: a device-side wait that runs past
 *    its limit records MUON_ERR_TIMEOUT in a sticky device status word that
 *    muon_last_device_status() reads (and clears).
 *  - Calls on the same stream are ordered; calls on different streams that
 *    share a workspace or a tensor race.
 */
#ifndef AURORA_MUON_H
#define AURORA_MUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad shape, bad config value */
  MUON_ERR_UNSUPPORTED = 2,  /* a valid request the library does not implement */
  MUON_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than muon_workspace_size() */
  MUON_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  MUON_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up (see muon_last_device_status) */
  MUON_ERR_BOUNDS = 6        /* checked build only: a kernel's index fell outside its buffer
                                (the access was skipped; see muon_build_checked) */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype;

/* Precision of the Newton-Schulz GEMMs.
 *  BF16      : bf16 operands, fp32 accumulation, tcgen05 tensor cores (the
 *              precision of the pages' zeropower_via_newtonschulz5).
 *  FP32      : fp32 operands and accumulation on the FMA pipes (reference
 *              precision; slow).
 *  BF16_SIMT : bf16 storage with fp32 FMA accumulation on the SIMT pipes; a
 *              diagnostic second implementation of the BF16 numerics. */
typedef enum { MUON_GEMM_BF16 = 0, MUON_GEMM_FP32 = 1, MUON_GEMM_BF16_SIMT = 2 } muon_gemm_mode;

typedef struct { int64_t rows, cols; } muon_shape;

/* Hyper-parameters of one step.  muon_config_default() fills the Track-3
 * result #17 locked values (section "完整的超参配置表"): lr 0.0375, mu 0.95,
 * Nesterov, 12 Newton-Schulz steps with (a,b,c) = (2, -1.5, 0.5) and eps
 * 1e-7, Aurora with pp_iterations 2, pp_beta 0.5, pp_eps 1e-7, CONTRA_MUON
 * 0.4 with 5 power iterations, TARGET_UW 0.35, weight_decay 0, BF16 GEMMs,
 * bf16 params and grads. */
typedef struct {
  float lr;             /* parameter step: W <- W - lr * V                         */
  float mu;             /* momentum: m <- lerp(m, g, 1 - mu)                        */
  int   nesterov;       /* 1: u = lerp(g, m, mu); 0: u = m                          */
  int   ns_steps;       /* Newton-Schulz iterations (>= 1)                          */
  float ns_a, ns_b, ns_c;  /* X <- a X + (b A + c A^2) X, A = X X^T                */
  float ns_eps;         /* X0 = G / (|G|_F + ns_eps)                                */
  int   aurora;         /* 1: polar(D G) row equilibration; 0: plain polar(G)       */
  int   pp_iterations;  /* number of polars per non-square matrix (>= 1)            */
  float pp_beta;        /* damping exponent of the D update                         */
  float pp_eps;         /* clamp of the row norms (row_sq clamp is pp_eps^2)        */
  float contra;         /* CONTRA_MUON; 0 disables the contra subtraction           */
  int   power_iters;    /* power iterations of the operator-norm estimate (>= 1)    */
  float target_uw;      /* TARGET_UW; 0 disables the u/w floor                      */
  float weight_decay;   /* must be 0 (the u/w floor replaces weight decay)          */
  int   gemm_mode;      /* muon_gemm_mode                                           */
  int   param_dtype;    /* muon_dtype of params                                     */
  int   grad_dtype;     /* muon_dtype of grads                                      */
} muon_config;

/* Fill *cfg with the locked Track-3 values listed above. */
void muon_config_default(muon_config* cfg);

/* Bytes of device workspace that every entry point below needs for these n
 * shapes and this config.  Returns 0 when n == 0.  Pure host function. */
size_t muon_workspace_size(const muon_config* cfg, int n, const muon_shape* shapes);

/* One full optimizer step on n matrices ("组合优化栈" + "u/w-floor"):
 *   m <- m + (1-mu)(g - m);  u = g + mu(m - g) (Nesterov) or m;
 *   N = u / sigma_hat(u)   (5-step power iteration, contra > 0 only);
 *   U = polar(u) (Newton-Schulz) or Aurora polar(D u) / polar(u D);
 *   V = (U - contra/2 N) |U|_F / |U - contra/2 N|_F;  V *= sqrt(max(1, m/n));
 *   if |V|_F / |W|_F < target_uw: V *= target_uw |W|_F / |V|_F;
 *   W <- W - lr V.
 * params   : n device pointers, param_dtype, updated in place.
 * grads    : n device pointers, grad_dtype, read only (the pages' grad.lerp_
 *            side effect on the gradient buffer is not reproduced).
 * momentum : n device pointers, fp32, updated in place.
 * update_out: NULL, or n device pointers (entries may be NULL) receiving V
 *            in fp32 (m x n), the applied update before the lr.
 * The call only enqueues kernel launches, and 4-byte memsets of the
 * workspace (the tensor-core GEMM's tile counter), on `stream` (no
 * allocation, no synchronisation, no host read of device data), so it can be
 * captured in a CUDA graph once the first call on the device has been made
 * outside capture; the captured launches carry this call's config.
 * Errors: INVALID_ARG, WORKSPACE, CUDA as described above. */
muon_status muon_step(const muon_config* cfg, int n, const muon_shape* shapes,
                      void* const* params, const void* const* grads,
                      float* const* momentum, float* const* update_out,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Newton-Schulz polar factor of each input ("源码实现",
 * zeropower_via_newtonschulz5): in (in_dtype, m x n) -> out (fp32, m x n).
 * Uses cfg->ns_* and cfg->gemm_mode; other fields are ignored. */
muon_status ns_polar(const muon_config* cfg, int n, const muon_shape* shapes,
                     const void* const* in, int in_dtype, float* const* out,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Aurora leverage-uniform polar ("Aurora 的迭代伪代码", "源码实现",
 * aurora_orthogonalize): square inputs take the plain polar; tall inputs
 * polar(D G); wide inputs polar(G D).  Uses cfg->ns_*, pp_iterations,
 * pp_beta, pp_eps, gemm_mode.  out is fp32 m x n. */
muon_status aurora_polar(const muon_config* cfg, int n, const muon_shape* shapes,
                         const void* const* in, int in_dtype, float* const* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Operator-norm normalisation ("组合优化栈", scale_to_unit_operator_norm):
 * sigma = |A v| after cfg->power_iters steps of v <- A^T A v / |A^T A v|
 * from v0 = ones(n)/sqrt(n); out = A / max(sigma, 1e-10).
 * sigma_out: device array of n floats (may be NULL).  out: NULL, or n device
 * pointers (entries may be NULL) receiving fp32 m x n. */
muon_status opnorm_normalize(const muon_config* cfg, int n, const muon_shape* shapes,
                             const void* const* in, int in_dtype, float* const* out,
                             float* sigma_out, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Workspace-free variant of opnorm_normalize (the pages have no counterpart;
 * it exists for callers that cannot allocate device memory where they need
 * this step: code under a framework whose memory manager owns the whole
 * device, or loops that must not enter the allocator after start-up).
 * Same results as opnorm_normalize within rounding: sigma = |A v| after
 * cfg->power_iters steps of v <- A^T A v / |A^T A v| from ones(n)/sqrt(n),
 * out = A / max(sigma, 1e-10), computed directly on the input in its own
 * dtype (in_dtype) and orientation.  Uses cfg->power_iters only.
 *  - Scratch: a 1 MiB file-scope device array inside the library (held by
 *    every GPU that loads the library until exit).  A call needs
 *    n * 128 bytes plus 4 * (round_up(rows, 64) + round_up(cols, 64)) bytes
 *    per matrix; larger requests return MUON_ERR_UNSUPPORTED before
 *    anything is launched.
 *  - Calls no cudaMalloc / cudaFree.  The first call on a device looks up
 *    the array's device address (cudaGetSymbolAddress, with that device
 *    current); make that first call before any stream capture.  The address
 *    is kept for the life of the process: no cudaDeviceReset may come
 *    between calls (a reset reloads the module and can move the array).
 *  - rows or cols above 2^31 return MUON_ERR_INVALID_ARG.
 *  - Every call shares the one array and it keeps the last call's contents;
 *    each call clears its scalar block first.  Calls that overlap on the
 *    GPU (different streams, or different host threads on one device) race
 *    on the array: serialise them. */
muon_status opnorm_normalize_noalloc(const muon_config* cfg, int n, const muon_shape* shapes,
                                     const void* const* in, int in_dtype, float* const* out,
                                     float* sigma_out, void* stream);

/* u/w floor ("u/w-floor"): for each matrix, with p = max(|W|_F, 1e-8) and
 * q = max(|U|_F, 1e-8), if q / p < cfg->target_uw the fp32 update U is
 * scaled in place by target_uw * p / q.  params are read only (param_dtype
 * = cfg->param_dtype). */
muon_status uw_floor_apply(const muon_config* cfg, int n, const muon_shape* shapes,
                           const void* const* params, float* const* updates,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Auxiliary AdamW for the parameters Muon does not step (the Track 3
 * write-up, "完整的超参配置表" and the hyper-parameter placement paragraph:
 * token embedding lr 0.3, output projection lr 1/320, 1-D parameters lr 0.01,
 * betas (0.8, 0.95), eps 1e-10, weight_decay 0, fused).  The pages name the
 * optimizer without printing its update; this is torch.optim.AdamW's
 * decoupled-weight-decay Adam at 1-based step count `step`:
 *   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *   p <- p - lr / (1 - b1^step) * m / (sqrt(v) / sqrt(1 - b2^step) + eps).
 * adamw_config_default() fills lr 0.01, betas (0.8, 0.95), eps 1e-10, wd 0,
 * step 1, bf16 params and grads. */
typedef struct {
  float lr;            /* used for every tensor when `lrs` is NULL */
  float beta1, beta2;  /* in [0, 1) */
  float eps;           /* >= 0 */
  float weight_decay;  /* >= 0 (decoupled) */
  int   step;          /* 1-based step count for the bias corrections */
  int   param_dtype;   /* muon_dtype of params */
  int   grad_dtype;    /* muon_dtype of grads */
} adamw_config;

void adamw_config_default(adamw_config* cfg);

/* One fused AdamW step over n contiguous tensors of any shape.
 * numels    : host array of n element counts (0 = skip the tensor).
 * lrs       : host array of n learning rates, or NULL (cfg->lr for all).
 * params    : n device pointers (param_dtype), updated in place.
 * grads     : n device pointers (grad_dtype), read only.
 * exp_avg, exp_avg_sq : n device pointers (fp32), updated in place.
 * Every device pointer must be 16-byte aligned.  No workspace.  Errors:
 * INVALID_ARG (before any launch), CUDA. */
muon_status adamw_step(const adamw_config* cfg, int n, const int64_t* numels, const float* lrs,
                       void* const* params, const void* const* grads, float* const* exp_avg,
                       float* const* exp_avg_sq, void* stream);

/* Synchronises `stream`, then returns and clears the sticky device status
 * words of the current device: MUON_OK, MUON_ERR_TIMEOUT after a bounded
 * device wait gave up, or (checked build) MUON_ERR_BOUNDS after an index
 * check failed. */
muon_status muon_last_device_status(void* stream);

/* Debugging aid without a counterpart on the pages (the pool has no memory
 * sanitizer).  libaurora_muon_checked.so is the same library compiled with
 * every global access of the streaming, power-iteration and GEMM-epilogue
 * kernels tested against the extent of the buffer it addresses (TMA loads
 * and stores are bounded by their tensor maps); a failed test skips the
 * access and records MUON_ERR_BOUNDS.  muon_build_checked() returns 1 in
 * that library and 0 in libaurora_muon.so.  muon_last_check_line() returns
 * (and clears) where the first failed test sits, 0 if none: file * 100000 +
 * line, files numbered 1 elementwise.cu, 2 powiter.cu, 3 gemm_tc.cu,
 * 4 gemm_simt.cu, 5 adamw.cu.
 * muon_selftest_bounds_check launches one thread that tests an element
 * range lying outside a 4-element extent without touching memory: in the
 * checked library the next muon_last_device_status returns MUON_ERR_BOUNDS,
 * in the normal one MUON_OK. */
int muon_build_checked(void);
int muon_last_check_line(void);
muon_status muon_selftest_bounds_check(void* stream);

/* Diagnostic of the failure-detection path (no counterpart on the pages):
 * launches one block whose thread waits, with the same bounded-wait routine
 * the GEMM kernels use, on a shared-memory barrier that nothing arrives on.
 * After max_cycles SM clock cycles (clamped to [1e3, 4e9]) the wait gives
 * up and records MUON_ERR_TIMEOUT in the sticky device status word, exactly
 * as a stalled pipeline would; the kernel then returns and the context stays
 * usable.  Returns MUON_OK when the launch succeeded (read the outcome with
 * muon_last_device_status), MUON_ERR_CUDA otherwise. */
muon_status muon_selftest_wait_timeout(long long max_cycles, void* stream);

/* Static English description of a status code. */
const char* muon_status_string(muon_status s);

/* Tracing of the library's own launches (no counterpart on the pages; it
 * serves measurement).  While enabled, every kernel launch of every entry
 * point is bracketed by two CUDA events recorded on the launch stream, and
 * attributed to a kernel class ("ns_gemm_tc", "ns_gemm_simt", "prologue",
 * "power_iter", "aurora_rows", "reductions", "epilogue") together with its
 * algorithmic floating-point operations and HBM bytes.
 * muon_profile_enable(1) clears earlier records and starts recording;
 * muon_profile_enable(0) stops.  Events are created on first use and reused.
 * muon_profile_read() waits for the recorded events, writes up to
 * max_entries per-class totals to `out` and returns the number of classes
 * written (or -1 on a CUDA error). */
typedef struct {
  char name[32];
  int64_t launches;
  double ms;      /* summed device time between each launch's two events      */
  double flops;   /* summed algorithmic floating-point operations            */
  double bytes;   /* summed algorithmic HBM bytes (reads + writes)           */
} muon_profile_entry;

void muon_profile_enable(int on);
int muon_profile_read(muon_profile_entry* out, int max_entries);

#ifdef __cplusplus
}
#endif

#endif /* AURORA_MUON_H */
