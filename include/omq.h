/*
 * libomq — OmniQuant fake-quantized linear calibration step on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [ICLR] "【ICLR 2024】OmniQuant: Omnidirectionally Calibrated Quantization for Large
 *          Language Models" (onecrewdev.com paper reading), sections 框架 (block-wise
 *          objective), LWC (W_q, h, z), LET (Y = [(X-δ)⊘s][s⊙W] + [B+δW]), 实验证据
 *          (AdamW, learning rates, per-channel / g128 weights, per-token activations).
 *   [AFF]  "LLM quantization tutorial" (devpress.csdn.net), section 2.2: affine
 *          (scale, zero-point) quantization.
 *   [EDGE] "OmniQuant：端侧大模型低比特量化的新思路与实战" (bjdmk.com.cn), section 2.2:
 *          the straight-through estimator.
 *
 * Notation. A linear layer Y = X W^T + B in PyTorch layout: W is [N, K] (N output rows,
 * K input channels), X is [M, K] (M tokens), Y is [M, N]. This is the paper's X W with
 * W_paper = W^T. s and δ have one entry per input channel (column of W, channel of X).
 * LWC groups are contiguous runs of `group` elements along K inside one row of W
 * (group == K is "per output channel"). Q = 2^bits - 1.
 *
 * Conventions for every entry point:
 *   - Memory. Every tensor pointer is a caller-owned DEVICE buffer, row-major and dense,
 *     16-byte aligned. Scalars are passed by value. The library allocates no device memory:
 *     scratch comes from a caller-provided workspace whose size omq_*_workspace_bytes
 *     reports.
 *   - Asynchrony. Work is enqueued on `stream` (0 = legacy default stream); calls return
 *     after validation and launch, before the GPU finishes.
 *   - Errors. Arguments are validated on the host before anything is launched; a rejected
 *     call returns a non-zero omq_status and enqueues nothing. A launch failure returns
 *     OMQ_ERR_CUDA (the CUDA code is kept in omq_last_cuda_error()). No call aborts, throws
 *     or traps. Kernels that wait on barriers give up after a bounded time and raise a
 *     device error flag that omq_sync_check() reports as OMQ_ERR_TIMEOUT.
 *   - Dtypes. W and X are stored as OMQ_BF16, OMQ_F16 or OMQ_F32; their fake-quant copies
 *     and dY (the GEMM operands) as OMQ_F16, OMQ_BF16 or OMQ_F32 (see omq_dtype); all
 *     learnable parameters, scales, gradients and losses are float32.
 *   - Rounding. round() is round-half-to-even. h, z and codes follow one fixed binary32
 *     operation order (no fused multiply-add, IEEE division):
 *        W~ = W*s;  h = max(((g*M) - (b*m)) / Q, 1e-8);  z = -round((b*m)/h)
 *        code = clamp(round(W~/h) + z, 0, Q);  W^ = (code - z)*h
 *     with g = sigmoid(γ), b = sigmoid(β) evaluated in binary64 and rounded once.
 */
#ifndef OMQ_H_
#define OMQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* omq_stream_t;   /* a cudaStream_t */

typedef enum {
  OMQ_OK = 0,
  OMQ_ERR_NULL = 1,         /* a required pointer is NULL */
  OMQ_ERR_SHAPE = 2,        /* a size is non-positive, too large, or not divisible as required */
  OMQ_ERR_DTYPE = 3,        /* unsupported dtype or dtype combination */
  OMQ_ERR_ALIGN = 4,        /* a pointer is not 16-byte aligned */
  OMQ_ERR_BITS = 5,         /* bits / abits out of range */
  OMQ_ERR_WORKSPACE = 6,    /* workspace NULL or smaller than required */
  OMQ_ERR_CUDA = 7,         /* a CUDA call failed; see omq_last_cuda_error() */
  OMQ_ERR_UNSUPPORTED = 8,  /* valid request this build does not implement */
  OMQ_ERR_TIMEOUT = 9       /* a kernel's bounded barrier wait expired (device flag) */
} omq_status;

/* Element types. W and X may be stored as F32, BF16 or F16. The GEMM operands (Xq, W_hat
 * and the residual dY) are F32 (CUDA-core path) or F16 / BF16 (tensor-core path); F16 keeps
 * 3 more mantissa bits than BF16 at the same speed and is the default of omq_calib_step
 * for 16-bit storage, its range (|x| < 65504) being ample for LET-scaled activations. */
typedef enum { OMQ_F32 = 0, OMQ_BF16 = 1, OMQ_F16 = 2 } omq_dtype;

/* Per-group (or per-token) range record written by the quantizers and read by the
 * backward: the group's max and min of the quantized values, and how many elements
 * attain each (ties share the range's gradient equally). */
typedef struct {
  float vmax;
  float vmin;
  int32_t nmax;
  int32_t nmin;
} omq_range;

/* Static description of a status code. Never NULL. */
const char* omq_status_str(int status);
/* CUDA error code (cudaError_t value) of the last OMQ_ERR_CUDA on this host thread. */
int omq_last_cuda_error(void);
/* Library version, major*10000 + minor*100 + patch. */
int omq_version(void);
/* Synchronize `stream`, then report and clear the device error flag raised by a kernel
 * whose bounded wait expired: OMQ_ERR_TIMEOUT if it was set, OMQ_ERR_CUDA if the
 * synchronization failed, OMQ_OK otherwise. */
omq_status omq_sync_check(omq_stream_t stream);
/* Longest time, in nanoseconds, that one barrier wait inside a kernel of this library may
 * take before the kernel gives up, raises the device error flag and returns (default 2 s).
 * Per device: applies to the current device. 1 ms <= ns <= 60 s, else OMQ_ERR_SHAPE.
 * Synchronous with respect to the device (a copy to a device variable); set it between
 * calls, not while kernels of the library run. */
omq_status omq_set_wait_limit_ns(uint64_t ns);
/* The current device's limit (0 if it cannot be read). */
uint64_t omq_wait_limit_ns(void);
/* Check of the bounded-wait path: one thread waits on a shared-memory barrier with the wait
 * the GEMM kernels use. arrive != 0: the thread completes the barrier itself and the wait
 * returns at once. arrive == 0: nothing completes it, so the wait gives up after the limit
 * and raises the device error flag; the kernel returns normally and omq_sync_check then
 * reports OMQ_ERR_TIMEOUT (and clears the flag). The context stays usable either way. */
omq_status omq_wait_probe(int arrive, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_lwc_quant — weight side of the step: LET weight scaling, then Learnable Weight
 * Clipping fake-quantization ([ICLR] sections LET and LWC).
 *
 *   W~[n,k] = W[n,k] * s[k]                                   (s == NULL: s = 1)
 *   per group (n, j):  M = max W~, m = min W~ over the group's `group` elements,
 *                      g = sigmoid(gamma_logit[n,j]), b = sigmoid(beta_logit[n,j]),
 *                      h = (g*M - b*m)/Q, z = -round(b*m/h)
 *   code[n,k] = clamp(round(W~/h) + z, 0, Q);   W_hat[n,k] = (code - z)*h
 *
 * W [N,K] in `wdt`; gamma_logit, beta_logit [N, K/group] float32; s [K] float32 or NULL.
 * Outputs: W_hat [N,K] in `hat_dt` (bf16 holds the binary32 value rounded to nearest
 * even); h [N, K/group] float32; z [N, K/group] int32; codes [N,K] uint8 or NULL;
 * grp_range [N, K/group] or NULL (needed by omq_fq_linear_bwd).
 * Requires K % group == 0, group % 8 == 0, bits in 2..8.
 * ------------------------------------------------------------------------------------ */
omq_status omq_lwc_quant(const void* W, omq_dtype wdt, int64_t N, int64_t K, int64_t group,
                         int bits, const float* gamma_logit, const float* beta_logit,
                         const float* s, void* W_hat, omq_dtype hat_dt, float* h, int32_t* z,
                         uint8_t* codes, omq_range* grp_range, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_let_apply — activation side of the step ([ICLR] section LET; per-token activation
 * quantization, section 实验证据).
 *
 *   X~[m,k] = (X[m,k] - delta[k]) / s[k]          (s == NULL: 1; delta == NULL: 0)
 *   abits < 16: per token m, MinMax affine fake-quant of row X~[m,:] with
 *               h_a = (max - min)/(2^abits - 1), z_a = -round(min/h_a),
 *               Xq = (clamp(round(X~/h_a) + z_a, 0, 2^abits-1) - z_a) * h_a
 *   abits == 16: Xq = X~ (h_a, z_a, tok_range are not written and may be NULL)
 *   B_tilde[n] = B[n] + sum_k W[n,k] delta[k]      (computed when B_tilde != NULL;
 *                                                   B == NULL means 0; uses the original W)
 *
 * X [M,K] in `xdt`; Xq [M,K] in `xq_dt`; h_a [M] float32, z_a [M] int32, tok_range [M].
 * W [N,K] in `wdt` is read only for B_tilde. abits in {2,3,4,6,8,16}.
 * ------------------------------------------------------------------------------------ */
omq_status omq_let_apply(const void* X, omq_dtype xdt, int64_t M, int64_t K, const float* s,
                         const float* delta, int abits, void* Xq, omq_dtype xq_dt, float* h_a,
                         int32_t* z_a, omq_range* tok_range, const void* W, omq_dtype wdt,
                         int64_t N, const float* B, float* B_tilde, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_fq_linear_fwd — fake-quantized linear forward and reconstruction loss
 * ([ICLR] section LET: Y = Q_a(X~) Q_w(W~) + B~; section 框架: the reconstruction
 * objective, taken as the mean squared error).
 *
 *   Y[m,n] = sum_k Xq[m,k] W_hat[n,k] + B_tilde[n]      (B_tilde == NULL: 0)
 *   if Y_ref != NULL:  loss = mean over M*N of (Y - Y_ref)^2     (device float32 scalar)
 *                      dY[m,n] = Y - Y_ref, the residual, stored in `dt`; the loss
 *                      gradient is dL/dY = 2 dY / (M N), a factor omq_fq_linear_bwd applies
 *                      (the residual keeps its precision in a 16-bit type)
 *
 * Xq [M,K], W_hat [N,K] in `dt`; Y_ref, Y [M,N] float32. Y may be NULL (not stored);
 * with Y_ref == NULL, `loss` and `dY` must be NULL and Y must not be.
 * 16-bit operands run on the tcgen05 tensor cores with float32 accumulation; float32
 * operands on CUDA cores in float32. K % 8 == 0 and N % 8 == 0.
 * Workspace: omq_fwd_workspace_bytes(M, N, K).
 * ------------------------------------------------------------------------------------ */
omq_status omq_fq_linear_fwd(const void* Xq, const void* W_hat, omq_dtype dt, int64_t M,
                             int64_t N, int64_t K, const float* B_tilde, const float* Y_ref,
                             float* Y, void* dY, float* loss, void* workspace, size_t ws_bytes,
                             omq_stream_t stream);
size_t omq_fwd_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* ------------------------------------------------------------------------------------
 * omq_fq_linear_fwd_noalloc — omq_fq_linear_fwd (with the loss) for callers that cannot
 * supply device scratch memory. The paper has no counterpart: this is a library convenience.
 *
 * Some hosts own every device allocation and give a plug-in library no way to obtain
 * scratch (a framework with its own memory pool and no allocation hook, or a runtime that
 * forbids device allocation after start-up). For them this call keeps its scratch (one
 * float per output tile) in a fixed array compiled into the library and allocates nothing.
 * Arguments are those of omq_fq_linear_fwd without the workspace; Y_ref, dY and loss are
 * required, Y may be NULL.
 *   - Limit: 2*ceil(M/256)*ceil(N/256) (16-bit operands) or ceil(M/64)*ceil(N/64) (float32)
 *     must not exceed 16384; larger problems return OMQ_ERR_SHAPE and launch nothing.
 *   - The array (64 KiB) is held on every GPU that loads the library until the process exits.
 *   - All calls on a device share it and it keeps the last call's contents; each call writes
 *     every slot it reads first, so nothing needs clearing. Calls that overlap on the GPU
 *     (unordered streams) race on it: order them on one stream.
 *   - Each call looks up the array's address in the calling thread's current context (a
 *     host-side lookup, no cached per-device pointer), so the call stays valid after
 *     cudaDeviceReset or under another context on the same device. The first call in a
 *     context also loads the library's module there: make it before any stream capture.
 * ------------------------------------------------------------------------------------ */
omq_status omq_fq_linear_fwd_noalloc(const void* Xq, const void* W_hat, omq_dtype dt, int64_t M,
                                     int64_t N, int64_t K, const float* B_tilde,
                                     const float* Y_ref, float* Y, void* dY, float* loss,
                                     omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_fq_linear_bwd — straight-through backward of the step ([EDGE] section 2.2; the
 * formulas of [ICLR] sections LWC and LET differentiated as written).
 *
 *   with G = 2 dY / (M N) the loss gradient (dY the forward's residual):
 *   dW_hat = G^T Xq,  dXq = G W_hat,  dB~ = sum_m G[m,:]
 *   Per LWC group, u = W~/h, c = code:
 *     in range (0 <= round(u)+z <= Q): dW_hat/dW~ = 1, dW_hat/dh = round(u) - u, dW_hat/dz = 0
 *     clipped:                          dW_hat/dW~ = 0, dW_hat/dh = c - z,        dW_hat/dz = -h
 *   and the chain through h = (g M - b m)/Q and z = -round(b m / h) into g, b and the
 *   group's max / min elements (ties split equally). Same rule per token for Q_a (g=b=1).
 *   d_gamma_logit = dL/dg * g(1-g), d_beta_logit = dL/db * b(1-b)
 *   d_s[k]     = sum_n dW~[n,k] W[n,k] - sum_m dX~[m,k] X~[m,k] / s[k]
 *   d_delta[k] = -sum_m dX~[m,k] / s[k] + sum_n dB~[n] W[n,k]
 *
 * Outputs that are NULL are skipped; d_s and d_delta need s, delta and X (LET learnable).
 * All reductions run in a fixed order: results are bitwise reproducible run to run.
 * Workspace: omq_bwd_workspace_bytes(M, N, K, group).
 * ------------------------------------------------------------------------------------ */
typedef struct {
  int64_t M, N, K, group;
  int bits, abits;
  omq_dtype dt;                   /* storage dtype of X and W */
  omq_dtype op_dt;                /* dtype of the GEMM operands Xq, W_hat and dY */
  const void* X;                  /* [M,K]   needed for d_s / d_delta */
  const void* W;                  /* [N,K] */
  const float* s;                 /* [K] or NULL (LET off) */
  const float* delta;             /* [K] or NULL */
  const float* gamma_logit;       /* [N, K/group] */
  const float* beta_logit;        /* [N, K/group] */
  const void* Xq;                 /* [M,K] forward GEMM operand */
  const void* W_hat;              /* [N,K] forward GEMM operand */
  const float* h;                 /* [N, K/group] from omq_lwc_quant */
  const int32_t* z;               /* [N, K/group] */
  const omq_range* grp_range;     /* [N, K/group] */
  const float* h_a;               /* [M] from omq_let_apply (abits < 16) */
  const int32_t* z_a;             /* [M] */
  const omq_range* tok_range;     /* [M] */
  const void* dY;                 /* [M,N] from omq_fq_linear_fwd */
  float* d_gamma_logit;           /* [N, K/group] or NULL */
  float* d_beta_logit;            /* [N, K/group] or NULL */
  float* d_s;                     /* [K] or NULL */
  float* d_delta;                 /* [K] or NULL */
  float* d_B_tilde;               /* [N] or NULL */
} omq_bwd_args;

omq_status omq_fq_linear_bwd(const omq_bwd_args* args, void* workspace, size_t ws_bytes,
                             omq_stream_t stream);
size_t omq_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group);

/* ------------------------------------------------------------------------------------
 * omq_adamw_step — one AdamW update ([ICLR] section 实验证据: AdamW, zero weight decay,
 * lr 5e-3 for the LWC logits and 1e-2 for s, δ), elementwise over n float32 values:
 *   p *= 1 - lr*wd;  m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2
 *   p -= lr/(1-b1^step) * m / (sqrt(v)/sqrt(1-b2^step) + eps)          (step >= 1)
 * ------------------------------------------------------------------------------------ */
omq_status omq_adamw_step(float* param, const float* grad, float* m, float* v, int64_t n,
                          float lr, float beta1, float beta2, float eps, float weight_decay,
                          int64_t step, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_fold_pack — fold the learned parameters into deployable integer weights
 * ([ICLR] section 框架: the learned transforms fold back into the weights).
 * codes as in omq_lwc_quant, packed row-major: element k of a row occupies bits
 * k*bits .. k*bits + bits - 1 of the row's little-endian bit string (it starts in byte
 * k*bits/8 at bit offset (k*bits) mod 8, least-significant bits first; 3-, 5-, 6- and 7-bit
 * codes may straddle two bytes). packed [N, K*bits/8] uint8; h, z [N, K/group]. bits 2..8.
 * ------------------------------------------------------------------------------------ */
omq_status omq_fold_pack(const void* W, omq_dtype wdt, int64_t N, int64_t K, int64_t group,
                         int bits, const float* gamma_logit, const float* beta_logit,
                         const float* s, uint8_t* packed, float* h, int32_t* z,
                         omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_qgemv — inference with the folded weights for a few tokens ([ICLR] section 框架: the
 * learned transforms fold into the weights; the quantized model runs as an ordinary low-bit
 * model):  y[m, n] = sum_k x[m, k] (c[n, k] - z[n, k/group]) h[n, k/group]
 * x [M, K] in xdt (the linear's input after its folded LET, i.e. (X - delta)/s), packed /
 * h / z as written by omq_fold_pack, y [M, N] float32 (add B~ for the bias). 1 <= M <= 8.
 * bits in {2, 4, 8}: CUDA-core kernel, group a multiple of 128/bits, K a multiple of group,
 * min(M, 4) (K + K bits/128) floats of shared memory at most 200 KiB (more than four tokens
 * run as two launches of at most four); decode-shaped, memory-bound on the codes. bits 3, 5, 6, 7 (codes straddling bytes): the omq_qgemm path below (16-bit x
 * only, its shape rules; OMQ_ERR_UNSUPPORTED for float32 x).
 * ------------------------------------------------------------------------------------ */
omq_status omq_qgemv(const void* x, omq_dtype xdt, int64_t M, int64_t K, const uint8_t* packed,
                     const float* h, const int32_t* z, int64_t N, int64_t group, int bits,
                     float* y, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_qgemm — the same product for any number of tokens (prefill) on the tcgen05 tensor
 * cores ([ICLR] section 框架: the quantized model runs as an ordinary low-bit model):
 *   y[m, n] = sum_k x[m, k] (c[n, k] - z[n, k/group]) h[n, k/group]  (+ bias[n])
 * The packed codes, h and z are read directly: converter warps expand each 64-column block
 * of codes into the 16-bit operand tile in shared memory ((c - z) h rounded once to xdt)
 * while the tensor cores consume the previous ones; no dequantized weight is stored.
 * x [M, K] F16 or BF16 (row-major, 16-byte aligned); packed [N, K bits/8] as written by
 * omq_fold_pack (16-byte aligned); h [N, K/group] float32, z [N, K/group] int32; bias [N]
 * float32 or NULL; y [M, N] float32. bits 2..8; K a multiple of 64; group a multiple of 8
 * dividing K; N a multiple of 8; M >= 1. float32 accumulation.
 * ------------------------------------------------------------------------------------ */
omq_status omq_qgemm(const void* x, omq_dtype xdt, int64_t M, int64_t K, const uint8_t* packed,
                     const float* h, const int32_t* z, int64_t N, int64_t group, int bits,
                     const float* bias, float* y, omq_stream_t stream);

/* ------------------------------------------------------------------------------------
 * omq_calib_step — one whole calibration step on one stream: omq_let_apply (when LET is
 * on or abits < 16), omq_lwc_quant, omq_fq_linear_fwd, omq_fq_linear_bwd, then AdamW on
 * the logits (lr_lwc) and, with LET, on s and delta (lr_let). `step` counts from 1.
 * All buffers are caller-owned device memory. When LET is off and abits == 16, X itself is
 * the GEMM operand and Xq is not used. When LET is off the step leaves the tie counts
 * (nmax, nmin) of grp_range at 0 where its row-staged LWC pass runs (16-bit W and W_hat):
 * only the LET gradients read them. Workspace: omq_step_workspace_bytes(M, N, K, group).
 *
 * Per-phase timing: `events` is NULL or an array of OMQ_PH_COUNT + 1 cudaEvent_t (passed
 * as void*). Event i is recorded on `stream` when phase i starts and event OMQ_PH_COUNT
 * when the step ends; phases that do not run are recorded back to back (zero length).
 * ------------------------------------------------------------------------------------ */
enum {
  OMQ_PH_LET = 0,       /* omq_let_apply: X~, per-token act quant, B~ */
  OMQ_PH_LWC,           /* omq_lwc_quant */
  OMQ_PH_FWD_GEMM,      /* forward GEMM with the bias / MSE / dY epilogue */
  OMQ_PH_LOSS,          /* loss reduction */
  OMQ_PH_DBIAS,         /* dB~ = column sums of dY */
  OMQ_PH_DW_GEMM,       /* dW^ = dY^T Xq */
  OMQ_PH_STE_W,         /* weight-side STE and LWC parameter gradients */
  OMQ_PH_DX_GEMM,       /* dXq = dY W^ */
  OMQ_PH_STE_X,         /* activation-side STE and LET column partials */
  OMQ_PH_LET_REDUCE,    /* d_s, d_delta reductions */
  OMQ_PH_ADAMW,         /* parameter updates */
  OMQ_PH_COUNT
};

typedef struct {
  int64_t M, N, K, group;
  int bits, abits, let;           /* let != 0: s, delta learnable */
  omq_dtype dt;                   /* storage dtype of X and W */
  omq_dtype op_dt;                /* GEMM operand dtype of Xq, W_hat, dY (F16 for 16-bit
                                     storage, F32 for F32 storage) */
  const void* X; const void* W; const float* B; const float* Y_ref;
  float* gamma_logit; float* beta_logit; float* s; float* delta;     /* learnable */
  float* m_gamma; float* v_gamma; float* m_beta; float* v_beta;      /* AdamW moments */
  float* m_s; float* v_s; float* m_delta; float* v_delta;
  void* Xq; void* W_hat; float* B_tilde;                             /* step buffers */
  float* h; int32_t* z; omq_range* grp_range;
  float* h_a; int32_t* z_a; omq_range* tok_range;
  void* dY;
  float* d_gamma_logit; float* d_beta_logit; float* d_s; float* d_delta;
  float* loss;                    /* device scalar */
  float lr_lwc, lr_let;
  int64_t step;
  void* const* events;            /* NULL, or OMQ_PH_COUNT + 1 cudaEvent_t */
} omq_step_args;

omq_status omq_calib_step(const omq_step_args* args, void* workspace, size_t ws_bytes,
                          omq_stream_t stream);
size_t omq_step_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group);

/* ====================================================================================
 * One transformer block ([ICLR] section 框架: calibration runs block by block, the loss is
 * the block output's error against the full-precision block; section LET: the transforms
 * of every linear's input except the FFN's second linear, the attention-affinity scaling
 * Q / s_a, s_a K, Q, K and V quantized, V transformed by the output projection's inverse
 * LET, softmax kept in full precision). The block, LLaMA-shaped:
 *
 *   a  = RMSNorm(x)  (weight 1, eps 1e-6);       qa = Q_a((a - δ1) / s1)        per token
 *   [q | k | v] = qa Ŵ_qkv^T + W_qkv δ1           (W~_qkv = W_qkv s1)
 *   q~ = RoPE(q) / s_a;  k~ = RoPE(k) s_a;  v~ = (v - δ_o) / s_o
 *   Qq, Qk, Qv = Q_a(q~), Q_a(k~), Q_a(v~)        per (token, head) row of 128
 *   P_h = softmax(causal(Qq_h Qk_h^T / sqrt(128)))   binary32;   O = [P_h Qv_h]_h
 *   x2 = x + Q_a(O) Ŵ_o^T + W_o δ_o               (W~_o = W_o s_o; Q_a per token)
 *   b  = RMSNorm(x2);  qb = Q_a((b - δ2) / s2);   [gate | up] = qb Ŵ_gu^T + W_gu δ2
 *   m  = SiLU(gate) up;  y = x2 + Q_a(m) Ŵ_d^T   (no LET on the down projection)
 *   loss = mean over M*D of (y - y_ref)^2
 * RoPE: rotate-half pairs (i, i + 64) of each head, angle = position * 10000^(-i/64),
 * positions 0..M-1. Each Ŵ is the LWC fake-quant of its W~ (omq_lwc_quant's rule).
 * The backward is the straight-through chain of every quantizer (omq_fq_linear_bwd's rule)
 * through the whole block; it fills d_theta for every learnable tensor.
 *
 * Storage: x and the weights BF16; the GEMM operands of the calibration step float16 (those
 * of omq_block_reference BF16, the weights' own type); y_ref, theta, gradients float32.
 * Weights: W_qkv [3D, D] (rows of q_proj, then k_proj, then v_proj), W_o [D, D],
 * W_gu [2I, D] (rows of gate_proj, then up_proj), W_d [D, I].
 * ==================================================================================== */
typedef struct {
  int64_t M;       /* tokens, a multiple of 8 */
  int64_t D;       /* hidden size = 128 H */
  int64_t H;       /* heads (head size 128) */
  int64_t I;       /* FFN size, a multiple of 32 */
  int64_t group;   /* LWC group length, a multiple of 32 dividing D and I; 0 = per channel */
  int wbits;       /* 2 .. 8 */
  int abits;       /* 2, 3, 4, 6, 8, or 16 (activations not quantized) */
} omq_block_dims;

/* The parameter vector theta: float32, these tensors back to back in this order. LWC
 * logits have one entry per (row, group) of their weight; LET vectors one per channel. */
enum {
  OMQ_TH_GAMMA_QKV = 0, OMQ_TH_BETA_QKV, OMQ_TH_GAMMA_O, OMQ_TH_BETA_O,
  OMQ_TH_GAMMA_GU, OMQ_TH_BETA_GU, OMQ_TH_GAMMA_D, OMQ_TH_BETA_D,
  OMQ_TH_S1, OMQ_TH_DELTA1, OMQ_TH_S_A, OMQ_TH_S_O, OMQ_TH_DELTA_O, OMQ_TH_S2, OMQ_TH_DELTA2,
  OMQ_TH_COUNT
};
/* Offset and length (in floats) of tensor `id` of theta; total length for id = OMQ_TH_COUNT. */
omq_status omq_block_theta_range(const omq_block_dims* dims, int id, int64_t* offset,
                                 int64_t* count);

/* Tensors the step keeps in its workspace (forward activations and the gradients that flow
 * between stages), at fixed offsets: omq_block_buffer reports offset and size in bytes. */
enum {
  OMQ_BB_ROPE = 0,   /* float32 [2, M, 64]: cos, then sin, of the rotation angles */
  OMQ_BB_A,          /* float32 [M, D]  RMSNorm(x) */
  OMQ_BB_QA,         /* F16 [M, D]      qa */
  OMQ_BB_WHAT_QKV,   /* F16 [3D, D]     Ŵ_qkv (then _O, _GU, _D) */
  OMQ_BB_WHAT_O, OMQ_BB_WHAT_GU, OMQ_BB_WHAT_D,
  OMQ_BB_QKV,        /* float32 [M, 3D] q | k | v */
  OMQ_BB_QQKV,       /* F16 [M, 3D]     Qq | Qk | Qv */
  OMQ_BB_P,          /* float32 [H, M, M] softmax (zero above the diagonal) */
  OMQ_BB_P16,        /* F16 [H, M, M]   the same, GEMM operand */
  OMQ_BB_O,          /* float32 [M, D]  attention output */
  OMQ_BB_QO,         /* F16 [M, D]      Q_a(O) */
  OMQ_BB_X2,         /* float32 [M, D]  x2 */
  OMQ_BB_B,          /* float32 [M, D]  RMSNorm(x2) */
  OMQ_BB_QB,         /* F16 [M, D]      qb */
  OMQ_BB_GU,         /* float32 [M, 2I] gate | up */
  OMQ_BB_MID,        /* float32 [M, I]  m = SiLU(gate) up */
  OMQ_BB_QM,         /* F16 [M, I]      Q_a(m) */
  OMQ_BB_RES,        /* F16 [M, D]      y - y_ref (the loss gradient is 2 res / (M D)) */
  /* The gradients below are those of (M D / 2) L, i.e. in units of res (float16 would not
   * hold the true ones, 2 / (M D) times smaller); d_theta carries the factor 2 / (M D). */
  OMQ_BB_DMID,       /* float32 [M, I]  dL/dm */
  OMQ_BB_DGU,        /* F16 [M, 2I]     dL/d[gate | up] */
  OMQ_BB_DB,         /* float32 [M, D]  dL/db */
  OMQ_BB_DX2,        /* F16 [M, D]      dL/dx2 */
  OMQ_BB_DO,         /* F16 [M, D]      dL/dO */
  OMQ_BB_DQQKV,      /* float32 [M, 3D] dL/d[Qq | Qk | Qv] */
  OMQ_BB_DQKV,       /* F16 [M, 3D]     dL/d[q | k | v] */
  OMQ_BB_COUNT
};
omq_status omq_block_buffer(const omq_block_dims* dims, int id, size_t* offset, size_t* bytes);
size_t omq_block_workspace_bytes(const omq_block_dims* dims);

/* Phases of omq_block_step for per-phase event timing (events: NULL or OMQ_BPH_COUNT + 1). */
enum {
  OMQ_BPH_WEIGHTS = 0,  /* LWC of the four weights, B~ */
  OMQ_BPH_ATTN_IN,      /* RMSNorm, LET, act quant, qkv GEMM, RoPE / affinity / head quant */
  OMQ_BPH_ATTN,         /* scores, softmax, P V */
  OMQ_BPH_FFN,          /* o_proj, RMSNorm, gate/up, SwiGLU, down + loss */
  OMQ_BPH_BWD_FFN,      /* down, SwiGLU, gate/up backward, RMSNorm backward */
  OMQ_BPH_BWD_ATTN,     /* o_proj backward, attention backward, head / RoPE STE */
  OMQ_BPH_BWD_QKV,      /* qkv backward */
  OMQ_BPH_REDUCE,       /* LET gradient reductions, loss */
  OMQ_BPH_ADAMW,
  OMQ_BPH_COUNT
};

typedef struct {
  omq_block_dims dims;
  const void* x;          /* [M, D] BF16 */
  const float* y_ref;     /* [M, D] the full-precision block output (omq_block_reference) */
  const void* W_qkv;      /* BF16 weights, shapes above */
  const void* W_o;
  const void* W_gu;
  const void* W_d;
  float* theta;           /* [P] parameters (omq_block_theta_range) */
  float* d_theta;         /* [P] gradient, written */
  float* loss;            /* device scalar, written */
  float* adam_m;          /* [P] AdamW moments, or both NULL: no update */
  float* adam_v;
  int64_t step;           /* AdamW step, from 1 */
  float lr_lwc, lr_let;   /* AdamW rates of the LWC logits and of the LET vectors */
  void* const* events;    /* NULL, or OMQ_BPH_COUNT + 1 cudaEvent_t */
} omq_block_args;

/* One calibration step of the block: forward, loss, straight-through backward, and (when
 * adam_m / adam_v are given) AdamW (beta 0.9 / 0.999, eps 1e-8, no weight decay) on theta.
 * Workspace: omq_block_workspace_bytes. The block's tensors stay in the workspace
 * (omq_block_buffer) until the next call. */
omq_status omq_block_step(const omq_block_args* args, void* workspace, size_t ws_bytes,
                          omq_stream_t stream);

/* The full-precision block (no quantizer, no transform): y [M, D] float32. Uses the same
 * workspace layout (omq_block_workspace_bytes of the same dims). */
omq_status omq_block_reference(const omq_block_dims* dims, const void* x, const void* W_qkv,
                               const void* W_o, const void* W_gu, const void* W_d, float* y,
                               void* workspace, size_t ws_bytes, omq_stream_t stream);

/* The block's output with the quantizers and transforms of theta (the fake-quantized block
 * the calibration optimises): y [M, D] in y_dt (OMQ_F32 or OMQ_BF16, rounded once from
 * binary32). This is what block-sequential calibration feeds to the next block ([ICLR]
 * section 框架: a block is calibrated, then its quantized weights compute the next block's
 * input). Same workspace as omq_block_step. */
omq_status omq_block_quant_forward(const omq_block_dims* dims, const void* x, const void* W_qkv,
                                   const void* W_o, const void* W_gu, const void* W_d,
                                   const float* theta, void* y, omq_dtype y_dt, void* workspace,
                                   size_t ws_bytes, omq_stream_t stream);

/* One block's calibration ([ICLR] sections 框架 and 实验证据: AdamW over the calibration
 * samples for a number of epochs, batch size 1): for epoch e < epochs, for sample i <
 * n_samples in order, omq_block_step on (x_i, y_ref_i) followed by AdamW with step counter
 * first_step + e * n_samples + i. Samples are stored back to back: xs [n_samples, M, D] BF16,
 * y_refs [n_samples, M, D] float32. losses [epochs * n_samples] float32 receives each step's
 * loss (device memory, written in step order). theta, adam_m, adam_v are updated in place;
 * d_theta holds the last step's gradient. All on `stream`, one step after another. */
typedef struct {
  omq_block_dims dims;
  const void* xs;
  const float* y_refs;
  int64_t n_samples;
  int64_t epochs;
  const void* W_qkv;
  const void* W_o;
  const void* W_gu;
  const void* W_d;
  float* theta;
  float* d_theta;
  float* adam_m;
  float* adam_v;
  int64_t first_step;     /* AdamW step counter of the first step, from 1 */
  float lr_lwc, lr_let;
  float* losses;
} omq_block_calib_args;
omq_status omq_block_calibrate(const omq_block_calib_args* args, void* workspace,
                               size_t ws_bytes, omq_stream_t stream);

/* Number of kernels this library has launched in this process (all threads, all devices),
 * counted on the host at each launch. */
uint64_t omq_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* OMQ_H_ */
