// Internal declarations shared by the libomq translation units: launch helpers, the
// device error flag, bf16 conversion, the clipping-strength sigmoid and the binary32
// encoder arithmetic (one fixed operation order, no contraction).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <cmath>
#include <utility>

#include "../../include/omq.h"

namespace omq {

// Raised (bitwise OR) by kernels whose bounded barrier waits expired; read by
// omq_sync_check(). Bit values say which wait gave up. The flag lives in gemm_tc.cu (the
// only translation unit with barrier waits); the host reads and clears it through this call.
enum : unsigned {
  DEV_ERR_TMA_WAIT = 1u, DEV_ERR_MMA_WAIT = 2u, DEV_ERR_EPI_WAIT = 4u, DEV_ERR_PROBE_WAIT = 8u
};
cudaError_t take_device_error(unsigned* flag);
// The device-side limit of one barrier wait, in nanoseconds (per device, default 2 s).
cudaError_t set_wait_limit(uint64_t ns);
cudaError_t get_wait_limit(uint64_t* ns);
omq_status launch_wait_probe(int arrive, cudaStream_t stream);

constexpr float H_FLOOR = 1e-8f;          // floor of the quantization step h
constexpr int Z_LIMIT = 1 << 30;          // |z| stored as int32 is clamped to this

// ---- element access --------------------------------------------------------------------
__device__ __forceinline__ float load_elem(const void* p, int64_t i, omq_dtype dt) {
  if (dt == OMQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  if (dt == OMQ_F16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void store_elem(void* p, int64_t i, float v, omq_dtype dt) {
  if (dt == OMQ_BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else if (dt == OMQ_F16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}
// 8 consecutive elements (16 B of a 16-bit type or 32 B of f32) starting at a multiple of 8.
__device__ __forceinline__ void load8(const void* p, int64_t i, omq_dtype dt, float (&v)[8]) {
  if (dt == OMQ_BF16) {
    uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(b2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  } else if (dt == OMQ_F16) {
    uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(p) + i);
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __half22float2(h2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  } else {
    const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    float4 a = q[0], b = q[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}
// 8 consecutive floats starting at a multiple of 4 (two 16-byte loads).
__device__ __forceinline__ void load_f8(const float* p, int64_t off, float (&v)[8]) {
  const float4* q = reinterpret_cast<const float4*>(p + off);
  const float4 a = q[0], b = q[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(void* p, int64_t i, omq_dtype dt, const float (&v)[8]) {
  if (dt == OMQ_BF16) {
    uint4 raw;
    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) b2[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = raw;
  } else if (dt == OMQ_F16) {
    uint4 raw;
    __half2* h2 = reinterpret_cast<__half2*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) h2[j] = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p) + i) = raw;
  } else {
    float4* q = reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i);
    q[0] = make_float4(v[0], v[1], v[2], v[3]);
    q[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// ---- encoder arithmetic ----------------------------------------------------------------
// Clipping strength in [0, 1] from its logit: evaluated in binary64, rounded once.
__device__ __forceinline__ float strength(float logit) {
  return __double2float_rn(1.0 / (1.0 + exp(-static_cast<double>(logit))));
}

struct GroupQ {
  float h;       // step (floored)
  float z;       // zero point, integral
  bool active;   // unfloored h >= H_FLOOR (h's gradient reaches g, b, max, min)
};

// h = max(((g*M) - (b*m)) / Q, 1e-8);  z = -round((b*m) / h)
__device__ __forceinline__ GroupQ group_params(float g, float b, float vmax, float vmin, float Q) {
  float hr = __fdiv_rn(__fsub_rn(__fmul_rn(g, vmax), __fmul_rn(b, vmin)), Q);
  GroupQ r;
  r.active = hr >= H_FLOOR;
  r.h = r.active ? hr : H_FLOOR;
  r.z = -rintf(__fdiv_rn(__fmul_rn(b, vmin), r.h));
  return r;
}

// Round to nearest, ties to even, for |x| < 2^22, with two additions: x + 1.5*2^23 lands in
// [2^23, 2^24) where the spacing of binary32 is 1, so the addition itself rounds x to an
// integer in round-to-nearest-even mode, and the subtraction is exact. Same result as rintf,
// on the FMA pipe.
__device__ __forceinline__ float rne_small(float x) {
  return __fsub_rn(__fadd_rn(x, 12582912.f), 12582912.f);
}

// round(v / h) with v / h the correctly rounded binary32 quotient.
//
// The quotient matters only through round(). With hinv = 1/h correctly rounded, the
// product v*hinv differs from v/h by at most 2^-23 |v/h| (two roundings), i.e. below
// 2.5e-4 while |v*hinv| < 2048. If the product's distance to its nearest integer r is at
// most 0.499, the quotient lies within 0.49925 of r and rounds to r as well; otherwise (the
// product within 1e-3 of a half-integer) and for large quotients the IEEE division itself is
// taken. The result is bitwise the level an exact-division implementation produces.
__device__ __forceinline__ float round_quotient(float v, float h, float hinv) {
  const float ua = __fmul_rn(v, hinv);
  if (fabsf(ua) < 2048.f) {
    const float r = rne_small(ua);
    if (fabsf(__fsub_rn(ua, r)) <= 0.499f) return r;
  }
  return rintf(__fdiv_rn(v, h));
}

// round(v / h) for 8 values, bitwise round_quotient's: the product with 1/h and its
// distance to the nearest integer, branch-free; one vote among the lanes that call it sends
// a lane holding a product near a half-integer (or a large quotient) to the exact quotient.
__device__ __forceinline__ void round_quotient8(const float (&v)[8], float h, float hinv,
                                                float (&r)[8]) {
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float ua = __fmul_rn(v[i], hinv);
    r[i] = rne_small(ua);
    slow |= !(fabsf(ua) < 2048.f) || !(fabsf(__fsub_rn(ua, r[i])) <= 0.499f);
  }
  if (__any_sync(__activemask(), slow)) {
    if (slow) {
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = round_quotient(v[i], h, hinv);
    }
  }
}

// Integer value of an integral binary32 c in [0, 2^23): adding 2^23 leaves c in the low
// mantissa bits.
__device__ __forceinline__ uint32_t small_uint(float c) {
  return __float_as_uint(__fadd_rn(c, 8388608.f)) & 0x7FFFFFu;
}

__device__ __forceinline__ int32_t z_to_i32(float z) {
  float c = fminf(fmaxf(z, -static_cast<float>(Z_LIMIT)), static_cast<float>(Z_LIMIT));
  return static_cast<int32_t>(c);
}

// ---- programmatic dependent launch -----------------------------------------------------
// Every kernel of the library is launched with programmatic stream serialization (launch_k)
// and opens with pdl_wait(): the grid may be scheduled while the previous kernel of the
// stream is still running (its launch and any prologue before the wait overlap that
// kernel's tail), but nothing it does to global memory precedes the previous grid's
// completion and memory flush. pdl_launch() then lets the next kernel be scheduled in turn.
// Both are no-ops for a grid launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- host-side helpers ------------------------------------------------------------------
void set_cuda_error(cudaError_t e);
omq_status launch_status();          // checks cudaGetLastError after a launch
int num_sms();

// kernel<<<grid, block, smem, stream>>>(args...) with programmatic stream serialization. A
// failed launch leaves its error for the launch_status() that follows every launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// A second stream of the calling host thread on the current device, for independent work
// inside one library call: fork() makes it wait for what the caller's stream has queued so
// far, join() makes the caller's stream wait for what it has queued. Created on first use
// (non-blocking, never destroyed); the event pair is reused from call to call, which stream
// order and graph capture both allow.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
  omq_status fork(cudaStream_t main) const;
  omq_status join(cudaStream_t main) const;
};
const SideStream* side_stream();   // nullptr (and the CUDA error recorded) if it cannot be made

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
// Groups handled lane-parallel inside a warp (16 to 256 elements, power of two); other group
// lengths take the block-per-group kernels.
inline bool small_group(int64_t g) { return g >= 16 && g <= 256 && (g & (g - 1)) == 0; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- GEMM front ends (gemm_tc.cu / gemm_simt.cu) -----------------------------------------
// C[i, j] = sum_k A(i, k) * B(j, k) for i < rows, j < cols, k < depth.
// An operand is "K-major" when A(i, k) = A[i*ld + k] and "MN-major" when A(i, k) = A[k*ld + i].
struct GemmOperand {
  const void* ptr;
  int64_t ld;         // elements between consecutive rows of the stored matrix
  bool mn_major;
};

enum class Epi { StoreF32 = 0, MseLoss = 1, SteW = 2 };

// Weight-side straight-through backward fused into the dW^ GEMM's epilogue (16-bit weights,
// group length a multiple of 32): the tile's accumulator is dW^ / out_scale. The epilogue
// writes per-(32-column chunk, row) partial sums; ste_w_finish / ste_w_corr complete them.
struct SteWEpi {
  const void* W;           // [N, K] BF16 or F16
  omq_dtype wdt;
  int64_t K, G, ng;
  float Q;
  const float* s;          // [K] or NULL
  const float* h;
  const int32_t* z;
  float* gh_part;          // [K/32, N]
  float* gc_part;          // [K/32, N]
  float* part_s;           // [ceil(N/32), K] or NULL: per 32-row block, sum (in range) dW~ W
};

// A B operand given as packed integer codes (omq_fold_pack's layout: row n of the weight is
// a little-endian bit string of `bits`-bit codes) with per-group step h and zero point z:
// B(n, k) = (code[n, k] - z[n, k / group]) h[n, k / group], expanded in the GEMM.
struct QuantB {
  const uint8_t* packed;   // [N, row_bytes]
  const float* h;          // [N, ng]
  const int32_t* z;        // [N, ng]
  int64_t row_bytes, ng, group, depth;
  int32_t kb_per_group;       // group / 64 when a group is whole 64-column k-blocks, else 0
  int32_t chunks_per_group;   // group / 8
};

struct GemmEpilogue {
  Epi kind;
  float* out;              // StoreF32: [rows, cols] fp32 (ld = cols); MseLoss: Y or NULL
  const float* bias;       // per column j, or NULL
  const float* y_ref;      // MseLoss: [rows, cols]
  void* dy;                // MseLoss: [rows, cols] residual in dy_dt
  omq_dtype dy_dt;
  float out_scale;         // StoreF32: out = out_scale * acc (+ bias); SteW: dW^ = out_scale * acc
  float* loss_partials;    // MseLoss: one per output tile (fixed order)
  SteWEpi ste;             // SteW
  int64_t ldo;             // row stride of out / y_ref / dy in elements (0: cols)
  // Scratch of the stream-K tail schedule of the tcgen05 GEMM (gemm_tc_sk_bytes), or NULL:
  // partial accumulators of split tiles and their arrival counters.
  void* sk_scratch;
  size_t sk_bytes;
  QuantB qb;               // gemm_tc_qb only
  // MseLoss, tcgen05 path, or NULL: [ceil(rows / 32), cols] column sums of the residual over
  // each 32-row block (its rows past the end count as zero)
  float* res_colsum;
};

// Group lengths whose weight-side STE runs in the dW^ GEMM's epilogue: whole 32-column
// chunks (per-channel groups included).
inline bool ste_fusable(int64_t g) { return g >= 32 && g % 32 == 0; }

// A batch of `count` GEMMs of one shape whose A, B and output origins are a_stride,
// b_stride and out_stride elements apart (attention: one problem per head), with an
// optional causal schedule for square problems over token positions:
//   causal 1: C[i, j] is needed only for j <= i: tiles wholly above the diagonal are skipped
//   causal 2: A(i, k) vanishes for k > i: the contraction stops at the tile's last row
//   causal 3: A(i, k) vanishes for k < i: the contraction starts at the tile's first row
struct GemmBatch {
  int64_t count;
  int64_t a_stride, b_stride, out_stride;
  int causal;
};
// The kernel's view of the schedule.
struct TileSched {
  int tiles_m, tiles_n;   // per problem
  int per_batch;          // tiles per problem (causal 1: the lower triangle)
  int num_tiles;          // all problems
  int causal;
  int a_bmode, b_bmode;   // operand maps: 0 2D; 1 / 2 3D, the problem index the middle / outer
  int64_t out_bstride;
  // stream-K tail: tiles [0, dp_tiles) go whole to pairs in turn; the k-blocks of tiles
  // [dp_tiles, dp_tiles + sk_tiles) are dealt out as contiguous runs of sk_len k-blocks per
  // pair (sk_tiles = 0: every tile whole)
  int dp_tiles, sk_tiles;
  int64_t sk_len;
  float* sk_part;         // [sk_tiles][2 splits][2 CTAs][128 x 256] partial accumulators
  int* sk_cnt;            // [sk_tiles][2 CTAs] arrivals
};

// 16-bit operands (BF16 or F16, both the same type) on tcgen05 (sm_100a). Reports the
// number of output tiles (loss partial slots). `batch` (StoreF32 epilogue only) may be NULL.
omq_status gemm_tc(omq_dtype dt, const GemmOperand& A, const GemmOperand& B, int64_t rows,
                   int64_t cols, int64_t depth, const GemmEpilogue& epi, int64_t* n_tiles,
                   cudaStream_t stream, const GemmBatch* batch = nullptr);
int64_t gemm_tc_tiles(int64_t rows, int64_t cols);
// Scratch that lets gemm_tc run the stream-K tail schedule on a rows x cols output (current
// device); GemmEpilogue::sk_scratch of at least this size enables it.
size_t gemm_tc_sk_bytes(int64_t rows, int64_t cols);
// C = A B^T with B expanded from packed codes in the GEMM (epi.qb; bits 2..8; epi.kind
// StoreF32): A [rows, depth] 16-bit K-major, depth a multiple of 64, B rows = cols.
omq_status gemm_tc_qb(omq_dtype dt, const GemmOperand& A, int64_t rows, int64_t cols,
                      int64_t depth, int bits, const GemmEpilogue& epi, cudaStream_t stream);
// f32 operands on CUDA cores.
omq_status gemm_f32_simt(const GemmOperand& A, const GemmOperand& B, int64_t rows, int64_t cols,
                         int64_t depth, const GemmEpilogue& epi, int64_t* n_tiles,
                         cudaStream_t stream);
int64_t gemm_f32_simt_tiles(int64_t rows, int64_t cols);


// ---- kernel parameter blocks and launchers (lwc.cu, let.cu, ste.cu) --------------------
struct LwcParams {
  const void* W;
  omq_dtype wdt;
  int64_t N, K, G, ng;
  float Q;
  const float* gl;
  const float* bl;
  const float* s;
  void* W_hat;
  omq_dtype hat_dt;
  float* h;
  int32_t* z;
  uint8_t* codes;
  omq_range* range;
  uint8_t* packed;
  int bits;
  // optional, fused into the same pass over W when the row-tile kernel runs (else a
  // separate launch): Bt[n] = B[n] + sum_k W[n,k] delta[k] with the original W
  const float* delta;
  const float* B;
  float* Bt;
  // the row-staged kernel leaves the tie counts of `range` at 0 (they feed only the LET
  // gradients, through the extremes' shares)
  bool no_ties;
};

struct LetParams {
  const void* X;
  omq_dtype xdt;
  int64_t M, K;
  const float* s;
  const float* d;
  float Qa;
  void* Xq;
  omq_dtype xq_dt;
  float* h_a;
  int32_t* z_a;
  omq_range* range;
};

struct SteWParams {
  const void* W;
  omq_dtype wdt;
  int64_t N, K, G, ng;
  float Q;
  const float* s;
  const float* gl;
  const float* bl;
  const float* h;
  const int32_t* z;
  const omq_range* range;
  const float* dWhat;   // [N,K] fp32
  const float* dBt;     // [N] or NULL
  float* d_gl;
  float* d_bl;
  float* part_s;        // [row blocks, K] or NULL: sum_n dW~[n,k] W[n,k]
  float* part_d;        // [row blocks, K] or NULL: sum_n dB~[n] W[n,k]
  int rows_per_block;
};

struct SteXParams {
  const void* X;
  omq_dtype xdt;
  int64_t M, K;
  float Qa;
  int quantized;        // abits < 16
  const float* s;
  const float* d;
  const float* h_a;
  const int32_t* z_a;
  const omq_range* range;
  const float* dXq;     // [M,K] fp32
  float* rowstat;       // [M, 2] scratch: gradient share of each token's max / min element
  float* part_s;        // [row blocks, K]: -sum_m dX~ X~ / s (NULL: skipped)
  float* part_d;        // [row blocks, K]: -sum_m dX~ / s (NULL: skipped)
  int rows_per_block;
  void* dX;             // [M, K] in dx_dt or NULL: the gradient of the LET's input, dX~ / s
  omq_dtype dx_dt;
};

// One parameter tensor of a fused AdamW launch.
struct AdamSeg {
  float* p;
  const float* g;
  float* m;
  float* v;
  int64_t n;
  float lr;
};
constexpr int kMaxAdamSegs = 4;

omq_status launch_lwc(const LwcParams& p, cudaStream_t stream);
omq_status launch_let(const LetParams& p, int abits, cudaStream_t stream);
omq_status launch_let_bias(const void* W, omq_dtype wdt, int64_t N, int64_t K, const float* delta,
                           const float* B, float* Bt, cudaStream_t stream);
omq_status launch_ste_w(const SteWParams& p, cudaStream_t stream);

// Completes the fused weight-side STE from the epilogue's partial sums: per group, G_h and
// G_z, the logit gradients and (emax / emin not NULL) the gradient share of each max / min
// element, dM / n_max and dm / n_min.
struct SteWFinish {
  int64_t N, G, ng;
  float Q;
  const float* gh_part;    // [K/32, N]
  const float* gc_part;
  const float* h;
  const omq_range* range;
  const float* gl;
  const float* bl;
  float* d_gl;
  float* d_bl;
  float* emax;             // [N, ng] or NULL
  float* emin;
};
omq_status launch_ste_w_finish(const SteWFinish& p, cudaStream_t stream);
// The W-side LET terms the fused epilogue leaves out, per 32-row block rb (one pass over W):
//   part_s[rb, k] += sum_n emax W[n,k] where W~[n,k] is its group's max, emin W[n,k] where it
//                    is the min (part_s NULL: skipped)
//   part_d[rb, k]  = sum_n dBt[n] W[n,k]  (part_d NULL: skipped)
struct SteWCorr {
  const void* W;
  omq_dtype wdt;
  int64_t N, K, G;
  const float* s;
  const omq_range* range;
  const float* emax;
  const float* emin;
  const float* dBt;
  float* part_s;
  float* part_d;
};
omq_status launch_ste_w_corr(const SteWCorr& p, cudaStream_t stream);
omq_status launch_ste_x(const SteXParams& p, cudaStream_t stream);
// part[rb, j] = sum over rows i of block rb (R rows) of w[i] A[i, j] (w NULL: 1).
omq_status launch_colsum(const void* A, omq_dtype dt, int64_t rows, int64_t cols, int R,
                         const float* w, float* part, cudaStream_t stream);
// out[j] = scale * sum over the rows of p0 [r0n, cols] and p1 [r1n, cols] (p1 may be NULL),
// binary64 in a fixed order, for one or two problems with the same cols in one launch pair;
// scratch holds 2 * kReduceChunks * cols doubles.
constexpr int kReduceChunks = 64;
struct ColReduce {
  const float* p0;
  int64_t r0n;
  const float* p1;
  int64_t r1n;
  float scale;
  float* out;
};
omq_status launch_reduce_cols(const ColReduce* probs, int nprob, int64_t cols, double* scratch,
                              cudaStream_t stream);
omq_status launch_loss_finalize(const float* part, int64_t n, double inv_count, float* loss,
                                cudaStream_t stream);
omq_status launch_adamw(const AdamSeg* segs, int nseg, float b1, float b2, float eps, float wd,
                        int64_t step, cudaStream_t stream);

}  // namespace omq
