// Internal declarations of the transformer-block step (block_kernels.cu, block_api.cu).
#pragma once

#include "omq_internal.cuh"

namespace omq {

constexpr int kAttnRows = 64;   // tokens per block of attn_prep_bwd_kernel (column partials)
constexpr int64_t kCausalTile = 256;   // output tile of the tcgen05 GEMM (rows = columns)

struct RmsParams {
  const void* x;        // [M, D] in xdt
  omq_dtype xdt;
  const float* add;     // [M, D] or NULL: v = x + add
  int64_t M, D;
  float eps;
  float* x2;            // [M, D] or NULL: v stored
  float* n;             // [M, D] v * rstd
  float* rstd;          // [M] or NULL
  const float* y_ref;   // [M, D] or NULL (zero)
  float* tgt;           // [M, D] or NULL: y_ref - v
};

struct RmsBwdParams {
  const float* dn;      // [M, D] gradient of the normalized values
  const float* n;       // [M, D] the normalized values
  const float* rstd;    // [M]
  const void* res;      // [M, D] residual-path gradient / res_scale, in dt16
  float res_scale;
  int64_t M, D;
  void* dx;             // [M, D] in dt16
  omq_dtype dt16;       // OMQ_F16 or OMQ_BF16: the block's 16-bit GEMM operand type
};

// q | k | v [M, 3D] float32 in, Qq | Qk | Qv [M, 3D] 16-bit out, per (which, token, head) stats.
struct AttnPrepParams {
  const float* qkv;
  const float* cos_t;   // [M, 64]
  const float* sin_t;
  const float* s_a;     // [D] or NULL (no affinity transform)
  const float* s_o;     // [D] or NULL (no V transform)
  const float* delta_o; // [D] (with s_o)
  int64_t M, D, H;
  int quantized;
  float Qa;
  omq_dtype dt16;       // OMQ_F16 or OMQ_BF16 for out and dout
  void* out;            // forward: the quantized (or transformed) q~, k~, v~
  float* h_s;           // [3, M, H]
  int32_t* z_s;
  omq_range* range_s;
  // backward
  const float* dq;      // [M, 3D] gradient of the quantized values
  void* dout;           // [M, 3D] gradient of q | k | v
  float* part_sa;       // [ceil(M / kAttnRows), D] or NULL
  float* part_so;
  float* part_do;
};

omq_status launch_rope_table(int64_t M, double base, float* cos_t, float* sin_t, cudaStream_t st);
omq_status launch_rms(const RmsParams& p, cudaStream_t st);
omq_status launch_rms_bwd(const RmsBwdParams& p, cudaStream_t st);
omq_status launch_attn_prep(const AttnPrepParams& p, bool backward, cudaStream_t st);
omq_status launch_softmax(float* S, void* P16, omq_dtype dt16, int64_t rows, int64_t M,
                          cudaStream_t st);
omq_status launch_softmax_bwd(const float* P, const float* dP, void* dS, omq_dtype dt16,
                              int64_t rows, int64_t M, float scale, cudaStream_t st);
omq_status launch_swiglu(const float* gu, float* mid, int64_t M, int64_t I, cudaStream_t st);
omq_status launch_swiglu_bwd(const float* gu, const float* dmid, void* dgu, omq_dtype dt16,
                             int64_t M, int64_t I, cudaStream_t st);
// x[i] *= s for i < n (float32), in place.
omq_status launch_scale(float* x, int64_t n, float s, cudaStream_t st);

}  // namespace omq
