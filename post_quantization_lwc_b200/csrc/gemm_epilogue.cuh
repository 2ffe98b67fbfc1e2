// Per-element GEMM epilogues shared by the tcgen05 and CUDA-core GEMMs.
//
// StoreF32: out[i, j] = out_scale * acc (+ bias[j]).
// Row i of out, y_ref and dy starts at i * ldo (ldo = 0: i * cols).
// MseLoss : the fake-quant forward's tail ("Y = Q_a(X~) Q_w(W~) + B~", then the squared
//           reconstruction error against the full-precision output):
//           Y = acc + bias[j]; optionally stored; R = Y - Y_ref written as the residual
//           (the loss gradient is 2 R / (rows cols), applied by the backward);
//           loss partial += R^2; optionally the column sums of R over each 32-row block
//           (the bias gradient's partials, res_colsum).
#pragma once

#include "omq_internal.cuh"

namespace omq {

// `out` is e.out, or the output of this tile's problem in a batch. Returns the residual
// (MseLoss; 0 for StoreF32).
__device__ __forceinline__ float epi_element(const GemmEpilogue& e, float* out, int64_t i,
                                             int64_t j, int64_t cols, float acc, float& lsum) {
  const int64_t o = i * (e.ldo ? e.ldo : cols) + j;
  if (e.kind == Epi::StoreF32) {
    out[o] = e.out_scale * acc + (e.bias ? e.bias[j] : 0.f);
    return 0.f;
  }
  const float y = acc + (e.bias ? e.bias[j] : 0.f);
  if (out) out[o] = y;
  const float d = y - e.y_ref[o];
  lsum += d * d;
  store_elem(e.dy, o, d, e.dy_dt);
  return d;
}

// 8 consecutive columns j0..j0+7 of row i, all in range, j0 % 8 == 0, cols % 8 == 0 and the
// row stride a multiple of 8.
__device__ __forceinline__ void epi_vec8(const GemmEpilogue& e, float* out, int64_t i,
                                         int64_t j0, int64_t cols, const float (&acc)[8],
                                         float& lsum, float (&res)[8]) {
  const int64_t o = i * (e.ldo ? e.ldo : cols) + j0;
  const float sc = e.kind == Epi::StoreF32 ? e.out_scale : 1.f;
  float y[8];
  if (e.bias) {
    const float4* bp = reinterpret_cast<const float4*>(e.bias + j0);
    float4 b0 = bp[0], b1 = bp[1];
    y[0] = sc * acc[0] + b0.x; y[1] = sc * acc[1] + b0.y; y[2] = sc * acc[2] + b0.z;
    y[3] = sc * acc[3] + b0.w; y[4] = sc * acc[4] + b1.x; y[5] = sc * acc[5] + b1.y;
    y[6] = sc * acc[6] + b1.z; y[7] = sc * acc[7] + b1.w;
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) y[t] = sc * acc[t];
  }
  if (e.kind == Epi::StoreF32) {
    store8(out, o, OMQ_F32, y);
#pragma unroll
    for (int t = 0; t < 8; ++t) res[t] = 0.f;
    return;
  }
  if (out) store8(out, o, OMQ_F32, y);
  float r[8];
  load8(e.y_ref, o, OMQ_F32, r);
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    res[t] = y[t] - r[t];
    lsum += res[t] * res[t];
  }
  store8(e.dy, o, e.dy_dt, res);
}

}  // namespace omq
