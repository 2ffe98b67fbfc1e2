// Straight-through-estimator arithmetic shared by the STE kernels (ste.cu) and the fused
// dW^ GEMM epilogue (gemm_tc.cu).
//
// For one group with step h, zero point z, range [m, M] and strengths g, b (g = b = 1 for
// the per-token activation quantizer), with u = v/h and level = round(u) + z:
//   in range (0 <= level <= Q): dq/dv = 1, dq/dh = round(u) - u, dq/dz = 0
//   clipped:                    dq/dv = 0, dq/dh = code - z,     dq/dz = -h
//   G_h = sum dq * dq/dh, G_z = sum dq * dq/dz
//   dh = G_h + G_z t/h (t = b m/h; zero where the floor of h is active)
//   dg = dh M/Q, db = -dh m/Q - G_z m/h, dM = dh g/Q, dm = -dh b/Q - G_z b/h
//   dv = dq * in_range + dM/n_max at the max elements + dm/n_min at the min elements
// ("【ICLR 2024】OmniQuant: ...", section LWC, formula differentiated as written; the
// rounding passes gradients straight through, "OmniQuant：端侧大模型低比特量化的新思路与实战"
// section 2.2.) The in-range / clipped decisions repeat the forward's binary32 arithmetic
// exactly; gradient values use a fast binary32 sigmoid for g and b.
#pragma once

#include "omq_internal.cuh"

namespace omq {

struct GroupGrad {
  float dM, dm;       // gradient reaching the range endpoints (before the tie split)
  float dg, db;       // gradient of the strengths
};

// (gradient values only: the quotients by h and Q are taken as products with the correctly
// rounded reciprocals, one rounding more than a division)
__device__ __forceinline__ GroupGrad group_grad(float Gh, float Gz, float g, float b, float h,
                                                float vmax, float vmin, float Q, bool active) {
  const float rh = __frcp_rn(h), rQ = __frcp_rn(Q);
  const float t = b * vmin * rh;
  const float dh = active ? Gh + Gz * t * rh : 0.f;
  const float dhq = dh * rQ, gzh = Gz * rh;
  GroupGrad r;
  r.dg = dhq * vmax;
  r.db = -dhq * vmin - gzh * vmin;
  r.dM = dhq * g;
  r.dm = -dhq * b - gzh * b;
  return r;
}

// Clipping strength used in gradient values (never in an integer decision); the correctly
// rounded reciprocal is the quotient 1 / (1 + e^-x) itself.
__device__ __forceinline__ float strength_value(float logit) {
  return __frcp_rn(1.f + __expf(-logit));
}

// Whether h's own gradient reaches g, b and the range: the stored h is max(h_raw, floor),
// so h above the floor means h == h_raw; at the floor h_raw is recomputed exactly.
__device__ __forceinline__ bool h_active(float h, float gl, float bl, float vmax, float vmin,
                                         float Q) {
  if (h > H_FLOOR) return true;
  return group_params(strength(gl), strength(bl), vmax, vmin, Q).active;
}

// Per-element STE pieces for 8 values: in-range mask and the G_h / G_z contributions.
__device__ __forceinline__ void ste8(const float (&v)[8], const float (&dq)[8], float h,
                                     float z, float Q, bool (&inr)[8], float& Gh, float& Gz) {
  const float hinv = __frcp_rn(h);
  float rq[8];
  round_quotient8(v, h, hinv, rq);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float r = rq[i];
    const float lvl = __fadd_rn(r, z);
    inr[i] = lvl >= 0.f && lvl <= Q;
    const float c = fminf(fmaxf(lvl, 0.f), Q);
    const float u = v[i] * hinv;
    Gh += dq[i] * (inr[i] ? (r - u) : (c - z));
    Gz += inr[i] ? 0.f : -dq[i] * h;
  }
}

__device__ __forceinline__ void in_range8(const float (&v)[8], float h, float z, float Q,
                                          bool (&inr)[8]) {
  const float hinv = __frcp_rn(h);
  float rq[8];
  round_quotient8(v, h, hinv, rq);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float lvl = __fadd_rn(rq[i], z);
    inr[i] = lvl >= 0.f && lvl <= Q;
  }
}

// Column sums over a warp's 32 rows: lane l holds 32 values (its row, 32 columns); on return
// lane l holds the sum of column l over the 32 lanes. Five butterfly rounds (31 shuffles),
// a fixed combination order.
__device__ __forceinline__ float warp_column_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

}  // namespace omq
