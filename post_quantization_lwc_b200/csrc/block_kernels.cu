// Elementwise and row kernels of the transformer-block calibration step ("【ICLR 2024】
// OmniQuant: ...", sections 框架 and LET): RMSNorm, the rotary embedding with the
// attention-affinity LET and the per-(token, head) activation quantizer, the causal softmax
// and its backward, SwiGLU and its backward, and the RMSNorm backward. The GEMMs, the weight
// quantizer and the per-token activation quantizer are the linear layer's kernels.
//
// Head size is 128: a warp holds one (token, head) row, lane l the elements 2l, 2l + 1,
// 64 + 2l, 65 + 2l, so each rotate-half pair (i, i + 64) sits in one lane.
#include <float.h>

#include "block_internal.cuh"
#include "ste_common.cuh"

namespace omq {

// ------------------------------------------------------------------ rotary table
// cos / sin of pos * base^(-2i/Dh) in binary64, rounded once: [M, Dh/2] each.
__global__ void rope_table_kernel(int64_t M, int half, double base, float* cos_t, float* sin_t) {
  pdl_wait();
  pdl_launch();
  const int64_t total = M * half;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = t / half;
    const int i = static_cast<int>(t % half);
    const double inv = pow(base, -2.0 * i / (2.0 * half));
    const double ang = static_cast<double>(m) * inv;
    cos_t[t] = static_cast<float>(cos(ang));
    sin_t[t] = static_cast<float>(sin(ang));
  }
}

// ------------------------------------------------------------------ RMSNorm
// Per row: v = x (+ add); x2 = v (stored if x2 != NULL); rstd = 1/sqrt(mean(v^2) + eps);
// n = v rstd; tgt = y_ref - v (tgt != NULL; y_ref NULL reads as zero). One 256-thread block per row, 8 values a thread
// per pass, binary32 with a fixed reduction order.
__device__ __forceinline__ float block_sum(float v, float* sm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sm[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += sm[i];
  return t;
}

__global__ void __launch_bounds__(256) rms_kernel(RmsParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float sm[32];
  const int chunks = static_cast<int>(p.D / 8);
  for (int64_t m = blockIdx.x; m < p.M; m += gridDim.x) {
    const int64_t base = m * p.D;
    float ss = 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8];
      load8(p.x, base + c * 8, p.xdt, v);
      if (p.add) {
        float a[8];
        load_f8(p.add, base + c * 8, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fadd_rn(v[i], a[i]);
        if (p.x2) store8(p.x2, base + c * 8, OMQ_F32, v);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
    }
    ss = block_sum(ss, sm);
    const float rstd = 1.f / sqrtf(ss / static_cast<float>(p.D) + p.eps);
    if (threadIdx.x == 0 && p.rstd) p.rstd[m] = rstd;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8], n[8];
      load8(p.x, base + c * 8, p.xdt, v);
      if (p.add) {
        float a[8];
        load_f8(p.add, base + c * 8, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fadd_rn(v[i], a[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) n[i] = v[i] * rstd;
      store8(p.n, base + c * 8, OMQ_F32, n);
      if (p.tgt) {
        float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (p.y_ref) load_f8(p.y_ref, base + c * 8, r);
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] = r[i] - v[i];
        store8(p.tgt, base + c * 8, OMQ_F32, r);
      }
    }
  }
}

// RMSNorm backward with the residual path: dx2 = res_scale res + rstd (dn - n mean(dn n)).
__global__ void __launch_bounds__(256) rms_bwd_kernel(RmsBwdParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float sm[32];
  const int chunks = static_cast<int>(p.D / 8);
  for (int64_t m = blockIdx.x; m < p.M; m += gridDim.x) {
    const int64_t base = m * p.D;
    float dot = 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float dn[8], n[8];
      load_f8(p.dn, base + c * 8, dn);
      load_f8(p.n, base + c * 8, n);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot += dn[i] * n[i];
    }
    dot = block_sum(dot, sm);
    const float mean = dot / static_cast<float>(p.D);
    const float rstd = p.rstd[m];
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float dn[8], n[8], r[8], o[8];
      load_f8(p.dn, base + c * 8, dn);
      load_f8(p.n, base + c * 8, n);
      load8(p.res, base + c * 8, p.dt16, r);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = p.res_scale * r[i] + rstd * (dn[i] - n[i] * mean);
      store8(p.dx, base + c * 8, p.dt16, o);
    }
  }
}

// ------------------------------------------------------------------ per-row quantizer
// One warp, one row of 128 values (4 per lane): MinMax affine fake-quant with g = b = 1.
struct RowQ {
  GroupQ q;
  omq_range rg;
};

__device__ __forceinline__ RowQ row_quant(const float (&v)[4], float Qa) {
  float vmax = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
  float vmin = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
  }
  int nmax = 0, nmin = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) { nmax += v[i] == vmax; nmin += v[i] == vmin; }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
    nmin += __shfl_xor_sync(0xffffffffu, nmin, o);
  }
  RowQ r;
  r.q = group_params(1.f, 1.f, vmax, vmin, Qa);
  r.rg = omq_range{vmax, vmin, nmax, nmin};
  return r;
}

__device__ __forceinline__ void row_dequant(float (&v)[4], const GroupQ& q, float Qa) {
  const float hinv = __frcp_rn(q.h);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lvl = __fadd_rn(round_quotient(v[i], q.h, hinv), q.z);
    const float c = fminf(fmaxf(lvl, 0.f), Qa);
    v[i] = __fmul_rn(__fsub_rn(c, q.z), q.h);
  }
}

// Straight-through gradient of row_quant's dequantized values with respect to its inputs
// (same rule as the per-token activation quantizer).
__device__ __forceinline__ void row_ste(const float (&v)[4], float (&d)[4], float h, float z,
                                        const omq_range& rg, float Qa) {
  const float hinv = __frcp_rn(h);
  bool inr[4];
  float Gh = 0.f, Gz = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float r = round_quotient(v[i], h, hinv);
    const float lvl = __fadd_rn(r, z);
    inr[i] = lvl >= 0.f && lvl <= Qa;
    const float c = fminf(fmaxf(lvl, 0.f), Qa);
    Gh += d[i] * (inr[i] ? (r - v[i] * hinv) : (c - z));
    Gz += inr[i] ? 0.f : -d[i] * h;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Gh += __shfl_xor_sync(0xffffffffu, Gh, o);
    Gz += __shfl_xor_sync(0xffffffffu, Gz, o);
  }
  const bool active = group_params(1.f, 1.f, rg.vmax, rg.vmin, Qa).active;
  const GroupGrad gg = group_grad(Gh, Gz, 1.f, 1.f, h, rg.vmax, rg.vmin, Qa, active);
  const float eM = gg.dM / static_cast<float>(rg.nmax);
  const float em = gg.dm / static_cast<float>(rg.nmin);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float g = inr[i] ? d[i] : 0.f;
    if (v[i] == rg.vmax) g += eM;
    if (v[i] == rg.vmin) g += em;
    d[i] = g;
  }
}

// Lane l's four columns of a head: 2l, 2l + 1, 64 + 2l, 65 + 2l.
__device__ __forceinline__ void load_head4(const float* row, int lane, float (&v)[4]) {
  const float2 lo = *reinterpret_cast<const float2*>(row + 2 * lane);
  const float2 hi = *reinterpret_cast<const float2*>(row + 64 + 2 * lane);
  v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}
// Two values rounded to the 16-bit type (nearest even), packed in one 32-bit word.
__device__ __forceinline__ uint32_t pack2(float a, float b, bool f16) {
  if (f16) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// Lane l's four columns of a head row of 16-bit values (element offset `off` from `base`).
__device__ __forceinline__ void store_head4(void* base, int64_t off, int lane, const float (&v)[4],
                                            bool f16) {
  uint16_t* row = static_cast<uint16_t*>(base) + off;
  *reinterpret_cast<uint32_t*>(row + 2 * lane) = pack2(v[0], v[1], f16);
  *reinterpret_cast<uint32_t*>(row + 64 + 2 * lane) = pack2(v[2], v[3], f16);
}
__device__ __forceinline__ void load_vec4(const float* vec, int lane, float (&v)[4]) {
  load_head4(vec, lane, v);
}

// Rotate-half RoPE of lane-held values in binary32, no contraction:
//   r[i] = x[i] c - x[i + 64] s,  r[i + 64] = x[i + 64] c + x[i] s
__device__ __forceinline__ void rope4(float (&v)[4], const float2 c, const float2 s) {
  const float a0 = v[0], a1 = v[1], b0 = v[2], b1 = v[3];
  v[0] = __fsub_rn(__fmul_rn(a0, c.x), __fmul_rn(b0, s.x));
  v[1] = __fsub_rn(__fmul_rn(a1, c.y), __fmul_rn(b1, s.y));
  v[2] = __fadd_rn(__fmul_rn(b0, c.x), __fmul_rn(a0, s.x));
  v[3] = __fadd_rn(__fmul_rn(b1, c.y), __fmul_rn(a1, s.y));
}
// Its transpose (gradient path).
__device__ __forceinline__ void rope4_t(float (&d)[4], const float2 c, const float2 s) {
  const float a0 = d[0], a1 = d[1], b0 = d[2], b1 = d[3];
  d[0] = a0 * c.x + b0 * s.x;
  d[1] = a1 * c.y + b1 * s.y;
  d[2] = b0 * c.x - a0 * s.x;
  d[3] = b1 * c.y - a1 * s.y;
}

// The forward transforms of one (token, head) row of q, k or v (which = 0, 1, 2), in the
// fixed binary32 order: q~ = RoPE(q) / s_a, k~ = RoPE(k) s_a, v~ = (v - delta_o) / s_o.
// rot receives RoPE(q) / RoPE(k) (the backward needs it).
__device__ __forceinline__ void head_forward(const AttnPrepParams& p, int which, int64_t m,
                                             int h, int lane, float (&v)[4], float (&rot)[4]) {
  const int64_t D = p.D;
  load_head4(p.qkv + m * 3 * D + which * D + h * 128, lane, v);
  if (which < 2) {
    const float2 c = *reinterpret_cast<const float2*>(p.cos_t + m * 64 + 2 * lane);
    const float2 s = *reinterpret_cast<const float2*>(p.sin_t + m * 64 + 2 * lane);
    rope4(v, c, s);
#pragma unroll
    for (int i = 0; i < 4; ++i) rot[i] = v[i];
    if (p.s_a) {
      float sa[4];
      load_vec4(p.s_a + h * 128, lane, sa);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = which == 0 ? __fdiv_rn(v[i], sa[i]) : __fmul_rn(v[i], sa[i]);
    }
  } else if (p.s_o) {
    float so[4], dl[4];
    load_vec4(p.s_o + h * 128, lane, so);
    load_vec4(p.delta_o + h * 128, lane, dl);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __fdiv_rn(__fsub_rn(v[i], dl[i]), so[i]);
  }
}

// grid (H, ceil(M / 8)), 8 warps: warp w takes token blockIdx.y * 8 + w of head blockIdx.x,
// for q, k and v in turn; stats index (which * M + m) * H + h.
__global__ void __launch_bounds__(256) attn_prep_kernel(AttnPrepParams p) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int h = blockIdx.x;
  const int64_t m = static_cast<int64_t>(blockIdx.y) * 8 + w;
  if (m >= p.M) return;
  const int64_t D = p.D;
  for (int which = 0; which < 3; ++which) {
    float v[4], rot[4];
    head_forward(p, which, m, h, lane, v, rot);
    if (p.quantized) {
      const RowQ r = row_quant(v, p.Qa);
      row_dequant(v, r.q, p.Qa);
      if (lane == 0) {
        const int64_t si = (which * p.M + m) * p.H + h;
        p.h_s[si] = r.q.h;
        p.z_s[si] = z_to_i32(r.q.z);
        p.range_s[si] = r.rg;
      }
    }
    store_head4(p.out, m * 3 * D + which * D + h * 128, lane, v, p.dt16 == OMQ_F16);
  }
}

// Backward of attn_prep: per (token, head) row, the quantizer's STE, then the transforms'
// transposes: dq = RoPE^T(dq~ / s_a), dk = RoPE^T(dk~ s_a), dv = dv~ / s_o; and the column
// partials of the LET gradients over the block's tokens:
//   part_sa[rb, c] = sum_m dk~ k_r - dq~ q~ / s_a
//   part_so[rb, c] = -sum_m dv~ v~ / s_o,  part_do[rb, c] = -sum_m dv~ / s_o
// grid (H, ceil(M / kAttnRows)); warp w takes tokens w, w + 8, ... of the block; the 8 warps'
// sums are added in warp order.
__global__ void __launch_bounds__(256) attn_prep_bwd_kernel(AttnPrepParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float red[3][8][128];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int h = blockIdx.x;
  const int64_t D = p.D;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kAttnRows;
  const int64_t r1 = min(p.M, r0 + kAttnRows);
  float sa[4] = {1.f, 1.f, 1.f, 1.f}, so[4] = {1.f, 1.f, 1.f, 1.f};
  if (p.s_a) load_vec4(p.s_a + h * 128, lane, sa);
  if (p.s_o) load_vec4(p.s_o + h * 128, lane, so);
  float acc_sa[4] = {}, acc_so[4] = {}, acc_do[4] = {};
  for (int64_t m = r0 + w; m < r1; m += 8) {
    const float2 c = *reinterpret_cast<const float2*>(p.cos_t + m * 64 + 2 * lane);
    const float2 s = *reinterpret_cast<const float2*>(p.sin_t + m * 64 + 2 * lane);
    for (int which = 0; which < 3; ++which) {
      float v[4], rot[4], d[4];
      head_forward(p, which, m, h, lane, v, rot);
      load_head4(p.dq + m * 3 * D + which * D + h * 128, lane, d);
      if (p.quantized) {
        const int64_t si = (which * p.M + m) * p.H + h;
        row_ste(v, d, p.h_s[si], static_cast<float>(p.z_s[si]), p.range_s[si], p.Qa);
      }
      if (which == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc_sa[i] -= d[i] * v[i] / sa[i];
          d[i] = d[i] / sa[i];
        }
        rope4_t(d, c, s);
      } else if (which == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc_sa[i] += d[i] * rot[i];
          d[i] = d[i] * sa[i];
        }
        rope4_t(d, c, s);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float q = d[i] / so[i];
          acc_so[i] -= q * v[i];
          acc_do[i] -= q;
          d[i] = q;
        }
      }
      store_head4(p.dout, m * 3 * D + which * D + h * 128, lane, d, p.dt16 == OMQ_F16);
    }
  }
  if (!p.part_sa) return;
  const int cols[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    red[0][w][cols[i]] = acc_sa[i];
    red[1][w][cols[i]] = acc_so[i];
    red[2][w][cols[i]] = acc_do[i];
  }
  __syncthreads();
  if (threadIdx.x < 128) {
    float a = 0.f, b = 0.f, e = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a += red[0][q][threadIdx.x];
      b += red[1][q][threadIdx.x];
      e += red[2][q][threadIdx.x];
    }
    const int64_t o = static_cast<int64_t>(blockIdx.y) * D + h * 128 + threadIdx.x;
    p.part_sa[o] = a;
    p.part_so[o] = b;
    p.part_do[o] = e;
  }
}

// ------------------------------------------------------------------ causal softmax
// Rows r of [H, M, M] (query i = r mod M): P[r, j] = exp(S - max) / sum over j <= i, in place
// (float32, written for the 4-column chunks holding j <= i) and as BF16 (the operand of the
// causal P V and P^T dO products, written up to the end of the row's 256-column GEMM tile,
// zero past the diagonal: the products read no further). S is read only at j <= i: the score
// GEMM skips tiles above the diagonal. One warp per row, 4 columns a lane per step; the row
// is read twice (the second read is served by L2).
__device__ __forceinline__ int64_t causal_span(int64_t i, int64_t M) {
  const int64_t e = (i / kCausalTile + 1) * kCausalTile;
  return e < M ? e : M;
}

__global__ void __launch_bounds__(256) softmax_kernel(float* S, uint16_t* P16, bool f16,
                                                      int64_t rows, int64_t M) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int64_t i = r % M;
  float* row = S + r * M;
  uint16_t* row16 = P16 + r * M;
  const int64_t nvalid = i + 1;
  float mx = -FLT_MAX;
  for (int64_t q = lane; q * 4 < nvalid; q += 32) {
    const float4 v = *reinterpret_cast<const float4*>(row + q * 4);
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (q * 4 + t < nvalid) mx = fmaxf(mx, e[t]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int64_t q = lane; q * 4 < nvalid; q += 32) {
    const float4 v = *reinterpret_cast<const float4*>(row + q * 4);
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (q * 4 + t < nvalid) sum += expf(e[t] - mx);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  const int64_t nq = causal_span(i, M) / 4;
  for (int64_t q = lane; q < nq; q += 32) {
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    if (q * 4 < nvalid) {
      const float4 v = *reinterpret_cast<const float4*>(row + q * 4);
      const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) e[t] = q * 4 + t < nvalid ? expf(x[t] - mx) * inv : 0.f;
      *reinterpret_cast<float4*>(row + q * 4) = make_float4(e[0], e[1], e[2], e[3]);
    }
    *reinterpret_cast<uint2*>(row16 + q * 4) =
        make_uint2(pack2(e[0], e[1], f16), pack2(e[2], e[3], f16));
  }
}

// dS[r, j] = scale P (dP - sum_j' P dP) for j <= i, zero above the diagonal up to the end of
// the row's 256-column tile (BF16; the causal dS Qk and dS^T Qq products read no further).
// P and dP are read only at j <= i.
__global__ void __launch_bounds__(256) softmax_bwd_kernel(const float* P, const float* dP,
                                                          uint16_t* dS, bool f16, int64_t rows,
                                                          int64_t M, float scale) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int64_t i = r % M;
  const float* prow = P + r * M;
  const float* drow = dP + r * M;
  uint16_t* orow = dS + r * M;
  const int64_t nvalid = i + 1;
  const int64_t nq = causal_span(i, M) / 4;
  float dot = 0.f;
  for (int64_t q = lane; q * 4 < nvalid; q += 32) {
    const float4 a = *reinterpret_cast<const float4*>(prow + q * 4);
    const float4 b = *reinterpret_cast<const float4*>(drow + q * 4);
    const float pa[4] = {a.x, a.y, a.z, a.w}, pb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (q * 4 + t < nvalid) dot += pa[t] * pb[t];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  for (int64_t q = lane; q < nq; q += 32) {
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    if (q * 4 < nvalid) {
      const float4 a = *reinterpret_cast<const float4*>(prow + q * 4);
      const float4 b = *reinterpret_cast<const float4*>(drow + q * 4);
      const float pa[4] = {a.x, a.y, a.z, a.w}, pb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) e[t] = q * 4 + t < nvalid ? scale * pa[t] * (pb[t] - dot) : 0.f;
    }
    *reinterpret_cast<uint2*>(orow + q * 4) =
        make_uint2(pack2(e[0], e[1], f16), pack2(e[2], e[3], f16));
  }
}

// ------------------------------------------------------------------ SwiGLU
// m[t, j] = SiLU(gu[t, j]) gu[t, I + j] (float32), 8 columns a thread.
__global__ void __launch_bounds__(256) swiglu_kernel(const float* gu, float* mid, int64_t M,
                                                     int64_t I) {
  pdl_wait();
  pdl_launch();
  const int64_t per_row = I / 8, total = M * per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = t / per_row, c = (t % per_row) * 8;
    float g[8], u[8], o[8];
    load_f8(gu, m * 2 * I + c, g);
    load_f8(gu, m * 2 * I + I + c, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = g[i] / (1.f + expf(-g[i])) * u[i];
    store8(mid, m * I + c, OMQ_F32, o);
  }
}

// d gate = dm up sigma(g) (1 + g (1 - sigma(g))), d up = dm SiLU(g)  ->  16-bit [M, 2I].
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const float* gu, const float* dmid,
                                                         void* dgu, omq_dtype dt16, int64_t M,
                                                         int64_t I) {
  pdl_wait();
  pdl_launch();
  const int64_t per_row = I / 8, total = M * per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = t / per_row, c = (t % per_row) * 8;
    float g[8], u[8], dm[8], dg[8], du[8];
    load_f8(gu, m * 2 * I + c, g);
    load_f8(gu, m * 2 * I + I + c, u);
    load_f8(dmid, m * I + c, dm);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float sg = 1.f / (1.f + expf(-g[i]));
      dg[i] = dm[i] * u[i] * sg * (1.f + g[i] * (1.f - sg));
      du[i] = dm[i] * g[i] * sg;
    }
    store8(dgu, m * 2 * I + c, dt16, dg);
    store8(dgu, m * 2 * I + I + c, dt16, du);
  }
}

// ------------------------------------------------------------------ launchers
static unsigned grid_for(int64_t work, int64_t per_block, int cap_per_sm) {
  const int64_t want = ceil_div(work, per_block);
  const int64_t cap = static_cast<int64_t>(num_sms()) * cap_per_sm;
  return static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap);
}

omq_status launch_rope_table(int64_t M, double base, float* cos_t, float* sin_t,
                             cudaStream_t st) {
  launch_k(rope_table_kernel, grid_for(M * 64, 256, 8), 256, 0, st, M, 64, base, cos_t, sin_t);
  return launch_status();
}

omq_status launch_rms(const RmsParams& p, cudaStream_t st) {
  launch_k(rms_kernel, grid_for(p.M, 1, 16), 256, 0, st, p);
  return launch_status();
}

omq_status launch_rms_bwd(const RmsBwdParams& p, cudaStream_t st) {
  launch_k(rms_bwd_kernel, grid_for(p.M, 1, 16), 256, 0, st, p);
  return launch_status();
}

omq_status launch_attn_prep(const AttnPrepParams& p, bool backward, cudaStream_t st) {
  if (backward) {
    const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(ceil_div(p.M, kAttnRows)));
    launch_k(attn_prep_bwd_kernel, grid, 256, 0, st, p);
  } else {
    const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(ceil_div(p.M, 8)));
    launch_k(attn_prep_kernel, grid, 256, 0, st, p);
  }
  return launch_status();
}

omq_status launch_softmax(float* S, void* P16, omq_dtype dt16, int64_t rows, int64_t M,
                          cudaStream_t st) {
  launch_k(softmax_kernel, static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, st, S,
      static_cast<uint16_t*>(P16), dt16 == OMQ_F16, rows, M);
  return launch_status();
}

omq_status launch_softmax_bwd(const float* P, const float* dP, void* dS, omq_dtype dt16,
                              int64_t rows, int64_t M, float scale, cudaStream_t st) {
  launch_k(softmax_bwd_kernel, static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, st,
      P, dP, static_cast<uint16_t*>(dS), dt16 == OMQ_F16, rows, M, scale);
  return launch_status();
}

omq_status launch_swiglu(const float* gu, float* mid, int64_t M, int64_t I, cudaStream_t st) {
  launch_k(swiglu_kernel, grid_for(M * I / 8, 256, 8), 256, 0, st, gu, mid, M, I);
  return launch_status();
}

omq_status launch_swiglu_bwd(const float* gu, const float* dmid, void* dgu, omq_dtype dt16,
                             int64_t M, int64_t I, cudaStream_t st) {
  launch_k(swiglu_bwd_kernel, grid_for(M * I / 8, 256, 8), 256, 0, st, gu, dmid, dgu, dt16, M, I);
  return launch_status();
}

__global__ void __launch_bounds__(256) scale_kernel(float* x, int64_t n, float s) {
  pdl_wait();
  pdl_launch();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    x[i] *= s;
}

omq_status launch_scale(float* x, int64_t n, float s, cudaStream_t st) {
  if (n <= 0) return OMQ_OK;
  launch_k(scale_kernel, grid_for(n, 256, 4), 256, 0, st, x, n, s);
  return launch_status();
}

}  // namespace omq
