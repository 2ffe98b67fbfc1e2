// Straight-through backward of the fake-quantizers and the LET gradient reductions.
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
// section 2.2.)
//
// LET gradients are column sums over rows; every kernel writes per-(row block, column)
// partial sums which reduce_cols_kernel adds in a fixed order, so results are bitwise
// reproducible (no floating-point atomics).
#include "omq_internal.cuh"

namespace omq {

struct GroupGrad {
  float dM, dm;       // gradient reaching the range endpoints (before the tie split)
  float dg, db;       // gradient of the strengths
};

__device__ __forceinline__ GroupGrad group_grad(float Gh, float Gz, float g, float b, float h,
                                                float vmax, float vmin, float Q, bool active) {
  const float t = b * vmin / h;
  const float dh = active ? Gh + Gz * t / h : 0.f;
  GroupGrad r;
  r.dg = dh * vmax / Q;
  r.db = -dh * vmin / Q - Gz * vmin / h;
  r.dM = dh * g / Q;
  r.dm = -dh * b / Q - Gz * b / h;
  return r;
}

// Per-element STE pieces for 8 values: in-range mask and the G_h / G_z contributions.
__device__ __forceinline__ void ste8(const float (&v)[8], const float (&dq)[8], float h,
                                     float z, float Q, bool (&inr)[8], float& Gh, float& Gz) {
  const float hinv = __frcp_rn(h);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float r = round_quotient(v[i], h, hinv);
    const float lvl = __fadd_rn(r, z);
    inr[i] = lvl >= 0.f && lvl <= Q;
    const float c = fminf(fmaxf(lvl, 0.f), Q);
    const float u = v[i] * hinv;
    Gh += dq[i] * (inr[i] ? (r - u) : (c - z));
    Gz += inr[i] ? 0.f : -dq[i] * h;
  }
}

__device__ __forceinline__ void load_f8(const float* p, int64_t off, float (&v)[8]) {
  const float4* q = reinterpret_cast<const float4*>(p + off);
  const float4 a = q[0], b = q[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ------------------------------------------------------------------ weight side, G <= 256
// grid (n_groups, row blocks); a sub-warp of G/8 lanes walks the rows of its block.
template <int LPG>
__global__ void __launch_bounds__(256) ste_w_small_kernel(SteWParams p) {
  constexpr int SPW = 32 / LPG;
  constexpr int NSUB = 8 * SPW;
  __shared__ float red_s[NSUB * LPG * 8];
  __shared__ float red_d[NSUB * LPG * 8];
  const int lane = threadIdx.x & 31;
  const int sw = (threadIdx.x >> 5) * SPW + lane / LPG;
  const int lig = lane % LPG;
  const int64_t j = blockIdx.x;
  const int64_t rb = blockIdx.y;
  const int64_t r0 = rb * p.rows_per_block;
  const int64_t r1 = min(p.N, r0 + p.rows_per_block);
  const int64_t col = j * p.G + lig * 8;
  float acc_s[8] = {}, acc_d[8] = {};
  float sv[8];
  if (p.s) load_f8(p.s, col, sv);
  // rows are visited in lockstep by all sub-warps of a warp (shuffles need full warps)
  for (int64_t nb = r0; nb < r1; nb += NSUB) {
    const int64_t n = nb + sw;
    const bool valid = n < r1;
    const int64_t gi = (valid ? n : r0) * p.ng + j;
    const int64_t off = (valid ? n : r0) * p.K + col;
    float w[8], wt[8], dq[8];
    load8(p.W, off, p.wdt, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) wt[i] = p.s ? __fmul_rn(w[i], sv[i]) : w[i];
    load_f8(p.dWhat, off, dq);
    const float h = p.h[gi];
    const float z = static_cast<float>(p.z[gi]);
    const omq_range rg = p.range[gi];
    bool inr[8];
    float Gh = 0.f, Gz = 0.f;
    ste8(wt, dq, h, z, p.Q, inr, Gh, Gz);
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) {
      Gh += __shfl_xor_sync(0xffffffffu, Gh, o);
      Gz += __shfl_xor_sync(0xffffffffu, Gz, o);
    }
    if (!valid) continue;
    const float g = strength(p.gl[gi]), b = strength(p.bl[gi]);
    const bool active = group_params(g, b, rg.vmax, rg.vmin, p.Q).active;
    const GroupGrad gg = group_grad(Gh, Gz, g, b, h, rg.vmax, rg.vmin, p.Q, active);
    if (lig == 0) {
      if (p.d_gl) p.d_gl[gi] = gg.dg * g * (1.f - g);
      if (p.d_bl) p.d_bl[gi] = gg.db * b * (1.f - b);
    }
    if (p.part_s) {
      const float eM = gg.dM / static_cast<float>(rg.nmax), em = gg.dm / static_cast<float>(rg.nmin);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float dwt = inr[i] ? dq[i] : 0.f;
        if (wt[i] == rg.vmax) dwt += eM;
        if (wt[i] == rg.vmin) dwt += em;
        acc_s[i] += dwt * w[i];
      }
    }
    if (p.part_d) {
      const float db_n = p.dBt[n];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc_d[i] += db_n * w[i];
    }
  }
  if (!p.part_s && !p.part_d) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red_s[sw * LPG * 8 + lig * 8 + i] = acc_s[i];
    red_d[sw * LPG * 8 + lig * 8 + i] = acc_d[i];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < LPG * 8; c += blockDim.x) {
    float a = 0.f, d = 0.f;
    for (int q = 0; q < NSUB; ++q) {
      a += red_s[q * LPG * 8 + c];
      d += red_d[q * LPG * 8 + c];
    }
    if (p.part_s) p.part_s[rb * p.K + j * p.G + c] = a;
    if (p.part_d) p.part_d[rb * p.K + j * p.G + c] = d;
  }
}

// Block-wide sum of two floats (fixed combination order); every thread gets the result.
__device__ __forceinline__ void block_sum2(float& a, float& b, float* sm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  __syncthreads();
  if (lane == 0) { sm[w] = a; sm[32 + w] = b; }
  __syncthreads();
  a = 0.f;
  b = 0.f;
  for (int i = 0; i < nw; ++i) { a += sm[i]; b += sm[32 + i]; }
}

// ------------------------------------------------------------------ weight side, G > 256
// grid (n_groups, row blocks); the block's 256 threads cover the group's columns in chunks
// of 8; column partial sums live in shared memory (each column owned by one thread).
__global__ void __launch_bounds__(256) ste_w_large_kernel(SteWParams p) {
  extern __shared__ float acc[];   // 2 * G floats
  __shared__ float sm[64];
  float* acc_s = acc;
  float* acc_d = acc + p.G;
  const int64_t j = blockIdx.x, rb = blockIdx.y;
  const int64_t r0 = rb * p.rows_per_block, r1 = min(p.N, r0 + p.rows_per_block);
  const int chunks = static_cast<int>(p.G / 8);
  for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
    for (int i = 0; i < 8; ++i) { acc_s[c * 8 + i] = 0.f; acc_d[c * 8 + i] = 0.f; }
  for (int64_t n = r0; n < r1; ++n) {
    const int64_t gi = n * p.ng + j;
    const float h = p.h[gi];
    const float z = static_cast<float>(p.z[gi]);
    const omq_range rg = p.range[gi];
    const int64_t base = n * p.K + j * p.G;
    float Gh = 0.f, Gz = 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float w[8], dq[8];
      load8(p.W, base + c * 8, p.wdt, w);
      if (p.s) {
        float sv[8];
        load_f8(p.s, j * p.G + c * 8, sv);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(w[i], sv[i]);
      }
      load_f8(p.dWhat, base + c * 8, dq);
      bool inr[8];
      ste8(w, dq, h, z, p.Q, inr, Gh, Gz);
    }
    block_sum2(Gh, Gz, sm);
    const float g = strength(p.gl[gi]), b = strength(p.bl[gi]);
    const bool active = group_params(g, b, rg.vmax, rg.vmin, p.Q).active;
    const GroupGrad gg = group_grad(Gh, Gz, g, b, h, rg.vmax, rg.vmin, p.Q, active);
    if (threadIdx.x == 0) {
      if (p.d_gl) p.d_gl[gi] = gg.dg * g * (1.f - g);
      if (p.d_bl) p.d_bl[gi] = gg.db * b * (1.f - b);
    }
    if (!p.part_s && !p.part_d) continue;
    const float eM = gg.dM / static_cast<float>(rg.nmax), em = gg.dm / static_cast<float>(rg.nmin);
    const float db_n = p.part_d ? p.dBt[n] : 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float w[8], wt[8], dq[8];
      load8(p.W, base + c * 8, p.wdt, w);
      if (p.s) {
        float sv[8];
        load_f8(p.s, j * p.G + c * 8, sv);
#pragma unroll
        for (int i = 0; i < 8; ++i) wt[i] = __fmul_rn(w[i], sv[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) wt[i] = w[i];
      }
      load_f8(p.dWhat, base + c * 8, dq);
      bool inr[8];
      float dummy_h = 0.f, dummy_z = 0.f;
      ste8(wt, dq, h, z, p.Q, inr, dummy_h, dummy_z);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float dwt = inr[i] ? dq[i] : 0.f;
        if (wt[i] == rg.vmax) dwt += eM;
        if (wt[i] == rg.vmin) dwt += em;
        acc_s[c * 8 + i] += dwt * w[i];
        acc_d[c * 8 + i] += db_n * w[i];
      }
    }
  }
  if (!p.part_s && !p.part_d) return;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (p.part_s) p.part_s[rb * p.K + j * p.G + c * 8 + i] = acc_s[c * 8 + i];
      if (p.part_d) p.part_d[rb * p.K + j * p.G + c * 8 + i] = acc_d[c * 8 + i];
    }
}

// ------------------------------------------------------------------ activation side
// grid (row blocks); one group per token row (K columns), g = b = 1, no parameters.
__global__ void __launch_bounds__(256) ste_x_kernel(SteXParams p) {
  extern __shared__ float acc[];   // 2 * K floats
  __shared__ float sm[64];
  float* acc_s = acc;
  float* acc_d = acc + p.K;
  const int64_t rb = blockIdx.x;
  const int64_t r0 = rb * p.rows_per_block, r1 = min(p.M, r0 + p.rows_per_block);
  const int chunks = static_cast<int>(p.K / 8);
  for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
    for (int i = 0; i < 8; ++i) { acc_s[c * 8 + i] = 0.f; acc_d[c * 8 + i] = 0.f; }

  auto xt8 = [&](int64_t off, int64_t col, float (&v)[8], float (&sv)[8]) {
    load8(p.X, off, p.xdt, v);
    float dv[8];
    if (p.s) load_f8(p.s, col, sv); else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sv[i] = 1.f;
    }
    if (p.d) load_f8(p.d, col, dv); else {
#pragma unroll
      for (int i = 0; i < 8; ++i) dv[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(__fsub_rn(v[i], dv[i]), sv[i]);
  };

  for (int64_t m = r0; m < r1; ++m) {
    const int64_t base = m * p.K;
    float eM = 0.f, em = 0.f, h = 1.f, z = 0.f;
    omq_range rg{0.f, 0.f, 1, 1};
    if (p.quantized) {
      h = p.h_a[m];
      z = static_cast<float>(p.z_a[m]);
      rg = p.range[m];
      float Gh = 0.f, Gz = 0.f;
      for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        float v[8], sv[8], dq[8];
        xt8(base + c * 8, c * 8, v, sv);
        load_f8(p.dXq, base + c * 8, dq);
        bool inr[8];
        ste8(v, dq, h, z, p.Qa, inr, Gh, Gz);
      }
      block_sum2(Gh, Gz, sm);
      const bool active = group_params(1.f, 1.f, rg.vmax, rg.vmin, p.Qa).active;
      const GroupGrad gg = group_grad(Gh, Gz, 1.f, 1.f, h, rg.vmax, rg.vmin, p.Qa, active);
      eM = gg.dM / static_cast<float>(rg.nmax);
      em = gg.dm / static_cast<float>(rg.nmin);
    }
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8], sv[8], dq[8];
      xt8(base + c * 8, c * 8, v, sv);
      load_f8(p.dXq, base + c * 8, dq);
      float dxt[8];
      if (p.quantized) {
        bool inr[8];
        float dh = 0.f, dz = 0.f;
        ste8(v, dq, h, z, p.Qa, inr, dh, dz);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dxt[i] = inr[i] ? dq[i] : 0.f;
          if (v[i] == rg.vmax) dxt[i] += eM;
          if (v[i] == rg.vmin) dxt[i] += em;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) dxt[i] = dq[i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float q = dxt[i] / sv[i];
        acc_s[c * 8 + i] -= q * v[i];
        acc_d[c * 8 + i] -= q;
      }
    }
  }
  for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      p.part_s[rb * p.K + c * 8 + i] = acc_s[c * 8 + i];
      p.part_d[rb * p.K + c * 8 + i] = acc_d[c * 8 + i];
    }
}

// ------------------------------------------------------------------ column sums
// part[rb, j] = sum over rows rb*R .. rb*R+R-1 of A[i, j]  (A [rows, cols] in dt)
__global__ void __launch_bounds__(256) colsum_kernel(const void* A, omq_dtype dt, int64_t rows,
                                                     int64_t cols, int R, float* part) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rb = blockIdx.y;
  if (j >= cols) return;
  const int64_t r0 = rb * R, r1 = min(rows, r0 + R);
  float a = 0.f;
  for (int64_t i = r0; i < r1; ++i) a += load_elem(A, i * cols + j, dt);
  part[rb * cols + j] = a;
}

// out[j] = sum_r p0[r, j] (+ sum_r p1[r, j]), binary64 accumulation in row order.
__global__ void __launch_bounds__(256) reduce_cols_kernel(const float* p0, int64_t r0n,
                                                          const float* p1, int64_t r1n,
                                                          int64_t cols, float* out) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= cols) return;
  double a = 0.0;
  for (int64_t r = 0; r < r0n; ++r) a += p0[r * cols + j];
  if (p1)
    for (int64_t r = 0; r < r1n; ++r) a += p1[r * cols + j];
  out[j] = static_cast<float>(a);
}

// loss = (sum of per-tile partials) / count, binary64, fixed order.
__global__ void __launch_bounds__(256) loss_finalize_kernel(const float* part, int64_t n,
                                                            double inv_count, float* loss) {
  __shared__ double sm[256];
  double a = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) a += part[i];
  sm[threadIdx.x] = a;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) sm[threadIdx.x] += sm[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(sm[0] * inv_count);
}

__global__ void __launch_bounds__(256) adamw_kernel(float* p, const float* g, float* m, float* v,
                                                    int64_t n, float lr, float b1, float b2,
                                                    float eps, float wd, float bc1, float bc2_sqrt) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float gi = g[i];
    float pi = p[i] * (1.f - lr * wd);
    const float mi = b1 * m[i] + (1.f - b1) * gi;
    const float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    pi -= (lr / bc1) * mi / (sqrtf(vi) / bc2_sqrt + eps);
    p[i] = pi;
    m[i] = mi;
    v[i] = vi;
  }
}

// ------------------------------------------------------------------ launchers

omq_status launch_ste_w(const SteWParams& p, cudaStream_t stream) {
  const int64_t rbs = ceil_div(p.N, p.rows_per_block);
  dim3 grid(static_cast<unsigned>(p.ng), static_cast<unsigned>(rbs));
  if (p.G <= 256 && (p.G & (p.G - 1)) == 0) {
    switch (p.G / 8) {
      case 1: ste_w_small_kernel<1><<<grid, 256, 0, stream>>>(p); break;
      case 2: ste_w_small_kernel<2><<<grid, 256, 0, stream>>>(p); break;
      case 4: ste_w_small_kernel<4><<<grid, 256, 0, stream>>>(p); break;
      case 8: ste_w_small_kernel<8><<<grid, 256, 0, stream>>>(p); break;
      case 16: ste_w_small_kernel<16><<<grid, 256, 0, stream>>>(p); break;
      default: ste_w_small_kernel<32><<<grid, 256, 0, stream>>>(p); break;
    }
    return launch_status();
  }
  const size_t smem = 2 * static_cast<size_t>(p.G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(ste_w_large_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) { set_cuda_error(e); return OMQ_ERR_CUDA; }
  }
  ste_w_large_kernel<<<grid, 256, smem, stream>>>(p);
  return launch_status();
}

omq_status launch_ste_x(const SteXParams& p, cudaStream_t stream) {
  const int64_t rbs = ceil_div(p.M, p.rows_per_block);
  const size_t smem = 2 * static_cast<size_t>(p.K) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(ste_x_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) { set_cuda_error(e); return OMQ_ERR_CUDA; }
  }
  ste_x_kernel<<<static_cast<unsigned>(rbs), 256, smem, stream>>>(p);
  return launch_status();
}

omq_status launch_colsum(const void* A, omq_dtype dt, int64_t rows, int64_t cols, int R,
                         float* part, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(ceil_div(cols, 256)), static_cast<unsigned>(ceil_div(rows, R)));
  colsum_kernel<<<grid, 256, 0, stream>>>(A, dt, rows, cols, R, part);
  return launch_status();
}

omq_status launch_reduce_cols(const float* p0, int64_t r0n, const float* p1, int64_t r1n,
                              int64_t cols, float* out, cudaStream_t stream) {
  reduce_cols_kernel<<<static_cast<unsigned>(ceil_div(cols, 256)), 256, 0, stream>>>(
      p0, r0n, p1, r1n, cols, out);
  return launch_status();
}

omq_status launch_loss_finalize(const float* part, int64_t n, double inv_count, float* loss,
                                cudaStream_t stream) {
  loss_finalize_kernel<<<1, 256, 0, stream>>>(part, n, inv_count, loss);
  return launch_status();
}

omq_status launch_adamw(float* p, const float* g, float* m, float* v, int64_t n, float lr,
                        float b1, float b2, float eps, float wd, int64_t step,
                        cudaStream_t stream) {
  const double bc1 = 1.0 - std::pow(static_cast<double>(b1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(b2), static_cast<double>(step));
  const int64_t want = ceil_div(n, 256);
  const int sms = num_sms();
  const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  adamw_kernel<<<grid > 0 ? grid : 1, 256, 0, stream>>>(p, g, m, v, n, lr, b1, b2, eps, wd,
                                                        static_cast<float>(bc1),
                                                        static_cast<float>(std::sqrt(bc2)));
  return launch_status();
}

}  // namespace omq
