// Straight-through backward of the fake-quantizers and the LET gradient reductions.
//
// The per-group STE arithmetic (dq/dv, dq/dh, dq/dz and the chain to g, b and the range)
// is in ste_common.cuh.
//
// The in-range / clipped decisions repeat the forward's binary32 arithmetic exactly; the
// gradient values use a fast binary32 sigmoid for g and b. LET gradients are column sums
// over rows: kernels write per-(row block, column) partial sums that reduce_cols_kernel adds
// in a fixed order, so results are bitwise reproducible (no floating-point atomics). The
// memory-bound kernels issue the loads of several rows before computing on any of them.
#include <algorithm>

#include "ste_common.cuh"

namespace omq {

// ------------------------------------------------------------------ weight side, G <= 256
// grid (256-column segments, row blocks); a warp covers one row of the segment (lane = 8
// columns; G/8 lanes per group), the 8 warps take every 8th row, U rows per iteration. A
// lane's columns (and so its column partial sums) stay fixed; the warps' partials are added
// in shared memory in warp order at the end.
template <int LPG, int U>
__global__ void __launch_bounds__(256, 2) ste_w_small_kernel(SteWParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float red_s[8][256];
  __shared__ float red_d[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int lig = lane % LPG;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  const bool cvalid = c0 < p.K;
  const int64_t j = c0 / (LPG * 8);
  const int64_t rb = blockIdx.y;
  const int64_t r0 = rb * p.rows_per_block;
  const int64_t r1 = min(p.N, r0 + p.rows_per_block);
  float acc_s[8] = {}, acc_d[8] = {};
  float sv[8];
  if (p.s && cvalid) {
    load_f8(p.s, c0, sv);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = 1.f;
  }
  for (int64_t nb = r0 + w; nb < r1; nb += 8 * U) {
    float wv[U][8], dq[U][8], h[U], z[U], glv[U], blv[U];
    omq_range rg[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t n = nb + 8 * u;
      if (n < r1 && cvalid) {
        const int64_t gi = n * p.ng + j;
        load8(p.W, n * p.K + c0, p.wdt, wv[u]);
        load_f8(p.dWhat, n * p.K + c0, dq[u]);
        h[u] = p.h[gi];
        z[u] = static_cast<float>(p.z[gi]);
        rg[u] = p.range[gi];
        glv[u] = p.gl[gi];
        blv[u] = p.bl[gi];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { wv[u][i] = 0.f; dq[u][i] = 0.f; }
        h[u] = 1.f;
        z[u] = 0.f;
        rg[u] = omq_range{0.f, 0.f, 1, 1};
        glv[u] = 0.f;
        blv[u] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t n = nb + 8 * u;
      float wt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) wt[i] = p.s ? __fmul_rn(wv[u][i], sv[i]) : wv[u][i];
      bool inr[8];
      float Gh = 0.f, Gz = 0.f;
      ste8(wt, dq[u], h[u], z[u], p.Q, inr, Gh, Gz);
#pragma unroll
      for (int o = LPG / 2; o > 0; o >>= 1) {
        Gh += __shfl_xor_sync(0xffffffffu, Gh, o);
        Gz += __shfl_xor_sync(0xffffffffu, Gz, o);
      }
      if (n >= r1 || !cvalid) continue;
      const float g = strength_value(glv[u]), b = strength_value(blv[u]);
      const bool active = h_active(h[u], glv[u], blv[u], rg[u].vmax, rg[u].vmin, p.Q);
      const GroupGrad gg = group_grad(Gh, Gz, g, b, h[u], rg[u].vmax, rg[u].vmin, p.Q, active);
      if (lig == 0) {
        const int64_t gi = n * p.ng + j;
        if (p.d_gl) p.d_gl[gi] = gg.dg * g * (1.f - g);
        if (p.d_bl) p.d_bl[gi] = gg.db * b * (1.f - b);
      }
      if (p.part_s) {
        const float eM = gg.dM / static_cast<float>(rg[u].nmax);
        const float em = gg.dm / static_cast<float>(rg[u].nmin);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float dwt = inr[i] ? dq[u][i] : 0.f;
          if (wt[i] == rg[u].vmax) dwt += eM;
          if (wt[i] == rg[u].vmin) dwt += em;
          acc_s[i] += dwt * wv[u][i];
        }
      }
      if (p.part_d) {
        const float db_n = p.dBt[n];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc_d[i] += db_n * wv[u][i];
      }
    }
  }
  if (!p.part_s && !p.part_d) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red_s[w][lane * 8 + i] = acc_s[i];
    red_d[w][lane * 8 + i] = acc_d[i];
  }
  __syncthreads();
  const int64_t col = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (col < p.K) {
    float a = 0.f, d = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a += red_s[q][threadIdx.x];
      d += red_d[q][threadIdx.x];
    }
    if (p.part_s) p.part_s[rb * p.K + col] = a;
    if (p.part_d) p.part_d[rb * p.K + col] = d;
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
  pdl_wait();
  pdl_launch();
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
    const float glv = p.gl[gi], blv = p.bl[gi];
    const float g = strength_value(glv), b = strength_value(blv);
    const bool active = h_active(h, glv, blv, rg.vmax, rg.vmin, p.Q);
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
      in_range8(wt, h, z, p.Q, inr);
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

// ------------------------------------------------------------------ fused weight side
constexpr int kFinishJ = 8;   // groups per tile of ste_w_finish_kernel (32 rows a tile)
// Completion of the STE that the dW^ GEMM's epilogue started. Grid (32-row tiles, kFinishJ-
// group tile strides), 256 threads; a tile of 32 rows x kFinishJ groups is read in two
// mappings so both layouts stay coalesced: the chunk partials ([K/32, N]) with the row
// fastest, staged in shared memory, then the per-group arrays ([N, ng]) with the group
// fastest. A group's
// chunk partials are added in chunk order (groups of up to 8 chunks) or as 8 interleaved
// partial sums added in a fixed order (longer groups).
__global__ void __launch_bounds__(256) ste_w_finish_kernel(SteWFinish p) {
  pdl_wait();
  pdl_launch();
  __shared__ float sgh[kFinishJ][33], sgc[kFinishJ][33];   // [group in tile][row in tile]
  __shared__ float wred[2][8][32];
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t cpg = p.G / 32;
  for (int64_t j0 = static_cast<int64_t>(blockIdx.y) * kFinishJ; j0 < p.ng;
       j0 += kFinishJ * gridDim.y) {
    if (cpg <= 8) {
      for (int e = threadIdx.x; e < 32 * kFinishJ; e += blockDim.x) {
        const int nl = e & 31, jl = e >> 5;
        const int64_t n = n0 + nl, j = j0 + jl;
        float Gh = 0.f, Gc = 0.f;
        if (n < p.N && j < p.ng)
#pragma unroll 8
          for (int64_t c = j * cpg; c < (j + 1) * cpg; ++c) {
            Gh += p.gh_part[c * p.N + n];
            Gc += p.gc_part[c * p.N + n];
          }
        sgh[jl][nl] = Gh;
        sgc[jl][nl] = Gc;
      }
    } else {
      // long groups (per-channel ones included): the 8 warps take every 8th chunk of a group
      // (lane = row), then warp 0 adds the 8 partial sums in warp order
      const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
      const int64_t n = n0 + lane;
      for (int jl = 0; jl < kFinishJ; ++jl) {
        const int64_t j = j0 + jl;
        float Gh = 0.f, Gc = 0.f;
        if (n < p.N && j < p.ng)
#pragma unroll 4
          for (int64_t c = j * cpg + w; c < (j + 1) * cpg; c += 8) {
            Gh += p.gh_part[c * p.N + n];
            Gc += p.gc_part[c * p.N + n];
          }
        wred[0][w][lane] = Gh;
        wred[1][w][lane] = Gc;
        __syncthreads();
        if (w == 0) {
          float a = 0.f, b = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            a += wred[0][q][lane];
            b += wred[1][q][lane];
          }
          sgh[jl][lane] = a;
          sgc[jl][lane] = b;
        }
        __syncthreads();
        if (j0 + jl + 1 >= p.ng) break;   // uniform
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * kFinishJ; e += blockDim.x) {
      const int jl = e % kFinishJ, nl = e / kFinishJ;
      const int64_t n = n0 + nl, j = j0 + jl;
      if (n >= p.N || j >= p.ng) continue;
      const int64_t gi = n * p.ng + j;
      const float h = p.h[gi];
      const float Gh = sgh[jl][nl];
      const float Gz = -h * sgc[jl][nl];
      const omq_range rg = p.range[gi];
      const float glv = p.gl[gi], blv = p.bl[gi];
      const float g = strength_value(glv), b = strength_value(blv);
      const bool active = h_active(h, glv, blv, rg.vmax, rg.vmin, p.Q);
      const GroupGrad gg = group_grad(Gh, Gz, g, b, h, rg.vmax, rg.vmin, p.Q, active);
      if (p.d_gl) p.d_gl[gi] = gg.dg * g * (1.f - g);
      if (p.d_bl) p.d_bl[gi] = gg.db * b * (1.f - b);
      if (p.emax) {
        p.emax[gi] = gg.dM / static_cast<float>(rg.nmax);
        p.emin[gi] = gg.dm / static_cast<float>(rg.nmin);
      }
    }
    __syncthreads();   // the tiles are rewritten for the next group stride
  }
}

// The W-side LET terms that the epilogue leaves out, in one pass over W. One warp per task
// (32-row block, 256-column segment), persistent warps; lane = 8 columns (one group), the
// block's 32 rows walked in order, eight row loads in flight before any is used:
//   part_s[rb, k] += sum_n (emax W[n,k] where W~[n,k] is its group's max, emin W[n,k] where
//                    it is the min)                       (the clipping-range terms of d s)
//   part_d[rb, k]  = sum_n dBt[n] W[n,k]                  (the bias term of d delta)
__global__ void __launch_bounds__(256, 2) ste_w_corr_kernel(SteWCorr p) {
  pdl_wait();
  pdl_launch();
  constexpr int U = 8;
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t segs = (p.K + 255) / 256, rbs = (p.N + 31) / 32;
  const int64_t ng = p.K / p.G;
  const bool f16 = p.wdt == OMQ_F16;
  for (int64_t task = warp_g; task < segs * rbs; task += n_warps) {
    const int64_t rb = task / segs, seg = task - rb * segs;
    const int64_t c0 = seg * 256 + lane * 8;
    const bool cvalid = c0 < p.K;
    const int64_t j = cvalid ? c0 / p.G : 0;
    const uint4* wcol = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.W) + c0);
    const int64_t wstride = p.K / 8;                 // uint4 per row
    float acc_s[8] = {}, acc_d[8] = {};
    for (int r = 0; r < 32; r += U) {
      // every load of the U rows (weights as packed 16-bit, the groups' records) before use
      uint4 raw[U];
      float2 mm[U];
      float eM[U], em[U], db[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t n = rb * 32 + r + u;
        const bool ok = n < p.N && cvalid;
        raw[u] = ok ? __ldg(wcol + n * wstride) : make_uint4(0, 0, 0, 0);
        const int64_t gi = ok ? n * ng + j : 0;
        mm[u] = make_float2(0.f, 0.f);
        eM[u] = em[u] = db[u] = 0.f;
        if (ok && p.part_s) {
          mm[u] = *reinterpret_cast<const float2*>(p.range + gi);   // vmax, vmin
          eM[u] = p.emax[gi];
          em[u] = p.emin[gi];
        }
        if (ok && p.part_d) db[u] = p.dBt[n];
      }
      float sv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) sv[i] = 1.f;
      if (p.s && cvalid) load_f8(p.s, c0, sv);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float v[8];
        if (f16) {
          const __half2* h2 = reinterpret_cast<const __half2*>(&raw[u]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(h2[q]);
            v[2 * q] = f.x;
            v[2 * q + 1] = f.y;
          }
        } else {
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b2[q]);
            v[2 * q] = f.x;
            v[2 * q + 1] = f.y;
          }
        }
        if (p.part_s) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float wt = p.s ? __fmul_rn(v[i], sv[i]) : v[i];
            if (wt == mm[u].x) acc_s[i] += eM[u] * v[i];
            if (wt == mm[u].y) acc_s[i] += em[u] * v[i];
          }
        }
        if (p.part_d) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc_d[i] += db[u] * v[i];
        }
      }
    }
    if (!cvalid) continue;
    if (p.part_s) {
      float cur[8];
      load_f8(p.part_s, rb * p.K + c0, cur);
#pragma unroll
      for (int i = 0; i < 8; ++i) cur[i] += acc_s[i];
      store8(p.part_s, rb * p.K + c0, OMQ_F32, cur);
    }
    if (p.part_d) store8(p.part_d, rb * p.K + c0, OMQ_F32, acc_d);
  }
}

// ------------------------------------------------------------------ activation side
__device__ __forceinline__ void xtilde8(const SteXParams& p, int64_t off, const float (&sv)[8],
                                        const float (&dv)[8], float (&v)[8]) {
  load8(p.X, off, p.xdt, v);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(__fsub_rn(v[i], dv[i]), sv[i]);
}

__device__ __forceinline__ void let_vectors(const SteXParams& p, int64_t col, float (&sv)[8],
                                            float (&dv)[8]) {
  if (p.s) {
    load_f8(p.s, col, sv);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = 1.f;
  }
  if (p.d) {
    load_f8(p.d, col, dv);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) dv[i] = 0.f;
  }
}

// Per token (quantized activations): the gradient share of the token's max and min elements,
// from the token's G_h and G_z sums (g = b = 1).
__global__ void __launch_bounds__(256) ste_x_rowstat_kernel(SteXParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float sm[64];
  const int chunks = static_cast<int>(p.K / 8);
  for (int64_t m = blockIdx.x; m < p.M; m += gridDim.x) {
    const int64_t base = m * p.K;
    const float h = p.h_a[m];
    const float z = static_cast<float>(p.z_a[m]);
    float Gh = 0.f, Gz = 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float sv[8], dv[8], v[8], dq[8];
      let_vectors(p, c * 8, sv, dv);
      xtilde8(p, base + c * 8, sv, dv, v);
      load_f8(p.dXq, base + c * 8, dq);
      bool inr[8];
      ste8(v, dq, h, z, p.Qa, inr, Gh, Gz);
    }
    block_sum2(Gh, Gz, sm);
    if (threadIdx.x == 0) {
      const omq_range rg = p.range[m];
      const bool active = group_params(1.f, 1.f, rg.vmax, rg.vmin, p.Qa).active;
      const GroupGrad gg = group_grad(Gh, Gz, 1.f, 1.f, h, rg.vmax, rg.vmin, p.Qa, active);
      p.rowstat[2 * m] = gg.dM / static_cast<float>(rg.nmax);
      p.rowstat[2 * m + 1] = gg.dm / static_cast<float>(rg.nmin);
    }
  }
}

// Column partials over row blocks: part_s[rb, k] = -sum_m dX~ X~ / s, part_d[rb, k] =
// -sum_m dX~ / s. grid (column segments of 256, row blocks); each warp covers the segment
// for every 8th row (lane = 8 columns), U rows per iteration.
template <int U>
__global__ void __launch_bounds__(256, 2) ste_x_cols_kernel(SteXParams p) {
  pdl_wait();
  pdl_launch();
  __shared__ float red_s[8][256];
  __shared__ float red_d[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  const bool cvalid = c0 < p.K;
  const int64_t rb = blockIdx.y;
  const int64_t r0 = rb * p.rows_per_block, r1 = min(p.M, r0 + p.rows_per_block);
  float sv[8], dv[8], rs[8];
  let_vectors(p, cvalid ? c0 : 0, sv, dv);
#pragma unroll
  for (int i = 0; i < 8; ++i) rs[i] = 1.f / sv[i];
  float acc_s[8] = {}, acc_d[8] = {};
  for (int64_t mb = r0 + w; mb < r1; mb += 8 * U) {
    float v[U][8], dq[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t m = mb + 8 * u;
      if (m < r1 && cvalid) {
        load8(p.X, m * p.K + c0, p.xdt, v[u]);
        load_f8(p.dXq, m * p.K + c0, dq[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { v[u][i] = 0.f; dq[u][i] = 0.f; }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t m = mb + 8 * u;
      if (m >= r1 || !cvalid) continue;
      float dxt[8];
      if (p.quantized) {
        // the in-range decisions need X~ exactly as the forward computed it
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = __fdiv_rn(__fsub_rn(v[u][i], dv[i]), sv[i]);
        const omq_range rg = p.range[m];
        bool inr[8];
        in_range8(v[u], p.h_a[m], static_cast<float>(p.z_a[m]), p.Qa, inr);
        const float eM = p.rowstat[2 * m], em = p.rowstat[2 * m + 1];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dxt[i] = inr[i] ? dq[u][i] : 0.f;
          if (v[u][i] == rg.vmax) dxt[i] += eM;
          if (v[u][i] == rg.vmin) dxt[i] += em;
        }
      } else {
        // values only: X~ through the reciprocal of s
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[u][i] = (v[u][i] - dv[i]) * rs[i];
          dxt[i] = dq[u][i];
        }
      }
      float dxs[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float q = dxt[i] * rs[i];
        dxs[i] = q;
        acc_s[i] += q * v[u][i];
        acc_d[i] += q;
      }
      if (p.dX) store8(p.dX, m * p.K + c0, p.dx_dt, dxs);
    }
  }
  if (!p.part_s && !p.part_d) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red_s[w][lane * 8 + i] = acc_s[i];
    red_d[w][lane * 8 + i] = acc_d[i];
  }
  __syncthreads();
  const int64_t col = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (col < p.K) {
    float a = 0.f, d = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a += red_s[q][threadIdx.x];
      d += red_d[q][threadIdx.x];
    }
    if (p.part_s) p.part_s[rb * p.K + col] = -a;
    if (p.part_d) p.part_d[rb * p.K + col] = -d;
  }
}

// ------------------------------------------------------------------ column sums
// part[rb, j] = sum of wrow[i] A[i, j] (wrow NULL: A[i, j]) over the rows of row block rb
// (A [rows, cols] in dt, cols % 8 == 0). Same launch shape as ste_x_cols_kernel.
template <int U>
__global__ void __launch_bounds__(256) colsum_kernel(const void* A, omq_dtype dt, int64_t rows,
                                                     int64_t cols, int R, const float* wrow,
                                                     float* part) {
  pdl_wait();
  pdl_launch();
  __shared__ float red[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  const bool cvalid = c0 < cols;
  const int64_t rb = blockIdx.y;
  const int64_t r0 = rb * R, r1 = min(rows, r0 + R);
  float acc[8] = {};
  for (int64_t mb = r0 + w; mb < r1; mb += 8 * U) {
    float v[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t m = mb + 8 * u;
      if (m < r1 && cvalid) {
        load8(A, m * cols + c0, dt, v[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t m = mb + 8 * u;
      const float f = wrow ? (m < r1 ? wrow[m] : 0.f) : 1.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f * v[u][i];
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[w][lane * 8 + i] = acc[i];
  __syncthreads();
  const int64_t col = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (col < cols) {
    float a = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) a += red[q][threadIdx.x];
    part[rb * cols + col] = a;
  }
}

// out[j] = scale * (sum_r p0[r, j] + sum_r p1[r, j]) for up to two such problems (blockIdx.z)
// in two levels, binary64, fixed order. Level 1, grid (32-column blocks, row chunks,
// problems): chunk c takes rows [c rpc, (c + 1) rpc) of p0 followed by p1; its 8 warps take
// every 8th row (lane = column) and are combined in warp order into scratch[problem, c, j],
// or, with a single chunk, straight into out.
struct ColReduceSet {
  ColReduce pr[2];
  int64_t cols, rpc;
  int chunks;
};

__global__ void __launch_bounds__(256) reduce_cols_partial_kernel(ColReduceSet rs,
                                                                  double* scratch) {
  pdl_wait();
  pdl_launch();
  __shared__ double red[8][32];
  const ColReduce& q = rs.pr[blockIdx.z];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  const int64_t r0n = q.r0n, total = q.r0n + (q.p1 ? q.r1n : 0);
  const int64_t ra = static_cast<int64_t>(blockIdx.y) * rs.rpc;
  const int64_t rb = min(total, ra + rs.rpc);
  double a = 0.0;
  if (j < rs.cols) {
#pragma unroll 4
    for (int64_t r = ra + w; r < rb; r += 8)
      a += r < r0n ? q.p0[r * rs.cols + j] : q.p1[(r - r0n) * rs.cols + j];
  }
  red[w][lane] = a;
  __syncthreads();
  if (w == 0 && j < rs.cols) {
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += red[k][lane];
    if (rs.chunks == 1)
      q.out[j] = static_cast<float>(t * static_cast<double>(q.scale));
    else
      scratch[(static_cast<int64_t>(blockIdx.z) * rs.chunks + blockIdx.y) * rs.cols + j] = t;
  }
}

// The same level 1 with four columns a thread (16-byte loads; cols a multiple of 4 and every
// matrix 16-byte aligned): grid (1024-column blocks, row chunks, problems); a thread walks its
// chunk's rows in order, so each column's chunk sum is one fixed-order binary64 sum.
__global__ void __launch_bounds__(256) reduce_cols4_partial_kernel(ColReduceSet rs,
                                                                   double* scratch) {
  pdl_wait();
  pdl_launch();
  const ColReduce& q = rs.pr[blockIdx.z];
  const int64_t j = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  if (j >= rs.cols) return;
  const int64_t r0n = q.r0n, total = q.r0n + (q.p1 ? q.r1n : 0);
  const int64_t ra = static_cast<int64_t>(blockIdx.y) * rs.rpc;
  const int64_t rb = min(total, ra + rs.rpc);
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll 8
  for (int64_t r = ra; r < rb; ++r) {
    const float* row = r < r0n ? q.p0 + r * rs.cols : q.p1 + (r - r0n) * rs.cols;
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + j));
    a0 += v.x;
    a1 += v.y;
    a2 += v.z;
    a3 += v.w;
  }
  if (rs.chunks == 1) {
    const double sc = static_cast<double>(q.scale);
    *reinterpret_cast<float4*>(q.out + j) = make_float4(
        static_cast<float>(a0 * sc), static_cast<float>(a1 * sc), static_cast<float>(a2 * sc),
        static_cast<float>(a3 * sc));
  } else {
    double* o = scratch + (static_cast<int64_t>(blockIdx.z) * rs.chunks + blockIdx.y) * rs.cols + j;
    o[0] = a0;
    o[1] = a1;
    o[2] = a2;
    o[3] = a3;
  }
}

// Level 2, grid (column blocks, problems): out[j] = scale * sum over chunks c (in order).
__global__ void __launch_bounds__(256) reduce_cols_final_kernel(ColReduceSet rs,
                                                                const double* scratch) {
  pdl_wait();
  pdl_launch();
  const ColReduce& q = rs.pr[blockIdx.y];
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= rs.cols) return;
  const double* sc = scratch + static_cast<int64_t>(blockIdx.y) * rs.chunks * rs.cols;
  // four interleaved sums (chunks c = 4 i + r), then (t0 + t1) + (t2 + t3): a fixed order
  // with four loads in flight
  double t[4] = {0.0, 0.0, 0.0, 0.0};
  int c = 0;
  for (; c + 4 <= rs.chunks; c += 4) {
#pragma unroll
    for (int r = 0; r < 4; ++r) t[r] += sc[(c + r) * rs.cols + j];
  }
  for (int r = 0; c < rs.chunks; ++c, ++r) t[r] += sc[c * rs.cols + j];
  const double sum = (t[0] + t[1]) + (t[2] + t[3]);
  q.out[j] = static_cast<float>(sum * static_cast<double>(q.scale));
}

// loss = (sum of per-tile partials) / count, binary64, fixed order.
__global__ void __launch_bounds__(256) loss_finalize_kernel(const float* part, int64_t n,
                                                            double inv_count, float* loss) {
  pdl_wait();
  pdl_launch();
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

struct AdamSegs {
  AdamSeg s[kMaxAdamSegs];
};

// AdamW over up to four parameter tensors in one launch (blockIdx.y selects the tensor).
__global__ void __launch_bounds__(256) adamw_kernel(AdamSegs segs, float b1, float b2, float eps,
                                                    float wd, float bc1, float bc2_sqrt) {
  pdl_wait();
  pdl_launch();
  const AdamSeg sg = segs.s[blockIdx.y];
  const float decay = 1.f - sg.lr * wd, step = sg.lr / bc1;
  auto update = [&](float gi, float& pi, float& mi, float& vi) {
    pi *= decay;
    mi = b1 * mi + (1.f - b1) * gi;
    vi = b2 * vi + (1.f - b2) * gi * gi;
    pi -= step * mi / (sqrtf(vi) / bc2_sqrt + eps);
  };
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // four elements a thread and 16-byte accesses when all four tensors are 16-byte aligned
  // (the same arithmetic per element as the scalar loop, which takes the rest)
  const bool vec = ((reinterpret_cast<uintptr_t>(sg.p) | reinterpret_cast<uintptr_t>(sg.g) |
                     reinterpret_cast<uintptr_t>(sg.m) | reinterpret_cast<uintptr_t>(sg.v)) &
                    15) == 0;
  const int64_t n4 = vec ? sg.n / 4 : 0;
  for (int64_t q = tid; q < n4; q += nthreads) {
    const float4 g4 = reinterpret_cast<const float4*>(sg.g)[q];
    float4 p4 = reinterpret_cast<float4*>(sg.p)[q];
    float4 m4 = reinterpret_cast<float4*>(sg.m)[q];
    float4 v4 = reinterpret_cast<float4*>(sg.v)[q];
    update(g4.x, p4.x, m4.x, v4.x);
    update(g4.y, p4.y, m4.y, v4.y);
    update(g4.z, p4.z, m4.z, v4.z);
    update(g4.w, p4.w, m4.w, v4.w);
    reinterpret_cast<float4*>(sg.p)[q] = p4;
    reinterpret_cast<float4*>(sg.m)[q] = m4;
    reinterpret_cast<float4*>(sg.v)[q] = v4;
  }
  for (int64_t i = 4 * n4 + tid; i < sg.n; i += nthreads) {
    float pi = sg.p[i], mi = sg.m[i], vi = sg.v[i];
    update(sg.g[i], pi, mi, vi);
    sg.p[i] = pi;
    sg.m[i] = mi;
    sg.v[i] = vi;
  }
}

// ------------------------------------------------------------------ launchers

omq_status launch_ste_w(const SteWParams& p, cudaStream_t stream) {
  const int64_t rbs = ceil_div(p.N, p.rows_per_block);
  if (small_group(p.G)) {
    dim3 grid(static_cast<unsigned>(ceil_div(p.K, 256)), static_cast<unsigned>(rbs));
    switch (p.G / 8) {
      case 2: launch_k(ste_w_small_kernel<2, 2>, grid, 256, 0, stream, p); break;
      case 4: launch_k(ste_w_small_kernel<4, 2>, grid, 256, 0, stream, p); break;
      case 8: launch_k(ste_w_small_kernel<8, 2>, grid, 256, 0, stream, p); break;
      case 16: launch_k(ste_w_small_kernel<16, 2>, grid, 256, 0, stream, p); break;
      default: launch_k(ste_w_small_kernel<32, 2>, grid, 256, 0, stream, p); break;
    }
    return launch_status();
  }
  dim3 grid(static_cast<unsigned>(p.ng), static_cast<unsigned>(rbs));
  const size_t smem = 2 * static_cast<size_t>(p.G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(ste_w_large_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) { set_cuda_error(e); return OMQ_ERR_CUDA; }
  }
  launch_k(ste_w_large_kernel, grid, 256, smem, stream, p);
  return launch_status();
}

omq_status launch_ste_w_finish(const SteWFinish& p, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(ceil_div(p.N, 32)),
                  static_cast<unsigned>(std::min<int64_t>(ceil_div(p.ng, kFinishJ), 65535)));
  launch_k(ste_w_finish_kernel, grid, 256, 0, stream, p);
  return launch_status();
}

omq_status launch_ste_w_corr(const SteWCorr& p, cudaStream_t stream) {
  const int64_t tasks = ceil_div(p.K, 256) * ceil_div(p.N, 32);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;    // resident warps
  const int64_t warps = tasks < cap ? tasks : cap;
  launch_k(ste_w_corr_kernel, static_cast<unsigned>(ceil_div(warps, 8)), 256, 0, stream, p);
  return launch_status();
}

omq_status launch_ste_x(const SteXParams& p, cudaStream_t stream) {
  if (p.quantized) {
    const int sms = num_sms();
    const unsigned grid = static_cast<unsigned>(p.M < int64_t(sms) * 8 ? p.M : int64_t(sms) * 8);
    launch_k(ste_x_rowstat_kernel, grid, 256, 0, stream, p);
    const omq_status st = launch_status();
    if (st != OMQ_OK) return st;
  }
  dim3 grid(static_cast<unsigned>(ceil_div(p.K, 256)),
            static_cast<unsigned>(ceil_div(p.M, p.rows_per_block)));
  launch_k(ste_x_cols_kernel<2>, grid, 256, 0, stream, p);
  return launch_status();
}

omq_status launch_colsum(const void* A, omq_dtype dt, int64_t rows, int64_t cols, int R,
                         const float* w, float* part, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(ceil_div(cols, 256)), static_cast<unsigned>(ceil_div(rows, R)));
  launch_k(colsum_kernel<4>, grid, 256, 0, stream, A, dt, rows, cols, R, w, part);
  return launch_status();
}

omq_status launch_reduce_cols(const ColReduce* probs, int nprob, int64_t cols, double* scratch,
                              cudaStream_t stream) {
  if (nprob < 1 || nprob > 2) return OMQ_ERR_SHAPE;
  ColReduceSet rs{};
  int64_t total = 0;
  for (int i = 0; i < nprob; ++i) {
    rs.pr[i] = probs[i];
    const int64_t t = probs[i].r0n + (probs[i].p1 ? probs[i].r1n : 0);
    total = t > total ? t : total;
  }
  rs.cols = cols;
  bool vec = cols % 4 == 0;
  for (int i = 0; i < nprob; ++i)
    vec = vec && aligned16(probs[i].p0) && aligned16(probs[i].out) &&
          (!probs[i].p1 || aligned16(probs[i].p1));
  if (vec) {
    // about two blocks of 1024 columns per SM, each chunk at least 8 rows long
    const int64_t colblocks = ceil_div(cols, 1024);
    const int64_t want = ceil_div(2 * static_cast<int64_t>(num_sms()), colblocks * nprob);
    rs.chunks = static_cast<int>(std::min<int64_t>(
        {kReduceChunks, std::max<int64_t>(1, want), std::max<int64_t>(1, ceil_div(total, 8))}));
    rs.rpc = ceil_div(std::max<int64_t>(total, 1), rs.chunks);
    rs.chunks = static_cast<int>(ceil_div(std::max<int64_t>(total, 1), rs.rpc));
    const dim3 grid(static_cast<unsigned>(colblocks), static_cast<unsigned>(rs.chunks),
                    static_cast<unsigned>(nprob));
    launch_k(reduce_cols4_partial_kernel, grid, 256, 0, stream, rs, scratch);
  } else {
    rs.chunks = static_cast<int>(
        std::min<int64_t>(16, std::max<int64_t>(1, ceil_div(total, 32))));
    rs.rpc = ceil_div(std::max<int64_t>(total, 1), rs.chunks);
    const dim3 grid(static_cast<unsigned>(ceil_div(cols, 32)), static_cast<unsigned>(rs.chunks),
                    static_cast<unsigned>(nprob));
    launch_k(reduce_cols_partial_kernel, grid, 256, 0, stream, rs, scratch);
  }
  const omq_status st = launch_status();
  if (st != OMQ_OK || rs.chunks == 1) return st;
  const dim3 g2(static_cast<unsigned>(ceil_div(cols, 64)), static_cast<unsigned>(nprob));
  launch_k(reduce_cols_final_kernel, g2, 64, 0, stream, rs, scratch);
  return launch_status();
}

omq_status launch_loss_finalize(const float* part, int64_t n, double inv_count, float* loss,
                                cudaStream_t stream) {
  launch_k(loss_finalize_kernel, 1, 256, 0, stream, part, n, inv_count, loss);
  return launch_status();
}

omq_status launch_adamw(const AdamSeg* segs, int nseg, float b1, float b2, float eps, float wd,
                        int64_t step, cudaStream_t stream) {
  if (nseg < 1 || nseg > kMaxAdamSegs) return OMQ_ERR_SHAPE;
  AdamSegs s{};
  int64_t nmax = 0;
  for (int i = 0; i < nseg; ++i) {
    s.s[i] = segs[i];
    nmax = segs[i].n > nmax ? segs[i].n : nmax;
  }
  const double bc1 = 1.0 - std::pow(static_cast<double>(b1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(b2), static_cast<double>(step));
  const int sms = num_sms();
  const int64_t want = ceil_div(nmax, 4 * 256);
  const unsigned gx = static_cast<unsigned>(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  dim3 grid(gx > 0 ? gx : 1, static_cast<unsigned>(nseg));
  launch_k(adamw_kernel, grid, 256, 0, stream,
      s, b1, b2, eps, wd, static_cast<float>(bc1), static_cast<float>(std::sqrt(bc2)));
  return launch_status();
}

}  // namespace omq
