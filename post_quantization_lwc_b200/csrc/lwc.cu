// Learnable Weight Clipping quantizer ("【ICLR 2024】OmniQuant: ...", section LWC), with
// the LET weight scaling W~ = s (.) W folded into the load (section LET), and the fold /
// pack of the final codes.
//
// Per group of G consecutive elements of one row of W~:
//   M = max, m = min, h = (g M - b m)/Q, z = -round(b m / h),
//   code = clamp(round(W~/h) + z, 0, Q),  W^ = (code - z) h
// in the binary32 operation order fixed in omq_internal.cuh.
//
// Two launch shapes, both one HBM pass (read W, write W^ / codes / packed):
//   small groups (G in {8,...,256}): G/8 lanes per group, 8 elements per lane held in
//     registers (one 16-byte load of bf16), max / min / tie counts by xor-shuffles inside
//     the sub-warp; a warp covers 32*8/G groups at once.
//   large groups (G > 256, e.g. one group per row): one 256-thread block per group, the
//     group staged in shared memory as fp32, block reductions.
#include <float.h>

#include "omq_internal.cuh"

namespace omq {

// Encode 8 values of one group; write W^, codes and packed codes of element `off`.
// round(v/h) of the correctly rounded quotient equals the rounding of the product v*hinv
// (hinv = 1/h correctly rounded) wherever the product is below 256 in magnitude and at most
// 0.49995 from its nearest integer: the product is within 2^-23 |v/h| of v/h (two roundings)
// and the quotient within 2^-24 |v/h|, so the two differ by less than 4.6e-5 and the
// quotient lies strictly inside the same rounding interval. The other elements (about 1e-4
// of them) take the IEEE quotient, in a branch the active lanes enter together only when one
// of them needs it.
__device__ __forceinline__ void encode8(const LwcParams& p, int64_t off, const float (&v)[8],
                                        const GroupQ& q) {
  const float hinv = __frcp_rn(q.h);
  float r[8];
  unsigned slow = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float ua = __fmul_rn(v[i], hinv);
    r[i] = rne_small(ua);
    const bool ok = fabsf(ua) < 256.f && fabsf(__fsub_rn(ua, r[i])) <= 0.49995f;
    slow |= ok ? 0u : (1u << i);
  }
  if (__any_sync(__activemask(), slow != 0)) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (slow & (1u << i)) r[i] = rintf(__fdiv_rn(v[i], q.h));
  }
  float deq[8];
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float cc = fminf(fmaxf(__fadd_rn(r[i], q.z), 0.f), p.Q);
    deq[i] = __fmul_rn(__fsub_rn(cc, q.z), q.h);
    c[i] = small_uint(cc);
  }
  if (p.W_hat) store8(p.W_hat, off, p.hat_dt, deq);
  if (p.codes) {
    uint2 w;
    w.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
    w.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
    *reinterpret_cast<uint2*>(p.codes + off) = w;
  }
  if (p.packed) {
    if (p.bits == 4) {
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) w |= c[i] << (4 * i);
      *reinterpret_cast<uint32_t*>(p.packed + off / 2) = w;
    } else if (p.bits == 2) {
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) w |= c[i] << (2 * i);
      *reinterpret_cast<uint16_t*>(p.packed + off / 4) = static_cast<uint16_t>(w);
    } else if (p.bits != 8) {
      // 3, 5, 6 or 7 bits: 8 codes fill `bits` bytes starting at byte bits * off / 8
      uint64_t w = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) w |= static_cast<uint64_t>(c[i]) << (p.bits * i);
      uint8_t* b = p.packed + off / 8 * p.bits;
      for (int k = 0; k < p.bits; ++k) b[k] = static_cast<uint8_t>(w >> (8 * k));
    } else {  // 8 bits
      uint2 w;
      w.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
      w.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
      *reinterpret_cast<uint2*>(p.packed + off) = w;
    }
  }
}

__device__ __forceinline__ void load_scaled8(const LwcParams& p, int64_t off, int64_t col,
                                             float (&v)[8]) {
  load8(p.W, off, p.wdt, v);
  if (p.s) {
    const float4* sp = reinterpret_cast<const float4*>(p.s + col);
    const float4 s0 = sp[0], s1 = sp[1];
    v[0] = __fmul_rn(v[0], s0.x); v[1] = __fmul_rn(v[1], s0.y);
    v[2] = __fmul_rn(v[2], s0.z); v[3] = __fmul_rn(v[3], s0.w);
    v[4] = __fmul_rn(v[4], s1.x); v[5] = __fmul_rn(v[5], s1.y);
    v[6] = __fmul_rn(v[6], s1.z); v[7] = __fmul_rn(v[7], s1.w);
  }
}

// Launch shape shared by the small-group kernels: grid (256-column segments, row blocks of
// rows_per_block rows); a warp covers one row of the segment (lane = 8 columns, one 16-byte
// load of bf16), the 8 warps of a block take every 8th row, U rows per iteration. A lane's
// columns, and so its group within the row, stay fixed: no index division in the loop.
constexpr int kLwcRows = 64;

template <int LPG, int U>
__global__ void __launch_bounds__(256, 3) lwc_small_kernel(LwcParams p) {
  constexpr int GPW = 32 / LPG;   // groups per segment
  // The clipping strengths (binary64 sigmoids) of the U rows' groups are spread over the
  // warp's lanes: SPR strengths a row (gamma, beta of each group), RPP rows a pass of 32
  // lanes, NP passes. Lane t of pass q evaluates row q*RPP + t/SPR, group t%SPR / 2, beta
  // for odd t.
  constexpr int SPR = 2 * GPW, RPP = 32 / SPR, NP = (U + RPP - 1) / RPP;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int sub = lane / LPG, lig = lane % LPG;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  const bool cvalid = c0 < p.K;
  const int64_t j = c0 / (LPG * 8);                        // this lane's group in the row
  const int64_t jt = static_cast<int64_t>(blockIdx.x) * GPW + (lane % SPR) / 2;
  const bool tvalid = jt < p.ng;
  const float* logit = (lane & 1) ? p.bl : p.gl;
  float sv[8];
  if (p.s && cvalid) {
    const float4* sp = reinterpret_cast<const float4*>(p.s + c0);
    const float4 s0 = sp[0], s1 = sp[1];
    sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
    sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
  }
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kLwcRows;
  const int64_t r1 = min(p.N, r0 + kLwcRows);
  for (int64_t nb = r0 + w; nb < r1; nb += 8 * U) {
    float v[U][8], st[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int u = q * RPP + lane / SPR;
      const int64_t n = nb + 8 * u;
      st[q] = (u < U && n < r1 && tvalid) ? strength(logit[n * p.ng + jt]) : 1.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t n = nb + 8 * u;
      if (n < r1 && cvalid) {
        load8(p.W, n * p.K + c0, p.wdt, v[u]);
        if (p.s) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[u][i] = __fmul_rn(v[u][i], sv[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t n = nb + 8 * u;
      float vmax = v[u][0], vmin = v[u][0];
#pragma unroll
      for (int i = 1; i < 8; ++i) { vmax = fmaxf(vmax, v[u][i]); vmin = fminf(vmin, v[u][i]); }
#pragma unroll
      for (int o = LPG / 2; o > 0; o >>= 1) {
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      }
      int nmax = 0, nmin = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { nmax += v[u][i] == vmax; nmin += v[u][i] == vmin; }
#pragma unroll
      for (int o = LPG / 2; o > 0; o >>= 1) {
        nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
        nmin += __shfl_xor_sync(0xffffffffu, nmin, o);
      }
      const int src = (u % RPP) * SPR + 2 * sub;
      const float g = __shfl_sync(0xffffffffu, st[u / RPP], src);
      const float b = __shfl_sync(0xffffffffu, st[u / RPP], src + 1);
      if (n >= r1 || !cvalid) continue;
      const GroupQ q = group_params(g, b, vmax, vmin, p.Q);
      encode8(p, n * p.K + c0, v[u], q);
      if (lig == 0) {
        const int64_t gi = n * p.ng + j;
        if (p.h) p.h[gi] = q.h;
        if (p.z) p.z[gi] = z_to_i32(q.z);
        if (p.range) p.range[gi] = omq_range{vmax, vmin, nmax, nmin};
      }
    }
  }
}

// Block-wide reduction of (max, min) or (sum, sum); every thread gets the result, combined
// in a fixed order.
__device__ __forceinline__ void block_maxmin(float& vmax, float& vmin, float* sm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
  }
  __syncthreads();
  if (lane == 0) { sm[w] = vmax; sm[32 + w] = vmin; }
  __syncthreads();
  vmax = sm[0];
  vmin = sm[32];
  for (int i = 1; i < nw; ++i) { vmax = fmaxf(vmax, sm[i]); vmin = fminf(vmin, sm[32 + i]); }
}
__device__ __forceinline__ void block_sum2i(int& a, int& b, int* sm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  __syncthreads();
  if (lane == 0) { sm[w] = a; sm[32 + w] = b; }
  __syncthreads();
  a = 0;
  b = 0;
  for (int i = 0; i < nw; ++i) { a += sm[i]; b += sm[32 + i]; }
}

__global__ void __launch_bounds__(256) lwc_large_kernel(LwcParams p) {
  extern __shared__ float buf[];   // G floats: the scaled group
  __shared__ float smf[64];
  __shared__ int smi[64];
  __shared__ float sgb[2];         // the group's strengths (read after the reductions' syncs)
  const int64_t total = p.N * p.ng;
  const int chunks = static_cast<int>(p.G / 8);
  for (int64_t gi = blockIdx.x; gi < total; gi += gridDim.x) {
    const int64_t n = gi / p.ng, j = gi % p.ng;
    const int64_t base = n * p.K + j * p.G;
    if (threadIdx.x < 2) sgb[threadIdx.x] = strength(threadIdx.x ? p.bl[gi] : p.gl[gi]);
    float vmax = -FLT_MAX, vmin = FLT_MAX;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8];
      load_scaled8(p, base + c * 8, j * p.G + c * 8, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        buf[c * 8 + i] = v[i];
        vmax = fmaxf(vmax, v[i]);
        vmin = fminf(vmin, v[i]);
      }
    }
    block_maxmin(vmax, vmin, smf);
    int nmax = 0, nmin = 0;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
      for (int i = 0; i < 8; ++i) { nmax += buf[c * 8 + i] == vmax; nmin += buf[c * 8 + i] == vmin; }
    block_sum2i(nmax, nmin, smi);
    const GroupQ q = group_params(sgb[0], sgb[1], vmax, vmin, p.Q);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = buf[c * 8 + i];
      encode8(p, base + c * 8, v, q);
    }
    if (threadIdx.x == 0) {
      if (p.h) p.h[gi] = q.h;
      if (p.z) p.z[gi] = z_to_i32(q.z);
      if (p.range) p.range[gi] = omq_range{vmax, vmin, nmax, nmin};
    }
    __syncthreads();   // buf is rewritten by the next group
  }
}

// 8 values of a 16-bit vector load.
__device__ __forceinline__ void unpack16x8(const uint4& q, bool f16, float (&v)[8]) {
  if (f16) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  } else {
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  }
}
// W~ = W s for 8 columns starting at col (binary32, one rounding).
__device__ __forceinline__ void scale8(const float* s, int64_t col, float (&v)[8]) {
  float sv[8];
  load_f8(s, col, sv);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], sv[i]);
}

// One group per row (per-channel), 16-bit W, K a multiple of 256 up to 4096: one warp per
// row, persistent warps taking rows in equal shares. Lane l holds columns 256 i + 8 l .. + 7
// of every 256-column segment i (coalesced 16-byte loads, all issued before any is used, the
// row kept packed in registers), so the max / min, the tie counts and the codes come from
// one read of W; B~[n] = B[n] + sum_k W[n,k] delta[k] (when requested) from the same data.
constexpr int kRowSegs = 16;

__global__ void __launch_bounds__(256, 2) lwc_row_kernel(LwcParams p, int64_t rows_per_warp) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int S = static_cast<int>(p.K / 256);
  const bool f16 = p.wdt == OMQ_F16;
  for (int64_t it = 0; it < rows_per_warp; ++it) {
    const int64_t n = warp_g + it * n_warps;
    if (n >= p.N) break;                                  // warp-uniform
    const uint4* wrow = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.W) + n * p.K) + lane;
    uint4 raw[kRowSegs];
#pragma unroll
    for (int i = 0; i < kRowSegs; ++i)
      if (i < S) raw[i] = __ldg(wrow + 32 * i);
    float vmax = -FLT_MAX, vmin = FLT_MAX;
#pragma unroll
    for (int i = 0; i < kRowSegs; ++i) {
      if (i >= S) break;
      float v[8];
      unpack16x8(raw[i], f16, v);
      if (p.s) scale8(p.s, 256 * i + 8 * lane, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) { vmax = fmaxf(vmax, v[e]); vmin = fminf(vmin, v[e]); }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    }
    float st = 1.f;
    if (lane < 2) st = strength((lane ? p.bl : p.gl)[n]);
    const float g = __shfl_sync(0xffffffffu, st, 0), b = __shfl_sync(0xffffffffu, st, 1);
    const GroupQ q = group_params(g, b, vmax, vmin, p.Q);
    int cnt = 0;                                          // nmax | nmin << 16
    float bias = 0.f;
#pragma unroll
    for (int i = 0; i < kRowSegs; ++i) {
      if (i >= S) break;
      const int64_t col = 256 * i + 8 * lane;
      float v[8];
      unpack16x8(raw[i], f16, v);
      if (p.Bt && p.delta) {
        float d[8];
        load_f8(p.delta, col, d);
#pragma unroll
        for (int e = 0; e < 8; ++e) bias += v[e] * d[e];
      }
      if (p.s) scale8(p.s, col, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) cnt += (v[e] == vmax ? 1 : 0) + (v[e] == vmin ? 0x10000 : 0);
      encode8(p, n * p.K + col, v, q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      bias += __shfl_xor_sync(0xffffffffu, bias, o);
    }
    if (lane == 0) {
      if (p.h) p.h[n] = q.h;
      if (p.z) p.z[n] = z_to_i32(q.z);
      if (p.range) p.range[n] = omq_range{vmax, vmin, cnt & 0xffff, cnt >> 16};
      if (p.Bt) p.Bt[n] = (p.B ? p.B[n] : 0.f) + bias;
    }
  }
}

omq_status launch_lwc(const LwcParams& p, cudaStream_t stream) {
  const int64_t total = p.N * p.ng;
  const int sms = num_sms();
  if ((p.wdt == OMQ_BF16 || p.wdt == OMQ_F16) && p.G == p.K && p.K % 256 == 0 &&
      p.K <= 256 * kRowSegs) {
    const int64_t max_warps = static_cast<int64_t>(sms) * 16;   // 2 blocks of 8 warps an SM
    const int64_t per = (p.N + max_warps - 1) / max_warps;
    const int64_t warps = (p.N + per - 1) / per;
    lwc_row_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(p, per);
    return launch_status();
  }
  if (p.Bt) {
    // B~ = B + W delta: its own pass over W
    const omq_status st = launch_let_bias(p.W, p.wdt, p.N, p.K, p.delta, p.B, p.Bt, stream);
    if (st != OMQ_OK) return st;
  }
  if (small_group(p.G)) {
    constexpr int U = 4;
    dim3 grid(static_cast<unsigned>(ceil_div(p.K, 256)),
              static_cast<unsigned>(ceil_div(p.N, kLwcRows)));
    switch (p.G / 8) {
      case 2: lwc_small_kernel<2, U><<<grid, 256, 0, stream>>>(p); break;
      case 4: lwc_small_kernel<4, U><<<grid, 256, 0, stream>>>(p); break;
      case 8: lwc_small_kernel<8, U><<<grid, 256, 0, stream>>>(p); break;
      case 16: lwc_small_kernel<16, U><<<grid, 256, 0, stream>>>(p); break;
      default: lwc_small_kernel<32, U><<<grid, 256, 0, stream>>>(p); break;
    }
    return launch_status();
  }
  const size_t smem = static_cast<size_t>(p.G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(lwc_large_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) { set_cuda_error(e); return OMQ_ERR_CUDA; }
  }
  const unsigned grid = static_cast<unsigned>(total < int64_t(sms) * 8 ? total : int64_t(sms) * 8);
  lwc_large_kernel<<<grid, 256, smem, stream>>>(p);
  return launch_status();
}

}  // namespace omq
