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
__device__ __forceinline__ void encode8(const LwcParams& p, int64_t off, const float (&v)[8],
                                        const GroupQ& q) {
  const float hinv = __frcp_rn(q.h);
  float deq[8];
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float lvl = __fadd_rn(round_quotient(v[i], q.h, hinv), q.z);
    const float cc = fminf(fmaxf(lvl, 0.f), p.Q);
    deq[i] = __fmul_rn(__fsub_rn(cc, q.z), q.h);
    c[i] = static_cast<uint32_t>(cc);
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

template <int LPG>
__global__ void __launch_bounds__(256) lwc_small_kernel(LwcParams p) {
  constexpr int SPW = 32 / LPG;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPG, lig = lane % LPG;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = p.N * p.ng;
  for (int64_t base = warp_g * SPW; base < total; base += n_warps * SPW) {
    const int64_t gi = base + sub;
    const bool valid = gi < total;
    const int64_t n = valid ? gi / p.ng : 0, j = valid ? gi % p.ng : 0;
    const int64_t col = j * p.G + lig * 8;
    const int64_t off = n * p.K + col;
    float v[8];
    if (valid) {
      load_scaled8(p, off, col, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    float vmax = v[0], vmin = v[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) { vmax = fmaxf(vmax, v[i]); vmin = fminf(vmin, v[i]); }
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) {
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    }
    int nmax = 0, nmin = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) { nmax += v[i] == vmax; nmin += v[i] == vmin; }
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) {
      nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
      nmin += __shfl_xor_sync(0xffffffffu, nmin, o);
    }
    if (!valid) continue;
    const float g = strength(p.gl[gi]), b = strength(p.bl[gi]);
    const GroupQ q = group_params(g, b, vmax, vmin, p.Q);
    encode8(p, off, v, q);
    if (lig == 0) {
      if (p.h) p.h[gi] = q.h;
      if (p.z) p.z[gi] = z_to_i32(q.z);
      if (p.range) p.range[gi] = omq_range{vmax, vmin, nmax, nmin};
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
  const int64_t total = p.N * p.ng;
  const int chunks = static_cast<int>(p.G / 8);
  for (int64_t gi = blockIdx.x; gi < total; gi += gridDim.x) {
    const int64_t n = gi / p.ng, j = gi % p.ng;
    const int64_t base = n * p.K + j * p.G;
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
    const float g = strength(p.gl[gi]), b = strength(p.bl[gi]);
    const GroupQ q = group_params(g, b, vmax, vmin, p.Q);
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

omq_status launch_lwc(const LwcParams& p, cudaStream_t stream) {
  const int64_t total = p.N * p.ng;
  const int sms = num_sms();
  if (p.G <= 256 && (p.G & (p.G - 1)) == 0) {
    const int lpg = static_cast<int>(p.G / 8);
    const int64_t groups_per_block = 8 * (32 / lpg);
    const int64_t want = ceil_div(total, groups_per_block);
    const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 16 ? want : int64_t(sms) * 16);
    switch (lpg) {
      case 1: lwc_small_kernel<1><<<grid, 256, 0, stream>>>(p); break;
      case 2: lwc_small_kernel<2><<<grid, 256, 0, stream>>>(p); break;
      case 4: lwc_small_kernel<4><<<grid, 256, 0, stream>>>(p); break;
      case 8: lwc_small_kernel<8><<<grid, 256, 0, stream>>>(p); break;
      case 16: lwc_small_kernel<16><<<grid, 256, 0, stream>>>(p); break;
      default: lwc_small_kernel<32><<<grid, 256, 0, stream>>>(p); break;
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
