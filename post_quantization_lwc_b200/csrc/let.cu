// Activation side of the step ("【ICLR 2024】OmniQuant: ...", section LET and the
// per-token activation quantizer of section 实验证据):
//   X~ = (X - delta) / s                       (one HBM pass, 16-byte vector accesses)
//   per token: MinMax affine fake-quant of the row X~[m, :]   (one block per token,
//     row staged in shared memory, warp-shuffle + shared-memory reductions)
//   B~ = B + W delta                            (one warp per output row)
#include <float.h>

#include "omq_internal.cuh"

namespace omq {

__device__ __forceinline__ void let8(const LetParams& p, int64_t off, int64_t col, float (&v)[8]) {
  load8(p.X, off, p.xdt, v);
  float sv[8], dv[8];
  if (p.s) {
    const float4* q = reinterpret_cast<const float4*>(p.s + col);
    const float4 a = q[0], b = q[1];
    sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w; sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = 1.f;
  }
  if (p.d) {
    const float4* q = reinterpret_cast<const float4*>(p.d + col);
    const float4 a = q[0], b = q[1];
    dv[0] = a.x; dv[1] = a.y; dv[2] = a.z; dv[3] = a.w; dv[4] = b.x; dv[5] = b.y; dv[6] = b.z; dv[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) dv[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(__fsub_rn(v[i], dv[i]), sv[i]);
}

// Unquantized activations (16-bit): X~ = (X - delta) / s stored in the operand type, or a
// plain conversion when there is no LET (AFFINE false). Grid (256-column segments, row
// blocks of kLetRows); a lane keeps 8 fixed columns (and their s, delta in registers), the 8
// warps take every 8th row, U rows loaded before any is converted.
constexpr int kLetRows = 64;

template <int U, bool AFFINE>
__global__ void __launch_bounds__(256, 2) let_elem_kernel(LetParams p) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  if (c0 >= p.K) return;
  float sv[8], dv[8];
  if (AFFINE) {
#pragma unroll
    for (int i = 0; i < 8; ++i) { sv[i] = 1.f; dv[i] = 0.f; }
    if (p.s) load_f8(p.s, c0, sv);
    if (p.d) load_f8(p.d, c0, dv);
  }
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kLetRows;
  const int64_t r1 = min(p.M, r0 + kLetRows);
  for (int64_t mb = r0 + w; mb < r1; mb += 8 * U) {
    float v[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (mb + 8 * u < r1) load8(p.X, (mb + 8 * u) * p.K + c0, p.xdt, v[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (mb + 8 * u >= r1) continue;
      if (AFFINE) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = __fdiv_rn(__fsub_rn(v[u][i], dv[i]), sv[i]);
      }
      store8(p.Xq, (mb + 8 * u) * p.K + c0, p.xq_dt, v[u]);
    }
  }
}

__global__ void __launch_bounds__(256) act_quant_kernel(LetParams p) {
  pdl_wait();
  pdl_launch();
  extern __shared__ float row[];   // K floats: X~[m, :]
  __shared__ float smf[64];
  __shared__ int smi[64];
  const int chunks = static_cast<int>(p.K / 8);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int64_t m = blockIdx.x; m < p.M; m += gridDim.x) {
    const int64_t base = m * p.K;
    float vmax = -FLT_MAX, vmin = FLT_MAX;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8];
      let8(p, base + c * 8, c * 8, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        row[c * 8 + i] = v[i];
        vmax = fmaxf(vmax, v[i]);
        vmin = fminf(vmin, v[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    }
    __syncthreads();
    if (lane == 0) { smf[w] = vmax; smf[32 + w] = vmin; }
    __syncthreads();
    vmax = smf[0];
    vmin = smf[32];
    for (int i = 1; i < nw; ++i) { vmax = fmaxf(vmax, smf[i]); vmin = fminf(vmin, smf[32 + i]); }
    int nmax = 0, nmin = 0;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x)
#pragma unroll
      for (int i = 0; i < 8; ++i) { nmax += row[c * 8 + i] == vmax; nmin += row[c * 8 + i] == vmin; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
      nmin += __shfl_xor_sync(0xffffffffu, nmin, o);
    }
    if (lane == 0) { smi[w] = nmax; smi[32 + w] = nmin; }
    __syncthreads();
    nmax = 0;
    nmin = 0;
    for (int i = 0; i < nw; ++i) { nmax += smi[i]; nmin += smi[32 + i]; }
    // gamma = beta = 1: h = (M - m)/Q, z = -round(m/h)
    const GroupQ q = group_params(1.f, 1.f, vmax, vmin, p.Qa);
    const float hinv = __frcp_rn(q.h);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float v[8], rq[8], o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = row[c * 8 + i];
      round_quotient8(v, q.h, hinv, rq);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float lvl = __fadd_rn(rq[i], q.z);
        const float cc = fminf(fmaxf(lvl, 0.f), p.Qa);
        o[i] = __fmul_rn(__fsub_rn(cc, q.z), q.h);
      }
      store8(p.Xq, base + c * 8, p.xq_dt, o);
    }
    if (threadIdx.x == 0) {
      if (p.h_a) p.h_a[m] = q.h;
      if (p.z_a) p.z_a[m] = z_to_i32(q.z);
      if (p.range) p.range[m] = omq_range{vmax, vmin, nmax, nmin};
    }
    __syncthreads();
  }
}

// B~[n] = B[n] + sum_k W[n,k] delta[k]. One warp per row, persistent warps taking rows in
// equal shares; the row is read in passes of 16 segments of 256 columns (lane = 8 columns of
// each), the 16 loads of a pass issued before any is used and kept packed.
constexpr int kBiasSegs = 16;

__global__ void __launch_bounds__(256, 2) let_bias_kernel(const void* W, omq_dtype wdt, int64_t N,
                                                          int64_t K, const float* delta,
                                                          const float* B, float* Bt,
                                                          int64_t rows_per_warp) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t nseg = (K + 255) / 256;
  for (int64_t it = 0; it < rows_per_warp; ++it) {
    const int64_t n = warp_g + it * n_warps;
    if (n >= N) break;                                     // warp-uniform
    float acc = 0.f;
    if (delta) {
      for (int64_t s0 = 0; s0 < nseg; s0 += kBiasSegs) {
        uint4 raw[kBiasSegs];
#pragma unroll
        for (int i = 0; i < kBiasSegs; ++i) {
          const int64_t col = (s0 + i) * 256 + lane * 8;
          raw[i] = col < K ? *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(W) +
                                                              n * K + col)
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kBiasSegs; ++i) {
          const int64_t col = (s0 + i) * 256 + lane * 8;
          if (col >= K) break;
          float v[8], d[8];
          const uint16_t* h = reinterpret_cast<const uint16_t*>(&raw[i]);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            v[e] = wdt == OMQ_F16 ? __half2float(__ushort_as_half(h[e]))
                                  : __bfloat162float(__ushort_as_bfloat16(h[e]));
          load_f8(delta, col, d);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc += v[e] * d[e];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    }
    if (lane == 0) Bt[n] = (B ? B[n] : 0.f) + acc;
  }
}

// float32 W (the CUDA-core path): one warp per row, lanes stride 8-element chunks.
__global__ void __launch_bounds__(256) let_bias_f32_kernel(const float* W, int64_t N, int64_t K,
                                                           const float* delta, const float* B,
                                                           float* Bt) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t n = warp_g; n < N; n += n_warps) {
    float acc = 0.f;
    if (delta) {
      for (int64_t c = lane; c < K / 8; c += 32) {
        float v[8], d[8];
        load_f8(W, n * K + c * 8, v);
        load_f8(delta, c * 8, d);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc += v[e] * d[e];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    }
    if (lane == 0) Bt[n] = (B ? B[n] : 0.f) + acc;
  }
}

omq_status launch_let(const LetParams& p, int abits, cudaStream_t stream) {
  const int sms = num_sms();
  if (abits >= 16) {
    const dim3 grid(static_cast<unsigned>(ceil_div(p.K, 256)),
                    static_cast<unsigned>(ceil_div(p.M, kLetRows)));
    if (p.s || p.d) launch_k(let_elem_kernel<4, true>, grid, 256, 0, stream, p);
    else launch_k(let_elem_kernel<4, false>, grid, 256, 0, stream, p);
    return launch_status();
  }
  const size_t smem = static_cast<size_t>(p.K) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(act_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) { set_cuda_error(e); return OMQ_ERR_CUDA; }
  }
  const unsigned grid = static_cast<unsigned>(p.M < int64_t(sms) * 8 ? p.M : int64_t(sms) * 8);
  launch_k(act_quant_kernel, grid, 256, smem, stream, p);
  return launch_status();
}

omq_status launch_let_bias(const void* W, omq_dtype wdt, int64_t N, int64_t K, const float* delta,
                           const float* B, float* Bt, cudaStream_t stream) {
  const int sms = num_sms();
  if (wdt == OMQ_F32) {
    const int64_t want = ceil_div(N, 8);
    const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 16 ? want : int64_t(sms) * 16);
    launch_k(let_bias_f32_kernel, grid, 256, 0, stream,
        static_cast<const float*>(W), N, K, delta, B, Bt);
    return launch_status();
  }
  const int64_t max_warps = static_cast<int64_t>(sms) * 16;
  const int64_t per = (N + max_warps - 1) / max_warps;
  const int64_t warps = (N + per - 1) / per;
  launch_k(let_bias_kernel, static_cast<unsigned>((warps + 7) / 8), 256, 0, stream,
      W, wdt, N, K, delta, B, Bt, per);
  return launch_status();
}

}  // namespace omq
