// Inference with the folded weights ("【ICLR 2024】OmniQuant: ...", section 框架: the learned
// transforms fold into the weights, and the quantized model is an ordinary low-bit model):
// y[m, n] = sum_k x[m, k] (c[n, k] - z[n, j(k)]) h[n, j(k)] for a few tokens (decode), from
// the packed codes of omq_fold_pack, h and z. Memory-bound on the codes: one warp per output
// row walks the row's packed bytes (16 bytes a lane a load, coalesced, all of a pass issued
// before any is used); the tokens' activations sit in shared memory as float32, stored
// chunk-minor (column t of every chunk side by side, so the lanes of a warp, which hold
// consecutive chunks, read consecutive banks), with their sums over each 16-byte chunk of
// columns, so a chunk contributes
//   h (sum_k c_k x[m, k] - z sum_k x[m, k])
// with one multiply-add per code and token.
#include <algorithm>
#include <type_traits>

#include "omq_internal.cuh"

namespace omq {

constexpr int kGemvMaxTokens = 8;
constexpr int kGemvPass = 4;          // 16-byte chunks a lane loads per pass

// MT: tokens rounded up to 1, 2, 4 or 8 (the accumulators held per lane)
template <int BITS, int MT>
__global__ void __launch_bounds__(256) qgemv_kernel(const void* x, omq_dtype xdt, int M,
                                                    int64_t K, const uint8_t* packed,
                                                    const float* h, const int32_t* z, int64_t N,
                                                    int64_t group, float* y,
                                                    int64_t rows_per_warp) {
  pdl_wait();
  pdl_launch();
  constexpr int CPC = 128 / BITS;     // codes per 16-byte chunk
  extern __shared__ float gsm[];      // xf [M][CPC][K / CPC], then xsum [M][K / CPC]
  const int64_t nch = K / CPC;
  float* xf = gsm;
  float* xsum = gsm + static_cast<int64_t>(M) * K;
  // stage the tokens: 8 consecutive columns a thread (one 16-byte load of 16-bit x), all of
  // a thread's loads issued before its stores
  {
    const int64_t n8 = static_cast<int64_t>(M) * K / 8;
    constexpr int SU = 4;
    for (int64_t i0 = threadIdx.x; i0 < n8; i0 += static_cast<int64_t>(blockDim.x) * SU) {
      float v[SU][8];
#pragma unroll
      for (int u = 0; u < SU; ++u) {
        const int64_t i = i0 + static_cast<int64_t>(u) * blockDim.x;
        if (i < n8) load8(x, i * 8, xdt, v[u]);
      }
#pragma unroll
      for (int u = 0; u < SU; ++u) {
        const int64_t i = i0 + static_cast<int64_t>(u) * blockDim.x;
        if (i >= n8) break;
        const int64_t m = i * 8 / K, k0 = i * 8 % K;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int64_t k = k0 + e;
          xf[m * K + (k % CPC) * nch + k / CPC] = v[u][e];
        }
      }
    }
  }
  __syncthreads();
  for (int64_t i = threadIdx.x; i < static_cast<int64_t>(M) * nch; i += blockDim.x) {
    const int64_t m = i / nch, c = i % nch;
    float s = 0.f;
#pragma unroll 8
    for (int t = 0; t < CPC; ++t) s += xf[m * K + t * nch + c];
    xsum[i] = s;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t ng = K / group;
  const int64_t row_bytes = K * BITS / 8;
  // two rows at a time, the loads of both issued before any use
  for (int64_t it = 0; it < rows_per_warp; it += 2) {
    const int64_t n0 = warp_g + it * n_warps;
    if (n0 >= N) break;                                     // warp-uniform
    const int64_t n1 = n0 + n_warps;
    const bool has1 = it + 1 < rows_per_warp && n1 < N;
    float acc[2][MT] = {};
    for (int64_t c0 = lane; c0 < nch; c0 += 32 * kGemvPass) {
      uint4 q[2][kGemvPass];
      float hq[2][kGemvPass], zq[2][kGemvPass];   // the chunks' group scales and zero points
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int64_t n = r ? n1 : n0;
        const uint4* prow = reinterpret_cast<const uint4*>(packed + n * row_bytes);
#pragma unroll
        for (int u = 0; u < kGemvPass; ++u) {
          const int64_t c = c0 + 32 * u;
          if (c < nch && (r == 0 || has1)) {
            q[r][u] = __ldg(prow + c);
            const int64_t gi = n * ng + c * CPC / group;
            hq[r][u] = __ldg(h + gi);
            zq[r][u] = static_cast<float>(__ldg(z + gi));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r == 1 && !has1) break;
#pragma unroll
        for (int u = 0; u < kGemvPass; ++u) {
          const int64_t c = c0 + 32 * u;
          if (c >= nch) break;
          const float hv = hq[r][u], zv = zq[r][u];
          const uint32_t wq[4] = {q[r][u].x, q[r][u].y, q[r][u].z, q[r][u].w};
          float dot[MT] = {};
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
            for (int e = 0; e < 32 / BITS; ++e) {
              const float code = static_cast<float>((wq[wi] >> (BITS * e)) & ((1u << BITS) - 1));
              const int64_t t = wi * (32 / BITS) + e;         // column within the chunk
#pragma unroll
              for (int m = 0; m < MT; ++m)
                if (m < M) dot[m] += code * xf[m * K + t * nch + c];
            }
          }
#pragma unroll
          for (int m = 0; m < MT; ++m)
            if (m < M) acc[r][m] += hv * (dot[m] - zv * xsum[m * nch + c]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float a = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0 && m < M && (r == 0 || has1))
          y[static_cast<int64_t>(m) * N + (r ? n1 : n0)] = a;
      }
    }
  }
}

}  // namespace omq

using namespace omq;

// Tensor-core product with the folded weights (prefill, or any token count): the weight's
// packed codes are expanded into the GEMM's B operand tiles in shared memory as they are
// consumed (gemm_tc_qb), so the codes, h and z are the only weight bytes read.
static omq_status qgemm_impl(const void* x, omq_dtype xdt, int64_t M, int64_t K,
                             const uint8_t* packed, const float* h, const int32_t* z, int64_t N,
                             int64_t group, int bits, const float* bias, float* y,
                             cudaStream_t st) {
  if (!x || !packed || !h || !z || !y) return OMQ_ERR_NULL;
  if (xdt != OMQ_BF16 && xdt != OMQ_F16) return OMQ_ERR_DTYPE;
  if (bits < 2 || bits > 8) return OMQ_ERR_BITS;
  const int64_t kMax = (int64_t(1) << 31) - 1;
  if (M < 1 || K < 64 || K % 64 || N < 8 || N % 8 || group < 8 || group % 8 || K % group ||
      M > kMax || N > kMax || K > kMax)
    return OMQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(y) || (bias && !aligned16(bias)))
    return OMQ_ERR_ALIGN;
  GemmEpilogue epi{};
  epi.kind = Epi::StoreF32;
  epi.out = y;
  epi.out_scale = 1.f;
  epi.bias = bias;
  if (K / group > (int64_t(1) << 31) - 1 || (K / 8) > (int64_t(1) << 31) - 1) return OMQ_ERR_SHAPE;
  epi.qb = QuantB{packed, h, z, K * bits / 8, K / group, group, K,
                  static_cast<int32_t>(group % 64 == 0 ? group / 64 : 0),
                  static_cast<int32_t>(group / 8)};
  return gemm_tc_qb(xdt, GemmOperand{x, K, false}, M, N, K, bits, epi, st);
}

extern "C" omq_status omq_qgemm(const void* x, omq_dtype xdt, int64_t M, int64_t K,
                                const uint8_t* packed, const float* h, const int32_t* z,
                                int64_t N, int64_t group, int bits, const float* bias, float* y,
                                omq_stream_t stream) {
  return qgemm_impl(x, xdt, M, K, packed, h, z, N, group, bits, bias, y,
                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" omq_status omq_qgemv(const void* x, omq_dtype xdt, int64_t M, int64_t K,
                                const uint8_t* packed, const float* h, const int32_t* z,
                                int64_t N, int64_t group, int bits, float* y,
                                omq_stream_t stream) {
  if (!x || !packed || !h || !z || !y) return OMQ_ERR_NULL;
  if (xdt != OMQ_F32 && xdt != OMQ_BF16 && xdt != OMQ_F16) return OMQ_ERR_DTYPE;
  if (bits < 2 || bits > 8) return OMQ_ERR_BITS;
  if (bits != 2 && bits != 4 && bits != 8) {
    // codes that straddle bytes: the tensor-core path (16-bit activations)
    if (xdt == OMQ_F32) return OMQ_ERR_UNSUPPORTED;
    if (M < 1 || M > kGemvMaxTokens) return OMQ_ERR_SHAPE;
    return qgemm_impl(x, xdt, M, K, packed, h, z, N, group, bits, nullptr, y,
                      reinterpret_cast<cudaStream_t>(stream));
  }
  const int64_t cpc = 128 / bits;
  if (M < 1 || M > kGemvMaxTokens || N < 1 || K < cpc || K % cpc || group < cpc ||
      group % cpc || K % group || N > (int64_t(1) << 31))
    return OMQ_ERR_SHAPE;
  // more than four tokens go as two launches of at most four (the eight-token variant needs
  // twice the registers, runs one block an SM and took 95 us for the q_proj fold against 27
  // for four tokens)
  const int64_t m_launch = M > 4 ? 4 : M;
  if (sizeof(float) * static_cast<size_t>(m_launch) * (K + K / cpc) > 200 * 1024)
    return OMQ_ERR_SHAPE;
  if (!aligned16(packed) || ((K * bits / 8) % 16)) return OMQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t xes = xdt == OMQ_F32 ? 4 : 2;
  // tokens [m0, m0 + mt) of x and y
  auto launch = [&](auto kernel, int64_t m0, int64_t mt) -> omq_status {
    const size_t smem = sizeof(float) * static_cast<size_t>(mt) * (K + K / cpc);
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem));
      if (e != cudaSuccess) {
        set_cuda_error(e);
        return OMQ_ERR_CUDA;
      }
    }
    const int64_t per_sm = std::max<int64_t>(1, std::min<int64_t>(2, (200 * 1024) / smem));
    const int64_t max_warps = static_cast<int64_t>(num_sms()) * 8 * per_sm;
    const int64_t per = (N + max_warps - 1) / max_warps;
    const int64_t warps = (N + per - 1) / per;
    launch_k(kernel, static_cast<unsigned>((warps + 7) / 8), 256, smem, st,
        static_cast<const void*>(static_cast<const char*>(x) + m0 * K * xes), xdt,
        static_cast<int>(mt), K, packed, h, z, N, group, y + m0 * N, per);
    return launch_status();
  };
  auto pick = [&](auto bits_c) -> omq_status {
    constexpr int B = decltype(bits_c)::value;
    for (int64_t m0 = 0; m0 < M; m0 += 4) {
      const int64_t mt = M - m0 < 4 ? M - m0 : 4;
      const omq_status st_m = mt == 1   ? launch(qgemv_kernel<B, 1>, m0, mt)
                              : mt == 2 ? launch(qgemv_kernel<B, 2>, m0, mt)
                                        : launch(qgemv_kernel<B, 4>, m0, mt);
      if (st_m != OMQ_OK) return st_m;
    }
    return OMQ_OK;
  };
  if (bits == 4) return pick(std::integral_constant<int, 4>{});
  if (bits == 2) return pick(std::integral_constant<int, 2>{});
  return pick(std::integral_constant<int, 8>{});
}
