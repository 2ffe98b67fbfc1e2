// float32 GEMM on CUDA cores for the float32 storage path (kept in float32 end to end so
// the float32 workloads keep full precision; the bf16 path uses the tensor cores).
// C[i, j] = sum_k A(i, k) B(j, k) with either operand K-major or MN-major; 64 x 64 tiles,
// 256 threads, 4 x 4 outputs per thread, shared-memory staged k-blocks of 16.
#include "gemm_epilogue.cuh"

namespace omq {
namespace simt {

constexpr int T = 64;
constexpr int TK = 16;

__device__ __forceinline__ float op_at(const GemmOperand& o, int64_t i, int64_t k) {
  const float* p = reinterpret_cast<const float*>(o.ptr);
  return o.mn_major ? p[k * o.ld + i] : p[i * o.ld + k];
}

__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmOperand A, GemmOperand B, int64_t rows,
                                                       int64_t cols, int64_t depth,
                                                       GemmEpilogue epi, int tiles_n) {
  pdl_wait();
  pdl_launch();
  __shared__ float As[TK][T + 1];
  __shared__ float Bs[TK][T + 1];
  __shared__ float red[8];
  const int tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  const int64_t i0 = static_cast<int64_t>(tm) * T, j0 = static_cast<int64_t>(tn) * T;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < depth; k0 += TK) {
    for (int e = threadIdx.x; e < T * TK; e += 256) {
      // MN-major operands are read along i (coalesced); K-major along k
      int ii, kk;
      if (A.mn_major) { ii = e % T; kk = e / T; } else { kk = e % TK; ii = e / TK; }
      const int64_t gi = i0 + ii, gk = k0 + kk;
      As[kk][ii] = (gi < rows && gk < depth) ? op_at(A, gi, gk) : 0.f;
      int jj, kb;
      if (B.mn_major) { jj = e % T; kb = e / T; } else { kb = e % TK; jj = e / TK; }
      const int64_t gj = j0 + jj, gk2 = k0 + kb;
      Bs[kb][jj] = (gj < cols && gk2 < depth) ? op_at(B, gj, gk2) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty * 4 + u];
        b[u] = Bs[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
    }
    __syncthreads();
  }
  float lsum = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int64_t i = i0 + ty * 4 + u, j = j0 + tx * 4 + w;
      if (i < rows && j < cols) epi_element(epi, epi.out, i, j, cols, acc[u][w], lsum);
    }
  if (epi.kind == Epi::MseLoss) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = lsum;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < 8; ++w) s += red[w];
      epi.loss_partials[blockIdx.x] = s;
    }
  }
}

}  // namespace simt

int64_t gemm_f32_simt_tiles(int64_t rows, int64_t cols) {
  return ceil_div(rows, simt::T) * ceil_div(cols, simt::T);
}

omq_status gemm_f32_simt(const GemmOperand& A, const GemmOperand& B, int64_t rows, int64_t cols,
                         int64_t depth, const GemmEpilogue& epi, int64_t* n_tiles,
                         cudaStream_t stream) {
  const int64_t tn = ceil_div(cols, simt::T);
  const int64_t tiles = ceil_div(rows, simt::T) * tn;
  if (n_tiles) *n_tiles = tiles;
  launch_k(simt::gemm_f32_kernel, static_cast<unsigned>(tiles), 256, 0, stream,
      A, B, rows, cols, depth, epi, static_cast<int>(tn));
  return launch_status();
}

}  // namespace omq
