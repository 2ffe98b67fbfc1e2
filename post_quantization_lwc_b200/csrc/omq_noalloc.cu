// omq_fq_linear_fwd_noalloc: the fake-quantized linear forward and loss of
// omq_fq_linear_fwd, for callers that cannot supply device scratch memory.
//
// Who needs it: some hosts own every device allocation themselves. Examples are a framework
// that routes all device memory through its own pool and gives plug-ins no allocation hook,
// or a runtime that forbids device allocation once it has started. Such a host cannot call
// cudaMalloc for this library's workspace and has no workspace of its own to lend. This entry
// point keeps its scratch (one float per output tile: the partial sums of the squared error)
// in a fixed array compiled into the library. The caller still passes every input and output
// buffer, and the call allocates nothing.
//
// Limits and sharing:
//   - The array holds kNoAllocTiles partial sums. A problem needs 2 * ceil(M/256) *
//     ceil(N/256) of them on the 16-bit tensor-core path (one per 128-row half of each
//     256 x 256 output tile), or ceil(M/64) * ceil(N/64) on the float32 path;
//     larger problems are rejected with OMQ_ERR_SHAPE before anything is launched.
//   - Every GPU that loads the library holds the array (64 KiB) until the process exits.
//   - All calls on a device share the one array, and it keeps the last call's contents.
//     Each call writes every slot it reads before reading it, so nothing needs clearing.
//     Calls whose work overlaps on the GPU (different streams with no ordering between them)
//     race on the array and may return a wrong loss; order such calls on one stream.
//   - Every call looks up the array's device address in the calling thread's current
//     context (cudaGetSymbolAddress, a host-side lookup) instead of caching it per device
//     ordinal: after cudaDeviceReset, or with another context current on the same device, a
//     cached address would name memory of a context that no longer owns it. The first call in
//     a context also loads the library's module there; make that first call before any
//     stream capture begins.
#include "omq_internal.cuh"

namespace omq {
namespace {

constexpr int64_t kNoAllocTiles = 16384;

static __device__ __align__(256) float g_noalloc_loss_partials[kNoAllocTiles];

// Device address of the fixed scratch array in the current context. Looked up on every call:
// the address belongs to the module instance of the context that is current now, which a
// cache keyed by device ordinal cannot tell apart from one that was reset or replaced.
omq_status noalloc_scratch(float** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_loss_partials);
  if (e != cudaSuccess || p == nullptr) {
    set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    return OMQ_ERR_CUDA;
  }
  *out = static_cast<float*>(p);
  return OMQ_OK;
}

}  // namespace
}  // namespace omq

using namespace omq;

extern "C" omq_status omq_fq_linear_fwd_noalloc(const void* Xq, const void* W_hat, omq_dtype dt,
                                                int64_t M, int64_t N, int64_t K,
                                                const float* B_tilde, const float* Y_ref,
                                                float* Y, void* dY, float* loss,
                                                omq_stream_t stream) {
  if (!Xq || !W_hat || !Y_ref || !dY || !loss) return OMQ_ERR_NULL;
  if (dt != OMQ_F32 && dt != OMQ_BF16 && dt != OMQ_F16) return OMQ_ERR_DTYPE;
  const int64_t kMax = (int64_t(1) << 31) - 1;
  if (M < 1 || N < 8 || K < 8 || N % 8 || K % 8 || M > kMax || N > kMax || K > kMax)
    return OMQ_ERR_SHAPE;
  if (!aligned16(Xq) || !aligned16(W_hat) || !aligned16(Y_ref) || !aligned16(dY) ||
      (B_tilde && !aligned16(B_tilde)) || (Y && !aligned16(Y)))
    return OMQ_ERR_ALIGN;
  const int64_t tiles = dt != OMQ_F32 ? gemm_tc_tiles(M, N) : gemm_f32_simt_tiles(M, N);
  if (tiles > kNoAllocTiles) return OMQ_ERR_SHAPE;
  float* partials = nullptr;
  omq_status st = noalloc_scratch(&partials);
  if (st != OMQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GemmOperand A{Xq, K, false}, B{W_hat, K, false};
  GemmEpilogue epi{};
  epi.kind = Epi::MseLoss;
  epi.bias = B_tilde;
  epi.out = Y;
  epi.y_ref = Y_ref;
  epi.dy = dY;
  epi.dy_dt = dt;
  epi.loss_partials = partials;
  int64_t launched = 0;
  st = dt != OMQ_F32 ? gemm_tc(dt, A, B, M, N, K, epi, &launched, s)
                     : gemm_f32_simt(A, B, M, N, K, epi, &launched, s);
  if (st != OMQ_OK) return st;
  return launch_loss_finalize(partials, launched,
                              1.0 / (static_cast<double>(M) * static_cast<double>(N)), loss, s);
}
