// bf16 x bf16 -> fp32 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// C[i, j] = sum_k A(i, k) B(j, k) over 128 x BN output tiles, persistent: one CTA per SM
// walks tiles t, t + grid, t + 2 grid, ... Warp roles (192 threads):
//   warp 0      TMA producer: one elected lane streams A and B k-blocks into a STAGES-deep
//               shared-memory ring (128-byte swizzle), completing "full" mbarriers.
//   warp 1      allocates TMEM for two accumulators (2 x BN columns); one lane issues
//               tcgen05.mma (M=128, N=BN, K=16) per k-slice, tcgen05.commit's each stage back
//               to its "empty" mbarrier and each finished tile to its accumulator's "full"
//               mbarrier. It starts a tile as soon as the epilogue has released the other
//               accumulator, so tile i+1's MMAs run while tile i is being stored.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time, fused epilogue (bias,
//               MSE loss, dY) and global stores; then release the accumulator.
// Operands may be K-major (row of the stored matrix runs along k) or MN-major (row runs
// along i / j), so the three contractions of the step read X, W and dY in their natural
// layouts without transposed copies:
//   forward   Y  = Xq  W^^T : A = Xq [M,K] K-major,        B = W^ [N,K] K-major
//   dW^       dW = dY^T Xq  : A = dY [M,N] MN-major,       B = Xq [M,K] MN-major
//   dXq       dX = dY W^    : A = dY [M,N] K-major,        B = W^ [N,K] MN-major
// Every mbarrier wait is bounded in time; on expiry the kernel raises the device error
// flag, every role stops, outstanding copies and MMAs are drained (bounded), and the TMEM
// is released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm_epilogue.cuh"

namespace omq {

__device__ unsigned g_dev_error = 0;

cudaError_t take_device_error(unsigned* flag) {
  unsigned zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_dev_error, sizeof(unsigned));
  if (e == cudaSuccess && *flag) e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(unsigned));
  return e;
}

namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                    // 64 bf16 = 128 bytes = one swizzle row
constexpr int UMMA_K = 16;
constexpr int NUM_THREADS = 192;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per barrier wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait until the phase with the given parity has completed, for at most WAIT_LIMIT_NS.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned err_bit) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > WAIT_LIMIT_NS) {
      atomicOr(&g_dev_error, err_bit);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start address,
// leading / stride byte offsets in 16-byte units, version 1 at bit 46, layout type 2 at
// bits 61-63).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Descriptor of the k-slice `kk` (16 elements) of an operand tile at `base`.
//  K-major tile: `rows` rows of 128 bytes (64 k), 8-row swizzle atoms 1024 bytes apart;
//                a k-slice starts 32 bytes further along the row.
//  MN-major tile: chunks of 64 rows(i/j) x 64 k, each BK rows of 128 bytes (one k per row),
//                 chunks 8192 bytes apart (LBO); 8-k atoms 1024 bytes apart (SBO); a k-slice
//                 starts 16 k-rows = 2048 bytes further.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, bool mn_major, int kk) {
  if (mn_major) return smem_desc(base + kk * 2048, BK * 128, 1024);
  return smem_desc(base + kk * 32, 16, 1024);
}

// Instruction descriptor of kind::f16: D fp32 (bits 4-5 = 1), A and B format (bits 7-9,
// 10-12: 0 = f16, 1 = bf16; always the same for both), A / B major (bits 15, 16), N >> 3
// (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t instr_desc(int m, int n, bool a_mn, bool b_mn,
                                                  uint32_t fmt) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

template <int BN, int STAGES>
struct Layout {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2], drain; then tmem slot, abort
  // flag, the epilogue's per-warp loss partials [2][4] and arrival counters [2]
  static constexpr int FULL = 0, EMPTY = 8 * STAGES, ACCF = 16 * STAGES, ACCE = ACCF + 16,
                       DRAIN = ACCE + 16, SLOT = DRAIN + 8, ABORT = SLOT + 4, RED = ABORT + 4,
                       CNT = RED + 32;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + BAR_OFF + 256;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int a_mn, int b_mn, uint32_t fmt, int64_t rows, int64_t cols, int64_t depth,
                   GemmEpilogue epi, int tiles_n, int num_tiles) {
  using L = Layout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* ctl = smem + L::BAR_OFF;
  const uint32_t bar_full = sbase + L::BAR_OFF + L::FULL;
  const uint32_t bar_empty = sbase + L::BAR_OFF + L::EMPTY;
  const uint32_t bar_accf = sbase + L::BAR_OFF + L::ACCF;
  const uint32_t bar_acce = sbase + L::BAR_OFF + L::ACCE;
  const uint32_t bar_drain = sbase + L::BAR_OFF + L::DRAIN;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + L::SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + L::ABORT);
  volatile float* red = reinterpret_cast<volatile float*>(ctl + L::RED);     // [2][4]
  int* cnt = reinterpret_cast<int*>(ctl + L::CNT);                           // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = static_cast<int>((depth + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);   // one arrival per epilogue warp
      cnt[b] = 0;
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      const int row0 = (t / tiles_n) * BM;
      const int col0 = (t % tiles_n) * BN;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (*abort_flag || !mbar_wait(bar_empty + 8 * s, ph ^ 1, DEV_ERR_TMA_WAIT)) {
          ok = false;
          break;
        }
        const uint32_t a_dst = sbase + s * L::STAGE_BYTES;
        const uint32_t b_dst = a_dst + L::A_BYTES;
        const uint32_t full = bar_full + 8 * s;
        mbar_expect_tx(full, L::STAGE_BYTES);
        const int k0 = kb * BK;
        if (a_mn) {
          for (int c = 0; c < BM / 64; ++c) tma_load_2d(a_dst + c * 8192, &tmA, full, row0 + 64 * c, k0);
        } else {
          tma_load_2d(a_dst, &tmA, full, k0, row0);
        }
        if (b_mn) {
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &tmB, full, col0 + 64 * c, k0);
        } else {
          tma_load_2d(b_dst, &tmB, full, k0, col0);
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      // let the copies already in flight land before the CTA can exit
      for (int j = it - STAGES < 0 ? 0 : it - STAGES; j < it; ++j)
        mbar_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1, DEV_ERR_TMA_WAIT);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = instr_desc(BM, BN, a_mn != 0, b_mn != 0, fmt);
    int it = 0, lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++lt) {
      const int buf = lt & 1;
      if (*abort_flag || !mbar_wait(bar_acce + 8 * buf, ((lt >> 1) & 1) ^ 1, DEV_ERR_MMA_WAIT)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (*abort_flag || !mbar_wait(bar_full + 8 * s, ph, DEV_ERR_MMA_WAIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = sbase + s * L::STAGE_BYTES;
        const uint32_t b_base = a_base + L::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
          umma_bf16(d, operand_desc(a_base, a_mn != 0, kk), operand_desc(b_base, b_mn != 0, kk),
                    idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(bar_empty + 8 * s);
      }
      if (!ok) break;
      umma_commit(bar_accf + 8 * buf);
    }
    if (!ok) *abort_flag = 1;
    // every MMA issued above has completed once this commit arrives
    umma_commit(bar_drain);
    mbar_wait(bar_drain, 0, DEV_ERR_MMA_WAIT);
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
    int lt = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++lt) {
      const int buf = lt & 1;
      // one lane polls; the decision is broadcast so the warp-wide tcgen05.ld stays uniform
      int go = 0;
      if (lane == 0)
        go = (mbar_wait(bar_accf + 8 * buf, (lt >> 1) & 1, DEV_ERR_EPI_WAIT) && *abort_flag == 0)
                 ? 1 : 0;
      go = __shfl_sync(0xffffffffu, go, 0);
      tc_fence_after();
      if (!go) break;
      const int64_t row0 = static_cast<int64_t>(t / tiles_n) * BM;
      const int64_t col0 = static_cast<int64_t>(t % tiles_n) * BN;
      const int64_t row = row0 + quad * 32 + lane;
      float lsum = 0.f;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(buf * BN);
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tbase + ch * 32, r);
        tmem_ld_wait();
        const int64_t cbase = col0 + ch * 32;
        if (row < rows && cbase < cols) {
          if (cbase + 32 <= cols) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float acc[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) acc[q] = __uint_as_float(r[v * 8 + q]);
              epi_vec8(epi, row, cbase + v * 8, cols, acc, lsum);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (cbase + q < cols) epi_element(epi, row, cbase + q, cols, __uint_as_float(r[q]), lsum);
          }
        }
      }
      if (epi.kind == Epi::MseLoss) {
        // per-tile partial: the last of the four warps adds the warps' sums in a fixed order.
        // red[buf] / cnt[buf] are next touched two tiles later, which cannot start before all
        // four warps have released this accumulator below.
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        if (lane == 0) {
          red[buf * 4 + quad] = lsum;
          __threadfence_block();
          if (atomicAdd(&cnt[buf], 1) == 3) {
            __threadfence_block();
            epi.loss_partials[t] = ((red[buf * 4 + 0] + red[buf * 4 + 1]) + red[buf * 4 + 2]) +
                                   red[buf * 4 + 3];
            cnt[buf] = 0;
          }
        }
      }
      // the accumulator has been read: hand it back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acce + 8 * buf);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(L::TMEM_COLS));
  }
}

// ------------------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map of one operand. K-major: stored [n_rows, depth] -> dims {depth, n_rows},
// box {64, box_rows}. MN-major: stored [depth, n_rows] -> dims {n_rows, depth}, box {64, 64}.
bool make_map(CUtensorMap* map, omq_dtype dt, const GemmOperand& op, int64_t n_rows,
              int64_t depth, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2];
  cuuint32_t box[2];
  if (op.mn_major) {
    dims[0] = static_cast<cuuint64_t>(n_rows);
    dims[1] = static_cast<cuuint64_t>(depth);
    box[0] = 64;
    box[1] = BK;
  } else {
    dims[0] = static_cast<cuuint64_t>(depth);
    dims[1] = static_cast<cuuint64_t>(n_rows);
    box[0] = BK;
    box[1] = static_cast<cuuint32_t>(box_rows);
  }
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(op.ld) * 2};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType ty =
      dt == OMQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, ty, 2, const_cast<void*>(op.ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kBN = 256;
constexpr int kStages = 4;

}  // namespace tc

int64_t gemm_tc_tiles(int64_t rows, int64_t cols) {
  return ceil_div(rows, tc::BM) * ceil_div(cols, tc::kBN);
}

omq_status gemm_tc(omq_dtype dt, const GemmOperand& A, const GemmOperand& B, int64_t rows,
                   int64_t cols, int64_t depth, const GemmEpilogue& epi, int64_t* n_tiles,
                   cudaStream_t stream) {
  using namespace tc;
  if (dt != OMQ_BF16 && dt != OMQ_F16) return OMQ_ERR_DTYPE;
  CUtensorMap ma, mb;
  if (!make_map(&ma, dt, A, rows, depth, BM) || !make_map(&mb, dt, B, cols, depth, kBN)) {
    set_cuda_error(cudaErrorInvalidValue);
    return OMQ_ERR_CUDA;
  }
  const int64_t tiles_m = ceil_div(rows, BM), tiles_n = ceil_div(cols, kBN);
  const int64_t tiles = tiles_m * tiles_n;
  if (n_tiles) *n_tiles = tiles;
  auto kern = gemm_tc_kernel<kBN, kStages>;
  const int smem = Layout<kBN, kStages>::SMEM_BYTES;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) {
    set_cuda_error(attr_err);
    return OMQ_ERR_CUDA;
  }
  const int64_t sms = num_sms();
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  kern<<<grid, NUM_THREADS, smem, stream>>>(ma, mb, A.mn_major ? 1 : 0, B.mn_major ? 1 : 0,
                                            dt == OMQ_F16 ? 0u : 1u, rows, cols, depth, epi,
                                            static_cast<int>(tiles_n), static_cast<int>(tiles));
  return launch_status();
}

}  // namespace omq
