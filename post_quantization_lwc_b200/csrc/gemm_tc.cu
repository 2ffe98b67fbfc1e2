// 16-bit x 16-bit -> fp32 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// C[i, j] = sum_k A(i, k) B(j, k) over 256 x 256 output tiles computed by CTA pairs
// (clusters of 2, tcgen05 cta_group::2), persistent: each pair walks tiles p, p + pairs, ...
// Each CTA of a pair keeps half of every operand tile in its shared memory (A rows
// 128 r .. 128 r + 127 and B rows 128 r .. 128 r + 127 of the tile, r = rank in the pair),
// and the pair's 256 x 256 x 16 MMA reads both halves, so a CTA streams 32 KB per k-block of
// 64 instead of the 48 KB a single-CTA 128 x 256 tile needs. The accumulator rows of CTA r
// live in its own TMEM (2 x 256 columns: two tiles in flight).
// Warp roles (320 threads per CTA):
//   warp 0      TMA producer (one lane): loads this CTA's halves of each k-block into a
//               STAGES-deep ring (128-byte swizzle); both CTAs complete the leader's "full"
//               mbarrier (cta_group::2 copies).
//   warp 1      allocates TMEM (both CTAs, cta_group::2); in the leader CTA one lane issues
//               the pair's tcgen05.mma (M=256, N=256, K=16) and commits each consumed stage
//               to both CTAs' "empty" mbarriers and each finished tile to both CTAs'
//               accumulator "full" mbarriers (tcgen05.commit multicast to the pair).
//   warps 2..17 epilogue: warp w reads TMEM lanes 32 (w mod 4) .. + 31 (its accumulator rows)
//               and one 64-column quarter of the tile ((w - 2) / 4), 32 x 32 at a time
//               (tcgen05.ld), applies the fused epilogue (bias, MSE loss and residual, scaled
//               store, or the weight-side STE backward), then releases the accumulator.
// Operands may be K-major (row of the stored matrix runs along k) or MN-major (row runs
// along i / j), so the three contractions of the step read X, W and dY in their natural
// layouts without transposed copies:
//   forward   Y  = Xq  W^^T : A = Xq [M,K] K-major,        B = W^ [N,K] K-major
//   dW^       dW = dY^T Xq  : A = dY [M,N] MN-major,       B = Xq [M,K] MN-major
//   dXq       dX = dY W^    : A = dY [M,N] K-major,        B = W^ [N,K] MN-major
// Loads never multicast. Every mbarrier wait is bounded in time; on expiry the kernel raises
// the device error flag, every role stops, outstanding copies and MMAs are drained
// (bounded), and both CTAs meet at the final cluster barrier before releasing TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm_epilogue.cuh"
#include "ste_common.cuh"

namespace omq {

__device__ unsigned g_dev_error = 0;
// Longest time one barrier wait may take before the waiting kernel gives up (nanoseconds).
__device__ uint64_t g_wait_limit_ns = 2000000000ull;

cudaError_t take_device_error(unsigned* flag) {
  unsigned zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_dev_error, sizeof(unsigned));
  if (e == cudaSuccess && *flag) e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(unsigned));
  return e;
}

cudaError_t set_wait_limit(uint64_t ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}
cudaError_t get_wait_limit(uint64_t* ns) {
  return cudaMemcpyFromSymbol(ns, g_wait_limit_ns, sizeof(*ns));
}

namespace tc {

constexpr int TILE_M = 256;               // rows of C per CTA pair
constexpr int TILE_N = 256;               // columns of C per CTA pair
constexpr int HALF = 128;                 // rows of A and of B held by each CTA
constexpr int BK = 64;                    // 64 16-bit values = 128 bytes = one swizzle row
constexpr int UMMA_K = 16;

// Epilogue variants: EV = 0 the store / MSE epilogue (epi.kind), light, with 8 epilogue warps
// of 128 columns; EV = 1 / 2 the weight-side STE epilogue (BF16 / F16 weights; 3 / 4 the same
// without the LET column sums, 32 registers a thread fewer), the step's
// heaviest per-element arithmetic, with 16 epilogue warps of 64 columns (four per scheduler,
// 96 registers a thread). One kernel per variant keeps each within its register budget.
//
// DQB (2..8): the B operand is a weight given as packed DQB-bit codes with per-group step h
// and zero point z (omq_fold_pack's layout); four converter warps per CTA expand each
// k-block of codes into the 16-bit values (c - z) h, written straight into the stage in the
// layout the TMA would have produced, and only A is copied by TMA.
template <int EV, int DQB = 0>
struct Cfg {
  static constexpr int EPI_WARPS = EV ? 16 : 8;
  static constexpr int EPI_COLS = TILE_N * 4 / EPI_WARPS;   // accumulator columns per warp
  static constexpr int CONV_WARPS = DQB ? 8 : 0;     // two groups of four (alternate k-blocks)
  static constexpr int CONV_ARRIVALS = DQB ? 2 * 4 : 0;   // a stage's: one group, both CTAs
  static constexpr int NUM_THREADS = 32 * (2 + EPI_WARPS + CONV_WARPS);
  // The STE variants give a 4 KB shared slice to each epilogue warp (its 32 x 64 block of W,
  // staged by coalesced copies). Ring depth, measured on B200: 6 stages (EV 0) and 4 (STE)
  // ran the GEMMs 1-5% faster than 7 and 5, the smaller shared-memory carve-out leaving the
  // L1 room for the epilogue's row-per-thread accesses; a shared-memory transpose of the
  // accumulator chunks (coalesced global accesses) was slower again on the forward.
  static constexpr int STAGES = EV ? 4 : 6;
  static constexpr int WST = EV ? 32 * 64 * 2 : 0;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of this shared variable in CTA `rank` of the cluster (shared::cluster window).
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
// Arrive on a barrier of any CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// One bounded-time probe: the thread may be suspended (not spinning on issue slots) for up
// to kSuspendNs while the phase is still pending.
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Wait until the phase with the given parity has completed, for at most g_wait_limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned err_bit) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t limit = *const_cast<volatile uint64_t*>(&g_wait_limit_ns);
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > limit) {
      atomicOr(&g_dev_error, err_bit);
      return false;
    }
  }
  return true;
}
// The same bounded wait for phases that typically take microseconds (a whole tile's MMAs or
// epilogue): between probes the thread sleeps, so waiting warps leave the issue slots to the
// epilogue warps that share their scheduler.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, unsigned err_bit,
                                                uint32_t sleep_ns) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t limit = *const_cast<volatile uint64_t*>(&g_wait_limit_ns);
  for (uint32_t n = 1;; ++n) {
    __nanosleep(sleep_ns);
    if (mbar_try(bar, parity)) return true;
    if ((n & 15) == 0 && globaltimer() - t0 > limit) {
      atomicOr(&g_dev_error, err_bit);
      return false;
    }
  }
}
__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Copy of this CTA's part of a pair's stage into its own shared memory, completing the
// transaction on the leader CTA's barrier (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int x, int y, int w) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y), "r"(w)
      : "memory");
}
// One operand box: 2D (bmode 0) or 3D with the batch as the middle (1) or outer (2)
// coordinate; (x, y) are the 2D coordinates (inner, outer) of the unbatched operand.
template <bool BATCH>
__device__ __forceinline__ void tma_load_op(uint32_t dst, const CUtensorMap* map,
                                            uint32_t leader_bar, int x, int y, int bmode,
                                            int b) {
  if (!BATCH || bmode == 0) tma_load_2d_pair(dst, map, leader_bar, x, y);
  else if (bmode == 1) tma_load_3d_pair(dst, map, leader_bar, x, b, y);
  else tma_load_3d_pair(dst, map, leader_bar, x, y, b);
}

// The pair's tile t: batch, origin, and the k-blocks it contracts. Causal modes (square
// batches of attention, rows and columns both token positions):
//   1 skip tiles wholly above the diagonal (columns > rows): the lower-triangle tiles are
//     enumerated row by row, tn <= tm
//   2 the contraction index is a column position: k < row0 + TILE_M
//   3 the contraction index is a row position: k >= row0
struct TileWork {
  int b, row0, col0, kb0, kb1;
};
template <bool BATCH>
__device__ __forceinline__ TileWork tile_of(const TileSched& sc, int t, int nk) {
  TileWork w;
  if (!BATCH) {   // one problem, no causal structure
    const int tm = t / sc.tiles_n;
    w.b = 0;
    w.row0 = tm * TILE_M;
    w.col0 = (t - tm * sc.tiles_n) * TILE_N;
    w.kb0 = 0;
    w.kb1 = nk;
    return w;
  }
  w.b = t / sc.per_batch;
  const int u = t - w.b * sc.per_batch;
  int tm, tn;
  if (sc.causal == 1) {
    tm = static_cast<int>((sqrtf(8.f * static_cast<float>(u) + 1.f) - 1.f) * 0.5f);
    while ((tm + 1) * (tm + 2) / 2 <= u) ++tm;
    while (tm * (tm + 1) / 2 > u) --tm;
    tn = u - tm * (tm + 1) / 2;
  } else {
    tm = u / sc.tiles_n;
    tn = u - tm * sc.tiles_n;
  }
  w.row0 = tm * TILE_M;
  w.col0 = tn * TILE_N;
  w.kb0 = 0;
  w.kb1 = nk;
  if (sc.causal == 2) w.kb1 = min(nk, (w.row0 + TILE_M + BK - 1) / BK);
  if (sc.causal == 3) w.kb0 = w.row0 / BK;
  return w;
}

// One unit of a pair's work: a whole tile, or a run of k-blocks of a stream-K tile (split
// `split` of `nsplit`, the pairs in k order; at most two, since a run is longer than a tile's
// contraction).
struct Unit {
  TileWork w;
  int t;        // tile index (its loss partial slots are 2 t and 2 t + 1)
  int tsk;      // index among the stream-K tiles, or -1
  int split, nsplit;
};
// The pair's u-th unit: its whole tiles pair, pair + pairs, ... below dp_tiles, then its run
// [pair sk_len, (pair + 1) sk_len) of the stream-K tiles' k-blocks (tile by tile, in order).
template <bool BATCH>
__device__ __forceinline__ bool next_unit(const TileSched& sc, int pair, int pairs, int u, int nk,
                                          Unit& un) {
  const int t = pair + u * pairs;
  if (t < sc.dp_tiles) {
    un.w = tile_of<BATCH>(sc, t, nk);
    un.t = t;
    un.tsk = -1;
    un.split = 0;
    un.nsplit = 1;
    return true;
  }
  if (sc.sk_tiles == 0) return false;
  const int s = u - sc.dp_tiles / pairs;            // dp_tiles is a multiple of pairs here
  const int64_t total = static_cast<int64_t>(sc.sk_tiles) * nk;
  const int64_t lo = static_cast<int64_t>(pair) * sc.sk_len;
  const int64_t hi = lo + sc.sk_len < total ? lo + sc.sk_len : total;
  const int64_t ts = lo / nk + s;
  const int64_t a = lo > ts * nk ? lo : ts * nk;
  const int64_t b = hi < (ts + 1) * nk ? hi : (ts + 1) * nk;
  if (a >= b) return false;
  un.t = sc.dp_tiles + static_cast<int>(ts);
  un.w = tile_of<BATCH>(sc, un.t, nk);
  un.w.kb0 = static_cast<int>(a - ts * nk);
  un.w.kb1 = static_cast<int>(b - ts * nk);
  un.tsk = static_cast<int>(ts);
  const int64_t first = (ts * nk) / sc.sk_len, last = ((ts + 1) * nk - 1) / sc.sk_len;
  un.nsplit = static_cast<int>(last - first + 1);
  un.split = static_cast<int>(pair - first);
  return true;
}
// One CTA's half of a partial accumulator: 128 rows x 256 columns, stored warp by warp as
// [epilogue warp][column][lane] so that a warp's stores and loads are 128-byte lines.
constexpr int64_t kSkSlot = 128 * 256;
__device__ __forceinline__ int64_t sk_slot(int tsk, int split, uint32_t rank) {
  return ((static_cast<int64_t>(tsk) * 2 + split) * 2 + rank) * kSkSlot;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrive (once each) on the barrier at this shared offset in both CTAs of the pair, when all
// previously issued tcgen05 operations of this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}
__device__ __forceinline__ void umma_commit_local(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
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
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
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

// Descriptor of the k-slice `kk` (16 elements) of a 128-row operand half at `base`.
//  K-major: 128 rows of 128 bytes (64 k), 8-row swizzle atoms 1024 bytes apart; a k-slice
//           starts 32 bytes further along the row.
//  MN-major: 2 chunks of 64 rows(i/j) x 64 k, each BK rows of 128 bytes (one k per row),
//           chunks 8192 bytes apart (LBO); 8-k atoms 1024 bytes apart (SBO); a k-slice
//           starts 16 k-rows = 2048 bytes further.
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

// 16-byte asynchronous copy global -> shared (no multicast), its group commit and wait.
__device__ __forceinline__ void cp16_async(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// 8 weights of one row from their 16-bit storage.
template <bool F16>
__device__ __forceinline__ void unpack8(const uint4& q, float (&w)[8]) {
  const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (F16) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[j]));
      w[2 * j] = f.x;
      w[2 * j + 1] = f.y;
    } else {
      w[2 * j] = __uint_as_float(u[j] << 16);
      w[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
  }
}

// Weight-side straight-through backward fused into the dW^ GEMM: one warp's 32 rows (lane =
// row n) x 64 columns of the accumulator, whose value times out_scale is dW^[n, k]; dW^ is
// never stored. The group length is a multiple of 32, so each 32-column chunk lies in one
// group (h, z of row n). Per chunk and row the epilogue writes
//   gh_part[chunk, n] = sum dq (round(u) - u) over in-range elements + dq (code - z) over
//                       clipped ones                                   (G_h's share)
//   gc_part[chunk, n] = sum dq over clipped elements                   (G_z = -h * that)
// and, with LET, the chunk's column sums over the warp's 32 rows of (in range ? dq : 0) W,
// one partial row per 32-row block for d s. The group's own terms (its G_h, G_z, the logit
// gradients and the max / min elements' shares) are finished by ste_w_finish_kernel and
// ste_w_corr_kernel after the GEMM. Rows past the end read as zero weights and zero
// accumulators (the operand loads fill zeros) and store nothing.
template <bool F16, bool LETSUM>
__device__ __forceinline__ void ste_w_epilogue(const GemmEpilogue& epi, uint32_t tcol,
                                               int64_t wrow0, int64_t col0, int64_t rows,
                                               int64_t cols, int lane, const uint8_t* wst,
                                               const float* other, const float (&hz)[4]) {
  const SteWEpi& p = epi.ste;
  const int64_t row = wrow0 + lane;
  const bool valid = row < rows;
  // this warp's weight block was staged in wst (chunk j of row r at (j ^ (r & 7)) * 16 bytes)
  cp_wait_all();
  __syncwarp();
  const uint8_t* wrow = wst + lane * 128;
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    const int64_t k0 = col0 + 32 * c;
    if (k0 >= cols) break;                           // warp-uniform
    // h and z of this chunk's group (loaded before the accumulator wait)
    const float h = hz[2 * c], z = hz[2 * c + 1];
    const float hinv = __frcp_rn(h);
    float Gh = 0.f, Gc = 0.f;
    float ps[LETSUM ? 32 : 1];
    // the chunk's 32 accumulator columns: both 16-column loads in flight, one wait
    uint32_t r[32];
    __syncwarp();
    tmem_ld16(tcol + 32 * c, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
    tmem_ld16(tcol + 32 * c + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
    tmem_ld_wait();
    if (other) {   // a stream-K tile: add the other pair's partial (this warp's layout)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        r[i] = __float_as_uint(__uint_as_float(r[i]) + __ldcg(other + (32 * c + i) * 32 + lane));
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int q = 4 * c + v;                       // 8-column chunk of the warp's 64
      const uint4 wq = valid ? *reinterpret_cast<const uint4*>(wrow + ((q ^ (lane & 7)) << 4))
                             : make_uint4(0, 0, 0, 0);
      // without the LET sums there is no LET at all (s is NULL): W~ = W
      float w[8], sv[8], wt[8], rq[8];
      unpack8<F16>(wq, w);
      if (LETSUM && p.s) load_f8(p.s, col0 + 8 * q, sv);
      // round(W~ / h) as the forward takes it: the product with 1/h, branch-free, its
      // distance to the nearest integer checked; one warp-wide vote sends the rare lane
      // with a product near a half-integer (or a large quotient) to the exact quotient
      bool slow = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wt[i] = (LETSUM && p.s) ? __fmul_rn(w[i], sv[i]) : w[i];
        const float ua = __fmul_rn(wt[i], hinv);
        rq[i] = rne_small(ua);
        slow |= !(fabsf(ua) < 2048.f) || !(fabsf(__fsub_rn(ua, rq[i])) <= 0.499f);
      }
      if (__any_sync(0xffffffffu, slow)) {
        if (slow) {
#pragma unroll
          for (int i = 0; i < 8; ++i) rq[i] = round_quotient(wt[i], h, hinv);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float dq = epi.out_scale * __uint_as_float(r[8 * v + i]);
        const float lvl = __fadd_rn(rq[i], z);
        const bool inr = lvl >= 0.f && lvl <= p.Q;
        const float cl = fminf(fmaxf(lvl, 0.f), p.Q);
        Gh += dq * (inr ? (rq[i] - wt[i] * hinv) : (cl - z));
        Gc += inr ? 0.f : dq;
        if constexpr (LETSUM) ps[8 * v + i] = inr ? dq * w[i] : 0.f;
      }
    }
    if (valid) {
      p.gh_part[(k0 >> 5) * rows + row] = Gh;
      p.gc_part[(k0 >> 5) * rows + row] = Gc;
    }
    if constexpr (LETSUM) {
      const float cs = warp_column_sum32(ps, lane);
      if (wrow0 < rows) p.part_s[(wrow0 >> 5) * cols + k0 + lane] = cs;
    }
  }
}

// h and z of the groups of a warp's two 32-column chunks of the STE epilogue (row per lane),
// loaded ahead of the accumulator.
__device__ __forceinline__ void ste_w_prefetch(const SteWEpi& p, int64_t row, bool valid,
                                               int64_t col0, int64_t cols, float (&hz)[4]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int64_t k0 = col0 + 32 * c;
    hz[2 * c] = 1.f;
    hz[2 * c + 1] = 0.f;
    if (valid && k0 < cols) {
      const int64_t gi = row * p.ng + static_cast<int>(k0) / static_cast<int>(p.G);
      hz[2 * c] = p.h[gi];
      hz[2 * c + 1] = static_cast<float>(p.z[gi]);
    }
  }
}

// ---- dequantizing B producer ---------------------------------------------------------
// The 64 DQB-bit codes of one row's k-block: 8 * DQB bytes, a little-endian bit string
// (code j at bits j DQB .. j DQB + DQB - 1), loaded as DQB 8-byte words.
template <int DQB>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[2 * DQB + 1], int j) {
  const int bit = j * DQB, word = bit >> 5, sh = bit & 31;
  uint32_t v = w[word] >> sh;
  if (sh + DQB > 32) v |= w[word + 1] << (32 - sh);
  return v & ((1u << DQB) - 1u);
}
// 2^23 + code as a float, the code's byte placed in the low mantissa byte by one permute.
__device__ __forceinline__ float magic_byte(uint32_t bytes, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(bytes), "r"(0x4B000000u), "r"(sel));
  return __uint_as_float(r);
}
// The 8 codes of chunk j (columns 8 j .. 8 j + 7 of the k-block) as floats 2^23 + c, exact.
// Byte-aligned widths take one permute a code (after a mask for 2 and 4 bits); the others
// the generic bit-string read.
template <int DQB>
__device__ __forceinline__ void codes8(const uint32_t (&w)[2 * DQB + 1], int j, float (&f)[8]) {
  if constexpr (DQB == 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = magic_byte(w[2 * j + i / 4], 0x7440u + (i & 3));
  } else if constexpr (DQB == 4) {
    const uint32_t x = w[j];                       // codes 8 j .. 8 j + 7, two a byte
    const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = magic_byte(lo, 0x7440u + i);
      f[2 * i + 1] = magic_byte(hi, 0x7440u + i);
    }
  } else if constexpr (DQB == 2) {
    const uint32_t x = (w[j / 2] >> (16 * (j & 1))) & 0xFFFFu;   // 8 codes, four a byte
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t m = (x >> (2 * i)) & 0x0303u;    // codes i and i + 4 in bytes 0 and 1
      f[i] = magic_byte(m, 0x7440u);
      f[i + 4] = magic_byte(m, 0x7441u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(0x4B000000u | code_at<DQB>(w, 8 * j + i));
  }
}

__device__ __forceinline__ uint32_t pack_pair(float a, float b, bool f16) {
  if (f16) {
    const __half2 x = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&x);
  }
  const __nv_bfloat162 x = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&x);
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Walks a pair's k-blocks in the order the producer and the MMA take them (unit by unit).
template <bool BATCH>
struct KbCursor {
  Unit un;
  int u = 0, kb = 0;
  bool ok = false;
  __device__ __forceinline__ void start(const TileSched& sc, int pair, int pairs, int nk) {
    u = 0;
    ok = next_unit<BATCH>(sc, pair, pairs, 0, nk, un);
    kb = ok ? un.w.kb0 : 0;
  }
  __device__ __forceinline__ void step(const TileSched& sc, int pair, int pairs, int nk) {
    if (!ok) return;
    if (++kb >= un.w.kb1) {
      ++u;
      ok = next_unit<BATCH>(sc, pair, pairs, u, nk, un);
      kb = ok ? un.w.kb0 : 0;
    }
  }
};

// One thread's inputs of a k-block: the row's 64 codes and the step / zero point of the group
// holding its first column.
template <int DQB>
struct KbCodes {
  uint32_t w[2 * DQB + 1];
  float h, z;
  int64_t n;
  bool valid;
};
template <int DQB>
__device__ __forceinline__ void load_kb(const QuantB& q, int64_t n, bool valid, int kb,
                                        KbCodes<DQB>& c) {
  c.n = n;
  c.valid = valid;
  c.w[2 * DQB] = 0u;
  c.h = 0.f;
  c.z = 0.f;
  if (valid) {
    const uint2* src = reinterpret_cast<const uint2*>(q.packed + n * q.row_bytes +
                                                      static_cast<int64_t>(kb) * 8 * DQB);
#pragma unroll
    for (int i = 0; i < DQB; ++i) {
      const uint2 v = __ldg(src + i);
      c.w[2 * i] = v.x;
      c.w[2 * i + 1] = v.y;
    }
    // the group of the k-block's first column (32-bit divisions by a group count)
    const uint32_t g = q.kb_per_group ? static_cast<uint32_t>(kb) / static_cast<uint32_t>(q.kb_per_group)
                                      : static_cast<uint32_t>(kb) * 8u /
                                            static_cast<uint32_t>(q.chunks_per_group);
    c.h = __ldg(q.h + n * q.ng + g);
    c.z = static_cast<float>(__ldg(q.z + n * q.ng + g));
  } else {
#pragma unroll
    for (int i = 0; i < 2 * DQB; ++i) c.w[i] = 0u;
  }
}

// The converter warps: two groups of four, taking alternate k-blocks, so each group has two
// stages' time for one; each thread prefetches its next k-block's codes before it waits for
// and fills the current stage. A code c becomes float by its bits in the low mantissa of
// 2^23 (exact), so (c - z) h = (float(2^23 + c) - (2^23 + z)) h, two full-rate operations.
template <int DQB, bool BATCH, int STAGES>
__device__ __forceinline__ void convert_b(const GemmEpilogue& epi, const TileSched& sc, int pair,
                                          int pairs, int nk, uint32_t rank, int64_t cols,
                                          uint32_t fmt, uint32_t sbase, int stage_bytes,
                                          int a_bytes, uint32_t bar_full, uint32_t bar_empty,
                                          volatile int* abort_flag, int cthread) {
  const int ct = cthread & 127, grp = cthread >> 7, lane = cthread & 31;
  const bool f16 = fmt == 0;
  const QuantB& q = epi.qb;
  KbCursor<BATCH> cur, nxt;
  cur.start(sc, pair, pairs, nk);
  int it = 0;
  if (grp) {
    cur.step(sc, pair, pairs, nk);
    it = 1;
  }
  nxt = cur;
  nxt.step(sc, pair, pairs, nk);
  nxt.step(sc, pair, pairs, nk);
  auto row_of = [&](const KbCursor<BATCH>& c, bool& valid) {
    const int64_t n = static_cast<int64_t>(c.un.w.col0) + rank * HALF + ct;
    valid = n < cols;
    return n;
  };
  KbCodes<DQB> a, b;
  if (cur.ok) {
    bool v;
    const int64_t n = row_of(cur, v);
    load_kb<DQB>(q, n, v, cur.kb, a);
  }
  while (cur.ok) {
    if (nxt.ok) {                                   // the next k-block of this group, early
      bool v;
      const int64_t n = row_of(nxt, v);
      load_kb<DQB>(q, n, v, nxt.kb, b);
    }
    const int s = it % STAGES;
    const uint32_t ph = (it / STAGES) & 1;
    int ok = 1;
    if (lane == 0)
      ok = (mbar_wait(bar_empty + 8 * s, ph ^ 1, DEV_ERR_TMA_WAIT) && *abort_flag == 0) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      *abort_flag = 1;
      return;
    }
    const uint32_t b_row = sbase + s * stage_bytes + a_bytes + ct * 128;
    // groups narrower than a k-block (a group is a multiple of 8 columns): each 8-column
    // chunk finds its own; otherwise the whole k-block is the group of load_kb
    const bool split_groups = q.kb_per_group == 0;
    const uint32_t ch0 = static_cast<uint32_t>(cur.kb) * 8u;
    const uint32_t g0 = split_groups ? ch0 / static_cast<uint32_t>(q.chunks_per_group) : 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float hh = a.h, zz = a.z;
      if (split_groups) {
        const uint32_t g = (ch0 + j) / static_cast<uint32_t>(q.chunks_per_group);
        if (g != g0 && a.valid) {
          hh = __ldg(q.h + a.n * q.ng + g);
          zz = static_cast<float>(__ldg(q.z + a.n * q.ng + g));
        }
      }
      const float bz = 8388608.f + zz;              // exact: |z| < 2^22 for these codes
      float f[8];
      codes8<DQB>(a.w, j, f);
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // (c - z) exact, one rounding of the product: the pair on the f32x2 pipe
        const float2 d = __fadd2_rn(make_float2(f[2 * e], f[2 * e + 1]), make_float2(-bz, -bz));
        const float2 v = __fmul2_rn(d, make_float2(hh, hh));
        o[e] = pack_pair(v.x, v.y, f16);
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(b_row + ((j ^ (ct & 7)) << 4)),
                   "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(peer_addr(bar_full + 8 * s, 0));
    cur = nxt;
    a = b;
    it += 2;
    nxt.step(sc, pair, pairs, nk);
    nxt.step(sc, pair, pairs, nk);
  }
}

template <int STAGES, int EPI_WARPS, int WST>
struct Layout {
  static constexpr int A_BYTES = HALF * BK * 2;          // 16 KB
  static constexpr int B_BYTES = HALF * BK * 2;          // 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // this CTA's part of a stage
  static constexpr int WST_OFF = STAGES * STAGE_BYTES;   // epilogue warps' weight slices
  static constexpr int BAR_OFF = WST_OFF + EPI_WARPS * WST;
  // control block: barriers full[S], empty[S], acc_full[2], acc_empty[2], drain; tmem slot,
  // abort flag, the epilogue's per-warp loss partials [2][EPI_WARPS] and arrival counters [2]
  static constexpr int CTL_BYTES = 512;
  // and, for stream-K tiles, the epilogue warps' arrival barrier, the decision barrier and
  // the decision
  static constexpr int FULL = 0, EMPTY = 8 * STAGES, ACCF = 16 * STAGES, ACCE = ACCF + 16,
                       DRAIN = ACCE + 16, SLOT = DRAIN + 8, ABORT = SLOT + 4, RED = ABORT + 4,
                       CNT = RED + 8 * EPI_WARPS, SKA = CNT + 8, SKB = SKA + 8, SKF = SKB + 8,
                       CTL_END = SKF + 8;
  static_assert(SKA % 8 == 0, "mbarrier alignment");
  static_assert(CTL_END <= CTL_BYTES, "control block");
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + BAR_OFF + CTL_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * TILE_N;
};

// BATCH: a batched and / or causal schedule (attention); false compiles the plain tile loop.
template <int EV, bool BATCH, int DQB = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<EV, DQB>::NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int a_mn, int b_mn, uint32_t fmt, int64_t rows, int64_t cols, int64_t depth,
                   GemmEpilogue epi, TileSched sc) {
  using C = Cfg<EV, DQB>;
  constexpr int STAGES = C::STAGES, EPI_WARPS = C::EPI_WARPS, EPI_COLS = C::EPI_COLS;
  using L = Layout<STAGES, EPI_WARPS, C::WST>;
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
  const uint32_t bar_ska = sbase + L::BAR_OFF + L::SKA;
  const uint32_t bar_skb = sbase + L::BAR_OFF + L::SKB;
  volatile int* sk_flag = reinterpret_cast<volatile int*>(ctl + L::SKF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + L::SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + L::ABORT);
  volatile float* red = reinterpret_cast<volatile float*>(ctl + L::RED);  // [2][EPI_WARPS]
  int* cnt = reinterpret_cast<int*>(ctl + L::CNT);                           // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();          // 0 = leader of the pair
  const int pair = static_cast<int>(cluster_id());
  const int pairs = static_cast<int>(cluster_count());
  const int nk = static_cast<int>((depth + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // leader's: one expect_tx arrival + both CTAs' bytes (+ both CTAs' converter warps)
      mbar_init(bar_full + 8 * s, 1 + C::CONV_ARRIVALS);
      mbar_init(bar_empty + 8 * s, 1);    // the leader's commit, multicast to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);     // the leader's commit, multicast to both CTAs
      mbar_init(bar_acce + 8 * b, 2 * EPI_WARPS);   // leader's: every epilogue warp of both
      cnt[b] = 0;
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_ska, EPI_WARPS);      // every epilogue warp has stored its partial
    mbar_init(bar_skb, 1);              // the decision who finishes the tile is published
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync();            // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the prologue above touches only shared memory and TMEM: it may overlap the previous
  // kernel of the stream; operands and outputs wait for that kernel's completion
  pdl_wait();
  pdl_launch();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs)
    int it = 0;
    bool ok = true;
    Unit un;
    for (int u = 0; ok && next_unit<BATCH>(sc, pair, pairs, u, nk, un); ++u) {
      const TileWork& tw = un.w;
      const int row0 = tw.row0 + static_cast<int>(rank) * HALF;
      const int col0 = tw.col0 + static_cast<int>(rank) * HALF;
      for (int kb = tw.kb0; kb < tw.kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const bool got = mbar_wait(bar_empty + 8 * s, ph ^ 1, DEV_ERR_TMA_WAIT);
        if (*abort_flag || !got) {
          ok = false;
          break;
        }
        const uint32_t a_dst = sbase + s * L::STAGE_BYTES;
        const uint32_t b_dst = a_dst + L::A_BYTES;
        const uint32_t full_leader = peer_addr(bar_full + 8 * s, 0);
        if (rank == 0) mbar_expect_tx(bar_full + 8 * s, 2 * (DQB ? L::A_BYTES : L::STAGE_BYTES));
        const int k0 = kb * BK;
        if (a_mn) {
          for (int c = 0; c < HALF / 64; ++c)
            tma_load_op<BATCH>(a_dst + c * 8192, &tmA, full_leader, row0 + 64 * c, k0, sc.a_bmode, tw.b);
        } else {
          tma_load_op<BATCH>(a_dst, &tmA, full_leader, k0, row0, sc.a_bmode, tw.b);
        }
        if (DQB) {
          // B is written by the converter warps
        } else if (b_mn) {
          for (int c = 0; c < HALF / 64; ++c)
            tma_load_op<BATCH>(b_dst + c * 8192, &tmB, full_leader, col0 + 64 * c, k0, sc.b_bmode, tw.b);
        } else {
          tma_load_op<BATCH>(b_dst, &tmB, full_leader, k0, col0, sc.b_bmode, tw.b);
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      // the leader waits for the copies already in flight before the pair can exit
      if (rank == 0)
        for (int j = it - STAGES < 0 ? 0 : it - STAGES; j < it; ++j)
          mbar_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1, DEV_ERR_TMA_WAIT);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------- MMA issuer (leader CTA only)
    const uint32_t idesc = instr_desc(TILE_M, TILE_N, a_mn != 0, b_mn != 0, fmt);
    int it = 0, lt = 0;
    bool ok = true;
    Unit un;
    for (int u = 0; ok && next_unit<BATCH>(sc, pair, pairs, u, nk, un); ++u, ++lt) {
      const int buf = lt & 1;
      const uint32_t pa = ((lt >> 1) & 1) ^ 1;
      const bool got = mbar_wait(bar_acce + 8 * buf, pa, DEV_ERR_MMA_WAIT);
      if (*abort_flag || !got) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + static_cast<uint32_t>(buf * TILE_N);
      const TileWork& tw = un.w;
      for (int kb = tw.kb0; kb < tw.kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        // the stage was written by the copy engine (async proxy) and published through the
        // barrier: no tcgen05 fence is needed before the MMAs read it
        if (*abort_flag || !mbar_wait(bar_full + 8 * s, ph, DEV_ERR_MMA_WAIT)) {
          ok = false;
          break;
        }
        const uint32_t a_base = sbase + s * L::STAGE_BYTES;
        const uint32_t b_base = a_base + L::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
          umma_pair(d, operand_desc(a_base, a_mn != 0, kk), operand_desc(b_base, b_mn != 0, kk),
                    idesc, (kb != tw.kb0 || kk != 0) ? 1u : 0u);
        }
        umma_commit_pair(bar_empty + 8 * s);
      }
      if (!ok) break;
      umma_commit_pair(bar_accf + 8 * buf);
    }
    if (!ok) *abort_flag = 1;
    // every MMA issued above has completed once this commit arrives
    umma_commit_local(bar_drain);
    mbar_wait(bar_drain, 0, DEV_ERR_MMA_WAIT);
  } else if (DQB != 0 && warp >= 2 + EPI_WARPS) {
    // ---------------- converter warps (both CTAs): this CTA's 128 rows of B (output
    // columns col0 + 128 rank + ct), one row a thread, each k-block's codes expanded into the
    // stage's B half: row ct at ct * 128 bytes, its 8-value chunk j at (j ^ (ct & 7)) * 16
    // (the 128-byte swizzle of the TMA copies), then a fence to the async proxy and one
    // arrival per warp on the leader's full barrier
    if constexpr (DQB != 0) convert_b<DQB, BATCH, STAGES>(epi, sc, pair, pairs, nk, rank, cols,
                                                          fmt, sbase, L::STAGE_BYTES, L::A_BYTES,
                                                          bar_full, bar_empty, abort_flag,
                                                          threadIdx.x - 32 * (2 + EPI_WARPS));
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs: this CTA's 128 rows of the tile)
    const int ew = warp - 2;                         // 0 .. EPI_WARPS-1
    const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
    const int cq = ew >> 2;                          // columns 64*cq .. 64*cq+63 of the tile
    const uint32_t acce_leader = peer_addr(bar_acce, 0);
    int lt = 0, sk_n = 0;
    Unit un;
    for (int u = 0; next_unit<BATCH>(sc, pair, pairs, u, nk, un); ++u, ++lt) {
      const int buf = lt & 1;
      const TileWork& tw = un.w;
      const int t = un.t;
      const int64_t wrow0 = static_cast<int64_t>(tw.row0) + rank * HALF + quad * 32;
      const int64_t col0 = static_cast<int64_t>(tw.col0) + cq * EPI_COLS;
      const int64_t row = wrow0 + lane;
      if constexpr (EV != 0) {
        // this warp's 32 x 64 block of W into its shared slice by 16-byte copies, 4 rows of
        // 128 bytes a warp instruction (the epilogue reads a row per lane, which straight
        // from global memory touches 32 lines an instruction); chunk j of row r goes to
        // (j ^ (r & 7)) * 16, so those row-per-lane reads are free of bank conflicts. Issued
        // before the accumulator wait: the copies overlap the tile's MMAs.
        const SteWEpi& sp = epi.ste;
        const uint32_t slice = sbase + L::WST_OFF + ew * C::WST;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int m = lane + 32 * k, r = m >> 3, j = m & 7;
          const int64_t grow = wrow0 + r, gcol = col0 + 8 * j;
          if (grow < rows && gcol < cols)
            cp16_async(slice + r * 128 + ((j ^ (r & 7)) << 4),
                       static_cast<const uint16_t*>(sp.W) + grow * sp.K + gcol);
        }
        cp_commit();
      }
      float hz[4] = {1.f, 0.f, 1.f, 0.f};
      if constexpr (EV != 0) ste_w_prefetch(epi.ste, row, row < rows, col0, cols, hz);
      // one lane polls; the decision is broadcast so the warp-wide tcgen05.ld stays uniform
      int go = 0;
      if (lane == 0)
        go = (mbar_wait_sleep(bar_accf + 8 * buf, (lt >> 1) & 1, DEV_ERR_EPI_WAIT, 128) &&
              *abort_flag == 0)
                 ? 1 : 0;
      go = __shfl_sync(0xffffffffu, go, 0);
      tc_fence_after();
      if (!go) break;
      float lsum = 0.f;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(buf * TILE_N + cq * EPI_COLS);
      const float* other = nullptr;
      // (the weight-side STE variants never take the stream-K schedule: their contraction
      // is over tokens, and the host keeps it off for them)
      if (EV == 0 && un.nsplit > 1) {
        // A stream-K tile: both contributing pairs store their partial accumulator, then
        // count their arrival on the tile's counter; the second to arrive adds the first's
        // partial to its own and runs the epilogue (own + other: the same sum whichever
        // pair comes second), the first hands its accumulator back and moves on.
        float* mine = sc.sk_part + sk_slot(un.tsk, un.split, rank) + ew * EPI_COLS * 32;
#pragma unroll 1
        for (int ch = 0; ch < EPI_COLS / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tbase + ch * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) __stcg(mine + (ch * 32 + q) * 32 + lane, __uint_as_float(r[q]));
        }
        __threadfence();
        __syncwarp();
        const uint32_t ph = static_cast<uint32_t>(sk_n & 1);
        ++sk_n;
        if (lane == 0) mbar_arrive_local(bar_ska);
        if (ew == 0 && lane == 0) {
          int last = 0;
          if (mbar_wait(bar_ska, ph, DEV_ERR_EPI_WAIT)) {
            __threadfence();
            int* c = sc.sk_cnt + 2 * un.tsk + static_cast<int>(rank);
            last = atomicAdd(c, 1) == un.nsplit - 1;
            if (last) atomicExch(c, 0);       // counters are zero again after the launch
            __threadfence();
          } else {
            *abort_flag = 1;
          }
          *sk_flag = last;
          mbar_arrive_local(bar_skb);
        }
        int fin = 0;
        if (lane == 0)
          fin = mbar_wait_sleep(bar_skb, ph, DEV_ERR_EPI_WAIT, 32) && *abort_flag == 0
                    ? (*sk_flag ? 1 : 2) : 0;
        fin = __shfl_sync(0xffffffffu, fin, 0);
        if (fin != 1) {
          if constexpr (EV != 0) cp_wait_all();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acce_leader + 8 * buf);
          if (fin == 0) break;
          continue;
        }
        other = sc.sk_part + sk_slot(un.tsk, 1 - un.split, rank) + ew * EPI_COLS * 32;
      }
      if constexpr (EV != 0) {
        // EV 1 / 2: bfloat16 / float16 W with the LET column sums; 3 / 4: without
        ste_w_epilogue<EV == 2 || EV == 4, EV <= 2>(epi, tbase, wrow0, col0, rows, cols, lane,
                                smem + L::WST_OFF + ew * C::WST, other, hz);
      } else {
        float* const out_b = BATCH ? epi.out + static_cast<int64_t>(tw.b) * sc.out_bstride : epi.out;
        for (int ch = 0; ch < EPI_COLS / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tbase + ch * 32, r);
          tmem_ld_wait();
          if (other) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              r[q] = __float_as_uint(__uint_as_float(r[q]) +
                                     __ldcg(other + (ch * 32 + q) * 32 + lane));
          }
          const int64_t cbase = col0 + ch * 32;
          float rc[32];                      // this row's residuals of the chunk (or zeros)
#pragma unroll
          for (int q = 0; q < 32; ++q) rc[q] = 0.f;
          if (row < rows && cbase < cols) {
            if (cbase + 32 <= cols) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                float acc[8], res[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = __uint_as_float(r[v * 8 + q]);
                epi_vec8(epi, out_b, row, cbase + v * 8, cols, acc, lsum, res);
#pragma unroll
                for (int q = 0; q < 8; ++q) rc[v * 8 + q] = res[q];
              }
            } else {
#pragma unroll
              for (int q = 0; q < 32; ++q)
                if (cbase + q < cols)
                  rc[q] = epi_element(epi, out_b, row, cbase + q, cols, __uint_as_float(r[q]), lsum);
            }
          }
          // warp-uniform: the bias gradient's partials, for row blocks that hold rows
          if (epi.res_colsum && cbase < cols && wrow0 < rows) {
            const float cs = warp_column_sum32(rc, lane);
            if (cbase + lane < cols) epi.res_colsum[(wrow0 >> 5) * cols + cbase + lane] = cs;
          }
        }
      }
      if (epi.kind == Epi::MseLoss) {
        // per-half-tile partial: the last of this CTA's epilogue warps adds the warps' sums in
        // a fixed order. red[buf] / cnt[buf] are next touched two tiles later, which cannot
        // start before every warp has released this accumulator below.
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        if (lane == 0) {
          red[buf * EPI_WARPS + ew] = lsum;
          __threadfence_block();
          if (atomicAdd(&cnt[buf], 1) == EPI_WARPS - 1) {
            __threadfence_block();
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < EPI_WARPS; ++q) sum += red[buf * EPI_WARPS + q];
            epi.loss_partials[2 * t + rank] = sum;
            cnt[buf] = 0;
          }
        }
      }
      // the accumulator has been read: hand it back to the leader's MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader + 8 * buf);
    }
    if constexpr (EV != 0) cp_wait_all();    // no copy in flight when the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // no CTA leaves while its partner may still signal it
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(L::TMEM_COLS));
  }
}

// Bounded-wait probe: one thread initialises a shared-memory barrier for one arrival, arrives
// on it only when `arrive` is set, and waits for its first phase with the same bounded wait
// the GEMM's roles use. Without the arrival nothing can complete the phase, so the wait gives
// up after g_wait_limit_ns, raises DEV_ERR_PROBE_WAIT and the kernel returns normally: the
// path a GEMM takes when one of its barriers never completes, without a GEMM around it.
__global__ void wait_probe_kernel(int arrive) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  if (arrive) mbar_arrive_local(b);
  mbar_wait(b, 0, DEV_ERR_PROBE_WAIT);
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

// Tensor map of one operand, boxes of one CTA's half tile. K-major: stored [n_rows, depth]
// -> dims {depth, n_rows}, box {64, 128}. MN-major: stored [depth, n_rows] ->
// dims {n_rows, depth}, box {64, 64}. A batch of `count` operands `bstride` elements apart
// adds a third dimension of extent `count`, placed by stride: in the middle when the batch
// stride is below the row stride (heads side by side in a row), else outermost; the box is
// one problem deep. *bmode reports the placement (0: 2D).
bool make_map(CUtensorMap* map, omq_dtype dt, const GemmOperand& op, int64_t n_rows,
              int64_t depth, int64_t count, int64_t bstride, int* bmode) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d2[2];
  cuuint32_t b2[2];
  if (op.mn_major) {
    d2[0] = static_cast<cuuint64_t>(n_rows);
    d2[1] = static_cast<cuuint64_t>(depth);
    b2[0] = 64;
    b2[1] = BK;
  } else {
    d2[0] = static_cast<cuuint64_t>(depth);
    d2[1] = static_cast<cuuint64_t>(n_rows);
    b2[0] = BK;
    b2[1] = HALF;
  }
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(op.ld) * 2;
  const CUtensorMapDataType ty =
      dt == OMQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r;
  if (count <= 1) {
    *bmode = 0;
    cuuint64_t strides[1] = {row_bytes};
    r = fn(map, ty, 2, const_cast<void*>(op.ptr), d2, strides, b2, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t batch_bytes = static_cast<cuuint64_t>(bstride) * 2;
    cuuint64_t d3[3], st3[2];
    cuuint32_t b3[3];
    if (batch_bytes < row_bytes) {
      *bmode = 1;
      d3[0] = d2[0]; d3[1] = static_cast<cuuint64_t>(count); d3[2] = d2[1];
      st3[0] = batch_bytes; st3[1] = row_bytes;
      b3[0] = b2[0]; b3[1] = 1; b3[2] = b2[1];
    } else {
      *bmode = 2;
      d3[0] = d2[0]; d3[1] = d2[1]; d3[2] = static_cast<cuuint64_t>(count);
      st3[0] = row_bytes; st3[1] = batch_bytes;
      b3[0] = b2[0]; b3[1] = b2[1]; b3[2] = 1;
    }
    r = fn(map, ty, 3, const_cast<void*>(op.ptr), d3, st3, b3, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

static_assert(Layout<Cfg<0>::STAGES, Cfg<0>::EPI_WARPS, Cfg<0>::WST>::SMEM_BYTES <= 232448, "smem");
static_assert(Layout<Cfg<1>::STAGES, Cfg<1>::EPI_WARPS, Cfg<1>::WST>::SMEM_BYTES <= 232448, "smem");
static_assert(Cfg<0, 4>::NUM_THREADS == 576, "converter warps");

using GemmKernel = void (*)(CUtensorMap, CUtensorMap, int, int, uint32_t, int64_t, int64_t,
                            int64_t, GemmEpilogue, TileSched);

struct KernelChoice {
  GemmKernel fn;
  int threads, smem;
};

template <int EV, bool BATCH = false, int DQB = 0>
KernelChoice choice() {
  using C = Cfg<EV, DQB>;
  return {gemm_tc_kernel<EV, BATCH, DQB>, C::NUM_THREADS,
          Layout<C::STAGES, C::EPI_WARPS, C::WST>::SMEM_BYTES};
}

// Opt each kernel variant into the large dynamic shared memory once.
cudaError_t kernel_attr(GemmKernel k, int smem) {
  static std::mutex mu;
  static GemmKernel done[16] = {};
  static int n_done = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i] == k) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && n_done < 16) done[n_done++] = k;
  return e;
}

}  // namespace tc

omq_status launch_wait_probe(int arrive, cudaStream_t stream) {
  tc::wait_probe_kernel<<<1, 1, 0, stream>>>(arrive);
  return launch_status();
}

// Loss partial slots: one per 128-row half of each 256 x 256 output tile.
int64_t gemm_tc_tiles(int64_t rows, int64_t cols) {
  return 2 * ceil_div(rows, tc::TILE_M) * ceil_div(cols, tc::TILE_N);
}

namespace {
// Scratch of `skt` stream-K tiles: the arrival counters (2 per tile), then the partial
// accumulators (2 splits x 2 CTAs x 128 x 256 floats per tile).
size_t sk_counter_bytes(int64_t skt) { return static_cast<size_t>((skt * 2 * 4 + 255) / 256 * 256); }
size_t sk_need(int64_t skt) {
  return sk_counter_bytes(skt) + static_cast<size_t>(skt) * 4 * tc::kSkSlot * sizeof(float);
}
}  // namespace

// The stream-K region holds fewer than two waves of tiles (the last whole wave and the tail).
// Sized for any contraction depth: the depth decides at launch whether the schedule is used.
size_t gemm_tc_sk_bytes(int64_t rows, int64_t cols) {
  const int64_t tiles = ceil_div(rows, tc::TILE_M) * ceil_div(cols, tc::TILE_N);
  const int64_t pairs = num_sms() / 2;
  if (tiles <= pairs) return 0;
  const int64_t skt = tiles < 2 * pairs - 1 ? tiles : 2 * pairs - 1;
  return sk_need(skt);
}

omq_status gemm_tc(omq_dtype dt, const GemmOperand& A, const GemmOperand& B, int64_t rows,
                   int64_t cols, int64_t depth, const GemmEpilogue& epi, int64_t* n_tiles,
                   cudaStream_t stream, const GemmBatch* batch) {
  using namespace tc;
  if (dt != OMQ_BF16 && dt != OMQ_F16) return OMQ_ERR_DTYPE;
  const int64_t count = batch ? batch->count : 1;
  const int causal = batch ? batch->causal : 0;
  if (count < 1 || causal < 0 || causal > 3) return OMQ_ERR_SHAPE;
  if ((count > 1 || causal) && epi.kind != Epi::StoreF32) return OMQ_ERR_UNSUPPORTED;
  if (causal && rows != (causal == 1 ? cols : depth)) return OMQ_ERR_SHAPE;
  CUtensorMap ma, mb;
  int amode = 0, bmode = 0;
  if (!make_map(&ma, dt, A, rows, depth, count, batch ? batch->a_stride : 0, &amode) ||
      !make_map(&mb, dt, B, cols, depth, count, batch ? batch->b_stride : 0, &bmode)) {
    set_cuda_error(cudaErrorInvalidValue);
    return OMQ_ERR_CUDA;
  }
  const int64_t tiles_m = ceil_div(rows, TILE_M), tiles_n = ceil_div(cols, TILE_N);
  const int64_t per = causal == 1 ? tiles_m * (tiles_m + 1) / 2 : tiles_m * tiles_n;
  const int64_t tiles = per * count;
  if (tiles > (int64_t(1) << 30)) return OMQ_ERR_SHAPE;
  if (n_tiles) *n_tiles = 2 * tiles;
  KernelChoice kc = (count > 1 || causal) ? choice<0, true>() : choice<0>();
  if (epi.kind == Epi::SteW) {
    if (!ste_fusable(epi.ste.G) || (epi.ste.wdt != OMQ_BF16 && epi.ste.wdt != OMQ_F16))
      return OMQ_ERR_SHAPE;
    const bool letsum = epi.ste.part_s != nullptr || epi.ste.s != nullptr;
    kc = epi.ste.wdt == OMQ_F16 ? (letsum ? choice<2>() : choice<4>())
                                : (letsum ? choice<1>() : choice<3>());
  }
  const cudaError_t attr_err = kernel_attr(kc.fn, kc.smem);
  if (attr_err != cudaSuccess) {
    set_cuda_error(attr_err);
    return OMQ_ERR_CUDA;
  }
  TileSched sc{static_cast<int>(tiles_m), static_cast<int>(tiles_n), static_cast<int>(per),
               static_cast<int>(tiles), causal, amode, bmode,
               batch ? batch->out_stride : 0};
  const int64_t max_pairs = num_sms() / 2;
  const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
  // Stream-K tail: when the last wave of whole tiles would leave more than a fifth of the
  // pairs idle, the last whole wave and the tail (fewer than 2 waves of tiles) are shared
  // out as equal runs of k-blocks, longer than one tile's contraction, so every tile of the
  // region has one or two contributing pairs. Only for long contractions (at least
  // kSkMinBlocks k-blocks) with at least one whole wave ahead of the region: measured on
  // B200, the split tiles' partial stores and the staggered k positions of the pairs cost
  // more than the idle tail saves when a tile's contraction is short (4096-deep: forward
  // 78 -> 98 us at 2048 x 4096) or when every tile of the problem is in the region (the
  // block's 22016-deep dX GEMM over 128 tiles got slower), and less on the down_proj forward
  // (13824-deep, 160 tiles: 287 -> 248 us).
  sc.dp_tiles = static_cast<int>(tiles);
  sc.sk_tiles = 0;
  sc.sk_len = 0;
  sc.sk_part = nullptr;
  sc.sk_cnt = nullptr;
  const int64_t nk = ceil_div(depth, BK);
  const int64_t rem = tiles % pairs;
  constexpr int64_t kSkMinBlocks = 128;
  if (count == 1 && !causal && epi.kind != Epi::SteW && epi.sk_scratch && tiles >= 2 * pairs &&
      rem != 0 && 5 * rem <= 4 * pairs && nk >= kSkMinBlocks) {
    const int64_t dp = (tiles / pairs - 1) * pairs, skt = tiles - dp;
    if (sk_need(skt) <= epi.sk_bytes) {
      sc.dp_tiles = static_cast<int>(dp);
      sc.sk_tiles = static_cast<int>(skt);
      sc.sk_len = ceil_div(skt * nk, pairs);
      sc.sk_cnt = static_cast<int*>(epi.sk_scratch);
      sc.sk_part = reinterpret_cast<float*>(static_cast<char*>(epi.sk_scratch) +
                                            sk_counter_bytes(skt));
      const cudaError_t me = cudaMemsetAsync(sc.sk_cnt, 0, static_cast<size_t>(skt) * 2 * 4, stream);
      if (me != cudaSuccess) {
        set_cuda_error(me);
        return OMQ_ERR_CUDA;
      }
    }
  }
  launch_k(kc.fn, static_cast<unsigned>(2 * pairs), kc.threads, kc.smem, stream,
      ma, mb, A.mn_major ? 1 : 0, B.mn_major ? 1 : 0, dt == OMQ_F16 ? 0u : 1u, rows, cols, depth,
      epi, sc);
  return launch_status();
}

omq_status gemm_tc_qb(omq_dtype dt, const GemmOperand& A, int64_t rows, int64_t cols,
                      int64_t depth, int bits, const GemmEpilogue& epi, cudaStream_t stream) {
  using namespace tc;
  if (dt != OMQ_BF16 && dt != OMQ_F16) return OMQ_ERR_DTYPE;
  if (A.mn_major || epi.kind != Epi::StoreF32 || depth % BK) return OMQ_ERR_UNSUPPORTED;
  if (bits < 2 || bits > 8) return OMQ_ERR_BITS;
  CUtensorMap ma;
  int amode = 0;
  if (!make_map(&ma, dt, A, rows, depth, 1, 0, &amode)) {
    set_cuda_error(cudaErrorInvalidValue);
    return OMQ_ERR_CUDA;
  }
  const int64_t tiles_m = ceil_div(rows, TILE_M), tiles_n = ceil_div(cols, TILE_N);
  const int64_t tiles = tiles_m * tiles_n;
  if (tiles > (int64_t(1) << 30)) return OMQ_ERR_SHAPE;
  KernelChoice kc{};
  switch (bits) {
    case 2: kc = choice<0, false, 2>(); break;
    case 3: kc = choice<0, false, 3>(); break;
    case 4: kc = choice<0, false, 4>(); break;
    case 5: kc = choice<0, false, 5>(); break;
    case 6: kc = choice<0, false, 6>(); break;
    case 7: kc = choice<0, false, 7>(); break;
    default: kc = choice<0, false, 8>(); break;
  }
  const cudaError_t attr_err = kernel_attr(kc.fn, kc.smem);
  if (attr_err != cudaSuccess) {
    set_cuda_error(attr_err);
    return OMQ_ERR_CUDA;
  }
  TileSched sc{static_cast<int>(tiles_m), static_cast<int>(tiles_n), static_cast<int>(tiles),
               static_cast<int>(tiles), 0, amode, 0, 0};
  sc.dp_tiles = static_cast<int>(tiles);
  sc.sk_tiles = 0;
  sc.sk_len = 0;
  sc.sk_part = nullptr;
  sc.sk_cnt = nullptr;
  const int64_t max_pairs = num_sms() / 2;
  const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
  // the B tensor map is not read (B comes from the converter warps): A's map stands in
  launch_k(kc.fn, static_cast<unsigned>(2 * pairs), kc.threads, kc.smem, stream,
      ma, ma, 0, 0, dt == OMQ_F16 ? 0u : 1u, rows, cols, depth, epi, sc);
  return launch_status();
}

}  // namespace omq
