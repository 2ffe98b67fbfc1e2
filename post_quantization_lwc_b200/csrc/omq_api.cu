// The libomq C ABI: host-side validation, workspace layout and launch sequencing of the
// fake-quantized linear calibration step. Nothing here allocates device memory.
#include <atomic>
#include <cstdio>
#include <mutex>
#include <vector>

#include "omq_internal.cuh"

namespace omq {

namespace {
thread_local int t_last_cuda_error = 0;

constexpr int64_t kMaxGroupLarge = 16384;   // group staged in shared memory (per group / row)
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int kRowsSmallW = 128;            // rows per block, weight STE, lane-parallel groups
constexpr int kRowsLargeW = 16;             // rows per block, weight STE, larger groups
constexpr int kRowsX = 64;                  // tokens per block, activation STE column sums
constexpr int kRowsColsum = 64;             // rows per block of the dY column sums
constexpr int kRowsFusedW = 32;             // rows per partial, weight STE in the dW^ epilogue

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

int64_t rows_per_block_w(int64_t group) { return small_group(group) ? kRowsSmallW : kRowsLargeW; }

// The weight-side STE runs inside the dW^ GEMM's epilogue for 16-bit operands and weights
// and group lengths that are multiples of 32 (per-channel groups included); otherwise it is
// a separate kernel reading a stored dW^.
bool fused_ste_w(omq_dtype op_dt, omq_dtype wdt, int64_t group) {
  return op_dt != OMQ_F32 && wdt != OMQ_F32 && ste_fusable(group);
}

struct BwdLayout {
  size_t dbt_part, dbt, dwhat, dxq, part_ws, part_wd, part_xs, part_xd, rowstat, red;
  size_t gh_part, gc_part, emax, emin;   // fused weight-side STE (group a multiple of 32)
  size_t sk_w, sk_w_bytes, sk_x, sk_x_bytes;   // stream-K scratch of the dW^ and dXq GEMMs
  size_t total;
  int64_t rb_colsum, rb_w, rb_x;
};

BwdLayout bwd_layout(int64_t M, int64_t N, int64_t K, int64_t group) {
  BwdLayout L{};
  L.rb_colsum = ceil_div(M, kRowsColsum);
  // enough partial rows for either weight-side STE (the fused one writes one per 32 rows)
  L.rb_w = ceil_div(N, rows_per_block_w(group));
  if (ste_fusable(group) && ceil_div(N, kRowsFusedW) > L.rb_w) L.rb_w = ceil_div(N, kRowsFusedW);
  L.rb_x = ceil_div(M, kRowsX);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  // dB~ partials: per 64-row block (colsum kernel) or per 32-row block (the forward GEMM's
  // residual column sums)
  L.dbt_part = take(sizeof(float) * ceil_div(M, 32) * N);
  L.dbt = take(sizeof(float) * N);
  L.dwhat = take(sizeof(float) * N * K);
  L.dxq = take(sizeof(float) * M * K);
  L.part_ws = take(sizeof(float) * L.rb_w * K);
  L.part_wd = take(sizeof(float) * L.rb_w * K);
  L.part_xs = take(sizeof(float) * L.rb_x * K);
  L.part_xd = take(sizeof(float) * L.rb_x * K);
  L.rowstat = take(sizeof(float) * 2 * M);
  L.red = take(sizeof(double) * 2 * kReduceChunks * (N > K ? N : K));
  const bool fusable = ste_fusable(group);
  L.gh_part = take(fusable ? sizeof(float) * (K / 32) * N : 0);
  L.gc_part = take(fusable ? sizeof(float) * (K / 32) * N : 0);
  L.emax = take(fusable ? sizeof(float) * N * (K / group) : 0);
  L.emin = take(fusable ? sizeof(float) * N * (K / group) : 0);
  // the two backward GEMMs may run at the same time (two streams): one region each
  L.sk_w_bytes = gemm_tc_sk_bytes(N, K);
  L.sk_w = take(L.sk_w_bytes);
  L.sk_x_bytes = gemm_tc_sk_bytes(M, K);
  L.sk_x = take(L.sk_x_bytes);
  L.total = off;
  return L;
}

// Forward workspace: the per-tile loss partials, then the GEMM's stream-K scratch.
size_t fwd_partial_bytes(int64_t M, int64_t N) {
  int64_t t = gemm_tc_tiles(M, N);
  int64_t t2 = gemm_f32_simt_tiles(M, N);
  return align256(sizeof(float) * static_cast<size_t>(t > t2 ? t : t2));
}
size_t fwd_bytes(int64_t M, int64_t N) {
  return fwd_partial_bytes(M, N) + align256(gemm_tc_sk_bytes(M, N));
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

bool dtype_ok(omq_dtype d) { return d == OMQ_F32 || d == OMQ_BF16 || d == OMQ_F16; }
bool wbits_ok(int b) { return b >= 2 && b <= 8; }
bool abits_ok(int b) { return b == 2 || b == 3 || b == 4 || b == 6 || b == 8 || b == 16; }
bool a16(const void* p) { return p == nullptr || aligned16(p); }

#define OMQ_TRY(expr)                 \
  do {                                \
    omq_status _s = (expr);           \
    if (_s != OMQ_OK) return _s;      \
  } while (0)

// Optional per-phase event recording of omq_calib_step (see OMQ_PH_* in omq.h).
struct Phases {
  void* const* ev = nullptr;
  cudaStream_t st = nullptr;
  omq_status mark(int i) const {
    if (!ev) return OMQ_OK;
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st);
    if (e != cudaSuccess) {
      t_last_cuda_error = static_cast<int>(e);
      return OMQ_ERR_CUDA;
    }
    return OMQ_OK;
  }
};

omq_status check_lwc(const void* W, omq_dtype wdt, int64_t N, int64_t K, int64_t group, int bits,
                     const float* gl, const float* bl, const float* s, omq_dtype hat_dt,
                     const void* W_hat, const void* codes, const void* h, const void* z) {
  if (!W || !gl || !bl || !h || !z) return OMQ_ERR_NULL;
  if (!dtype_ok(wdt) || !dtype_ok(hat_dt)) return OMQ_ERR_DTYPE;
  if (!wbits_ok(bits)) return OMQ_ERR_BITS;
  if (N < 1 || K < 8 || group < 8 || N > kMaxDim || K > kMaxDim) return OMQ_ERR_SHAPE;
  if (group % 8 || K % group) return OMQ_ERR_SHAPE;
  if (!small_group(group) && group > kMaxGroupLarge) return OMQ_ERR_SHAPE;
  if (!a16(W) || !a16(W_hat) || !a16(codes) || !a16(s)) return OMQ_ERR_ALIGN;
  return OMQ_OK;
}

}  // namespace

void set_cuda_error(cudaError_t e) { t_last_cuda_error = static_cast<int>(e); }

omq_status SideStream::fork(cudaStream_t main) const {
  cudaError_t e = cudaEventRecord(fork_ev, main);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, fork_ev, 0);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  return OMQ_OK;
}

omq_status SideStream::join(cudaStream_t main) const {
  cudaError_t e = cudaEventRecord(join_ev, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(main, join_ev, 0);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  return OMQ_OK;
}

const SideStream* side_stream() {
  thread_local std::vector<SideStream> per_device;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return nullptr;
  }
  if (static_cast<int>(per_device.size()) <= dev) per_device.resize(dev + 1);
  SideStream& ss = per_device[dev];
  if (!ss.s) {
    SideStream n;
    e = cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.fork_ev, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.join_ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      set_cuda_error(e);
      return nullptr;
    }
    ss = n;
  }
  return &ss;
}

static std::atomic<uint64_t> g_launches{0};

omq_status launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  return OMQ_OK;
}

int num_sms() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

}  // namespace omq

using namespace omq;

extern "C" {

const char* omq_status_str(int status) {
  switch (status) {
    case OMQ_OK: return "ok";
    case OMQ_ERR_NULL: return "required pointer is NULL";
    case OMQ_ERR_SHAPE: return "invalid shape";
    case OMQ_ERR_DTYPE: return "unsupported dtype";
    case OMQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case OMQ_ERR_BITS: return "bit width out of range";
    case OMQ_ERR_WORKSPACE: return "workspace missing or too small";
    case OMQ_ERR_CUDA: return "CUDA error";
    case OMQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case OMQ_ERR_TIMEOUT: return "device barrier wait timed out";
    default: return "unknown status";
  }
}

int omq_last_cuda_error(void) { return t_last_cuda_error; }

int omq_version(void) { return 10000; }

omq_status omq_set_wait_limit_ns(uint64_t ns) {
  if (ns < 1000000ull || ns > 60000000000ull) return OMQ_ERR_SHAPE;
  const cudaError_t e = set_wait_limit(ns);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  return OMQ_OK;
}

uint64_t omq_wait_limit_ns(void) {
  uint64_t ns = 0;
  return get_wait_limit(&ns) == cudaSuccess ? ns : 0;
}

omq_status omq_wait_probe(int arrive, omq_stream_t stream) {
  return launch_wait_probe(arrive != 0, reinterpret_cast<cudaStream_t>(stream));
}

omq_status omq_sync_check(omq_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  unsigned flag = 0;
  e = take_device_error(&flag);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  return flag ? OMQ_ERR_TIMEOUT : OMQ_OK;
}

omq_status omq_lwc_quant(const void* W, omq_dtype wdt, int64_t N, int64_t K, int64_t group,
                         int bits, const float* gamma_logit, const float* beta_logit,
                         const float* s, void* W_hat, omq_dtype hat_dt, float* h, int32_t* z,
                         uint8_t* codes, omq_range* grp_range, omq_stream_t stream) {
  OMQ_TRY(check_lwc(W, wdt, N, K, group, bits, gamma_logit, beta_logit, s, hat_dt, W_hat, codes,
                    h, z));
  LwcParams p{W, wdt, N, K, group, K / group, static_cast<float>((1 << bits) - 1), gamma_logit,
              beta_logit, s, W_hat, hat_dt, h, z, codes, grp_range, nullptr, bits};
  return launch_lwc(p, reinterpret_cast<cudaStream_t>(stream));
}

omq_status omq_fold_pack(const void* W, omq_dtype wdt, int64_t N, int64_t K, int64_t group,
                         int bits, const float* gamma_logit, const float* beta_logit,
                         const float* s, uint8_t* packed, float* h, int32_t* z,
                         omq_stream_t stream) {
  if (!packed) return OMQ_ERR_NULL;
  OMQ_TRY(check_lwc(W, wdt, N, K, group, bits, gamma_logit, beta_logit, s, OMQ_F32, nullptr,
                    packed, h, z));
  LwcParams p{W, wdt, N, K, group, K / group, static_cast<float>((1 << bits) - 1), gamma_logit,
              beta_logit, s, nullptr, OMQ_F32, h, z, nullptr, nullptr, packed, bits};
  return launch_lwc(p, reinterpret_cast<cudaStream_t>(stream));
}

omq_status omq_let_apply(const void* X, omq_dtype xdt, int64_t M, int64_t K, const float* s,
                         const float* delta, int abits, void* Xq, omq_dtype xq_dt, float* h_a,
                         int32_t* z_a, omq_range* tok_range, const void* W, omq_dtype wdt,
                         int64_t N, const float* B, float* B_tilde, omq_stream_t stream) {
  if (!X || !Xq) return OMQ_ERR_NULL;
  if (!dtype_ok(xdt) || !dtype_ok(xq_dt)) return OMQ_ERR_DTYPE;
  if (!abits_ok(abits)) return OMQ_ERR_BITS;
  if (M < 1 || K < 8 || K % 8 || M > kMaxDim || K > kMaxDim) return OMQ_ERR_SHAPE;
  if (abits < 16 && K > 49152) return OMQ_ERR_SHAPE;
  if (!a16(X) || !a16(Xq) || !a16(s) || !a16(delta)) return OMQ_ERR_ALIGN;
  if (B_tilde) {
    if (delta && !W) return OMQ_ERR_NULL;
    if (N < 1 || N > kMaxDim) return OMQ_ERR_SHAPE;
    if (delta && !dtype_ok(wdt)) return OMQ_ERR_DTYPE;
    if (!a16(W)) return OMQ_ERR_ALIGN;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LetParams p{X, xdt, M, K, s, delta, static_cast<float>((1 << (abits < 16 ? abits : 1)) - 1), Xq,
              xq_dt, h_a, z_a, tok_range};
  OMQ_TRY(launch_let(p, abits, st));
  if (B_tilde) OMQ_TRY(launch_let_bias(W, wdt, N, K, delta, B, B_tilde, st));
  return OMQ_OK;
}

size_t omq_fwd_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)K;
  if (M < 1 || N < 1) return 0;
  return fwd_bytes(M, N);
}

static omq_status run_gemm(omq_dtype dt, const GemmOperand& A, const GemmOperand& B, int64_t rows,
                           int64_t cols, int64_t depth, const GemmEpilogue& epi, int64_t* tiles,
                           cudaStream_t st) {
  if (dt == OMQ_F32) return gemm_f32_simt(A, B, rows, cols, depth, epi, tiles, st);
  return gemm_tc(dt, A, B, rows, cols, depth, epi, tiles, st);
}

// The forward GEMM and, unless loss_stream is given, the loss reduction after it on the same
// stream; with loss_stream the reduction runs there (forked after the GEMM; the caller joins).
static omq_status fwd_impl(const void* Xq, const void* W_hat, omq_dtype dt, int64_t M, int64_t N,
                           int64_t K, const float* B_tilde, const float* Y_ref, float* Y, void* dY,
                           float* loss, void* workspace, size_t ws_bytes, omq_stream_t stream,
                           const Phases& ph, const SideStream* loss_stream = nullptr,
                           float* res_colsum = nullptr) {
  if (!Xq || !W_hat) return OMQ_ERR_NULL;
  if (!dtype_ok(dt)) return OMQ_ERR_DTYPE;
  if (M < 1 || N < 8 || K < 8 || N % 8 || K % 8 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
    return OMQ_ERR_SHAPE;
  if (Y_ref) {
    if (!dY) return OMQ_ERR_NULL;
  } else {
    if (!Y) return OMQ_ERR_NULL;
    if (dY || loss) return OMQ_ERR_NULL;
  }
  if (!a16(Xq) || !a16(W_hat) || !a16(B_tilde) || !a16(Y_ref) || !a16(Y) || !a16(dY))
    return OMQ_ERR_ALIGN;
  if (Y_ref && (!workspace || ws_bytes < fwd_bytes(M, N))) return OMQ_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  GemmOperand A{Xq, K, false}, B{W_hat, K, false};
  GemmEpilogue epi{};
  epi.bias = B_tilde;
  const size_t part_bytes = fwd_partial_bytes(M, N);
  if (workspace && ws_bytes > part_bytes) {
    epi.sk_scratch = static_cast<char*>(workspace) + part_bytes;
    epi.sk_bytes = ws_bytes - part_bytes;
  }
  if (Y_ref) {
    epi.kind = Epi::MseLoss;
    epi.out = Y;
    epi.y_ref = Y_ref;
    epi.dy = dY;
    epi.dy_dt = dt;
    epi.loss_partials = static_cast<float*>(workspace);
    if (dt != OMQ_F32) epi.res_colsum = res_colsum;
  } else {
    epi.kind = Epi::StoreF32;
    epi.out = Y;
    epi.out_scale = 1.f;
  }
  int64_t tiles = 0;
  OMQ_TRY(ph.mark(OMQ_PH_FWD_GEMM));
  OMQ_TRY(run_gemm(dt, A, B, M, N, K, epi, &tiles, st));
  OMQ_TRY(ph.mark(OMQ_PH_LOSS));
  if (Y_ref && loss) {
    cudaStream_t ls = st;
    if (loss_stream) {
      OMQ_TRY(loss_stream->fork(st));
      ls = loss_stream->s;
    }
    OMQ_TRY(launch_loss_finalize(epi.loss_partials, tiles,
                                 1.0 / (static_cast<double>(M) * static_cast<double>(N)), loss, ls));
  }
  return OMQ_OK;
}

omq_status omq_fq_linear_fwd(const void* Xq, const void* W_hat, omq_dtype dt, int64_t M,
                             int64_t N, int64_t K, const float* B_tilde, const float* Y_ref,
                             float* Y, void* dY, float* loss, void* workspace, size_t ws_bytes,
                             omq_stream_t stream) {
  return fwd_impl(Xq, W_hat, dt, M, N, K, B_tilde, Y_ref, Y, dY, loss, workspace, ws_bytes, stream,
                  Phases{});
}

size_t omq_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group) {
  if (M < 1 || N < 1 || K < 1 || group < 1) return 0;
  return bwd_layout(M, N, K, group).total;
}

// dbias_rows > 0: the forward already left the column sums of the residual over blocks of
// dbias_rows rows in the dB~ partials (its MSE epilogue), so no pass over dY is needed.
static omq_status bwd_impl(const omq_bwd_args* a, void* workspace, size_t ws_bytes,
                           omq_stream_t stream, const Phases& ph, int dbias_rows = 0) {
  if (!a) return OMQ_ERR_NULL;
  const int64_t M = a->M, N = a->N, K = a->K, G = a->group;
  if (!a->W || !a->Xq || !a->W_hat || !a->h || !a->z || !a->grp_range || !a->dY ||
      !a->gamma_logit || !a->beta_logit)
    return OMQ_ERR_NULL;
  if (!dtype_ok(a->dt) || !dtype_ok(a->op_dt)) return OMQ_ERR_DTYPE;
  if (!wbits_ok(a->bits) || !abits_ok(a->abits)) return OMQ_ERR_BITS;
  if (M < 1 || N < 8 || K < 8 || G < 8 || N % 8 || K % 8 || G % 8 || K % G || M > kMaxDim ||
      N > kMaxDim || K > kMaxDim)
    return OMQ_ERR_SHAPE;
  // the loss gradient is 2 R / (M N) for the forward's residual R
  const float gscale = static_cast<float>(2.0 / (static_cast<double>(M) * static_cast<double>(N)));
  if (!small_group(G) && G > kMaxGroupLarge) return OMQ_ERR_SHAPE;
  const bool need_let = a->d_s || a->d_delta;
  if (need_let) {
    if (!a->X || !a->s || !a->delta) return OMQ_ERR_NULL;
    if (2 * K * sizeof(float) > 200 * 1024) return OMQ_ERR_SHAPE;
    if (a->abits < 16 && (!a->h_a || !a->z_a || !a->tok_range)) return OMQ_ERR_NULL;
  }
  if (!a16(a->X) || !a16(a->W) || !a16(a->s) || !a16(a->delta) || !a16(a->Xq) ||
      !a16(a->W_hat) || !a16(a->dY))
    return OMQ_ERR_ALIGN;
  const BwdLayout L = bwd_layout(M, N, K, G);
  if (!workspace || ws_bytes < L.total) return OMQ_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  float* dbt_part = at<float>(workspace, L.dbt_part);
  float* dbt = a->d_B_tilde ? a->d_B_tilde : at<float>(workspace, L.dbt);
  float* dwhat = at<float>(workspace, L.dwhat);
  float* dxq = at<float>(workspace, L.dxq);
  float* part_ws = at<float>(workspace, L.part_ws);
  float* part_wd = at<float>(workspace, L.part_wd);
  float* part_xs = at<float>(workspace, L.part_xs);
  float* part_xd = at<float>(workspace, L.part_xd);
  double* red = at<double>(workspace, L.red);

  const float Q = static_cast<float>((1 << a->bits) - 1);
  const bool fused = fused_ste_w(a->op_dt, a->dt, G);
  const int64_t rb_w = fused ? ceil_div(N, kRowsFusedW) : ceil_div(N, rows_per_block_w(G));

  // Weight side: dB~, the dW^ GEMM and the weight-side STE.
  auto weight_side = [&](cudaStream_t s) -> omq_status {
    // dB~ = column sums of dY (needed for d_delta, or when asked for)
    OMQ_TRY(ph.mark(OMQ_PH_DBIAS));
    if (a->d_delta || a->d_B_tilde) {
      int64_t blocks = ceil_div(M, dbias_rows);
      if (dbias_rows <= 0) {
        OMQ_TRY(launch_colsum(a->dY, a->op_dt, M, N, kRowsColsum, nullptr, dbt_part, s));
        blocks = L.rb_colsum;
      }
      const ColReduce r{dbt_part, blocks, nullptr, 0, gscale, dbt};
      OMQ_TRY(launch_reduce_cols(&r, 1, N, red, s));
    }
    // dW^ = G^T Xq   [N, K]
    OMQ_TRY(ph.mark(OMQ_PH_DW_GEMM));
    {
      GemmOperand A{a->dY, N, true}, B{a->Xq, K, true};
      GemmEpilogue epi{};
      epi.out_scale = gscale;
      epi.sk_scratch = at<char>(workspace, L.sk_w);
      epi.sk_bytes = L.sk_w_bytes;
      if (fused) {
        // weight-side STE in the epilogue: per-chunk partial sums and the W-side LET column
        // partials straight from the accumulator
        epi.kind = Epi::SteW;
        epi.ste = SteWEpi{a->W, a->dt, K, G, K / G, Q, a->s, a->h, a->z,
                          at<float>(workspace, L.gh_part), at<float>(workspace, L.gc_part),
                          a->d_s ? part_ws : nullptr};
      } else {
        epi.kind = Epi::StoreF32;
        epi.out = dwhat;
      }
      OMQ_TRY(run_gemm(a->op_dt, A, B, N, K, M, epi, nullptr, s));
    }
    // weight-side STE: d gamma / d beta logits and the W-side LET column partials
    OMQ_TRY(ph.mark(OMQ_PH_STE_W));
    if (fused) {
      float* emax = a->d_s ? at<float>(workspace, L.emax) : nullptr;
      float* emin = a->d_s ? at<float>(workspace, L.emin) : nullptr;
      const SteWFinish f{N, G, K / G, Q, at<float>(workspace, L.gh_part),
                         at<float>(workspace, L.gc_part), a->h, a->grp_range, a->gamma_logit,
                         a->beta_logit, a->d_gamma_logit, a->d_beta_logit, emax, emin};
      OMQ_TRY(launch_ste_w_finish(f, s));
      if (a->d_s || a->d_delta) {
        const SteWCorr c{a->W, a->dt, N, K, G, a->s, a->grp_range, emax, emin, dbt,
                         a->d_s ? part_ws : nullptr, a->d_delta ? part_wd : nullptr};
        OMQ_TRY(launch_ste_w_corr(c, s));
      }
    } else {
      SteWParams p{a->W, a->dt, N, K, G, K / G, Q, a->s, a->gamma_logit, a->beta_logit, a->h,
                   a->z, a->grp_range, dwhat, a->d_delta ? dbt : nullptr, a->d_gamma_logit,
                   a->d_beta_logit, a->d_s ? part_ws : nullptr, a->d_delta ? part_wd : nullptr,
                   static_cast<int>(rows_per_block_w(G))};
      OMQ_TRY(launch_ste_w(p, s));
    }
    return OMQ_OK;
  };
  // Activation side (LET only): the dXq GEMM and the activation-side STE.
  auto act_side = [&](cudaStream_t s) -> omq_status {
    OMQ_TRY(ph.mark(OMQ_PH_DX_GEMM));
    // dXq = G W^   [M, K]
    {
      GemmOperand A{a->dY, N, false}, B{a->W_hat, K, true};
      GemmEpilogue epi{};
      epi.kind = Epi::StoreF32;
      epi.out = dxq;
      epi.out_scale = gscale;
      epi.sk_scratch = at<char>(workspace, L.sk_x);
      epi.sk_bytes = L.sk_x_bytes;
      OMQ_TRY(run_gemm(a->op_dt, A, B, M, K, N, epi, nullptr, s));
    }
    OMQ_TRY(ph.mark(OMQ_PH_STE_X));
    SteXParams p{a->X, a->dt, M, K,
                 static_cast<float>((1 << (a->abits < 16 ? a->abits : 1)) - 1),
                 a->abits < 16 ? 1 : 0, a->s, a->delta, a->h_a, a->z_a, a->tok_range, dxq,
                 at<float>(workspace, L.rowstat), part_xs, part_xd, kRowsX};
    return launch_ste_x(p, s);
  };

  // The two sides share only dY (read) and write disjoint buffers: without phase events
  // the activation side runs on a second stream, so each side's kernels fill the other's
  // pipeline fill, epilogue tails and launch gaps.
  const SideStream* ss = (!ph.ev && need_let) ? side_stream() : nullptr;
  if (ss) {
    OMQ_TRY(ss->fork(st));
    const omq_status sa = act_side(ss->s);
    const omq_status sw = weight_side(st);
    const omq_status sj = ss->join(st);
    OMQ_TRY(sa);
    OMQ_TRY(sw);
    OMQ_TRY(sj);
  } else {
    OMQ_TRY(weight_side(st));
    if (!need_let) {
      OMQ_TRY(ph.mark(OMQ_PH_DX_GEMM));
      OMQ_TRY(ph.mark(OMQ_PH_STE_X));
      return ph.mark(OMQ_PH_LET_REDUCE);
    }
    OMQ_TRY(act_side(st));
  }
  OMQ_TRY(ph.mark(OMQ_PH_LET_REDUCE));
  ColReduce r[2];
  int nr = 0;
  if (a->d_s) r[nr++] = ColReduce{part_ws, rb_w, part_xs, L.rb_x, 1.f, a->d_s};
  if (a->d_delta) r[nr++] = ColReduce{part_wd, rb_w, part_xd, L.rb_x, 1.f, a->d_delta};
  if (nr) OMQ_TRY(launch_reduce_cols(r, nr, K, red, st));
  return OMQ_OK;
}

omq_status omq_fq_linear_bwd(const omq_bwd_args* a, void* workspace, size_t ws_bytes,
                             omq_stream_t stream) {
  return bwd_impl(a, workspace, ws_bytes, stream, Phases{});
}

omq_status omq_adamw_step(float* param, const float* grad, float* m, float* v, int64_t n, float lr,
                          float beta1, float beta2, float eps, float weight_decay, int64_t step,
                          omq_stream_t stream) {
  if (n < 0) return OMQ_ERR_SHAPE;
  if (n == 0) return OMQ_OK;
  if (!param || !grad || !m || !v) return OMQ_ERR_NULL;
  if (step < 1) return OMQ_ERR_SHAPE;
  const AdamSeg seg{param, grad, m, v, n, lr};
  return launch_adamw(&seg, 1, beta1, beta2, eps, weight_decay, step,
                      reinterpret_cast<cudaStream_t>(stream));
}

size_t omq_step_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group) {
  if (M < 1 || N < 1 || K < 1 || group < 1) return 0;
  return fwd_bytes(M, N) + bwd_layout(M, N, K, group).total;
}

omq_status omq_calib_step(const omq_step_args* a, void* workspace, size_t ws_bytes,
                          omq_stream_t stream) {
  if (!a) return OMQ_ERR_NULL;
  const int64_t M = a->M, N = a->N, K = a->K, G = a->group;
  if (!a->X || !a->W || !a->Y_ref || !a->gamma_logit || !a->beta_logit || !a->W_hat || !a->h ||
      !a->z || !a->grp_range || !a->dY || !a->d_gamma_logit || !a->d_beta_logit || !a->loss ||
      !a->m_gamma || !a->v_gamma || !a->m_beta || !a->v_beta)
    return OMQ_ERR_NULL;
  if (M < 1 || N < 1 || K < 1 || G < 1) return OMQ_ERR_SHAPE;
  if (a->step < 1) return OMQ_ERR_SHAPE;
  const bool let = a->let != 0;
  if (!dtype_ok(a->dt) || !dtype_ok(a->op_dt)) return OMQ_ERR_DTYPE;
  // X itself is the GEMM operand only without LET, activation quantization or conversion
  const bool need_act = let || a->abits < 16 || a->op_dt != a->dt;
  if (let && (!a->s || !a->delta || !a->d_s || !a->d_delta || !a->m_s || !a->v_s || !a->m_delta ||
              !a->v_delta || !a->B_tilde))
    return OMQ_ERR_NULL;
  if (need_act && (!a->Xq || a->Xq == a->X)) return OMQ_ERR_NULL;
  if (a->abits < 16 && (!a->h_a || !a->z_a || !a->tok_range)) return OMQ_ERR_NULL;
  const size_t fwd_ws = fwd_bytes(M, N);
  if (!workspace || ws_bytes < omq_step_workspace_bytes(M, N, K, G)) return OMQ_ERR_WORKSPACE;
  const void* Xq = need_act ? a->Xq : a->X;
  const float* Bt = let ? a->B_tilde : a->B;
  Phases ph{a->events, reinterpret_cast<cudaStream_t>(stream)};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  OMQ_TRY(check_lwc(a->W, a->dt, N, K, G, a->bits, a->gamma_logit, a->beta_logit,
                    let ? a->s : nullptr, a->op_dt, a->W_hat, nullptr, a->h, a->z));
  auto act = [&](cudaStream_t s) -> omq_status {
    if (!need_act) return OMQ_OK;
    return omq_let_apply(a->X, a->dt, M, K, let ? a->s : nullptr, let ? a->delta : nullptr,
                         a->abits, a->Xq, a->op_dt, a->h_a, a->z_a, a->tok_range, nullptr, a->dt,
                         N, nullptr, nullptr, s);
  };
  auto lwc = [&](cudaStream_t s) -> omq_status {
    // LWC, with B~ = B + W delta out of the same pass over W
    LwcParams p{a->W, a->dt, N, K, G, K / G, static_cast<float>((1 << a->bits) - 1),
                a->gamma_logit, a->beta_logit, let ? a->s : nullptr, a->W_hat, a->op_dt, a->h,
                a->z, nullptr, a->grp_range, nullptr, a->bits};
    if (let) {
      p.delta = a->delta;
      p.B = a->B;
      p.Bt = a->B_tilde;
    }
    p.no_ties = !let;     // without LET no gradient reads the tie counts
    return launch_lwc(p, s);
  };
  // The activation and weight sides of the forward are independent: without phase events
  // the weight side runs on a second stream.
  const SideStream* ss = (!ph.ev && need_act) ? side_stream() : nullptr;
  if (ss) {
    OMQ_TRY(ss->fork(st));
    const omq_status sl = lwc(ss->s);
    const omq_status sa = act(st);
    const omq_status sj = ss->join(st);
    OMQ_TRY(sl);
    OMQ_TRY(sa);
    OMQ_TRY(sj);
  } else {
    OMQ_TRY(ph.mark(OMQ_PH_LET));
    OMQ_TRY(act(st));
    OMQ_TRY(ph.mark(OMQ_PH_LWC));
    OMQ_TRY(lwc(st));
  }
  // without phase events the loss reduction runs on the second stream, beside the backward
  // (which does not read it); the stream is joined before AdamW
  const SideStream* ls = ph.ev ? nullptr : side_stream();
  // with LET the backward needs dB~ = column sums of the residual: the forward GEMM's MSE
  // epilogue forms them per 32-row block (tensor-core path) in the backward's partials
  const bool fused_dbias = let && a->op_dt != OMQ_F32;
  float* dbias_part = fused_dbias ? reinterpret_cast<float*>(
                                        static_cast<char*>(workspace) + fwd_ws +
                                        bwd_layout(M, N, K, G).dbt_part)
                                  : nullptr;
  OMQ_TRY(fwd_impl(Xq, a->W_hat, a->op_dt, M, N, K, Bt, a->Y_ref, nullptr, a->dY, a->loss,
                   workspace, fwd_ws, stream, ph, ls, dbias_part));
  omq_bwd_args b{};
  b.M = M; b.N = N; b.K = K; b.group = G; b.bits = a->bits; b.abits = a->abits; b.dt = a->dt;
  b.op_dt = a->op_dt;
  b.X = a->X; b.W = a->W; b.s = let ? a->s : nullptr; b.delta = let ? a->delta : nullptr;
  b.gamma_logit = a->gamma_logit; b.beta_logit = a->beta_logit;
  b.Xq = Xq; b.W_hat = a->W_hat; b.h = a->h; b.z = a->z; b.grp_range = a->grp_range;
  b.h_a = a->h_a; b.z_a = a->z_a; b.tok_range = a->tok_range; b.dY = a->dY;
  b.d_gamma_logit = a->d_gamma_logit; b.d_beta_logit = a->d_beta_logit;
  b.d_s = let ? a->d_s : nullptr; b.d_delta = let ? a->d_delta : nullptr;
  OMQ_TRY(bwd_impl(&b, static_cast<char*>(workspace) + fwd_ws, ws_bytes - fwd_ws, stream, ph,
                   fused_dbias ? 32 : 0));
  if (ls) OMQ_TRY(ls->join(st));
  OMQ_TRY(ph.mark(OMQ_PH_ADAMW));
  const int64_t ng = N * (K / G);
  const AdamSeg segs[kMaxAdamSegs] = {
      {a->gamma_logit, a->d_gamma_logit, a->m_gamma, a->v_gamma, ng, a->lr_lwc},
      {a->beta_logit, a->d_beta_logit, a->m_beta, a->v_beta, ng, a->lr_lwc},
      {a->s, a->d_s, a->m_s, a->v_s, K, a->lr_let},
      {a->delta, a->d_delta, a->m_delta, a->v_delta, K, a->lr_let}};
  OMQ_TRY(launch_adamw(segs, let ? 4 : 2, 0.9f, 0.999f, 1e-8f, 0.f, a->step,
                       reinterpret_cast<cudaStream_t>(stream)));
  return ph.mark(OMQ_PH_COUNT);
}

uint64_t omq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
