// The transformer-block calibration step ("【ICLR 2024】OmniQuant: ...", sections 框架, LET,
// LWC): validation, parameter and workspace layout, and the launch sequence of the forward,
// the loss, the straight-through backward and AdamW. Every tensor lives in caller memory
// (the parameter vector, the gradient, the workspace); nothing here allocates.
//
// The four linears are fake-quant linears of the single-layer step (LWC with the LET
// weight scale folded into the load, per-token activation quantizer, tcgen05 GEMMs, the
// weight-side STE fused into the dW GEMM). Attention runs on the same GEMM, all heads of a
// product in one launch, the causal structure skipping the tiles and contraction blocks the
// mask zeroes; scores and probabilities are materialised in float32.
#include <algorithm>
#include <cmath>
#include <initializer_list>
#include <vector>

#include "block_internal.cuh"

namespace omq {
namespace {

constexpr int kRowsX = 64;        // tokens per block, activation STE column partials
constexpr int kRowsColsum = 64;   // rows per block of the dY column sums
constexpr int kRowsFusedW = 32;   // rows per partial, weight STE in the dW epilogue
constexpr int64_t kHead = 128;
constexpr double kRopeBase = 10000.0;
constexpr float kEps = 1e-6f;

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

#define BLK_TRY(expr)                 \
  do {                                \
    omq_status _s = (expr);           \
    if (_s != OMQ_OK) return _s;      \
  } while (0)

bool dims_ok(const omq_block_dims& d) {
  if (d.M < 8 || d.M % 8 || d.H < 1 || d.D != kHead * d.H || d.I < 32 || d.I % 32) return false;
  if (d.M > (int64_t(1) << 20) || d.D > 65536 || d.I > 65536) return false;
  if (d.group != 0 && (d.group % 32 || d.D % d.group || d.I % d.group)) return false;
  return true;
}
bool bits_ok(const omq_block_dims& d) {
  const bool w = d.wbits >= 2 && d.wbits <= 8;
  const bool a = d.abits == 2 || d.abits == 3 || d.abits == 4 || d.abits == 6 || d.abits == 8 ||
                 d.abits == 16;
  return w && a;
}

int64_t group_of(const omq_block_dims& d, int64_t K) { return d.group == 0 ? K : d.group; }

// The linears: rows, depth, which LET vectors act on them.
enum { L_QKV = 0, L_O, L_GU, L_D, L_COUNT };
struct LinShape {
  int64_t N, K;
};
LinShape lin_shape(const omq_block_dims& d, int l) {
  switch (l) {
    case L_QKV: return {3 * d.D, d.D};
    case L_O: return {d.D, d.D};
    case L_GU: return {2 * d.I, d.D};
    default: return {d.D, d.I};
  }
}

void theta_ranges(const omq_block_dims& d, int64_t* off, int64_t* cnt) {
  int64_t o = 0;
  for (int l = 0; l < L_COUNT; ++l) {
    const LinShape s = lin_shape(d, l);
    const int64_t ng = s.N * (s.K / group_of(d, s.K));
    for (int t = 0; t < 2; ++t) {
      off[2 * l + t] = o;
      cnt[2 * l + t] = ng;
      o += ng;
    }
  }
  for (int i = OMQ_TH_S1; i < OMQ_TH_COUNT; ++i) {
    off[i] = o;
    cnt[i] = d.D;
    o += d.D;
  }
  off[OMQ_TH_COUNT] = o;
  cnt[OMQ_TH_COUNT] = o;
}

// Workspace: the named tensors of omq.h, then internal scratch.
struct LinScratch {
  size_t h, z, range, bt, part_ws, part_wd, part_xs, part_xd;
};
struct BlockLayout {
  size_t bb[OMQ_BB_COUNT];
  size_t bb_bytes[OMQ_BB_COUNT];
  LinScratch lin[L_COUNT];
  size_t act_h[4], act_z[4], act_range[4];   // qa, Qo, qb, qm
  size_t head_h, head_z, head_range;
  size_t rstd2, tgt, o_out, loss_part, dP, dS, dxq;
  size_t gh_part, gc_part, emax, emin, dbt_part, dbt, rowstat, red;
  size_t part_sa, part_so, part_do;
  size_t sk, sk_bytes;   // stream-K scratch of the linears' GEMMs (one at a time)
  size_t total;
  int64_t loss_tiles;
};

BlockLayout block_layout(const omq_block_dims& d) {
  BlockLayout L{};
  const int64_t M = d.M, D = d.D, H = d.H, I = d.I;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  auto named = [&](int id, size_t bytes) { L.bb[id] = take(bytes); L.bb_bytes[id] = bytes; };
  const size_t f4 = sizeof(float), b2 = 2;
  named(OMQ_BB_ROPE, f4 * 2 * M * 64);
  named(OMQ_BB_A, f4 * M * D);
  named(OMQ_BB_QA, b2 * M * D);
  named(OMQ_BB_WHAT_QKV, b2 * 3 * D * D);
  named(OMQ_BB_WHAT_O, b2 * D * D);
  named(OMQ_BB_WHAT_GU, b2 * 2 * I * D);
  named(OMQ_BB_WHAT_D, b2 * D * I);
  named(OMQ_BB_QKV, f4 * M * 3 * D);
  named(OMQ_BB_QQKV, b2 * M * 3 * D);
  named(OMQ_BB_P, f4 * H * M * M);
  named(OMQ_BB_P16, b2 * H * M * M);
  named(OMQ_BB_O, f4 * M * D);
  named(OMQ_BB_QO, b2 * M * D);
  named(OMQ_BB_X2, f4 * M * D);
  named(OMQ_BB_B, f4 * M * D);
  named(OMQ_BB_QB, b2 * M * D);
  named(OMQ_BB_GU, f4 * M * 2 * I);
  named(OMQ_BB_MID, f4 * M * I);
  named(OMQ_BB_QM, b2 * M * I);
  named(OMQ_BB_RES, b2 * M * D);
  named(OMQ_BB_DMID, f4 * M * I);
  named(OMQ_BB_DGU, b2 * M * 2 * I);
  named(OMQ_BB_DB, f4 * M * D);
  named(OMQ_BB_DX2, b2 * M * D);
  named(OMQ_BB_DO, b2 * M * D);
  named(OMQ_BB_DQQKV, f4 * M * 3 * D);
  named(OMQ_BB_DQKV, b2 * M * 3 * D);
  int64_t max_gh = 0, max_ng = 0, max_n = 0;
  for (int l = 0; l < L_COUNT; ++l) {
    const LinShape s = lin_shape(d, l);
    const int64_t ng = s.N * (s.K / group_of(d, s.K));
    LinScratch& c = L.lin[l];
    c.h = take(f4 * ng);
    c.z = take(sizeof(int32_t) * ng);
    c.range = take(sizeof(omq_range) * ng);
    c.bt = take(f4 * s.N);
    c.part_ws = take(f4 * ceil_div(s.N, kRowsFusedW) * s.K);
    c.part_wd = take(f4 * ceil_div(s.N, kRowsFusedW) * s.K);
    c.part_xs = take(f4 * ceil_div(M, kRowsX) * s.K);
    c.part_xd = take(f4 * ceil_div(M, kRowsX) * s.K);
    max_gh = std::max<int64_t>(max_gh, (s.K / 32) * s.N);
    max_ng = std::max<int64_t>(max_ng, ng);
    max_n = std::max<int64_t>(max_n, std::max(s.N, s.K));
  }
  for (int a = 0; a < 4; ++a) {
    L.act_h[a] = take(f4 * M);
    L.act_z[a] = take(sizeof(int32_t) * M);
    L.act_range[a] = take(sizeof(omq_range) * M);
  }
  L.head_h = take(f4 * 3 * M * H);
  L.head_z = take(sizeof(int32_t) * 3 * M * H);
  L.head_range = take(sizeof(omq_range) * 3 * M * H);
  L.rstd2 = take(f4 * M);
  L.tgt = take(f4 * M * D);
  L.o_out = take(f4 * M * D);
  L.loss_tiles = gemm_tc_tiles(M, D);
  L.loss_part = take(f4 * L.loss_tiles);
  L.dP = take(f4 * H * M * M);
  L.dS = take(b2 * H * M * M);
  L.dxq = take(f4 * M * std::max(D, I));
  L.gh_part = take(f4 * max_gh);
  L.gc_part = take(f4 * max_gh);
  L.emax = take(f4 * max_ng);
  L.emin = take(f4 * max_ng);
  L.dbt_part = take(f4 * ceil_div(M, kRowsColsum) * max_n);
  L.dbt = take(f4 * max_n);
  L.rowstat = take(f4 * 2 * M);
  L.red = take(sizeof(double) * 2 * kReduceChunks * max_n);
  L.part_sa = take(f4 * ceil_div(M, kAttnRows) * D);
  L.part_so = take(f4 * ceil_div(M, kAttnRows) * D);
  L.part_do = take(f4 * ceil_div(M, kAttnRows) * D);
  L.sk_bytes = 0;
  for (int l = 0; l < L_COUNT; ++l) {
    const LinShape s = lin_shape(d, l);
    L.sk_bytes = std::max({L.sk_bytes, gemm_tc_sk_bytes(M, s.N), gemm_tc_sk_bytes(s.N, s.K),
                           gemm_tc_sk_bytes(M, s.K)});
  }
  L.sk = take(L.sk_bytes);
  L.total = off;
  return L;
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

struct Marks {
  void* const* ev = nullptr;
  cudaStream_t st = nullptr;
  omq_status mark(int i) const {
    if (!ev) return OMQ_OK;
    const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st);
    if (e != cudaSuccess) {
      set_cuda_error(e);
      return OMQ_ERR_CUDA;
    }
    return OMQ_OK;
  }
};


omq_status gemm_store(omq_dtype op, const GemmOperand& A, const GemmOperand& B, int64_t rows,
                      int64_t cols, int64_t depth, float* out, int64_t ldo, float scale,
                      const float* bias, void* sk, size_t sk_bytes, cudaStream_t st) {
  GemmEpilogue e{};
  e.sk_scratch = sk;
  e.sk_bytes = sk_bytes;
  e.kind = Epi::StoreF32;
  e.out = out;
  e.ldo = ldo;
  e.out_scale = scale;
  e.bias = bias;
  return gemm_tc(op, A, B, rows, cols, depth, e, nullptr, st);
}

// The attention products, all heads in one launch each (heads are the batch).
omq_status gemm_heads(omq_dtype op, const GemmOperand& A, int64_t a_stride, const GemmOperand& B,
                      int64_t b_stride, int64_t rows, int64_t cols, int64_t depth, float* out,
                      int64_t ldo, int64_t out_stride, float scale, int64_t heads, int causal,
                      cudaStream_t st) {
  GemmEpilogue e{};
  e.kind = Epi::StoreF32;
  e.out = out;
  e.ldo = ldo;
  e.out_scale = scale;
  const GemmBatch b{heads, a_stride, b_stride, out_stride, causal};
  return gemm_tc(op, A, B, rows, cols, depth, e, nullptr, st, &b);
}

omq_status act_quant(omq_dtype op, const void* X, omq_dtype xdt, int64_t M, int64_t K,
                     const float* s, const float* d, int abits, void* Xq, float* h_a, int32_t* z_a,
                     omq_range* range, cudaStream_t st) {
  LetParams p{X, xdt, M, K, s, d, static_cast<float>((1 << (abits < 16 ? abits : 1)) - 1), Xq,
              op, h_a, z_a, range};
  return launch_let(p, abits, st);
}

// Views of the workspace for one call.
struct View {
  const omq_block_dims& d;
  const BlockLayout& L;
  void* ws;
  template <class T>
  T* bb(int id) const { return at<T>(ws, L.bb[id]); }
  template <class T>
  T* in(size_t off) const { return at<T>(ws, off); }
};

struct Inputs {
  const void* x;
  const void* W[L_COUNT];
  const float* y_ref;   // NULL: forward only, y written to y_out
  void* y_out;
  const float* theta;   // NULL: the full-precision block
  omq_dtype y_dt;       // of y_out
};

// Forward of the block (the formulas of omq.h). With theta NULL every quantizer and transform
// is off and the GEMMs take the weights themselves.
omq_status block_forward(const View& v, const Inputs& in, const Marks& mk, cudaStream_t st) {
  const omq_block_dims& d = v.d;
  const BlockLayout& L = v.L;
  const int64_t M = d.M, D = d.D, H = d.H, I = d.I;
  const bool fp = in.theta == nullptr;
  const int abits = fp ? 16 : d.abits;
  // GEMM operands: float16 for the fake-quantized block (its operands and the gradients
  // that flow back through them keep 3 more mantissa bits than bfloat16); the full-precision
  // block multiplies the bfloat16 weights themselves
  const omq_dtype op = fp ? OMQ_BF16 : OMQ_F16;
  const float Qw = static_cast<float>((1 << d.wbits) - 1);
  int64_t toff[OMQ_TH_COUNT + 1], tcnt[OMQ_TH_COUNT + 1];
  theta_ranges(d, toff, tcnt);
  auto th = [&](int id) -> const float* { return fp ? nullptr : in.theta + toff[id]; };
  const float* s_w[L_COUNT] = {th(OMQ_TH_S1), th(OMQ_TH_S_O), th(OMQ_TH_S2), nullptr};
  const float* dl_w[L_COUNT] = {th(OMQ_TH_DELTA1), th(OMQ_TH_DELTA_O), th(OMQ_TH_DELTA2), nullptr};
  const int what_id[L_COUNT] = {OMQ_BB_WHAT_QKV, OMQ_BB_WHAT_O, OMQ_BB_WHAT_GU, OMQ_BB_WHAT_D};
  const void* Wop[L_COUNT];
  float* cos_t = v.bb<float>(OMQ_BB_ROPE);
  float* sin_t = cos_t + M * 64;

  BLK_TRY(mk.mark(OMQ_BPH_WEIGHTS));
  BLK_TRY(launch_rope_table(M, kRopeBase, cos_t, sin_t, st));
  for (int l = 0; l < L_COUNT; ++l) {
    const LinShape s = lin_shape(d, l);
    if (fp) {
      Wop[l] = in.W[l];
      continue;
    }
    const int64_t G = group_of(d, s.K);
    const LinScratch& c = L.lin[l];
    LwcParams p{in.W[l], OMQ_BF16, s.N, s.K, G, s.K / G, Qw, th(OMQ_TH_GAMMA_QKV + 2 * l),
                th(OMQ_TH_BETA_QKV + 2 * l), s_w[l], v.bb<void>(what_id[l]), op,
                v.in<float>(c.h), v.in<int32_t>(c.z), nullptr, v.in<omq_range>(c.range), nullptr,
                d.wbits};
    if (dl_w[l]) {   // B~ = W delta out of the same pass over W
      p.delta = dl_w[l];
      p.Bt = v.in<float>(c.bt);
    }
    BLK_TRY(launch_lwc(p, st));
    Wop[l] = v.bb<void>(what_id[l]);
  }
  auto bias = [&](int l) -> const float* { return fp || !dl_w[l] ? nullptr : v.in<float>(L.lin[l].bt); };

  // attention input: RMSNorm, LET, act quant, q | k | v, RoPE / affinity / V transform, head quant
  BLK_TRY(mk.mark(OMQ_BPH_ATTN_IN));
  {
    RmsParams r{in.x, OMQ_BF16, nullptr, M, D, kEps, nullptr, v.bb<float>(OMQ_BB_A), nullptr,
                nullptr, nullptr};
    BLK_TRY(launch_rms(r, st));
  }
  BLK_TRY(act_quant(op, v.bb<float>(OMQ_BB_A), OMQ_F32, M, D, th(OMQ_TH_S1), th(OMQ_TH_DELTA1), abits,
                    v.bb<void>(OMQ_BB_QA), v.in<float>(L.act_h[0]), v.in<int32_t>(L.act_z[0]),
                    v.in<omq_range>(L.act_range[0]), st));
  BLK_TRY(gemm_store(op, GemmOperand{v.bb<void>(OMQ_BB_QA), D, false}, GemmOperand{Wop[L_QKV], D, false},
                     M, 3 * D, D, v.bb<float>(OMQ_BB_QKV), 0, 1.f, bias(L_QKV), v.in<char>(L.sk),
                     L.sk_bytes, st));
  {
    AttnPrepParams p{};
    p.qkv = v.bb<float>(OMQ_BB_QKV);
    p.cos_t = cos_t;
    p.sin_t = sin_t;
    p.s_a = th(OMQ_TH_S_A);
    p.s_o = th(OMQ_TH_S_O);
    p.delta_o = th(OMQ_TH_DELTA_O);
    p.M = M; p.D = D; p.H = H;
    p.quantized = abits < 16 ? 1 : 0;
    p.Qa = static_cast<float>((1 << (abits < 16 ? abits : 1)) - 1);
    p.out = v.bb<void>(OMQ_BB_QQKV);
    p.dt16 = op;
    p.h_s = v.in<float>(L.head_h);
    p.z_s = v.in<int32_t>(L.head_z);
    p.range_s = v.in<omq_range>(L.head_range);
    BLK_TRY(launch_attn_prep(p, false, st));
  }
  // attention, one head at a time: S = Qq Qk^T / sqrt(128), P = causal softmax, O = P Qv
  BLK_TRY(mk.mark(OMQ_BPH_ATTN));
  {
    const uint16_t* qqkv = v.bb<uint16_t>(OMQ_BB_QQKV);
    float* P = v.bb<float>(OMQ_BB_P);
    uint16_t* P16 = v.bb<uint16_t>(OMQ_BB_P16);
    const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(kHead)));
    BLK_TRY(gemm_heads(op, GemmOperand{qqkv, 3 * D, false}, kHead,
                       GemmOperand{qqkv + D, 3 * D, false}, kHead, M, M, kHead, P, 0, M * M, scale,
                       H, 1, st));
    BLK_TRY(launch_softmax(P, P16, op, H * M, M, st));
    BLK_TRY(gemm_heads(op, GemmOperand{P16, M, false}, M * M,
                       GemmOperand{qqkv + 2 * D, 3 * D, true}, kHead, M, kHead, M,
                       v.bb<float>(OMQ_BB_O), D, kHead, 1.f, H, 2, st));
  }
  // o_proj, residual, RMSNorm, gate / up, SwiGLU, down (+ loss)
  BLK_TRY(mk.mark(OMQ_BPH_FFN));
  BLK_TRY(act_quant(op, v.bb<float>(OMQ_BB_O), OMQ_F32, M, D, nullptr, nullptr, abits,
                    v.bb<void>(OMQ_BB_QO), v.in<float>(L.act_h[1]), v.in<int32_t>(L.act_z[1]),
                    v.in<omq_range>(L.act_range[1]), st));
  BLK_TRY(gemm_store(op, GemmOperand{v.bb<void>(OMQ_BB_QO), D, false}, GemmOperand{Wop[L_O], D, false},
                     M, D, D, v.in<float>(L.o_out), 0, 1.f, bias(L_O), v.in<char>(L.sk),
                     L.sk_bytes, st));
  {
    RmsParams r{in.x, OMQ_BF16, v.in<float>(L.o_out), M, D, kEps, v.bb<float>(OMQ_BB_X2),
                v.bb<float>(OMQ_BB_B), v.in<float>(L.rstd2), in.y_ref, v.in<float>(L.tgt)};
    BLK_TRY(launch_rms(r, st));
  }
  BLK_TRY(act_quant(op, v.bb<float>(OMQ_BB_B), OMQ_F32, M, D, th(OMQ_TH_S2), th(OMQ_TH_DELTA2), abits,
                    v.bb<void>(OMQ_BB_QB), v.in<float>(L.act_h[2]), v.in<int32_t>(L.act_z[2]),
                    v.in<omq_range>(L.act_range[2]), st));
  BLK_TRY(gemm_store(op, GemmOperand{v.bb<void>(OMQ_BB_QB), D, false}, GemmOperand{Wop[L_GU], D, false},
                     M, 2 * I, D, v.bb<float>(OMQ_BB_GU), 0, 1.f, bias(L_GU), v.in<char>(L.sk),
                     L.sk_bytes, st));
  BLK_TRY(launch_swiglu(v.bb<float>(OMQ_BB_GU), v.bb<float>(OMQ_BB_MID), M, I, st));
  BLK_TRY(act_quant(op, v.bb<float>(OMQ_BB_MID), OMQ_F32, M, I, nullptr, nullptr, abits,
                    v.bb<void>(OMQ_BB_QM), v.in<float>(L.act_h[3]), v.in<int32_t>(L.act_z[3]),
                    v.in<omq_range>(L.act_range[3]), st));
  {
    // y = x2 + qm Ŵ_d^T. With y_ref: the residual y - y_ref = acc - (y_ref - x2) and its
    // squares; without: the same epilogue against -x2 gives y itself.
    GemmEpilogue e{};
    e.kind = Epi::MseLoss;
    e.y_ref = v.in<float>(L.tgt);
    e.dy = in.y_ref ? v.bb<void>(OMQ_BB_RES) : in.y_out;
    e.dy_dt = in.y_ref ? op : in.y_dt;
    e.loss_partials = v.in<float>(L.loss_part);
    e.sk_scratch = v.in<char>(L.sk);
    e.sk_bytes = L.sk_bytes;
    BLK_TRY(gemm_tc(op, GemmOperand{v.bb<void>(OMQ_BB_QM), I, false},
                    GemmOperand{Wop[L_D], I, false}, M, D, I, e, nullptr, st));
  }
  return OMQ_OK;
}


// Backward of one fake-quant linear Y = Q_a(X~) Ŵ^T + B~ given dL/dY = dy_scale dY:
// dB~ (when the linear has a shift), the dŴ GEMM with the weight-side STE in its epilogue
// and its completion (LWC logit gradients, W-side LET column partials), the dX GEMM and the
// activation-side STE (dX~ / s_x stored in dX when asked, X-side LET column partials).
struct LinBwd {
  omq_dtype op;            // GEMM operand type of Xq, W_hat, dY (and dX when 16-bit)
  int64_t M, N, K, G;
  float Q;
  const void* W;
  const void* W_hat;
  const float* s_w;        // W~ = W s_w, or NULL
  const float* gl;
  const float* bl;
  const float* h;
  const int32_t* z;
  const omq_range* range;
  const void* Xq;
  const void* dY;
  float dy_scale;
  float* d_gl;
  float* d_bl;
  bool shift;              // B~ = W delta: dB~ and part_wd
  float* part_ws;          // [ceil(N/32), K] (s_w)
  float* part_wd;          // (shift)
  const void* X;           // activation side: the quantizer's input before its LET
  omq_dtype xdt;
  const float* s_x;
  const float* d_x;
  int quantized;
  float Qa;
  const float* h_a;
  const int32_t* z_a;
  const omq_range* tok_range;
  void* dX;                // or NULL
  omq_dtype dx_dt;
  float* part_xs;          // [ceil(M/64), K] or NULL
  float* part_xd;
};

omq_status lin_bwd(const LinBwd& a, const View& v, cudaStream_t st) {
  const BlockLayout& L = v.L;
  float* dbt = v.in<float>(L.dbt);
  float* gh = v.in<float>(L.gh_part);
  float* gc = v.in<float>(L.gc_part);
  float* emax = a.s_w ? v.in<float>(L.emax) : nullptr;
  float* emin = a.s_w ? v.in<float>(L.emin) : nullptr;
  if (a.shift) {
    float* part = v.in<float>(L.dbt_part);
    BLK_TRY(launch_colsum(a.dY, a.op, a.M, a.N, kRowsColsum, nullptr, part, st));
    const ColReduce r{part, ceil_div(a.M, kRowsColsum), nullptr, 0, a.dy_scale, dbt};
    BLK_TRY(launch_reduce_cols(&r, 1, a.N, v.in<double>(L.red), st));
  }
  {
    GemmEpilogue e{};
    e.kind = Epi::SteW;
    e.out_scale = a.dy_scale;
    e.ste = SteWEpi{a.W, OMQ_BF16, a.K, a.G, a.K / a.G, a.Q, a.s_w, a.h, a.z, gh, gc,
                    a.s_w ? a.part_ws : nullptr};
    e.sk_scratch = v.in<char>(L.sk);
    e.sk_bytes = L.sk_bytes;
    BLK_TRY(gemm_tc(a.op, GemmOperand{a.dY, a.N, true}, GemmOperand{a.Xq, a.K, true}, a.N, a.K,
                    a.M, e, nullptr, st));
  }
  {
    const SteWFinish f{a.N, a.G, a.K / a.G, a.Q, gh, gc, a.h, a.range, a.gl, a.bl, a.d_gl,
                       a.d_bl, emax, emin};
    BLK_TRY(launch_ste_w_finish(f, st));
  }
  if (a.s_w || a.shift) {
    const SteWCorr c{a.W, OMQ_BF16, a.N, a.K, a.G, a.s_w, a.range, emax, emin,
                     a.shift ? dbt : nullptr, a.s_w ? a.part_ws : nullptr,
                     a.shift ? a.part_wd : nullptr};
    BLK_TRY(launch_ste_w_corr(c, st));
  }
  float* dxq = v.in<float>(L.dxq);
  BLK_TRY(gemm_store(a.op, GemmOperand{a.dY, a.N, false}, GemmOperand{a.W_hat, a.K, true}, a.M, a.K, a.N,
                     dxq, 0, a.dy_scale, nullptr, v.in<char>(L.sk), L.sk_bytes, st));
  SteXParams p{a.X, a.xdt, a.M, a.K, a.Qa, a.quantized, a.s_x, a.d_x, a.h_a, a.z_a, a.tok_range,
               dxq, v.in<float>(L.rowstat), a.part_xs, a.part_xd, kRowsX, a.dX, a.dx_dt};
  return launch_ste_x(p, st);
}

omq_status block_backward(const View& v, const Inputs& in, float* d_theta, const Marks& mk,
                          cudaStream_t st) {
  const omq_block_dims& d = v.d;
  const BlockLayout& L = v.L;
  const int64_t M = d.M, D = d.D, H = d.H, I = d.I;
  int64_t toff[OMQ_TH_COUNT + 1], tcnt[OMQ_TH_COUNT + 1];
  theta_ranges(d, toff, tcnt);
  auto th = [&](int id) { return in.theta + toff[id]; };
  auto dth = [&](int id) { return d_theta + toff[id]; };
  const int quantized = d.abits < 16 ? 1 : 0;
  const float Qa = static_cast<float>((1 << (d.abits < 16 ? d.abits : 1)) - 1);
  const float Qw = static_cast<float>((1 << d.wbits) - 1);
  // The activation gradients flow back unscaled: in units of the residual res = y - y*, i.e.
  // as gradients of (M D / 2) L. They are stored as float16 GEMM operands, whose range then
  // holds them (the true gradients, 2 / (M D) times smaller, would fall into float16's
  // subnormals); the factor 2 / (M D) is applied once, to the parameter gradients.
  const float gscale = static_cast<float>(2.0 / (static_cast<double>(M) * static_cast<double>(D)));
  const omq_dtype op = OMQ_F16;
  const int what_id[L_COUNT] = {OMQ_BB_WHAT_QKV, OMQ_BB_WHAT_O, OMQ_BB_WHAT_GU, OMQ_BB_WHAT_D};
  auto base = [&](int l) {
    const LinShape s = lin_shape(d, l);
    const LinScratch& c = L.lin[l];
    LinBwd a{};
    a.op = op;
    a.M = M; a.N = s.N; a.K = s.K; a.G = group_of(d, s.K); a.Q = Qw;
    a.W = in.W[l]; a.W_hat = v.bb<void>(what_id[l]);
    a.gl = th(OMQ_TH_GAMMA_QKV + 2 * l); a.bl = th(OMQ_TH_BETA_QKV + 2 * l);
    a.d_gl = dth(OMQ_TH_GAMMA_QKV + 2 * l); a.d_bl = dth(OMQ_TH_BETA_QKV + 2 * l);
    a.h = v.in<float>(c.h); a.z = v.in<int32_t>(c.z); a.range = v.in<omq_range>(c.range);
    a.part_ws = v.in<float>(c.part_ws); a.part_wd = v.in<float>(c.part_wd);
    a.xdt = OMQ_F32; a.quantized = quantized; a.Qa = Qa;
    a.dx_dt = OMQ_F32;
    return a;
  };
  auto act = [&](LinBwd& a, int k) {
    a.h_a = v.in<float>(L.act_h[k]);
    a.z_a = v.in<int32_t>(L.act_z[k]);
    a.tok_range = v.in<omq_range>(L.act_range[k]);
  };

  // down projection: the gradient of (M D / 2) L with respect to y is res; no LET
  BLK_TRY(mk.mark(OMQ_BPH_BWD_FFN));
  {
    LinBwd a = base(L_D);
    a.Xq = v.bb<void>(OMQ_BB_QM); a.dY = v.bb<void>(OMQ_BB_RES); a.dy_scale = 1.f;
    a.X = v.bb<void>(OMQ_BB_MID); act(a, 3);
    a.dX = v.bb<void>(OMQ_BB_DMID);
    BLK_TRY(lin_bwd(a, v, st));
  }
  BLK_TRY(launch_swiglu_bwd(v.bb<float>(OMQ_BB_GU), v.bb<float>(OMQ_BB_DMID),
                            v.bb<void>(OMQ_BB_DGU), op, M, I, st));
  {
    LinBwd a = base(L_GU);
    a.Xq = v.bb<void>(OMQ_BB_QB); a.dY = v.bb<void>(OMQ_BB_DGU); a.dy_scale = 1.f;
    a.s_w = th(OMQ_TH_S2); a.shift = true;
    a.X = v.bb<void>(OMQ_BB_B); act(a, 2);
    a.s_x = th(OMQ_TH_S2); a.d_x = th(OMQ_TH_DELTA2);
    a.dX = v.bb<void>(OMQ_BB_DB);
    a.part_xs = v.in<float>(L.lin[L_GU].part_xs); a.part_xd = v.in<float>(L.lin[L_GU].part_xd);
    BLK_TRY(lin_bwd(a, v, st));
  }
  {
    RmsBwdParams r{v.bb<float>(OMQ_BB_DB), v.bb<float>(OMQ_BB_B), v.in<float>(L.rstd2),
                   v.bb<void>(OMQ_BB_RES), 1.f, M, D, v.bb<void>(OMQ_BB_DX2), op};
    BLK_TRY(launch_rms_bwd(r, st));
  }
  // output projection (its LET acts on V), then attention
  BLK_TRY(mk.mark(OMQ_BPH_BWD_ATTN));
  {
    LinBwd a = base(L_O);
    a.Xq = v.bb<void>(OMQ_BB_QO); a.dY = v.bb<void>(OMQ_BB_DX2); a.dy_scale = 1.f;
    a.s_w = th(OMQ_TH_S_O); a.shift = true;
    a.X = v.bb<void>(OMQ_BB_O); act(a, 1);
    a.dX = v.bb<void>(OMQ_BB_DO); a.dx_dt = op;
    BLK_TRY(lin_bwd(a, v, st));
  }
  {
    const uint16_t* qqkv = v.bb<uint16_t>(OMQ_BB_QQKV);
    const uint16_t* P16 = v.bb<uint16_t>(OMQ_BB_P16);
    const uint16_t* dO = v.bb<uint16_t>(OMQ_BB_DO);
    float* dP = v.in<float>(L.dP);
    uint16_t* dS = v.in<uint16_t>(L.dS);
    float* dq = v.bb<float>(OMQ_BB_DQQKV);
    // dQv_h = P_h^T dO_h;  dP_h = dO_h Qv_h^T
    BLK_TRY(gemm_heads(op, GemmOperand{P16, M, true}, M * M, GemmOperand{dO, D, true}, kHead, M,
                       kHead, M, dq + 2 * D, 3 * D, kHead, 1.f, H, 3, st));
    BLK_TRY(gemm_heads(op, GemmOperand{dO, D, false}, kHead,
                       GemmOperand{qqkv + 2 * D, 3 * D, false}, kHead, M, M, kHead, dP, 0, M * M,
                       1.f, H, 1, st));
    const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(kHead)));
    BLK_TRY(launch_softmax_bwd(v.bb<float>(OMQ_BB_P), dP, dS, op, H * M, M, scale, st));
    // dQq_h = dS_h Qk_h;  dQk_h = dS_h^T Qq_h
    BLK_TRY(gemm_heads(op, GemmOperand{dS, M, false}, M * M, GemmOperand{qqkv + D, 3 * D, true},
                       kHead, M, kHead, M, dq, 3 * D, kHead, 1.f, H, 2, st));
    BLK_TRY(gemm_heads(op, GemmOperand{dS, M, true}, M * M, GemmOperand{qqkv, 3 * D, true}, kHead,
                       M, kHead, M, dq + D, 3 * D, kHead, 1.f, H, 3, st));
    AttnPrepParams p{};
    p.qkv = v.bb<float>(OMQ_BB_QKV);
    p.cos_t = v.bb<float>(OMQ_BB_ROPE);
    p.sin_t = p.cos_t + M * 64;
    p.s_a = th(OMQ_TH_S_A);
    p.s_o = th(OMQ_TH_S_O);
    p.delta_o = th(OMQ_TH_DELTA_O);
    p.M = M; p.D = D; p.H = H;
    p.quantized = quantized;
    p.Qa = Qa;
    p.h_s = v.in<float>(L.head_h);
    p.z_s = v.in<int32_t>(L.head_z);
    p.range_s = v.in<omq_range>(L.head_range);
    p.dq = dq;
    p.dout = v.bb<void>(OMQ_BB_DQKV);
    p.dt16 = op;
    p.part_sa = v.in<float>(L.part_sa);
    p.part_so = v.in<float>(L.part_so);
    p.part_do = v.in<float>(L.part_do);
    BLK_TRY(launch_attn_prep(p, true, st));
  }
  BLK_TRY(mk.mark(OMQ_BPH_BWD_QKV));
  {
    LinBwd a = base(L_QKV);
    a.Xq = v.bb<void>(OMQ_BB_QA); a.dY = v.bb<void>(OMQ_BB_DQKV); a.dy_scale = 1.f;
    a.s_w = th(OMQ_TH_S1); a.shift = true;
    a.X = v.bb<void>(OMQ_BB_A); act(a, 0);
    a.s_x = th(OMQ_TH_S1); a.d_x = th(OMQ_TH_DELTA1);
    a.part_xs = v.in<float>(L.lin[L_QKV].part_xs); a.part_xd = v.in<float>(L.lin[L_QKV].part_xd);
    BLK_TRY(lin_bwd(a, v, st));
  }
  // LET gradients: weight-side + activation-side (or V-side) partials, fixed order
  BLK_TRY(mk.mark(OMQ_BPH_REDUCE));
  {
    const int64_t rw_qkv = ceil_div(3 * D, kRowsFusedW), rw_o = ceil_div(D, kRowsFusedW),
                  rw_gu = ceil_div(2 * I, kRowsFusedW), rx = ceil_div(M, kRowsX),
                  ra = ceil_div(M, kAttnRows);
    const LinScratch &q = L.lin[L_QKV], &o = L.lin[L_O], &g = L.lin[L_GU];
    const float gs = gscale;
    const ColReduce r[8] = {
        {v.in<float>(q.part_ws), rw_qkv, v.in<float>(q.part_xs), rx, gs, dth(OMQ_TH_S1)},
        {v.in<float>(q.part_wd), rw_qkv, v.in<float>(q.part_xd), rx, gs, dth(OMQ_TH_DELTA1)},
        {v.in<float>(o.part_ws), rw_o, v.in<float>(L.part_so), ra, gs, dth(OMQ_TH_S_O)},
        {v.in<float>(o.part_wd), rw_o, v.in<float>(L.part_do), ra, gs, dth(OMQ_TH_DELTA_O)},
        {v.in<float>(g.part_ws), rw_gu, v.in<float>(g.part_xs), rx, gs, dth(OMQ_TH_S2)},
        {v.in<float>(g.part_wd), rw_gu, v.in<float>(g.part_xd), rx, gs, dth(OMQ_TH_DELTA2)},
        {v.in<float>(L.part_sa), ra, nullptr, 0, gs, dth(OMQ_TH_S_A)},
        {v.in<float>(L.part_sa), ra, nullptr, 0, gs, dth(OMQ_TH_S_A)}};
    for (int k = 0; k < 7; k += 2)
      BLK_TRY(launch_reduce_cols(r + k, k == 6 ? 1 : 2, D, v.in<double>(L.red), st));
    // the LWC logit gradients, written by the weight-side STE completion of each linear
    BLK_TRY(launch_scale(d_theta, toff[OMQ_TH_S1], gscale, st));
  }
  return OMQ_OK;
}

}  // namespace
}  // namespace omq

using namespace omq;

extern "C" {

omq_status omq_block_theta_range(const omq_block_dims* dims, int id, int64_t* offset,
                                 int64_t* count) {
  if (!dims || !offset || !count) return OMQ_ERR_NULL;
  if (!dims_ok(*dims)) return OMQ_ERR_SHAPE;
  if (id < 0 || id > OMQ_TH_COUNT) return OMQ_ERR_SHAPE;
  int64_t off[OMQ_TH_COUNT + 1], cnt[OMQ_TH_COUNT + 1];
  theta_ranges(*dims, off, cnt);
  *offset = id == OMQ_TH_COUNT ? 0 : off[id];
  *count = cnt[id];
  return OMQ_OK;
}

size_t omq_block_workspace_bytes(const omq_block_dims* dims) {
  if (!dims || !dims_ok(*dims)) return 0;
  return block_layout(*dims).total;
}

omq_status omq_block_buffer(const omq_block_dims* dims, int id, size_t* offset, size_t* bytes) {
  if (!dims || !offset || !bytes) return OMQ_ERR_NULL;
  if (!dims_ok(*dims) || id < 0 || id >= OMQ_BB_COUNT) return OMQ_ERR_SHAPE;
  const BlockLayout L = block_layout(*dims);
  *offset = L.bb[id];
  *bytes = L.bb_bytes[id];
  return OMQ_OK;
}

static omq_status check_common(const omq_block_dims& d, const void* x, const void* const* W,
                               void* ws, size_t ws_bytes) {
  if (!x || !W[0] || !W[1] || !W[2] || !W[3]) return OMQ_ERR_NULL;
  if (!dims_ok(d)) return OMQ_ERR_SHAPE;
  if (!bits_ok(d)) return OMQ_ERR_BITS;
  if (!aligned16(x) || !aligned16(W[0]) || !aligned16(W[1]) || !aligned16(W[2]) || !aligned16(W[3]))
    return OMQ_ERR_ALIGN;
  if (!ws || ws_bytes < block_layout(d).total) return OMQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return OMQ_ERR_ALIGN;
  return OMQ_OK;
}

omq_status omq_block_step(const omq_block_args* a, void* workspace, size_t ws_bytes,
                          omq_stream_t stream) {
  if (!a) return OMQ_ERR_NULL;
  const omq_block_dims& d = a->dims;
  const void* W[L_COUNT] = {a->W_qkv, a->W_o, a->W_gu, a->W_d};
  BLK_TRY(check_common(d, a->x, W, workspace, ws_bytes));
  if (!a->y_ref || !a->theta || !a->d_theta || !a->loss) return OMQ_ERR_NULL;
  if ((a->adam_m == nullptr) != (a->adam_v == nullptr)) return OMQ_ERR_NULL;
  if (a->adam_m && a->step < 1) return OMQ_ERR_SHAPE;
  if (!aligned16(a->y_ref) || !aligned16(a->theta) || !aligned16(a->d_theta)) return OMQ_ERR_ALIGN;
  const BlockLayout L = block_layout(d);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const View v{d, L, workspace};
  const Inputs in{a->x, {W[0], W[1], W[2], W[3]}, a->y_ref, nullptr, a->theta, OMQ_F32};
  const Marks mk{a->events, st};
  BLK_TRY(block_forward(v, in, mk, st));
  BLK_TRY(block_backward(v, in, a->d_theta, mk, st));
  BLK_TRY(launch_loss_finalize(v.in<float>(L.loss_part), L.loss_tiles,
                               1.0 / (static_cast<double>(d.M) * static_cast<double>(d.D)), a->loss,
                               st));
  BLK_TRY(mk.mark(OMQ_BPH_ADAMW));
  if (a->adam_m) {
    int64_t off[OMQ_TH_COUNT + 1], cnt[OMQ_TH_COUNT + 1];
    theta_ranges(d, off, cnt);
    const int64_t n_lwc = off[OMQ_TH_S1], n_all = cnt[OMQ_TH_COUNT];
    const AdamSeg segs[2] = {
        {a->theta, a->d_theta, a->adam_m, a->adam_v, n_lwc, a->lr_lwc},
        {a->theta + n_lwc, a->d_theta + n_lwc, a->adam_m + n_lwc, a->adam_v + n_lwc, n_all - n_lwc,
         a->lr_let}};
    BLK_TRY(launch_adamw(segs, 2, 0.9f, 0.999f, 1e-8f, 0.f, a->step, st));
  }
  return mk.mark(OMQ_BPH_COUNT);
}

omq_status omq_block_reference(const omq_block_dims* dims, const void* x, const void* W_qkv,
                               const void* W_o, const void* W_gu, const void* W_d, float* y,
                               void* workspace, size_t ws_bytes, omq_stream_t stream) {
  if (!dims || !y) return OMQ_ERR_NULL;
  const void* W[L_COUNT] = {W_qkv, W_o, W_gu, W_d};
  BLK_TRY(check_common(*dims, x, W, workspace, ws_bytes));
  if (!aligned16(y)) return OMQ_ERR_ALIGN;
  const BlockLayout L = block_layout(*dims);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const View v{*dims, L, workspace};
  const Inputs in{x, {W[0], W[1], W[2], W[3]}, nullptr, y, nullptr, OMQ_F32};
  return block_forward(v, in, Marks{}, st);
}

omq_status omq_block_quant_forward(const omq_block_dims* dims, const void* x, const void* W_qkv,
                                   const void* W_o, const void* W_gu, const void* W_d,
                                   const float* theta, void* y, omq_dtype y_dt, void* workspace,
                                   size_t ws_bytes, omq_stream_t stream) {
  if (!dims || !y || !theta) return OMQ_ERR_NULL;
  if (y_dt != OMQ_F32 && y_dt != OMQ_BF16) return OMQ_ERR_DTYPE;
  const void* W[L_COUNT] = {W_qkv, W_o, W_gu, W_d};
  BLK_TRY(check_common(*dims, x, W, workspace, ws_bytes));
  if (!aligned16(y) || !aligned16(theta)) return OMQ_ERR_ALIGN;
  const BlockLayout L = block_layout(*dims);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const View v{*dims, L, workspace};
  // with theta and no target: every quantizer on, the down GEMM's epilogue writes y itself
  const Inputs in{x, {W[0], W[1], W[2], W[3]}, nullptr, y, theta, y_dt};
  return block_forward(v, in, Marks{}, st);
}

omq_status omq_block_calibrate(const omq_block_calib_args* c, void* workspace, size_t ws_bytes,
                               omq_stream_t stream) {
  if (!c) return OMQ_ERR_NULL;
  if (!c->xs || !c->y_refs || !c->theta || !c->d_theta || !c->adam_m || !c->adam_v ||
      !c->losses)
    return OMQ_ERR_NULL;
  if (c->n_samples < 1 || c->epochs < 1 || c->first_step < 1) return OMQ_ERR_SHAPE;
  const omq_block_dims& d = c->dims;
  if (!dims_ok(d)) return OMQ_ERR_SHAPE;
  const int64_t xs_stride = d.M * d.D;                 // elements per sample
  for (int64_t e = 0; e < c->epochs; ++e) {
    for (int64_t i = 0; i < c->n_samples; ++i) {
      const int64_t k = e * c->n_samples + i;
      omq_block_args a{};
      a.dims = d;
      a.x = static_cast<const uint16_t*>(c->xs) + i * xs_stride;
      a.y_ref = c->y_refs + i * xs_stride;
      a.W_qkv = c->W_qkv;
      a.W_o = c->W_o;
      a.W_gu = c->W_gu;
      a.W_d = c->W_d;
      a.theta = c->theta;
      a.d_theta = c->d_theta;
      a.loss = c->losses + k;
      a.adam_m = c->adam_m;
      a.adam_v = c->adam_v;
      a.step = c->first_step + k;
      a.lr_lwc = c->lr_lwc;
      a.lr_let = c->lr_let;
      BLK_TRY(omq_block_step(&a, workspace, ws_bytes, stream));
    }
  }
  return OMQ_OK;
}

}  // extern "C"
