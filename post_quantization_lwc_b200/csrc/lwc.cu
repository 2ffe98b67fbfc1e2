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

#include <algorithm>
#include <mutex>

#include "omq_internal.cuh"
#include "stage_common.cuh"

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
  pdl_wait();
  pdl_launch();
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
  pdl_wait();
  pdl_launch();
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

// ---- row-staged launch shape -----------------------------------------------------------
// 16-bit W and W^, groups of 32, 64, 128 or 256 columns or one group per row. One warp per
// row, persistent warps: the row is copied into the warp's shared-memory buffer by 16-byte
// cp.async copies (the next piece's copies in flight while this one is encoded, when two
// buffers fit), then walked in 256-column segments by a rolled loop, lane l holding columns
// 256 i + 8 l .. + 7 of segment i. A group of G = 8 LPG columns is a sub-warp of LPG lanes;
// one group per row (LPG = 0) takes two passes over the staged row (max / min, then the
// encoder), so its piece is the whole row; grouped rows are staged in pieces of `pcols`
// columns (whole groups, whole segments), so that a long row does not take a warp's whole
// share of shared memory and the warps per SM stay many. B~[n] = B[n] + sum_k W[n,k]
// delta[k] comes out of the same pass over the row, so with B~ a warp takes whole rows
// (`per` rows: all pieces of rows wg, wg + n_warps, ...); without it the (row, piece) items
// themselves are dealt out (`per` items: wg, wg + n_warps, ...), which keeps every warp of
// the SM busy when the rows do not divide evenly among them.

constexpr int kStageSegs = 4;   // 256-column segments a grouped batch holds in registers
constexpr int64_t kStagePiece = 2048;   // columns a grouped piece holds

// Warps a block may hold: one group per row keeps few registers and takes more warps.
constexpr int stage_max_warps(int lpg) { return lpg == 0 ? 24 : 16; }

template <int LPG, bool F16>
__global__ void __launch_bounds__(32 * stage_max_warps(LPG))
    lwc_stage_kernel(LwcParams p, int nbuf, int64_t per, int64_t pcols, int by_rows) {
  pdl_wait();
  pdl_launch();
  extern __shared__ __align__(16) unsigned char lsm[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5, wpb = blockDim.x >> 5;
  const int64_t K = p.K, ng = p.ng;
  const int64_t pieces = (K + pcols - 1) / pcols, png = pcols / p.G;   // groups a piece holds
  uint16_t* rows = reinterpret_cast<uint16_t*>(lsm) + static_cast<int64_t>(wib) * nbuf * pcols;
  // grouped: per warp, nbuf staged copies of the piece's logits (gamma then beta), then the
  // piece's strengths (gamma, beta of each group interleaved)
  float* lgb = reinterpret_cast<float*>(lsm + static_cast<size_t>(wpb) * nbuf * pcols * 2) +
               static_cast<int64_t>(wib) * (nbuf + 1) * 2 * png;
  float* sst = lgb + nbuf * 2 * png;
  // warp w of block b is warp w * gridDim.x + b, so a partial last round of rows spreads
  // over all blocks
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * wpb;
  const int64_t wg = static_cast<int64_t>(wib) * gridDim.x + blockIdx.x;
  const bool hat_f16 = p.hat_dt == OMQ_F16;
  const bool let = p.s != nullptr, bias_on = p.Bt != nullptr && p.delta != nullptr;
  const int64_t items = by_rows ? per * pieces : per;   // this warp's (row, piece) items
  // row and piece of this warp's item `it`
  auto row_of = [&](int64_t it) {
    return by_rows ? wg + (it / pieces) * n_warps : (wg + it * n_warps) / pieces;
  };
  auto piece_of = [&](int64_t it) {
    return by_rows ? it % pieces : (wg + it * n_warps) % pieces;
  };
  auto issue = [&](int64_t it) {
    const int64_t n = row_of(it);
    if (it < items && n < p.N) {
      const int64_t pc0 = piece_of(it) * pcols;
      const int64_t nc = K - pc0 < pcols ? K - pc0 : pcols;
      const unsigned char* src = static_cast<const unsigned char*>(p.W) + (n * K + pc0) * 2;
      uint16_t* dst = rows + (it % nbuf) * pcols;
      for (int64_t c = lane; c < nc / 8; c += 32) cp_async16(dst + c * 8, src + c * 16);
      if constexpr (LPG != 0) {
        const int64_t g0 = pc0 / p.G, gn = nc / p.G;
        float* lg = lgb + (it % nbuf) * 2 * png;
        for (int64_t i = lane; i < 2 * gn; i += 32)
          cp_async4(lg + i, i < gn ? p.gl + n * ng + g0 + i : p.bl + n * ng + g0 + (i - gn));
      }
    }
    cp_async_commit();
  };
  issue(0);
  float2 bias2 = make_float2(0.f, 0.f);
  for (int64_t it = 0; it < items; ++it) {
    const int64_t n = row_of(it);
    if (n >= p.N) break;                                       // warp-uniform
    const int64_t pc = piece_of(it), pc0 = pc * pcols;
    const int64_t nc = K - pc0 < pcols ? K - pc0 : pcols;
    if (nbuf == 2) {
      issue(it + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint16_t* row = rows + (it % nbuf) * pcols;        // columns pc0 .. pc0 + nc - 1
    uint16_t* hat = static_cast<uint16_t*>(p.W_hat) + n * K + pc0;
    if (pc == 0) bias2 = make_float2(0.f, 0.f);
    if constexpr (LPG == 0) {
      // one group per row (the piece is the whole row): max / min over the staged row, then
      // the encoder
      const int64_t chunks = nc / 8;
      float st = 1.f;
      if (lane < 2) st = strength((lane ? p.bl : p.gl)[n]);
      float vmax = -FLT_MAX, vmin = FLT_MAX;
#pragma unroll 2
      for (int64_t c0 = 0; c0 < chunks; c0 += 32) {
        const int64_t c = c0 + lane;
        if (c < chunks) {
          float2 V[4];
          unpack16x8_x2(*reinterpret_cast<const uint4*>(row + c * 8), F16, V);
          if (let) {
            float2 S[4];
            load_f8_x2(p.s, c * 8, S);
#pragma unroll
            for (int j = 0; j < 4; ++j) V[j] = __fmul2_rn(V[j], S[j]);
          }
          vmax = max8(V, vmax);
          vmin = min8(V, vmin);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      }
      const float g = __shfl_sync(0xffffffffu, st, 0), b = __shfl_sync(0xffffffffu, st, 1);
      const GroupQ gq = group_params(g, b, vmax, vmin, p.Q);
      const StageQ q = stage_q(gq, vmax, vmin);
      int nmax = 0, nmin = 0;
      // the next round's row chunk, scale and shift are loaded before this round's store
      uint4 nraw = make_uint4(0u, 0u, 0u, 0u);
      float2 nS[4], nD[4];
      auto fetch = [&](int64_t c) {
        nraw = *reinterpret_cast<const uint4*>(row + c * 8);
        if (let) load_f8_x2(p.s, c * 8, nS);
        if (bias_on) load_f8_x2(p.delta, c * 8, nD);
      };
      if (lane < chunks) fetch(lane);
      for (int64_t c0 = 0; c0 < chunks; c0 += 32) {
        const int64_t c = c0 + lane;
        const bool ok = c < chunks;
        const uint4 raw = nraw;
        float2 S[4], D[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) { S[j] = nS[j]; D[j] = nD[j]; }
        if (c + 32 < chunks) fetch(c + 32);
        float2 V[4];
        if (ok) {
          unpack16x8_x2(raw, F16, V);
          if (bias_on) {
#pragma unroll
            for (int j = 0; j < 4; ++j) bias2 = __ffma2_rn(V[j], D[j], bias2);
          }
          if (let) {
#pragma unroll
            for (int j = 0; j < 4; ++j) V[j] = __fmul2_rn(V[j], S[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) V[j] = make_float2(0.f, 0.f);
        }
        // ties are counted only in the rare rounds where some lane's 8 values reach an
        // extreme of the row
        const bool ext = ok && !p.no_ties && (max8(V, V[0].x) == vmax || min8(V, V[0].x) == vmin);
        if (__any_sync(0xffffffffu, ext)) {
          if (ext) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              nmax += (V[j].x == vmax) + (V[j].y == vmax);
              nmin += (V[j].x == vmin) + (V[j].y == vmin);
            }
          }
        }
        const uint4 out = encode8_x2(V, q, p.Q, hat_f16);
        if (ok) *reinterpret_cast<uint4*>(hat + c * 8) = out;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
        nmin += __shfl_xor_sync(0xffffffffu, nmin, o);
      }
      if (lane == 0) {
        if (p.h) p.h[n] = q.h;
        if (p.z) p.z[n] = z_to_i32(q.z);
        if (p.range) p.range[n] = omq_range{vmax, vmin, nmax, nmin};
      }
    } else {
      // groups of 8 LPG columns: kStageSegs segments at a time; the batch's GPB groups get
      // their parameters from one lane each (lane t serves group t % GPB) and hand them back
      // by shuffles. Columns are local to the piece (global column pc0 + lc), groups too
      // (group j of the piece is group pg0 + j of the row).
      constexpr int GPS = 32 / LPG, GPB = kStageSegs * GPS;
      static_assert(GPB <= 32, "one lane per group of a batch");
      const int64_t pg0 = pc0 / p.G, gn = nc / p.G;
      const float* lg = lgb + (it % nbuf) * 2 * png;
      for (int64_t i = lane; i < 2 * gn; i += 32)
        sst[i] = strength(lg[(i & 1) * gn + (i >> 1)]);
      __syncwarp();
      const int64_t nseg = (nc + 255) / 256;
      for (int64_t s0 = 0; s0 < nseg; s0 += kStageSegs) {
        float2 V[kStageSegs][4];
        float vmx[kStageSegs], vmn[kStageSegs], cnt[kStageSegs];
#pragma unroll
        for (int u = 0; u < kStageSegs; ++u) {
          const int64_t lc = (s0 + u) * 256 + lane * 8;
          if (lc < nc) {     // whole groups: a group's lanes are all in or all out
            unpack16x8_x2(*reinterpret_cast<const uint4*>(row + lc), F16, V[u]);
            if (bias_on) {
              float2 D[4];
              load_f8_x2(p.delta, pc0 + lc, D);
#pragma unroll
              for (int j = 0; j < 4; ++j) bias2 = __ffma2_rn(V[u][j], D[j], bias2);
            }
            if (let) {
              float2 S[4];
              load_f8_x2(p.s, pc0 + lc, S);
#pragma unroll
              for (int j = 0; j < 4; ++j) V[u][j] = __fmul2_rn(V[u][j], S[j]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) V[u][j] = make_float2(0.f, 0.f);
          }
          vmx[u] = max8(V[u], V[u][0].x);
          vmn[u] = min8(V[u], V[u][0].x);
#pragma unroll
          for (int o = LPG / 2; o > 0; o >>= 1) {
            vmx[u] = fmaxf(vmx[u], __shfl_xor_sync(0xffffffffu, vmx[u], o));
            vmn[u] = fminf(vmn[u], __shfl_xor_sync(0xffffffffu, vmn[u], o));
          }
          cnt[u] = 0.f;
          if (!p.no_ties) {                                  // uniform
            cnt[u] = ties8(V[u], vmx[u], vmn[u]);
#pragma unroll
            for (int o = LPG / 2; o > 0; o >>= 1)
              cnt[u] = __fadd_rn(cnt[u], __shfl_xor_sync(0xffffffffu, cnt[u], o));
          }
        }
        // this lane's group of the batch: segment ut, sub-warp sg
        const int gb = lane % GPB, ut = gb / GPS, sg = gb % GPS, src = sg * LPG;
        float gmx = 0.f, gmn = 0.f, gc = 0.f;
#pragma unroll
        for (int u = 0; u < kStageSegs; ++u) {
          const float x = __shfl_sync(0xffffffffu, vmx[u], src);
          const float y = __shfl_sync(0xffffffffu, vmn[u], src);
          const float c = __shfl_sync(0xffffffffu, cnt[u], src);
          if (u == ut) { gmx = x; gmn = y; gc = c; }
        }
        const int64_t j = (s0 + ut) * GPS + sg;                  // group within the piece
        StageQ gq{H_FLOOR, 0.f, 0.f, 0.4f};
        if (j < gn) {
          const GroupQ q = group_params(sst[2 * j], sst[2 * j + 1], gmx, gmn, p.Q);
          gq = stage_q(q, gmx, gmn);
          if (lane < GPB) {
            const int64_t gi = n * ng + pg0 + j;
            const int ic = static_cast<int>(gc);
            if (p.h) p.h[gi] = q.h;
            if (p.z) p.z[gi] = z_to_i32(q.z);
            if (p.range) p.range[gi] = omq_range{gmx, gmn, ic & 511, ic >> 9};
          }
        }
#pragma unroll
        for (int u = 0; u < kStageSegs; ++u) {
          const int holder = u * GPS + lane / LPG;
          StageQ q;
          q.h = __shfl_sync(0xffffffffu, gq.h, holder);
          q.hinv = __shfl_sync(0xffffffffu, gq.hinv, holder);
          q.z = __shfl_sync(0xffffffffu, gq.z, holder);
          q.thr = __shfl_sync(0xffffffffu, gq.thr, holder);
          const uint4 out = encode8_x2(V[u], q, p.Q, hat_f16);
          const int64_t lc = (s0 + u) * 256 + lane * 8;
          if (lc < nc) *reinterpret_cast<uint4*>(hat + lc) = out;
        }
      }
    }
    if (p.Bt && pc == pieces - 1) {
      float bias = __fadd_rn(bias2.x, bias2.y);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bias += __shfl_xor_sync(0xffffffffu, bias, o);
      if (lane == 0) p.Bt[n] = (p.B ? p.B[n] : 0.f) + bias;
    }
    __syncwarp();                      // every lane is done with the buffer before it refills
    if (nbuf == 1) issue(it + 1);
  }
  cp_async_wait<0>();
}

// Shared memory of the row-staged shape: buffers per warp and warps per block.
struct StageShape {
  int lpg = -1;          // lanes per group (0: one group per row); -1: shape not applicable
  int nbuf = 0, wpb = 0;
  int64_t pcols = 0;     // columns a staged piece holds (the row when one group per row)
  size_t smem = 0;
};
constexpr size_t kStageSmem = 200 * 1024;

StageShape stage_shape(const LwcParams& p) {
  StageShape s;
  const bool w16 = p.wdt == OMQ_BF16 || p.wdt == OMQ_F16;
  const bool h16 = p.hat_dt == OMQ_BF16 || p.hat_dt == OMQ_F16;
  if (!w16 || !h16 || !p.W_hat || p.codes || p.packed || p.K % 8 || p.N < 1) return s;
  if (p.G == p.K) {
    if (p.K > 16384) return s;               // tie counts are packed in 16 bits
    s.lpg = 0;
  } else if (p.K % p.G == 0 && (p.G == 32 || p.G == 64 || p.G == 128 || p.G == 256)) {
    s.lpg = static_cast<int>(p.G / 8);
  } else {
    return s;
  }
  s.pcols = s.lpg == 0 ? p.K : std::min<int64_t>((p.K + 255) / 256 * 256, kStagePiece);
  const size_t row = static_cast<size_t>(s.pcols) * 2;
  // logits or strengths of a piece's groups
  const size_t lg = s.lpg ? static_cast<size_t>(s.pcols / p.G) * 8 : 0;
  const size_t cap = static_cast<size_t>(s.lpg == 0 ? stage_max_warps(0) : stage_max_warps(8));
  // two staged pieces a warp only when that still leaves room for the most warps
  s.nbuf = cap * (2 * row + 3 * lg) <= kStageSmem ? 2 : 1;
  const size_t per_warp = s.nbuf * (row + lg) + lg;
  s.wpb = static_cast<int>(std::min<size_t>(cap, kStageSmem / per_warp));
  if (s.wpb < 1) { s.lpg = -1; return s; }
  s.smem = per_warp * s.wpb;
  return s;
}

template <int LPG, bool F16>
omq_status launch_stage(const LwcParams& p, const StageShape& s, cudaStream_t stream) {
  auto kernel = lwc_stage_kernel<LPG, F16>;
  static std::mutex mu;
  static uint64_t done = 0;                  // devices opted into the large shared memory
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 64 || !(done >> dev & 1)) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kStageSmem));
      if (e == cudaSuccess && dev < 64) done |= uint64_t(1) << dev;
    }
  }
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return OMQ_ERR_CUDA;
  }
  // rows (with B~: a row's pieces stay in one warp) or (row, piece) items per warp from the
  // most warps that fit, then those warps spread over every SM
  const int64_t pieces = (p.K + s.pcols - 1) / s.pcols;
  const int by_rows = p.Bt != nullptr || pieces == 1;
  const int64_t units = by_rows ? p.N : p.N * pieces;
  const int64_t sms = num_sms();
  const int64_t per = (units + sms * s.wpb - 1) / (sms * s.wpb);
  const int64_t warps = (units + per - 1) / per;
  const int64_t wpb = std::min<int64_t>(s.wpb, (warps + sms - 1) / sms);
  const int64_t blocks = (warps + wpb - 1) / wpb;
  const size_t smem = s.smem / s.wpb * wpb;
  launch_k(kernel, static_cast<unsigned>(blocks), static_cast<unsigned>(32 * wpb), smem, stream,
      p, s.nbuf, per, s.pcols, by_rows);
  return launch_status();
}

omq_status launch_stage_any(const LwcParams& p, const StageShape& s, cudaStream_t stream) {
  const bool f16 = p.wdt == OMQ_F16;
  switch (s.lpg) {
    case 0: return f16 ? launch_stage<0, true>(p, s, stream) : launch_stage<0, false>(p, s, stream);
    case 4: return f16 ? launch_stage<4, true>(p, s, stream) : launch_stage<4, false>(p, s, stream);
    case 8: return f16 ? launch_stage<8, true>(p, s, stream) : launch_stage<8, false>(p, s, stream);
    case 16:
      return f16 ? launch_stage<16, true>(p, s, stream) : launch_stage<16, false>(p, s, stream);
    default:
      return f16 ? launch_stage<32, true>(p, s, stream) : launch_stage<32, false>(p, s, stream);
  }
}

omq_status launch_lwc(const LwcParams& p, cudaStream_t stream) {
  const int64_t total = p.N * p.ng;
  const int sms = num_sms();
  const StageShape shape = stage_shape(p);
  if (shape.lpg >= 0) return launch_stage_any(p, shape, stream);
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
      case 2: launch_k(lwc_small_kernel<2, U>, grid, 256, 0, stream, p); break;
      case 4: launch_k(lwc_small_kernel<4, U>, grid, 256, 0, stream, p); break;
      case 8: launch_k(lwc_small_kernel<8, U>, grid, 256, 0, stream, p); break;
      case 16: launch_k(lwc_small_kernel<16, U>, grid, 256, 0, stream, p); break;
      default: launch_k(lwc_small_kernel<32, U>, grid, 256, 0, stream, p); break;
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
  launch_k(lwc_large_kernel, grid, 256, smem, stream, p);
  return launch_status();
}

}  // namespace omq
