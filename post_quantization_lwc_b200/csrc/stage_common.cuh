// Device helpers of the row-staged encoders (the LWC weight quantizer and the per-token
// activation quantizer): cp.async copies, three-input min / max, packed f32x2 loads, tie
// counts and the binary32 encoder of omq_internal.cuh in its packed fast-path form
// ("【ICLR 2024】OmniQuant: ...", section LWC: h = (g M - b m)/Q, z = -round(b m / h),
// code = clamp(round(x / h) + z, 0, Q), x^ = (code - z) h).
#pragma once

#include "omq_internal.cuh"

namespace omq {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(a), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(a), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// three-input maximum / minimum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed binary32 pairs (the sm_100 f32x2 operations: two IEEE round-to-nearest results
// per instruction, each exactly the scalar operation's).
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ void unpack16x8_x2(const uint4& q, bool f16, float2 (&V)[4]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    V[j] = f16 ? __half22float2(*reinterpret_cast<const __half2*>(&w[j]))
               : __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
}
__device__ __forceinline__ void load_f8_x2(const float* p, int64_t off, float2 (&S)[4]) {
  const float4* q = reinterpret_cast<const float4*>(p + off);
  const float4 a = q[0], b = q[1];
  S[0] = make_float2(a.x, a.y); S[1] = make_float2(a.z, a.w);
  S[2] = make_float2(b.x, b.y); S[3] = make_float2(b.z, b.w);
}
__device__ __forceinline__ float max8(const float2 (&V)[4], float init) {
  return max3f(max3f(V[0].x, V[0].y, V[1].x), max3f(V[1].y, V[2].x, V[2].y),
               max3f(V[3].x, V[3].y, init));
}
__device__ __forceinline__ float min8(const float2 (&V)[4], float init) {
  return min3f(min3f(V[0].x, V[0].y, V[1].x), min3f(V[1].y, V[2].x, V[2].y),
               min3f(V[3].x, V[3].y, init));
}
// 1.0f where a == b, else 0.0f (one compare-and-set)
__device__ __forceinline__ float eqf(float a, float b) {
  float d;
  asm("set.eq.f32.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
// ties at the extremes of 8 values: count(v == vmax) + 512 count(v == vmin), exact in
// binary32 while the counts stay below 512
__device__ __forceinline__ float ties8(const float2 (&V)[4], float vmax, float vmin) {
  float2 t[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    t[j] = __ffma2_rn(make_float2(eqf(V[j].x, vmin), eqf(V[j].y, vmin)), f2(512.f),
                      make_float2(eqf(V[j].x, vmax), eqf(V[j].y, vmax)));
  const float2 u = __fadd2_rn(__fadd2_rn(t[0], t[1]), __fadd2_rn(t[2], t[3]));
  return __fadd_rn(u.x, u.y);
}

// A group's encoder constants. thr: the largest |ua - r| the fast path accepts (see
// encode8_x2), 0.49999 - A 2^-22 with A = max(|vmax|, |vmin|) / h bounding |ua| over the
// group; -1 (no element fast) unless A < 2^20 and |z| < 2^21.
struct StageQ {
  float h, hinv, z, thr;
};
__device__ __forceinline__ StageQ stage_q(const GroupQ& q, float vmax, float vmin) {
  StageQ r{q.h, __frcp_rn(q.h), q.z, -1.f};
  const float A = __fmul_rn(fmaxf(fabsf(vmax), fabsf(vmin)), r.hinv);
  if (fabsf(q.z) < 2097152.f && A < 1048576.f)
    r.thr = __fsub_rn(0.49999f, __fmul_rn(A, 2.384185791015625e-07f));
  return r;
}

// The encoder of encode8 for 8 values of one group, W^ packed as 16-bit values.
//
// Fast path: ua = v*hinv (hinv = 1/h correctly rounded) is within 3.0001*2^-24 |ua| <
// 2^-22 A of the correctly rounded quotient v/h (A bounds |ua| over the group, A < 2^20).
// t = ua + (B + z), B = 1.5*2^23, |z| < 2^21, lies in [2^23, 2^24) where binary32 integers
// are spaced 1 apart, so t - (B + z) = r is an integer next to ua and d = ua - r is exact;
// |d| <= thr = 0.49999 - 2^-22 A (thr itself within 2^-25 of that) then puts v/h strictly
// inside r's rounding interval, so r = rint(v/h) (a tie of ua, or of the addition, has
// |d| = 1/2 and fails the check). The code stays biased: clamp(t, B, B + Q) = B + clamp(r
// + z, 0, Q), and W^ = (clamp - (B + z)) h, every sum exact, so the result is bitwise that
// of the plain order (round, add z, clamp, subtract z, multiply by h). A lane with an
// element outside the check (about 2e-5 + 5e-7 A of them), or of a group outside the
// bounds, redoes its 8 values in the plain order with the IEEE quotient where needed.
__device__ __forceinline__ uint4 encode8_x2(const float2 (&V)[4], const StageQ& q, float Q,
                                            bool hat_f16) {
  constexpr float kBias = 12582912.f;                  // 1.5 * 2^23
  const float cz = __fadd_rn(kBias, q.z), top = __fadd_rn(kBias, Q);
  bool slow = false;
  float2 deq[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 ua = __fmul2_rn(V[j], f2(q.hinv));
    const float2 t = __fadd2_rn(ua, f2(cz));
    const float2 r = __fadd2_rn(t, f2(-cz));
    const float2 d = __ffma2_rn(r, f2(-1.f), ua);
    slow |= !(fabsf(d.x) <= q.thr) || !(fabsf(d.y) <= q.thr);
    const float2 cb = make_float2(fminf(fmaxf(t.x, kBias), top), fminf(fmaxf(t.y, kBias), top));
    deq[j] = __fmul2_rn(__fadd2_rn(cb, f2(-cz)), f2(q.h));
  }
  if (__any_sync(0xffffffffu, slow)) {
    if (slow) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float* dj = reinterpret_cast<float*>(&deq[j]);
        const float vj[2] = {V[j].x, V[j].y};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float r = round_quotient(vj[e], q.h, q.hinv);
          const float cc = fminf(fmaxf(__fadd_rn(r, q.z), 0.f), Q);
          dj[e] = __fmul_rn(__fsub_rn(cc, q.z), q.h);
        }
      }
    }
  }
  uint4 out;
  uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (hat_f16) {
      const __half2 x = __float22half2_rn(deq[j]);
      w[j] = *reinterpret_cast<const uint32_t*>(&x);
    } else {
      const __nv_bfloat162 x = __float22bfloat162_rn(deq[j]);
      w[j] = *reinterpret_cast<const uint32_t*>(&x);
    }
  }
  return out;
}

}  // namespace omq
