// Device helpers shared by the decode and prefill kernels: input loads, the
// state QDQ codecs, and the per-device error word.
//
// Codecs (GatedDeltaNet / KDA state-QAT pages): FP8 E4M3 with scale =
// amax / 448 and a zero guard (PR #2497 What section); INT8 with scale =
// amax / 127, round half to even and clamp to [-127, 127] (PR #2519 commit
// notes).  Every step that decides a code is an explicitly rounded IEEE fp32
// operation (__fdiv_rn, __fmul_rn, rintf, the satfinite E4M3 conversion), so
// the result does not depend on contraction or approximate division.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Error bits of the device error word.
constexpr unsigned kErrBadSeqlens = 1u;
constexpr unsigned kErrTimeout = 2u;

enum QdqKind : int { kQdqNone = 0, kQdqFp8Tile = 1, kQdqInt8 = 2 };

// ---------------------------------------------------------------- loads ----
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Four consecutive elements (16-byte aligned for fp32, 8-byte for bf16).
__device__ __forceinline__ float4 load4(const float *p) {
  return __ldg(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  uint2 r = __ldg(reinterpret_cast<const uint2 *>(p));
  float4 f;
  f.x = __uint_as_float(r.x << 16);
  f.y = __uint_as_float(r.x & 0xffff0000u);
  f.z = __uint_as_float(r.y << 16);
  f.w = __uint_as_float(r.y & 0xffff0000u);
  return f;
}

__device__ __forceinline__ void store4(float *p, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b);
  __nv_bfloat162 hi = __floats2bfloat162_rn(c, d);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t *>(&lo);
  r.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(p) = r;
}

// --------------------------------------------------------------- codecs ----
// Correctly rounded quotient x / s from y = RN(1/s): one product and
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with q0 = RN(x*y) within one ulp of x/s, the residual r = x - s*q0 is
// exact in an FMA and RN(q0 + r*y) = RN(x/s) for normal operands.
//
// A scale below 2^-100 (an all-but-zero group or tile) is first multiplied,
// together with x, by 2^64; power-of-two scaling is exact in both and keeps
// 1/s finite, so the quotient is unchanged.  Quotients small enough to be
// subnormal round to code 0 either way.
// Packed fp32 pairs (sm_100 f32x2 arithmetic: each lane rounds exactly as
// the scalar instruction, two lanes per instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
struct ScaleRecip {
  float s;    // the scale itself (dequantization multiplies by it)
  float pre;  // exact power-of-two pre-scale of x and s (1 or 2^64)
  float s2;   // s * pre
  float r;    // RN(1 / s2)
};

__device__ __forceinline__ ScaleRecip make_scale(float s) {
  ScaleRecip sr;
  sr.s = s;
  sr.pre = s < 0x1p-100f ? 0x1p64f : 1.0f;
  sr.s2 = __fmul_rn(s, sr.pre);
  sr.r = __frcp_rn(sr.s2);
  return sr;
}

__device__ __forceinline__ float div_by_scale(float x, const ScaleRecip &sr) {
  const float xs = __fmul_rn(x, sr.pre);
  const float q0 = __fmul_rn(xs, sr.r);
  const float r = __fmaf_rn(-q0, sr.s2, xs);
  return __fmaf_rn(r, sr.r, q0);
}

// div_by_scale of two values in packed f32x2 arithmetic (the same roundings).
__device__ __forceinline__ void div_by_scale2(float x0, float x1, const ScaleRecip &sr, float &q0,
                                              float &q1) {
  const uint64_t xs = f2_mul(f2_pack(x0, x1), f2_pack(sr.pre, sr.pre));
  const uint64_t rr = f2_pack(sr.r, sr.r);
  const uint64_t q = f2_mul(xs, rr);
  const uint64_t res = f2_fma(q, f2_pack(-sr.s2, -sr.s2), xs);
  f2_unpack(f2_fma(res, rr, q), q0, q1);
}

// INT8: c = clamp(rint(x / s), -127, 127); y = c * s.  s > 0.
__device__ __forceinline__ float qdq_int8(float x, const ScaleRecip &sr) {
  float c = rintf(div_by_scale(x, sr));
  c = fminf(fmaxf(c, -127.0f), 127.0f);
  return __fmul_rn(c, sr.s);
}

// The two fp32 values of an fp16 pair (exact): mixed-precision adds of -0 on
// the FMA pipe instead of two conversions.
__device__ __forceinline__ void h2_to_f32(uint32_t h2, float &a, float &b) {
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, 0f80000000;\n\tadd.rn.f32.f16 %1, h, 0f80000000;\n\t}"
      : "=f"(a), "=f"(b) : "r"(h2));
}

// E4M3 round trip of two values: RNE with saturation to +-448 (the
// conversion's satfinite mode), then back to fp32 exactly.
__device__ __forceinline__ float2 e4m3_round2(float a, float b) {
  __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(p, __NV_E4M3);
  float2 r;
  h2_to_f32(*reinterpret_cast<const uint32_t *>(&h), r.x, r.y);
  return r;
}

// FP8 tile codec for two values sharing scale s > 0.
__device__ __forceinline__ float2 qdq_fp8_2(float x0, float x1, const ScaleRecip &sr) {
  float2 c = e4m3_round2(div_by_scale(x0, sr), div_by_scale(x1, sr));
  return make_float2(__fmul_rn(c.x, sr.s), __fmul_rn(c.y, sr.s));
}

__device__ __forceinline__ float4 mul4(float4 c, float s) {
  const uint64_t s2 = f2_pack(s, s);
  float4 y;
  f2_unpack(f2_mul(f2_pack(c.x, c.y), s2), y.x, y.y);
  f2_unpack(f2_mul(f2_pack(c.z, c.w), s2), y.z, y.w);
  return y;
}

// The packed state's codes: code * s is exactly the dequantized value of the
// codecs above.  Integer-valued floats in [-2^22, 2^22] <-> their low byte /
// value through the magic constant 1.5 * 2^23: adding it rounds to the
// nearest integer (ties to even, the fp32 addition's own rounding) and leaves
// the integer in the low mantissa bits, so neither direction needs a
// float <-> int conversion instruction.
constexpr float kMagicRound = 12582912.0f;  // 1.5 * 2^23
// The four INT8 codes in the bytes of w (two's complement), exactly, as
// floats: flipping each byte's sign bit gives u = c + 128 in 0 .. 255, prmt
// puts u under the upper bytes of 1.5 * 2^23 (the float 1.5 * 2^23 + u, an
// integer where the fp32 ulp is 1), and one packed subtraction of
// 1.5 * 2^23 + 128 leaves c.
__device__ __forceinline__ float4 int8x4_to_f32(uint32_t w) {
  const uint32_t u = w ^ 0x80808080u;
  uint32_t b0, b1, b2, b3;
  asm("prmt.b32 %0, %1, 0x4B400000, 0x7650;" : "=r"(b0) : "r"(u));
  asm("prmt.b32 %0, %1, 0x4B400000, 0x7651;" : "=r"(b1) : "r"(u));
  asm("prmt.b32 %0, %1, 0x4B400000, 0x7652;" : "=r"(b2) : "r"(u));
  asm("prmt.b32 %0, %1, 0x4B400000, 0x7653;" : "=r"(b3) : "r"(u));
  const uint64_t off = f2_pack(-(kMagicRound + 128.0f), -(kMagicRound + 128.0f));
  float4 c;
  f2_unpack(f2_add(f2_pack(__uint_as_float(b0), __uint_as_float(b1)), off), c.x, c.y);
  f2_unpack(f2_add(f2_pack(__uint_as_float(b2), __uint_as_float(b3)), off), c.z, c.w);
  return c;
}

// INT8 codes of four quotients q = x / s already correctly rounded, with
// s = RN(amax / 127) of a group whose |x| <= amax: then |x| / s <=
// 127 / (1 - 2^-24) < 127 + 2^-16, so RN(q) stays below 127.5 and rounding to
// the nearest integer lands in [-127, 127] by itself; the codec's clamp is
// the identity there and is left out.  Returns the codes' two's-complement
// bytes packed low byte first; c receives the codes as floats.
__device__ __forceinline__ uint32_t int8_round4(uint64_t q01, uint64_t q23, float4 &c) {
  const uint64_t m2 = f2_pack(kMagicRound, kMagicRound);
  float t0, t1, t2, t3;
  f2_unpack(f2_add(q01, m2), t0, t1);
  f2_unpack(f2_add(q23, m2), t2, t3);
  uint32_t lo, hi, w;
  asm("prmt.b32 %0, %1, %2, 0x3340;" : "=r"(lo) : "r"(__float_as_uint(t0)), "r"(__float_as_uint(t1)));
  asm("prmt.b32 %0, %1, %2, 0x4033;" : "=r"(hi) : "r"(__float_as_uint(t2)), "r"(__float_as_uint(t3)));
  asm("prmt.b32 %0, %1, %2, 0x7610;" : "=r"(w) : "r"(lo), "r"(hi));
  const uint64_t nm2 = f2_pack(-kMagicRound, -kMagicRound);
  f2_unpack(f2_add(f2_pack(t0, t1), nm2), c.x, c.y);
  f2_unpack(f2_add(f2_pack(t2, t3), nm2), c.z, c.w);
  return w;
}

// Two E4M3 bytes (low byte first) -> their values, exactly.
__device__ __forceinline__ float2 e4m3_pair_to_f2(unsigned short p) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)p, __NV_E4M3);
  float2 r;
  h2_to_f32(*reinterpret_cast<const uint32_t *>(&h), r.x, r.y);
  return r;
}

__device__ __forceinline__ float int8_scale(float amax) { return __fdiv_rn(amax, 127.0f); }
__device__ __forceinline__ float fp8_scale(float amax) { return __fdiv_rn(amax, 448.0f); }

// Reductions over aligned lane groups of size W (power of two <= 32).
template <int W>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
  for (int off = 1; off < W; off <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}


// ------------------------------------------------------------ scheduling ----
// Longest-first order for packed batches: the CTAs of a grid are dispatched
// roughly in index order, so CTA group b takes the sequence whose length
// ranks b (descending; ties by index), which lets the long sequences start
// first and the short ones fill the tail.  Ranks are a permutation of
// 0 .. n_seq-1 for any lengths, so exactly one sequence matches.  Called by
// every thread of the block; needs n_seq <= blockDim.x (each of the first
// n_seq threads ranks one candidate).
__device__ __forceinline__ int seq_of_rank(const int *__restrict__ cu, int n_seq, int rank) {
  __shared__ int s_pick;
  const int t = threadIdx.x;
  if (t == 0) s_pick = rank;
  __syncthreads();
  if (t < n_seq) {
    const long long lt = (long long)cu[t + 1] - cu[t];
    int r = 0;
    for (int v = 0; v < n_seq; ++v) {
      const long long lv = (long long)cu[v + 1] - cu[v];
      r += (lv > lt) || (lv == lt && v < t);
    }
    if (r == rank) s_pick = t;
  }
  __syncthreads();
  return s_pick;
}

}  // namespace gdn
