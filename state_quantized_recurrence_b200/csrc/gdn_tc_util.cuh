// Helpers shared by the tensor-core prefill kernels: 128-byte-swizzled
// shared-memory addressing, fp16 hi/lo operand splits, the FP8 code pair of
// the state codec, smem descriptors, and the per-chunk gate block.
#pragma once

#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tcu {

// 16-byte aligned so that both buffers of Small::gt allow float4 loads.
struct __align__(16) Gates {
  float G[64], beta[64], gam[64], dec[64], ep[64], em[64];
  float gn_exp;  // exp(G_{n-1}): decay of the chunk-start state over the chunk
  int direct;    // 1: per-element exp of gate differences (wide gate span)
};

// Byte address of 16-byte chunk `ch` of row `r` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(uint32_t tile, int r, int ch) {
  return tile + (uint32_t)r * 128u + ((uint32_t)(ch ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// x - (the low / high fp16 of an fp16 pair), exactly, as one mixed-precision
// FMA (fp16 operands, fp32 addend and result) on the FMA pipe instead of a
// conversion.
__device__ __forceinline__ float sub_h_lo(float x, uint32_t h2) {
  float d;
  asm("{\n\t.reg .f16 l, h, m;\n\tmov.b32 {l, h}, %1;\n\tmov.b16 m, 0xBC00;\n\t"
      "fma.rn.f32.f16 %0, l, m, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(x));
  return d;
}
__device__ __forceinline__ float sub_h_hi(float x, uint32_t h2) {
  float d;
  asm("{\n\t.reg .f16 l, h, m;\n\tmov.b32 {l, h}, %1;\n\tmov.b16 m, 0xBC00;\n\t"
      "fma.rn.f32.f16 %0, h, m, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(x));
  return d;
}
// hi = fp16(x), lo = fp16(x - hi), packed in pairs (x - hi is exact in fp32).
__device__ __forceinline__ void split_h2(float a, float b, uint32_t &hi, uint32_t &lo) {
  hi = pack_h2(a, b);
  lo = pack_h2(sub_h_lo(a, hi), sub_h_hi(b, hi));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// 32 fp32 values -> chunks ch0 .. ch0+3 of row r of a hi and a lo tile.
__device__ __forceinline__ void store32_hl(uint32_t thi, uint32_t tlo, int r, int ch0,
                                           const float *x) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
    split_h2(x[8 * c], x[8 * c + 1], h0, l0);
    split_h2(x[8 * c + 2], x[8 * c + 3], h1, l1);
    split_h2(x[8 * c + 4], x[8 * c + 5], h2, l2);
    split_h2(x[8 * c + 6], x[8 * c + 7], h3, l3);
    st_shared_v4(sw128(thi, r, ch0 + c), h0, h1, h2, h3);
    st_shared_v4(sw128(tlo, r, ch0 + c), l0, l1, l2, l3);
  }
}

// y[i] *= s for 32 values.
__device__ __forceinline__ void scale32(float *y, float s) {
  const uint64_t s2 = f2_pack(s, s);
#pragma unroll
  for (int i = 0; i < 32; i += 2) f2_unpack(f2_mul(f2_pack(y[i], y[i + 1]), s2), y[i], y[i + 1]);
}

// E4M3 codes of x0/s2 and x1/s2 (correctly rounded quotients from r = RN(1/s2),
// Markstein's correction), returned as an fp16 pair (exact); y0, y1 receive
// code * sd (the dequantized values for sd = the scale, possibly times a
// decay).  The fp16 -> fp32 widening runs on the FMA pipe (h2_to_f32).
__device__ __forceinline__ uint32_t fp8_code_pair(float x0, float x1, float s2, float r, float &y0,
                                                  float &y1, float sd) {
  const uint64_t x = f2_pack(x0, x1), rr = f2_pack(r, r);
  const uint64_t q = f2_mul(x, rr);
  const uint64_t t = f2_fma(f2_fma(q, f2_pack(-s2, -s2), x), rr, q);
  float t0, t1;
  f2_unpack(t, t0, t1);
  const __nv_fp8x2_storage_t f8 =
      __nv_cvt_float2_to_fp8x2(make_float2(t0, t1), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(f8, __NV_E4M3);
  const uint32_t h2 = *reinterpret_cast<const uint32_t *>(&hr);
  float c0, c1;
  h2_to_f32(h2, c0, c1);
  f2_unpack(f2_mul(f2_pack(c0, c1), f2_pack(sd, sd)), y0, y1);
  return h2;
}

// max(m, |a|, |b|) in one three-input max.
__device__ __forceinline__ float max_abs2(float m, float a, float b) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(m), "f"(fabsf(a)), "f"(fabsf(b)));
  return d;
}

// In-place bf16 -> fp16 conversion of half `part` (the key columns
// 64 part .. + 63) of one [K;Q] buffer by 256 threads, this one being `t`:
// 1024 16-byte chunks in their swizzled positions, four per thread with the
// loads in flight together; rows of tokens past n are zeroed.
__device__ __forceinline__ void convert_kq_half(uint8_t *buf, int n, int t, int part) {
  uint4 x[4];
  uint8_t *ad[4];
  bool live[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int e = u * 256 + t;  // < 1024
    const int rw = e >> 3, ch = e & 7;
    ad[u] = buf + part * 16384 + rw * 128 + ch * 16;
    live[u] = (rw & 63) < n;
    x[u] = *reinterpret_cast<const uint4 *>(ad[u]);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t in[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (live[u]) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = pack_h2(__uint_as_float(in[j] << 16), __uint_as_float(in[j] & 0xffff0000u));
    }
    *reinterpret_cast<uint4 *>(ad[u]) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// After an abort: the lane of this (converged) warp that issued its MMAs
// makes `bar` (count 1, unused so far) track all of them and waits for them
// (bounded, 2 s), so that no MMA still reads shared memory or writes TMEM
// when the CTA releases both.
__device__ __forceinline__ void drain_mmas(uint64_t *bar) {
  if (sm100::elect_one()) {
    sm100::mma_commit(bar);
    (void)sm100::mbar_wait(bar, 0, 2000000000ull);
  }
  __syncwarp();
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) {
  return sm100::smem_desc_sw128(addr, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) {
  return sm100::smem_desc_sw128(addr, lbo, 1024);
}

// Raw per-token gate inputs of one chunk held by one warp (lane t: tokens t
// and t + 32), loaded a chunk ahead so that the global-load latency is hidden.
struct GateRaw {
  float g0, g1, b0, b1;
};

__device__ __forceinline__ GateRaw load_gates_raw(const float *__restrict__ g,
                                                  const float *__restrict__ beta, long long tb,
                                                  int n, int H, int h, int lane) {
  GateRaw r;
  r.g0 = lane < n ? __ldg(g + (tb + lane) * H + h) : 0.0f;
  r.g1 = lane + 32 < n ? __ldg(g + (tb + lane + 32) * H + h) : 0.0f;
  r.b0 = lane < n ? __ldg(beta + (tb + lane) * H + h) : 0.0f;
  r.b1 = lane + 32 < n ? __ldg(beta + (tb + lane + 32) * H + h) : 0.0f;
  return r;
}

// Gates of one chunk (one warp): G = inclusive cumsum of the log gates,
// gamma = exp(G), dec = exp(G_{n-1} - G), the factors exp(+-(G - G_ref))
// around the middle token, and beta; rows past n are zero-gated.
__device__ __forceinline__ void finish_gates(Gates *gt, GateRaw r, int n, int lane) {
  float x0 = r.g0, x1 = r.g1;
  gt->beta[lane] = r.b0;
  gt->beta[lane + 32] = r.b1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
    const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
    if (lane >= off) { x0 += y0; x1 += y1; }
  }
  x1 += __shfl_sync(0xffffffffu, x0, 31);
  const int rref = (n - 1) >> 1;
  const float gref = __shfl_sync(0xffffffffu, rref < 32 ? x0 : x1, rref & 31);
  const float gn = __shfl_sync(0xffffffffu, (n - 1) < 32 ? x0 : x1, (n - 1) & 31);
  const float g0 = __shfl_sync(0xffffffffu, x0, 0);
  gt->G[lane] = x0;
  gt->G[lane + 32] = x1;
  gt->gam[lane] = expf(x0);
  gt->gam[lane + 32] = expf(x1);
  gt->dec[lane] = expf(gn - x0);
  gt->dec[lane + 32] = expf(gn - x1);
  gt->ep[lane] = expf(x0 - gref);
  gt->ep[lane + 32] = expf(x1 - gref);
  gt->em[lane] = expf(gref - x0);
  gt->em[lane + 32] = expf(gref - x1);
  if (lane == 0) {
    gt->gn_exp = expf(gn);
    gt->direct = (g0 - gref > 80.0f || gref - gn > 80.0f) ? 1 : 0;
  }
}

__device__ __forceinline__ void load_gates(Gates *gt, const float *__restrict__ g,
                                           const float *__restrict__ beta, long long tb, int n,
                                           int H, int h, int lane) {
  finish_gates(gt, load_gates_raw(g, beta, tb, n, H, h, lane), n, lane);
}

}  // namespace tcu
}  // namespace gdn
