// Chunked prefix of the gated delta rule (GDN, scalar gate) with a QDQ state
// on the sm_100a tensor cores: TMA staging, tcgen05.mma with TMEM
// accumulators, one CTA per (sequence, head) for d_k = d_v = 128.
//
// Algebra per 64-token chunk (PR #2497 What section: 64-token chunks, the
// WY-transformed form; PR #2507 What section: exact triangular solve), with
// G_t the within-chunk cumulative log gate, gamma_t = exp(G_t), H0 = S^T the
// chunk-start state [d_k, d_v]:
//
//   A     = strict_lower(diag(beta) (K K^T) * exp(G_r - G_i))
//   Aqk   = lower((Q K^T) * exp(G_r - G_i))
//   T     = (I + A)^-1                            (exact, blocked substitution)
//   P     = K H0,  R = diag(beta) (V - diag(gamma) P)
//   Vn    = T R                                   (= U - W H0 of the WY form)
//   O     = scale (diag(gamma) Q H0 + Aqk Vn)
//   H     = gamma_n H0 + K^T diag(exp(G_n - G_t)) Vn,   H = QDQ(H)
//
// Every product is issued transposed so that its M side is 128 (the value or
// key axis): [K;Q] K^T, H0^T [K;Q]^T, R^T T^T, Vn^T Aqk^T and K^T (dVn) each
// have M = 128.  Operands are fp16 in 128-byte-swizzled shared memory tiles;
// q/k/v (bf16) convert exactly for |x| in the fp16 range, the codes of a QDQ'd
// state are exact, and fp32 operands that are not exact (H0, R, T, dVn) are
// split into hi + lo fp16 pairs (about 22 significant bits), so the state
// chain keeps near-fp32 accuracy; output-only terms use the hi part.
//
// Roles: warps 0-3 own TMEM lanes 0-127 and run every accumulator epilogue;
// all 8 warps convert inputs and run the triangular solve; thread 0 issues
// TMA loads and MMAs.  Every mbarrier wait is bounded; on a timeout the CTA
// records kErrTimeout, stops, releases its TMEM and returns.
#pragma once

#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tc {

constexpr int kThreads = 256;
constexpr int kC = 64;      // chunk length
constexpr int kD = 128;     // d_k = d_v
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded waits give up after 2 s

// Shared-memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_KQ = 0;          // [K;Q] fp16, 2 blocks x [128 rows x 128 B]
constexpr uint32_t OFF_H = 32768;       // H0 hi (2 blocks), lo (2 blocks): [k][v]
constexpr uint32_t OFF_X = 98304;       // 48 KB, reused within a chunk (see below)
constexpr uint32_t OFF_AQK = 147456;    // Aqk fp16 [64 x 64]
constexpr uint32_t OFF_STG = 155648;    // TMA staging: Q0 Q1 K0 K1 V0 V1 (8 KB each)
constexpr uint32_t OFF_SMALL = 204800;  // gates, flags, barriers
constexpr uint32_t kSmemBytes = OFF_SMALL + 2048 + 1024;  // + alignment slack
// Region X, first half of a chunk:  R^T hi [0,16K) | R^T lo [16K,32K) |
//   T hi [32K,40K) | T lo [40K,48K); the solve uses A fp32 at [0, 16640) and
//   its partial products at [16640, 29120) before R^T is written.
// Region X, second half: Vn^T hi [0,16K) | dVn^T hi [16K,32K) | dVn^T lo [32K,48K).
constexpr uint32_t X_RHI = 0, X_RLO = 16384, X_THI = 32768, X_TLO = 40960;
constexpr uint32_t X_VN = 0, X_DVHI = 16384, X_DVLO = 32768;
constexpr uint32_t X_A32 = 0, X_P32 = 16640;
constexpr int LDS = 65;  // fp32 row stride of the solve's matrices
// TMEM columns.
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 192, TM_D4 = 256, TM_COLS = 512;

struct Small {
  float G[64], beta[64], gam[64], dec[64], ep[64], em[64];
  float red[8];
  float gn_exp;
  int direct;  // 1: per-element exp of gate differences (wide gate span)
  int abort;
  uint32_t tmem;
  uint64_t bar_qk, bar_v, bar_m1, bar_m2, bar_m3, bar_m4;
};

// Byte address of 16-byte chunk `ch` of row `r` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(uint32_t tile, int r, int ch) {
  return tile + (uint32_t)r * 128u + ((uint32_t)(ch ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// hi = fp16(x), lo = fp16(x - hi), packed in pairs.
__device__ __forceinline__ void split_h2(float a, float b, uint32_t &hi, uint32_t &lo) {
  __half2 h = __floats2half2_rn(a, b);
  float2 hf = __half22float2(h);
  hi = *reinterpret_cast<uint32_t *>(&h);
  lo = pack_h2(a - hf.x, b - hf.y);
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

// Write 64 fp32 values of one tile row as fp16 (hi only) into a [rows x 64]
// 128B-swizzled tile.
__device__ __forceinline__ void store_row_h(uint32_t tile, int r, const float *x) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    st_shared_v4(sw128(tile, r, ch), pack_h2(x[8 * ch], x[8 * ch + 1]),
                 pack_h2(x[8 * ch + 2], x[8 * ch + 3]), pack_h2(x[8 * ch + 4], x[8 * ch + 5]),
                 pack_h2(x[8 * ch + 6], x[8 * ch + 7]));
}

// Same, split into hi and lo tiles.
__device__ __forceinline__ void store_row_hl(uint32_t thi, uint32_t tlo, int r, const float *x) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
    split_h2(x[8 * ch], x[8 * ch + 1], h0, l0);
    split_h2(x[8 * ch + 2], x[8 * ch + 3], h1, l1);
    split_h2(x[8 * ch + 4], x[8 * ch + 5], h2, l2);
    split_h2(x[8 * ch + 6], x[8 * ch + 7], h3, l3);
    st_shared_v4(sw128(thi, r, ch), h0, h1, h2, h3);
    st_shared_v4(sw128(tlo, r, ch), l0, l1, l2, l3);
  }
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) {
  return sm100::smem_desc_sw128(addr, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) {
  return sm100::smem_desc_sw128(addr, lbo, 1024);
}

// Bounded wait by every calling thread; a timeout marks the CTA aborted.
__device__ __forceinline__ void wait_or_abort(uint64_t *bar, uint32_t parity, Small *sm,
                                              unsigned *err) {
  if (!sm100::mbar_wait(bar, parity, kWaitNs)) {
    sm->abort = 1;
    atomicOr(err, kErrTimeout);
  }
}

template <int QK, int GROUP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
                  const float *__restrict__ beta, const float *__restrict__ state_in,
                  const int *__restrict__ cu_seqlens, int T, int H, float scale,
                  __nv_bfloat16 *__restrict__ o, float *__restrict__ state_out,
                  unsigned *__restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw_addr);
  Small *sm = reinterpret_cast<Small *>(gbase + OFF_SMALL);
  float *sA = reinterpret_cast<float *>(gbase + OFF_X + X_A32);
  float *sP = reinterpret_cast<float *>(gbase + OFF_X + X_P32);
  float *sT = reinterpret_cast<float *>(gbase + OFF_STG);  // solve output, fp32 [64][LDS]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;  // seq * H + head
  const int h = unit % H, s = unit / H;

  long long t0, t1;
  if (cu_seqlens) {
    t0 = cu_seqlens[s];
    t1 = cu_seqlens[s + 1];
    const int n_seq = gridDim.x / H;
    if (t0 < 0 || t1 < t0 || t1 > T || (s == 0 && t0 != 0) || (s == n_seq - 1 && t1 != T)) {
      if (tid == 0) atomicOr(err, kErrBadSeqlens);
      return;
    }
  } else {
    t0 = (long long)s * T;
    t1 = t0 + T;
  }
  const long long L = t1 - t0;
  const long long st_off = (long long)unit * kD * kD;

  if (L == 0) {  // no token: the state passes through unchanged
    for (int i = tid; i < kD * kD / 4; i += kThreads) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (state_in) x = reinterpret_cast<const float4 *>(state_in + st_off)[i];
      reinterpret_cast<float4 *>(state_out + st_off)[i] = x;
    }
    return;
  }

  if (tid == 0) {
    sm100::mbar_init(&sm->bar_qk, 1);
    sm100::mbar_init(&sm->bar_v, 1);
    sm100::mbar_init(&sm->bar_m1, 1);
    sm100::mbar_init(&sm->bar_m2, 1);
    sm100::mbar_init(&sm->bar_m3, 1);
    sm100::mbar_init(&sm->bar_m4, 1);
    sm100::fence_mbar_init();
    sm->abort = 0;
  }
  if (warp == 0) {
    sm100::tmem_alloc(&sm->tmem, TM_COLS);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sm->tmem;
  const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;  // this warp's TMEM lanes

  auto issue_qk = [&](long long tb) {
    sm100::mbar_arrive_expect_tx(&sm->bar_qk, 4 * 8192);
    sm100::tma_load_3d(gbase + OFF_STG + 0, &tm_q, &sm->bar_qk, 0, h, (int)tb);
    sm100::tma_load_3d(gbase + OFF_STG + 8192, &tm_q, &sm->bar_qk, 64, h, (int)tb);
    sm100::tma_load_3d(gbase + OFF_STG + 16384, &tm_k, &sm->bar_qk, 0, h, (int)tb);
    sm100::tma_load_3d(gbase + OFF_STG + 24576, &tm_k, &sm->bar_qk, 64, h, (int)tb);
  };
  auto issue_v = [&](long long tb) {
    sm100::mbar_arrive_expect_tx(&sm->bar_v, 2 * 8192);
    sm100::tma_load_3d(gbase + OFF_STG + 32768, &tm_v, &sm->bar_v, 0, h, (int)tb);
    sm100::tma_load_3d(gbase + OFF_STG + 40960, &tm_v, &sm->bar_v, 64, h, (int)tb);
  };
  // Thread 0 tracks TMA loads issued but not yet waited for, so that an
  // aborted CTA can let them land before it exits.
  int qk_pending = 0, v_pending = 0;  // 1 + parity of the pending phase, or 0
  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    issue_qk(t0);
    issue_v(t0);
    qk_pending = v_pending = 1;
  }

  // ---- initial state: TMEM D4 (fp32) and the hi/lo fp16 operand tiles ----
  if (tid < 128) {
    const int k = tid;
    for (int p = 0; p < 4; ++p) {
      float x[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (state_in) v4 = *reinterpret_cast<const float4 *>(state_in + st_off + k * kD + 32 * p + i);
        x[i] = v4.x; x[i + 1] = v4.y; x[i + 2] = v4.z; x[i + 3] = v4.w;
      }
      sm100::tmem_st32(tmem + lane_off + TM_D4 + 32 * p, x);
      const uint32_t blk = (uint32_t)(p >> 1) * 16384u;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        split_h2(x[8 * c4], x[8 * c4 + 1], h0, l0);
        split_h2(x[8 * c4 + 2], x[8 * c4 + 3], h1, l1);
        split_h2(x[8 * c4 + 4], x[8 * c4 + 5], h2, l2);
        split_h2(x[8 * c4 + 6], x[8 * c4 + 7], h3, l3);
        const int ch = (p & 1) * 4 + c4;
        st_shared_v4(sw128(base + OFF_H + blk, k, ch), h0, h1, h2, h3);
        st_shared_v4(sw128(base + OFF_H + 32768 + blk, k, ch), l0, l1, l2, l3);
      }
    }
  }
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();

  const uint32_t ID_KQ = sm100::idesc_f16_f32(128, 64, 0, 0);
  const uint32_t ID_H2 = sm100::idesc_f16_f32(128, 128, 1, 0);
  const uint32_t ID_H2LO = sm100::idesc_f16_f32(128, 64, 1, 0);
  const uint32_t ID_64 = sm100::idesc_f16_f32(128, 64, 0, 0);
  const uint32_t ID_KV = sm100::idesc_f16_f32(128, 128, 1, 0);

  int it = 0;
  for (long long c0 = 0; c0 < L; c0 += kC, ++it) {
    const int n = (int)min((long long)kC, L - c0);
    const long long tb = t0 + c0;
    const bool last = c0 + kC >= L;
    const uint32_t par = (uint32_t)(it & 1);

    // ---- gates of this chunk (warp 0) ----
    if (warp == 0) {
      float x0 = lane < n ? __ldg(g + (tb + lane) * H + h) : 0.0f;
      float x1 = lane + 32 < n ? __ldg(g + (tb + lane + 32) * H + h) : 0.0f;
      sm->beta[lane] = lane < n ? __ldg(beta + (tb + lane) * H + h) : 0.0f;
      sm->beta[lane + 32] = lane + 32 < n ? __ldg(beta + (tb + lane + 32) * H + h) : 0.0f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
        if (lane >= off) { x0 += y0; x1 += y1; }
      }
      x1 += __shfl_sync(0xffffffffu, x0, 31);
      sm->G[lane] = x0;
      sm->G[lane + 32] = x1;
      __syncwarp();
      const float gref = sm->G[(n - 1) >> 1], gn = sm->G[n - 1], g0 = sm->G[0];
      sm->gam[lane] = expf(x0);
      sm->gam[lane + 32] = expf(x1);
      sm->dec[lane] = expf(gn - x0);
      sm->dec[lane + 32] = expf(gn - x1);
      sm->ep[lane] = expf(x0 - gref);
      sm->ep[lane + 32] = expf(x1 - gref);
      sm->em[lane] = expf(gref - x0);
      sm->em[lane + 32] = expf(gref - x1);
      if (lane == 0) {
        sm->gn_exp = expf(gn);
        sm->direct = (g0 - gref > 80.0f || gref - gn > 80.0f) ? 1 : 0;
      }
    }
    // ---- wait for Q, K; convert to fp16 [K;Q] (rows past n zeroed) ----
    wait_or_abort(&sm->bar_qk, par, sm, err);
    if (tid == 0 && !sm->abort) qk_pending = 0;
    __syncthreads();
    if (sm->abort) break;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = tid + kThreads * i;  // 2048 16-byte chunks
      const int mat = e >> 10, rem = e & 1023;
      const int blk = rem >> 9, row = (rem >> 3) & 63, ch = rem & 7;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (row < n) {
        const uint4 src = ld_shared_v4(base + OFF_STG + (uint32_t)((1 - mat) * 2 + blk) * 8192u +
                                       (uint32_t)row * 128u + (uint32_t)ch * 16u);
        const uint32_t in[4] = {src.x, src.y, src.z, src.w};
        uint32_t outw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          outw[j] = pack_h2(__uint_as_float(in[j] << 16), __uint_as_float(in[j] & 0xffff0000u));
        w = make_uint4(outw[0], outw[1], outw[2], outw[3]);
      }
      const int drow = mat * 64 + row;  // mat 0 = K rows 0-63, mat 1 = Q rows 64-127
      st_shared_v4(sw128(base + OFF_KQ + (uint32_t)blk * 16384u, drow, ch), w.x, w.y, w.z, w.w);
    }
    sm100::fence_proxy_async();
    __syncthreads();

    // ---- MMA 1: D1 = [K;Q] K^T;  MMA 2: D2 = H0^T [K;Q]^T (hi), + H0lo^T K^T ----
    if (tid == 0) {
      sm100::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a = base + OFF_KQ + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
        sm100::mma_f16_ss(tmem + TM_D1, kdesc(a), kdesc(a), ID_KQ, ks > 0);
      }
      sm100::mma_commit(&sm->bar_m1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t b = base + OFF_KQ + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
        sm100::mma_f16_ss(tmem + TM_D2, mndesc(base + OFF_H + (uint32_t)ks * 2048u, 16384),
                          kdesc(b), ID_H2, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t b = base + OFF_KQ + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
        sm100::mma_f16_ss(tmem + TM_D2, mndesc(base + OFF_H + 32768u + (uint32_t)ks * 2048u, 16384),
                          kdesc(b), ID_H2LO, 1);
      }
      sm100::mma_commit(&sm->bar_m2);
    }

    // ---- epilogue 1: A (fp32, for the solve) and Aqk (fp16 operand) ----
    if (tid < 128) {
      wait_or_abort(&sm->bar_m1, par, sm, err);
      sm100::tc_fence_after();
      float v[64];
      sm100::tmem_ld32(tmem + lane_off + TM_D1, *reinterpret_cast<float(*)[32]>(v));
      sm100::tmem_ld32(tmem + lane_off + TM_D1 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
      const bool direct = sm->direct != 0;
      if (tid < 64) {
        const int r = tid;
        const float br = sm->beta[r], epr = sm->ep[r], Gr = sm->G[r];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float e = direct ? expf(Gr - sm->G[i]) : epr * sm->em[i];
          sA[r * LDS + i] = i < r ? br * e * v[i] : 0.0f;
        }
      } else {
        const int r = tid - 64;
        const float epr = sm->ep[r], Gr = sm->G[r];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float e = direct ? expf(Gr - sm->G[i]) : epr * sm->em[i];
          v[i] = i <= r ? e * v[i] : 0.0f;
        }
        store_row_h(base + OFF_AQK, r, v);
      }
    }
    sm100::fence_proxy_async();
    __syncthreads();
    if (sm->abort) break;

    // ---- triangular solve T = (I + A)^-1, blocked by 16 ----
    // Diagonal blocks: column substitution, one thread per column.
    if (tid < 64) {
      const int b = tid >> 4, jj = tid & 15, j0 = 16 * b;
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        float acc = rr == jj ? 1.0f : 0.0f;
        if (rr > jj) {
#pragma unroll
          for (int m = 0; m < rr; ++m) acc -= sA[(j0 + rr) * LDS + j0 + m] * x[m];
        }
        x[rr] = acc;
      }
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) sT[(j0 + rr) * LDS + j0 + jj] = x[rr];
    }
    __syncthreads();
    // Block rows 1..3: P = A[rows, :] T[:, cols] over the solved part, then
    // T[rows, cols] = -T_ii P.
    for (int bi = 1; bi < 4; ++bi) {
      const int r0 = 16 * bi, ncol = 16 * bi, nel = 16 * ncol;
      for (int e = tid; e < nel; e += kThreads) {
        const int rr = e / ncol, c = e % ncol;
        float acc = 0.0f;
        for (int m = c; m < r0; ++m) acc += sA[(r0 + rr) * LDS + m] * sT[m * LDS + c];
        sP[rr * LDS + c] = acc;
      }
      __syncthreads();
      for (int e = tid; e < nel; e += kThreads) {
        const int rr = e / ncol, c = e % ncol;
        float acc = 0.0f;
        for (int m = 0; m <= rr; ++m) acc += sT[(r0 + rr) * LDS + r0 + m] * sP[m * LDS + c];
        sT[(r0 + rr) * LDS + c] = -acc;
      }
      __syncthreads();
    }
    // T -> hi/lo fp16 tiles [tok][tok'] (upper triangle zero).
    {
      const int r = tid >> 2, cpart = (tid & 3) * 16;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = cpart + i;
        x[i] = c <= r ? sT[r * LDS + c] : 0.0f;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        const float *y = x + 8 * half;
        split_h2(y[0], y[1], h0, l0);
        split_h2(y[2], y[3], h1, l1);
        split_h2(y[4], y[5], h2, l2);
        split_h2(y[6], y[7], h3, l3);
        const int ch = (cpart >> 3) + half;
        st_shared_v4(sw128(base + OFF_X + X_THI, r, ch), h0, h1, h2, h3);
        st_shared_v4(sw128(base + OFF_X + X_TLO, r, ch), l0, l1, l2, l3);
      }
    }
    sm100::fence_proxy_async();
    __syncthreads();
    // staging Q/K (which held the solve's fp32 T) is free: prefetch the next chunk
    if (tid == 0 && !last) {
      issue_qk(tb + kC);
      qk_pending = 1 + ((it + 1) & 1);
    }

    // ---- epilogue 2: R = diag(beta) (V - diag(gamma) P) -> R^T hi/lo;
    //      O accumulator initialised with gamma-scaled (Q H0)^T ----
    wait_or_abort(&sm->bar_v, par, sm, err);
    if (tid == 0 && !sm->abort) v_pending = 0;
    if (tid < 128) {
      wait_or_abort(&sm->bar_m2, par, sm, err);
      sm100::tc_fence_after();
      const int vv = tid;
      const uint8_t *stgv = gbase + OFF_STG + 32768 + (vv >> 6) * 8192 + (vv & 63) * 2;
      float x[64];
      sm100::tmem_ld32(tmem + lane_off + TM_D2, *reinterpret_cast<float(*)[32]>(x));
      sm100::tmem_ld32(tmem + lane_off + TM_D2 + 32, *reinterpret_cast<float(*)[32]>(x + 32));
#pragma unroll
      for (int t = 0; t < 64; ++t) {
        const float vt = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(stgv + t * 128));
        x[t] = t < n ? sm->beta[t] * (vt - sm->gam[t] * x[t]) : 0.0f;
      }
      store_row_hl(base + OFF_X + X_RHI, base + OFF_X + X_RLO, vv, x);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        float y[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D2 + 64 + 32 * p, y);
#pragma unroll
        for (int t = 0; t < 32; ++t) y[t] *= sm->gam[32 * p + t];
        sm100::tmem_st32(tmem + lane_off + TM_D2 + 64 + 32 * p, y);
      }
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (sm->abort) break;
    if (tid == 0 && !last) {
      issue_v(tb + kC);
      v_pending = 1 + ((it + 1) & 1);
    }

    // ---- MMA 3: Vn^T = R^T T^T (hi*hi + hi*lo + lo*hi) ----
    if (tid == 0) {
      sm100::tc_fence_after();
      const uint32_t rA[3] = {X_RHI, X_RHI, X_RLO}, tB[3] = {X_THI, X_TLO, X_THI};
#pragma unroll
      for (int pass = 0; pass < 3; ++pass)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          sm100::mma_f16_ss(tmem + TM_D3, kdesc(base + OFF_X + rA[pass] + 32u * ks),
                            kdesc(base + OFF_X + tB[pass] + 32u * ks), ID_64, pass + ks > 0);
      sm100::mma_commit(&sm->bar_m3);
    }

    // ---- epilogue 3: Vn^T hi and decayed dVn^T hi/lo; H accumulator *= gamma_n ----
    if (tid < 128) {
      wait_or_abort(&sm->bar_m3, par, sm, err);
      sm100::tc_fence_after();
      const int vv = tid;
      float x[64];
      sm100::tmem_ld32(tmem + lane_off + TM_D3, *reinterpret_cast<float(*)[32]>(x));
      sm100::tmem_ld32(tmem + lane_off + TM_D3 + 32, *reinterpret_cast<float(*)[32]>(x + 32));
      store_row_h(base + OFF_X + X_VN, vv, x);
#pragma unroll
      for (int t = 0; t < 64; ++t) x[t] *= sm->dec[t];
      store_row_hl(base + OFF_X + X_DVHI, base + OFF_X + X_DVLO, vv, x);
      const float gnx = sm->gn_exp;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float y[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D4 + 32 * p, y);
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] *= gnx;
        sm100::tmem_st32(tmem + lane_off + TM_D4 + 32 * p, y);
      }
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (sm->abort) break;

    // ---- MMA 4: O^T += Vn^T Aqk^T;  MMA 5: H += K^T dVn (hi, lo) ----
    if (tid == 0) {
      sm100::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        sm100::mma_f16_ss(tmem + TM_D2 + 64, kdesc(base + OFF_X + X_VN + 32u * ks),
                          kdesc(base + OFF_AQK + 32u * ks), ID_64, 1);
#pragma unroll
      for (int pass = 0; pass < 2; ++pass)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          sm100::mma_f16_ss(tmem + TM_D4, mndesc(base + OFF_KQ + (uint32_t)ks * 2048u, 16384),
                            kdesc(base + OFF_X + (pass ? X_DVLO : X_DVHI) + 32u * ks), ID_KV, 1);
      sm100::mma_commit(&sm->bar_m4);
    }

    // ---- epilogue 4: outputs, state QDQ, next chunk's H0 operands ----
    if (tid < 128) {
      wait_or_abort(&sm->bar_m4, par, sm, err);
      sm100::tc_fence_after();
      // O^T[v][t] -> o[t][h][v]
      const int vv = tid;
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        float y[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D2 + 64 + 32 * p, y);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int tok = 32 * p + t;
          if (tok < n) o[((tb + tok) * H + h) * kD + vv] = __float2bfloat16_rn(scale * y[t]);
        }
      }
      // H rows: this thread owns key row k = tid.  Pass 1 (FP8 tiles, INT8
      // groups of 64): amax of the two 64-column halves of the row; FP8 then
      // reduces them over all 128 rows (the tile spans every key).
      const int k = tid;
      float mh[2] = {0.f, 0.f};
      if (QK == kQdqFp8Tile || (QK == kQdqInt8 && GROUP == 64)) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float y[32];
          sm100::tmem_ld32(tmem + lane_off + TM_D4 + 32 * p, y);
          float m = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(y[i]));
          mh[p >> 1] = fmaxf(mh[p >> 1], m);
        }
      }
      if (QK == kQdqFp8Tile) {
        const float m0 = group_max<32>(mh[0]), m1 = group_max<32>(mh[1]);
        if (lane == 0) { sm->red[2 * warp] = m0; sm->red[2 * warp + 1] = m1; }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        mh[0] = fmaxf(fmaxf(sm->red[0], sm->red[2]), fmaxf(sm->red[4], sm->red[6]));
        mh[1] = fmaxf(fmaxf(sm->red[1], sm->red[3]), fmaxf(sm->red[5], sm->red[7]));
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      // Pass 2: quantize, write back the fp32 state, its hi/lo operand tiles
      // and, after the last chunk, state_out.
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float y[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D4 + 32 * p, y);
        if (QK == kQdqInt8) {
          constexpr int GW = GROUP < 32 ? GROUP : 32;  // group width inside this piece
#pragma unroll
          for (int g0 = 0; g0 < 32; g0 += GW) {
            float m = 0.f;
            if (GROUP == 64) {
              m = mh[p >> 1];
            } else {
#pragma unroll
              for (int i = 0; i < GW; ++i) m = fmaxf(m, fabsf(y[g0 + i]));
            }
            if (m == 0.0f) {
#pragma unroll
              for (int i = 0; i < GW; ++i) y[g0 + i] = 0.0f;
            } else {
              const ScaleRecip sr = make_scale(int8_scale(m));
#pragma unroll
              for (int i = 0; i < GW; ++i) y[g0 + i] = qdq_int8(y[g0 + i], sr);
            }
          }
          sm100::tmem_st32(tmem + lane_off + TM_D4 + 32 * p, y);
        } else if (QK == kQdqFp8Tile) {
          const float m = mh[p >> 1];
          if (m == 0.0f) {
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = 0.0f;
          } else {
            const ScaleRecip sr = make_scale(fp8_scale(m));
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 r2 = qdq_fp8_2(y[i], y[i + 1], sr);
              y[i] = r2.x;
              y[i + 1] = r2.y;
            }
          }
          sm100::tmem_st32(tmem + lane_off + TM_D4 + 32 * p, y);
        }
        const uint32_t blk = (uint32_t)(p >> 1) * 16384u;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          split_h2(y[8 * c4], y[8 * c4 + 1], h0, l0);
          split_h2(y[8 * c4 + 2], y[8 * c4 + 3], h1, l1);
          split_h2(y[8 * c4 + 4], y[8 * c4 + 5], h2, l2);
          split_h2(y[8 * c4 + 6], y[8 * c4 + 7], h3, l3);
          const int ch = (p & 1) * 4 + c4;
          st_shared_v4(sw128(base + OFF_H + blk, k, ch), h0, h1, h2, h3);
          st_shared_v4(sw128(base + OFF_H + 32768 + blk, k, ch), l0, l1, l2, l3);
        }
        if (last) {
          float *dst = state_out + st_off + k * kD + 32 * p;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(dst + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
        }
      }
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (sm->abort) break;
  }

  // An aborted CTA lets its outstanding TMA loads land (again bounded)
  // before its shared memory is released.
  if (tid == 0 && sm->abort) {
    if (qk_pending) (void)sm100::mbar_wait(&sm->bar_qk, (uint32_t)(qk_pending - 1), kWaitNs);
    if (v_pending) (void)sm100::mbar_wait(&sm->bar_v, (uint32_t)(v_pending - 1), kWaitNs);
  }
  __syncthreads();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace tc
}  // namespace gdn
