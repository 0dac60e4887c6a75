// Chunked prefix of the gated delta rule with a QDQ state, fp32 CUDA-core
// (FFMA) kernel.  It serves the fp32 input dtype, where the tensor-core
// operand precisions cannot meet a 1e-5 tolerance.
//
// Per (sequence, head, 64-column value tile) one CTA walks the sequence in
// 64-token chunks (PR #2497 What section: "64-token chunks", the
// "WY-transformed W"; PR #2507 What section: exact triangular solve).  With
// G_r the within-chunk cumulative log gate (per key channel; a broadcast
// scalar for GDN), a reference G_ref = G[(n-1)/2] and the factored operands
//   Kp = K * exp(G - G_ref),  Km = K * exp(G_ref - G),  Qp = Q * exp(G - G_ref)
// (so Kp_r . Km_i = sum_c k_rc k_ic exp(G_rc - G_ic), bounded for i <= r),
// one chunk of n <= 64 tokens from state H0 ([d_k, 64] tile) computes
//   A     = strict_lower(diag(beta) Kp Km^T),  Aqk = lower(Qp Km^T)
//   [W|U] = (I + A)^-1 [diag(beta) K*exp(G) | diag(beta) V]   (forward subst.)
//   Vn    = U - W H0
//   O     = scale * ((Q*exp(G)) H0 + Aqk Vn)
//   H     = diag(exp(G_n)) H0 + (K*exp(G_n - G))^T Vn
//   H     = QDQ(H)                                   (every chunk end)
// Rows past the end of a partial chunk are zero-filled, which makes every
// product above ignore them without special cases.
#pragma once

#include "gdn_common.cuh"

namespace gdn {
namespace simt {

constexpr int kChunk = 64;
constexpr int kThreads = 256;
constexpr int LDV = 68;  // row stride (floats) of [64 x 64] tiles
constexpr int LDA = 66;  // row stride of A / Aqk

constexpr int LDT = 68;  // row stride of the Neumann product-form matrices

template <int DK, bool NEU = false>
struct Smem {
  static constexpr int LDK = DK + 4;
  static constexpr int kRegion = (64 * LDK > 2 * 64 * LDA) ? 64 * LDK : 2 * 64 * LDA;
  static constexpr int oK = 0;                     // K -> Kp -> diag(b) K e^G -> W
  static constexpr int oX = oK + 64 * LDK;         // Km -> Kc = K e^(Gn - G)
  static constexpr int oQ = oX + 64 * LDK;         // Q -> Qp -> Q e^G
  static constexpr int oR = oQ + 64 * LDK;         // G (cumsum) -> A | Aqk
  static constexpr int oV = oR + kRegion;          // V -> diag(b) V -> U -> Vn
  static constexpr int oH = oV + 64 * LDV;         // state tile [DK x 64]
  static constexpr int oBeta = oH + DK * LDV;
  static constexpr int oGs = oBeta + 64;           // scalar-gate cumsum
  static constexpr int oEref = oGs + 64;           // exp(G_ref)
  static constexpr int oEn = oEref + DK;           // exp(G_n)
  static constexpr int oEnr = oEn + DK;            // exp(G_n - G_ref)
  static constexpr int oGref = oEnr + DK;
  static constexpr int oGn = oGref + DK;
  static constexpr int oRed = oGn + DK;
  // Neumann solve only: T and the running power X^(2^i), [64 x LDT] each
  static constexpr int oT = (oRed + 32 + 3) & ~3;
  static constexpr int oP = oT + 64 * LDT;
  static constexpr int kFloats = NEU ? oP + 64 * LDT : oRed + 32;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

static_assert(Smem<128, true>::kBytes <= 232448, "Neumann variant exceeds shared memory");
static_assert(Smem<128, true>::oT % 4 == 0 && (LDT * 4) % 16 == 0, "float4 rows of T and P");

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// The products below run as packed f32x2 FMAs (two lanes per instruction,
// each rounded as the scalar FMA): the kernel is bound by instruction issue.
__device__ __forceinline__ uint64_t lo2(float4 v) { return f2_pack(v.x, v.y); }
__device__ __forceinline__ uint64_t hi2(float4 v) { return f2_pack(v.z, v.w); }
__device__ __forceinline__ uint64_t bc2(float x) { return f2_pack(x, x); }

// C = M1 M2 for lower-triangular 64 x 64 operands (row stride LDT), the 4 x 4
// block (rows 4 R .., columns 4 C ..) of this thread into `acc` (zero above
// the diagonal): terms with i outside [4 C, 4 R + 3] vanish because the
// operands' upper triangles are zero.
__device__ __forceinline__ void lower_mul_block(const float *M1, const float *M2, int R, int C,
                                                float (&acc)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
  if (C > R) return;
  uint64_t a01[4] = {0ull, 0ull, 0ull, 0ull}, a23[4] = {0ull, 0ull, 0ull, 0ull};
  for (int i0 = 4 * C; i0 <= 4 * R; i0 += 4) {
    float4 m2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) m2[e] = *reinterpret_cast<const float4 *>(M2 + (i0 + e) * LDT + 4 * C);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float4 m1 = *reinterpret_cast<const float4 *>(M1 + (4 * R + a) * LDT + i0);
      const float w[4] = {m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a01[a] = f2_fma(bc2(w[e]), lo2(m2[e]), a01[a]);
        a23[a] = f2_fma(bc2(w[e]), hi2(m2[e]), a23[a]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    f2_unpack(a01[a], acc[a][0], acc[a][1]);
    f2_unpack(a23[a], acc[a][2], acc[a][3]);
  }
}

// Stage one chunk's k, q (and per-key log gates) and this CTA's v columns
// into shared memory, rows past n zero.  All of a thread's global loads are
// issued before its first store, so their latencies overlap; FULL (n = 64)
// drops the row guards.
template <bool FULL, int DK, bool PER_KEY, typename Tin>
__device__ __forceinline__ void stage_chunk(const Tin *__restrict__ k, const Tin *__restrict__ q,
                                            const float *__restrict__ g,
                                            const Tin *__restrict__ v, long long tb, int n, int H,
                                            int h, int DV, int vt, int tid, float *sK, float *sQ,
                                            float *sR, float *sV) {
  constexpr int LDK = Smem<DK>::LDK;
  constexpr int KIT = 64 * (DK / 4) / kThreads, VIT = 64 * 16 / kThreads;
  static_assert(64 * (DK / 4) % kThreads == 0 && 64 * 16 % kThreads == 0, "staging split");
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 kx[KIT], qx[KIT], gx[PER_KEY ? KIT : 1], vx[VIT];
#pragma unroll
  for (int j = 0; j < KIT; ++j) {
    const int idx = tid + j * kThreads, r = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
    kx[j] = qx[j] = zero;
    if (PER_KEY) gx[j] = zero;
    if (FULL || r < n) {
      const long long off = ((tb + r) * H + h) * DK + c4;
      kx[j] = load4(k + off);
      qx[j] = load4(q + off);
      if (PER_KEY) gx[j] = load4(g + off);
    }
  }
#pragma unroll
  for (int j = 0; j < VIT; ++j) {
    const int idx = tid + j * kThreads, r = idx >> 4, c4 = (idx & 15) * 4;
    vx[j] = zero;
    if (FULL || r < n) vx[j] = load4(v + ((tb + r) * H + h) * DV + vt * 64 + c4);
  }
#pragma unroll
  for (int j = 0; j < KIT; ++j) {
    const int idx = tid + j * kThreads, r = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
    *reinterpret_cast<float4 *>(sK + r * LDK + c4) = kx[j];
    *reinterpret_cast<float4 *>(sQ + r * LDK + c4) = qx[j];
    if (PER_KEY) *reinterpret_cast<float4 *>(sR + r * LDK + c4) = gx[j];
  }
#pragma unroll
  for (int j = 0; j < VIT; ++j) {
    const int idx = tid + j * kThreads, r = idx >> 4, c4 = (idx & 15) * 4;
    *reinterpret_cast<float4 *>(sV + r * LDV + c4) = vx[j];
  }
}

// NEU: the approximate solve of the GDN/KDA approximate-inverse PR (#2507,
// What section: an explicit Neumann polynomial degree) in place of the exact
// one: T = sum_{n <= d} (-A)^n with d = 2^neu_m - 1, evaluated as
// prod_{i < neu_m} (I + X^(2^i)), X = -A.
template <typename Tin, int DK, bool PER_KEY, bool NEU>
__global__ void __launch_bounds__(kThreads, 1)
prefill_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const Tin *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta,
                    const float *__restrict__ state_in,
                    const int *__restrict__ cu_seqlens, int T, int H, int DV,
                    float scale, int qdq_kind, int qdq_group,
                    Tin *__restrict__ o, float *__restrict__ state_out,
                    unsigned *__restrict__ err, int neu_m) {
  using L = Smem<DK, NEU>;
  constexpr int LDK = L::LDK;
  extern __shared__ __align__(16) float sm[];
  float *sK = sm + L::oK, *sX = sm + L::oX, *sQ = sm + L::oQ, *sR = sm + L::oR;
  float *sA = sR, *sAqk = sR + 64 * LDA;
  float *sV = sm + L::oV, *sH = sm + L::oH, *sBeta = sm + L::oBeta;
  float *sGs = sm + L::oGs, *sEref = sm + L::oEref, *sEn = sm + L::oEn;
  float *sEnr = sm + L::oEnr, *sGref = sm + L::oGref, *sGn = sm + L::oGn;
  float *sRed = sm + L::oRed;

  const int nvt = DV >> 6;
  const int vt = blockIdx.x % nvt;
  const int h = (blockIdx.x / nvt) % H;
  int s = (blockIdx.x / nvt) / H;
  if (cu_seqlens && (int)gridDim.x / (H * nvt) <= kThreads)  // packed: longest sequences first
    s = seq_of_rank(cu_seqlens, (int)gridDim.x / (H * nvt), s);
  const int unit = s * H + h;  // (sequence, head)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rb = tid >> 4, cb = tid & 15;

  long long t0, t1;
  if (cu_seqlens) {
    t0 = cu_seqlens[s];
    t1 = cu_seqlens[s + 1];
    const int n_seq = gridDim.x / (H * nvt);
    if (t0 < 0 || t1 < t0 || t1 > T || (s == 0 && t0 != 0) || (s == n_seq - 1 && t1 != T)) {
      if (tid == 0) atomicOr(err, kErrBadSeqlens);
      return;
    }
  } else {
    t0 = (long long)s * T;
    t1 = t0 + T;
  }
  const long long L_seq = t1 - t0;

  // ---- initial state tile ----
  const long long st_off = (long long)unit * DK * DV + vt * 64;
  for (int idx = tid; idx < DK * 16; idx += kThreads) {
    const int r = idx >> 4, c4 = (idx & 15) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) x = *reinterpret_cast<const float4 *>(state_in + st_off + (long long)r * DV + c4);
    *reinterpret_cast<float4 *>(sH + r * LDV + c4) = x;
  }

  for (long long c0 = 0; c0 < L_seq; c0 += kChunk) {
    const int n = (int)min((long long)kChunk, L_seq - c0);
    const long long tb = t0 + c0;
    __syncthreads();  // previous chunk fully consumed

    // ---- P0: stage the chunk (zero rows past n) ----
    if (n == kChunk)
      stage_chunk<true, DK, PER_KEY>(k, q, g, v, tb, n, H, h, DV, vt, tid, sK, sQ, sR, sV);
    else
      stage_chunk<false, DK, PER_KEY>(k, q, g, v, tb, n, H, h, DV, vt, tid, sK, sQ, sR, sV);
    if (tid < 64) {
      sBeta[tid] = tid < n ? __ldg(beta + (tb + tid) * H + h) : 0.0f;
      if (!PER_KEY) sGs[tid] = tid < n ? __ldg(g + (tb + tid) * H + h) : 0.0f;
    }
    __syncthreads();

    // ---- P1: within-chunk cumulative log gate, reference and end rows ----
    if (PER_KEY) {
      if (tid < DK) {
        float acc = 0.0f;
        for (int r = 0; r < 64; ++r) {
          acc += sR[r * LDK + tid];
          sR[r * LDK + tid] = acc;
        }
      }
    } else if (warp == 0) {
      float x0 = sGs[lane], x1 = sGs[lane + 32];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        float y0 = __shfl_up_sync(0xffffffffu, x0, off);
        float y1 = __shfl_up_sync(0xffffffffu, x1, off);
        if (lane >= off) { x0 += y0; x1 += y1; }
      }
      x1 += __shfl_sync(0xffffffffu, x0, 31);
      sGs[lane] = x0;
      sGs[lane + 32] = x1;
    }
    __syncthreads();
    const int rref = (n - 1) >> 1;
    if (tid < DK) {
      const float gr = PER_KEY ? sR[rref * LDK + tid] : sGs[rref];
      const float gn = PER_KEY ? sR[(n - 1) * LDK + tid] : sGs[n - 1];
      sGref[tid] = gr;
      sGn[tid] = gn;
      sEref[tid] = expf(gr);
      sEn[tid] = expf(gn);
      sEnr[tid] = expf(gn - gr);
    }
    __syncthreads();

    // ---- P2: factored operands Kp, Km, Qp ----
    for (int idx = tid; idx < 64 * (DK / 4); idx += kThreads) {
      const int r = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
      float4 kx = *reinterpret_cast<float4 *>(sK + r * LDK + c4);
      float4 qx = *reinterpret_cast<float4 *>(sQ + r * LDK + c4);
      float gg[4];
      if (PER_KEY) {
        float4 gx = *reinterpret_cast<float4 *>(sR + r * LDK + c4);
        gg[0] = gx.x; gg[1] = gx.y; gg[2] = gx.z; gg[3] = gx.w;
      } else {
        gg[0] = gg[1] = gg[2] = gg[3] = sGs[r];
      }
      float ep[4], em[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ep[e] = expf(gg[e] - sGref[c4 + e]);
        em[e] = expf(sGref[c4 + e] - gg[e]);
      }
      *reinterpret_cast<float4 *>(sK + r * LDK + c4) =
          make_float4(kx.x * ep[0], kx.y * ep[1], kx.z * ep[2], kx.w * ep[3]);
      *reinterpret_cast<float4 *>(sX + r * LDK + c4) =
          make_float4(kx.x * em[0], kx.y * em[1], kx.z * em[2], kx.w * em[3]);
      *reinterpret_cast<float4 *>(sQ + r * LDK + c4) =
          make_float4(qx.x * ep[0], qx.y * ep[1], qx.z * ep[2], qx.w * ep[3]);
    }
    __syncthreads();

    // ---- P3: A = strict_lower(diag(b) Kp Km^T), Aqk = lower(Qp Km^T) ----
    {
      // each dot product as two packed partial sums (even / odd keys),
      // folded at the end
      uint64_t pA[4][4], pQ[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) pA[m][mm] = pQ[m][mm] = 0ull;
      for (int c = 0; c < DK; c += 4) {
        float4 kp[4], qp[4], km[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          kp[m] = *reinterpret_cast<float4 *>(sK + (rb + 16 * m) * LDK + c);
          qp[m] = *reinterpret_cast<float4 *>(sQ + (rb + 16 * m) * LDK + c);
          km[m] = *reinterpret_cast<float4 *>(sX + (cb + 16 * m) * LDK + c);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) {
            pA[m][mm] = f2_fma(hi2(kp[m]), hi2(km[mm]), f2_fma(lo2(kp[m]), lo2(km[mm]), pA[m][mm]));
            pQ[m][mm] = f2_fma(hi2(qp[m]), hi2(km[mm]), f2_fma(lo2(qp[m]), lo2(km[mm]), pQ[m][mm]));
          }
      }
      float accA[4][4], accQ[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          float a0, a1, q0, q1;
          f2_unpack(pA[m][mm], a0, a1);
          f2_unpack(pQ[m][mm], q0, q1);
          accA[m][mm] = a0 + a1;
          accQ[m][mm] = q0 + q1;
        }
      __syncthreads();  // the gate cumsum in sR is consumed; A/Aqk overwrite it
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = rb + 16 * m;
        const float br = sBeta[r];
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          const int i = cb + 16 * mm;
          sA[r * LDA + i] = i < r ? br * accA[m][mm] : 0.0f;
          sAqk[r * LDA + i] = i <= r ? accQ[m][mm] : 0.0f;
        }
      }
    }
    __syncthreads();

    // ---- P4: right-hand sides and the remaining scaled operands ----
    for (int idx = tid; idx < 64 * (DK / 4); idx += kThreads) {
      const int r = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
      const float br = sBeta[r];
      float4 kx = *reinterpret_cast<float4 *>(sK + r * LDK + c4);
      float4 qx = *reinterpret_cast<float4 *>(sQ + r * LDK + c4);
      float4 mx = *reinterpret_cast<float4 *>(sX + r * LDK + c4);
      const float e0 = sEref[c4], e1 = sEref[c4 + 1], e2 = sEref[c4 + 2], e3 = sEref[c4 + 3];
      *reinterpret_cast<float4 *>(sK + r * LDK + c4) =
          make_float4(br * (kx.x * e0), br * (kx.y * e1), br * (kx.z * e2), br * (kx.w * e3));
      *reinterpret_cast<float4 *>(sQ + r * LDK + c4) =
          make_float4(qx.x * e0, qx.y * e1, qx.z * e2, qx.w * e3);
      *reinterpret_cast<float4 *>(sX + r * LDK + c4) =
          make_float4(mx.x * sEnr[c4], mx.y * sEnr[c4 + 1], mx.z * sEnr[c4 + 2], mx.w * sEnr[c4 + 3]);
    }
    for (int idx = tid; idx < 64 * 16; idx += kThreads) {
      const int r = idx >> 4, c4 = (idx & 15) * 4;
      const float br = sBeta[r];
      float4 vx = *reinterpret_cast<float4 *>(sV + r * LDV + c4);
      *reinterpret_cast<float4 *>(sV + r * LDV + c4) =
          make_float4(br * vx.x, br * vx.y, br * vx.z, br * vx.w);
    }
    __syncthreads();

    if (NEU) {
      // ---- P5 (Neumann): T = prod_{i < m} (I + X^(2^i)), X = -A, then
      //      [W | U] = T RHS, one column per thread held in registers ----
      float *sT = sm + L::oT, *sP = sm + L::oP;
      for (int idx = tid; idx < 64 * 64; idx += kThreads) {
        const int r = idx >> 6, c = idx & 63;
        const float x = c < r ? -sA[r * LDA + c] : 0.0f;
        sP[r * LDT + c] = x;
        sT[r * LDT + c] = r == c ? 1.0f : x;
      }
      const int R = tid >> 4, C = tid & 15;
      for (int i = 1; i < neu_m; ++i) {
        float acc[4][4];
        __syncthreads();
        lower_mul_block(sP, sP, R, C, acc);  // P <- P P
        __syncthreads();
        if (C <= R) {
#pragma unroll
          for (int a = 0; a < 4; ++a)
            *reinterpret_cast<float4 *>(sP + (4 * R + a) * LDT + 4 * C) =
                make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        }
        __syncthreads();
        lower_mul_block(sT, sP, R, C, acc);  // T <- T + T P
        __syncthreads();
        if (C <= R) {
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            float4 *t = reinterpret_cast<float4 *>(sT + (4 * R + a) * LDT + 4 * C);
            const float4 tv = *t;
            *t = make_float4(tv.x + acc[a][0], tv.y + acc[a][1], tv.z + acc[a][2], tv.w + acc[a][3]);
          }
        }
      }
      __syncthreads();
      if (tid < DK + 64) {
        float *colp = tid < DK ? sK + tid : sV + (tid - DK);
        const int ld = tid < DK ? LDK : LDV;
        float x[kChunk];
#pragma unroll
        for (int r = 0; r < kChunk; ++r) x[r] = colp[r * ld];
        // rows past n: T is the identity there and the right-hand side zero
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
          const float *trow = sT + r * LDT;
          float p0 = 0.f, p1 = 0.f;
#pragma unroll
          for (int i = 0; i <= r; i += 2) {
            if (i + 1 <= r) {
              const float2 tt = *reinterpret_cast<const float2 *>(trow + i);
              p0 += tt.x * x[i];
              p1 += tt.y * x[i + 1];
            } else {
              p0 += trow[i] * x[i];
            }
          }
          colp[r * ld] = p0 + p1;
        }
      }
    } else {
      // ---- P5: [W | U] = (I + A)^-1 RHS by forward substitution, one column
      //      per thread held in registers ----
      if (tid < DK + 64) {
        float *colp = tid < DK ? sK + tid : sV + (tid - DK);
        const int ld = tid < DK ? LDK : LDV;
        // Rows past n are zero in A and in both right-hand sides (staged
        // zero, beta = 0), so they solve to x = 0 without a guard, and the
        // unguarded body lets rows overlap.
        float x[kChunk];
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
          // partial sums (p0, p1) and (p2, p3) as packed pairs
          uint64_t p01 = 0ull, p23 = 0ull;
          const float *arow = sA + r * LDA;
#pragma unroll
          for (int i = 0; i + 1 < r; i += 2) {
            const uint64_t aa = *reinterpret_cast<const uint64_t *>(arow + i);
            if (i & 2) p23 = f2_fma(aa, f2_pack(x[i], x[i + 1]), p23);
            else       p01 = f2_fma(aa, f2_pack(x[i], x[i + 1]), p01);
          }
          float p0, p1, p2, p3;
          f2_unpack(p01, p0, p1);
          f2_unpack(p23, p2, p3);
          if (r & 1) p0 += arow[r - 1] * x[r - 1];
          const float xr = colp[r * ld] - ((p0 + p1) + (p2 + p3));
          x[r] = xr;
          colp[r * ld] = xr;
        }
      }
    }
    __syncthreads();

    // ---- P6: Vn = U - W H0 (in place in sV), and in the same pass over H0
    //      the outputs' first term (Q e^G) H0, kept packed in o01 / o23 ----
    uint64_t o01[4], o23[4];
    {
      float acc[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float4 u4 = *reinterpret_cast<float4 *>(sV + (rb + 16 * m) * LDV + 4 * cb);
        acc[m][0] = u4.x; acc[m][1] = u4.y; acc[m][2] = u4.z; acc[m][3] = u4.w;
      }
      uint64_t a01[4], a23[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        a01[m] = f2_pack(acc[m][0], acc[m][1]);
        a23[m] = f2_pack(acc[m][2], acc[m][3]);
        o01[m] = o23[m] = 0ull;
      }
      for (int c = 0; c < DK; c += 4) {
        float4 hh[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) hh[e] = *reinterpret_cast<float4 *>(sH + (c + e) * LDV + 4 * cb);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float4 w = *reinterpret_cast<float4 *>(sK + (rb + 16 * m) * LDK + c);
          float4 qq = *reinterpret_cast<float4 *>(sQ + (rb + 16 * m) * LDK + c);
          const float we[4] = {w.x, w.y, w.z, w.w};
          const float qe[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t nw = bc2(-we[e]), q2 = bc2(qe[e]);
            a01[m] = f2_fma(nw, lo2(hh[e]), a01[m]);
            a23[m] = f2_fma(nw, hi2(hh[e]), a23[m]);
            o01[m] = f2_fma(q2, lo2(hh[e]), o01[m]);
            o23[m] = f2_fma(q2, hi2(hh[e]), o23[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        f2_unpack(a01[m], acc[m][0], acc[m][1]);
        f2_unpack(a23[m], acc[m][2], acc[m][3]);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<float4 *>(sV + (rb + 16 * m) * LDV + 4 * cb) =
            make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
    }
    __syncthreads();

    // ---- P7: O = scale ((Q e^G) H0 + Aqk Vn), the first term from P6 ----
    {
      float acc[4][4];
      uint64_t *a01 = o01, *a23 = o23;
      for (int i = 0; i < 64; i += 2) {
        float4 v0 = *reinterpret_cast<float4 *>(sV + i * LDV + 4 * cb);
        float4 v1 = *reinterpret_cast<float4 *>(sV + (i + 1) * LDV + 4 * cb);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float2 aa = *reinterpret_cast<float2 *>(sAqk + (rb + 16 * m) * LDA + i);
          const uint64_t x2 = bc2(aa.x), y2 = bc2(aa.y);
          a01[m] = f2_fma(y2, lo2(v1), f2_fma(x2, lo2(v0), a01[m]));
          a23[m] = f2_fma(y2, hi2(v1), f2_fma(x2, hi2(v0), a23[m]));
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        f2_unpack(a01[m], acc[m][0], acc[m][1]);
        f2_unpack(a23[m], acc[m][2], acc[m][3]);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = rb + 16 * m;
        if (r < n)
          store4(o + ((tb + r) * H + h) * DV + vt * 64 + 4 * cb, scale * acc[m][0],
                 scale * acc[m][1], scale * acc[m][2], scale * acc[m][3]);
      }
    }
    __syncthreads();

    // ---- P8: H = diag(e^Gn) H0 + Kc^T Vn, then QDQ (P9) ----
    {
      constexpr int RPT = DK / 16;  // rows rb*RPT .. +RPT-1, cols 4*cb .. +3
      float acc[RPT][4];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int r = rb * RPT + j;
        float4 h0 = *reinterpret_cast<float4 *>(sH + r * LDV + 4 * cb);
        const float en = sEn[r];
        acc[j][0] = en * h0.x; acc[j][1] = en * h0.y; acc[j][2] = en * h0.z; acc[j][3] = en * h0.w;
      }
      uint64_t a01[RPT], a23[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        a01[j] = f2_pack(acc[j][0], acc[j][1]);
        a23[j] = f2_pack(acc[j][2], acc[j][3]);
      }
      for (int i = 0; i < 64; ++i) {
        float4 vn = *reinterpret_cast<float4 *>(sV + i * LDV + 4 * cb);
        const uint64_t v01 = lo2(vn), v23 = hi2(vn);
#pragma unroll
        for (int j4 = 0; j4 < RPT; j4 += 4) {
          float4 kc = *reinterpret_cast<float4 *>(sX + i * LDK + rb * RPT + j4);
          const float ke[4] = {kc.x, kc.y, kc.z, kc.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t k2 = bc2(ke[e]);
            a01[j4 + e] = f2_fma(k2, v01, a01[j4 + e]);
            a23[j4 + e] = f2_fma(k2, v23, a23[j4 + e]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        f2_unpack(a01[j], acc[j][0], acc[j][1]);
        f2_unpack(a23[j], acc[j][2], acc[j][3]);
      }
      if (qdq_kind == kQdqInt8) {
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          float m = fmaxf(fmaxf(fabsf(acc[j][0]), fabsf(acc[j][1])),
                          fmaxf(fabsf(acc[j][2]), fabsf(acc[j][3])));
          for (int off = 1; off < (qdq_group >> 2); off <<= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          if (m == 0.0f) {
            acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
          } else {
            const ScaleRecip sr = make_scale(int8_scale(m));
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = qdq_int8(acc[j][e], sr);
          }
        }
      } else if (qdq_kind == kQdqFp8Tile) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < RPT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) m = fmaxf(m, fabsf(acc[j][e]));
        m = group_max<32>(m);
        if (lane == 0) sRed[warp] = m;
        __syncthreads();
        m = sRed[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, sRed[w]);
        if (m == 0.0f) {
#pragma unroll
          for (int j = 0; j < RPT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
        } else {
          const ScaleRecip sr = make_scale(fp8_scale(m));
#pragma unroll
          for (int j = 0; j < RPT; ++j) {
            float2 lo = qdq_fp8_2(acc[j][0], acc[j][1], sr);
            float2 hi = qdq_fp8_2(acc[j][2], acc[j][3], sr);
            acc[j][0] = lo.x; acc[j][1] = lo.y; acc[j][2] = hi.x; acc[j][3] = hi.y;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        *reinterpret_cast<float4 *>(sH + (rb * RPT + j) * LDV + 4 * cb) =
            make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
    }
  }
  __syncthreads();

  // ---- state out ----
  for (int idx = tid; idx < DK * 16; idx += kThreads) {
    const int r = idx >> 4, c4 = (idx & 15) * 4;
    *reinterpret_cast<float4 *>(state_out + st_off + (long long)r * DV + c4) =
        *reinterpret_cast<float4 *>(sH + r * LDV + c4);
  }
}

}  // namespace simt
}  // namespace gdn
