// Decode step of the gated delta rule with a QDQ state (one token per
// sequence), following the recurrent suffix of the GatedDeltaNet / KDA
// state-QAT pages (recurrent_decode, PR #2519 What section):
//
//   Ht = diag(alpha) H            (alpha = exp(g) on the key rows)
//   a  = Ht^T k,  b = Ht^T q
//   u  = beta (v - a)
//   H  = Ht + k u^T
//   o  = (H^T q) / sqrt(d_k) = (b + (k^T q) u) / sqrt(d_k)
//   H  = QDQ(H)                   (after every decode token)
//
// with H = S^T stored [d_k, d_v].  The path is HBM-bound: each call reads and
// writes every state once, so the kernel streams the state once with
// coalesced loads and stores, keeps it in registers across the two key-axis
// reductions, and writes it back in place.
//
// Two state storages share the kernel:
//   fp32    the QDQ'd values, 4 bytes per element (the pages' layout);
//   packed  the codes of the same QDQ (int8, or E4M3 bytes) plus one fp32
//           scale per INT8 group / FP8 tile.  code * scale is exactly the
//           fp32 value the other storage holds, so both give bit-identical
//           results, with 1 + 4/group bytes per element moved instead of 4.
//           (The pages keep fp32 storage and mark compressed storage as not
//           done, PR #2497 What section; it is an added interface.)
//
// Work split: one 256-thread CTA per (sequence, head, 64-column value tile),
// i.e. a d_k x 64 slab - exactly one FP8 scale tile.  Thread t owns columns
// 4*(t % 16) .. +3 of rows (t / 16) + 16 j, so a warp reads two full row
// segments per load instruction, an INT8 group of 32 columns lives in 8
// consecutive lanes, and the key-axis reductions are one xor-16 shuffle plus
// an 8-warp shared-memory pass.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

// Where the state of one (sequence, head) lives.
struct StateRef {
  float *vals;     // fp32 storage: [d_k, d_v]
  uint8_t *codes;  // packed storage: [d_k, d_v] one byte per element
  float *scales;   // packed storage: INT8 [d_k, d_v / GROUP], FP8 [d_v / 64]
};

// Reduce-scatter of row maxima over the 2 D lanes of a group: on entry w
// holds this lane's maxima of K rows; each exchange at lane distance d
// halves the rows a lane keeps (the upper half where bit d of its lane index
// is set) and merges in its partner's maxima of them, until SPL rows are
// left; further exchanges only merge.  On exit w[0 .. SPL) are the group
// maxima of the rows scatter_owner names.
template <int D, int K, int SPL, int N>
__device__ __forceinline__ void scatter_max(float (&w)[N], int li) {
  if constexpr (D >= 1) {
    if constexpr (K > SPL) {
      const bool up = (li & D) != 0;
#pragma unroll
      for (int i = 0; i < K / 2; ++i) {
        const float send = up ? w[i] : w[i + K / 2];
        const float keep = up ? w[i + K / 2] : w[i];
        w[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, D));
      }
      scatter_max<D / 2, K / 2, SPL, N>(w, li);
    } else {
#pragma unroll
      for (int i = 0; i < SPL; ++i) w[i] = fmaxf(w[i], __shfl_xor_sync(0xffffffffu, w[i], D));
      scatter_max<D / 2, K, SPL, N>(w, li);
    }
  }
}
// The lane (within its group) that holds row j's group maximum after
// scatter_max<D, K, SPL>, in slot j % SPL: the halving exchanges map row bit
// K / 2 to lane bit D, row bit K / 4 to lane bit D / 2, and so on.
template <int D, int K, int SPL>
__host__ __device__ constexpr int scatter_owner(int j) {
  if constexpr (D >= 1 && K > SPL)
    return ((j & (K / 2)) ? D : 0) + scatter_owner<D / 2, K / 2, SPL>(j);
  else
    return 0;
}

template <int DK, int DV, int QK, int GROUP, bool PACKED>
struct StateIO {
  static constexpr int RPT = DK / 16;  // state rows per thread

  // The fp32 values code * scale of a thread's packed codes: cw[j] holds
  // the four codes of row rg + 16 j, sc[j] its INT8 group scale (FP8: sc[0]
  // is the tile scale).
  __device__ __forceinline__ static void dequant(const uint32_t (&cw)[RPT], const float (&sc)[RPT],
                                                 float4 (&h)[RPT]) {
    if (QK == kQdqInt8) {
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const uint32_t w = cw[j];
        h[j] = mul4(int8x4_to_f32(w), sc[j]);
      }
    } else {
      const float st = sc[0];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const float2 lo = e4m3_pair_to_f2((unsigned short)(cw[j] & 0xffffu));
        const float2 hi = e4m3_pair_to_f2((unsigned short)(cw[j] >> 16));
        h[j] = mul4(make_float4(lo.x, lo.y, hi.x, hi.y), st);
      }
    }
  }

  // Row `r`, columns col .. col+3 of the state, as fp32 values.
  __device__ __forceinline__ static void load(const StateRef &sr, int rg, int col, float4 (&h)[RPT]) {
    if (!PACKED) {
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        h[j] = __ldcs(reinterpret_cast<const float4 *>(sr.vals + (rg + 16 * j) * DV + col));
    } else {
      uint32_t cw[RPT];
      float s[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        cw[j] = __ldcs(reinterpret_cast<const unsigned int *>(sr.codes + (rg + 16 * j) * DV + col));
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        s[j] = QK == kQdqInt8 ? __ldg(sr.scales + (rg + 16 * j) * (DV / GROUP) + col / GROUP)
                              : (j == 0 ? __ldg(sr.scales + col / 64) : 0.0f);
      dequant(cw, s, h);
    }
  }

  // QDQ of the slab and store: fp32 values, or codes + scales.  `red` is 8
  // floats of shared memory (FP8 tile amax); called by all 256 threads.
  __device__ __forceinline__ static void qdq_store(const StateRef &sr, int rg, int col, int lane,
                                                   int warp, float *red, float4 (&h)[RPT]) {
    uint32_t cw[RPT];  // packed codes, 4 per row
    if (QK == kQdqInt8) {
      // Row maxima over each group (GROUP / 4 consecutive lanes hold one
      // group of a row), reduced and scattered at once: after the exchange
      // each lane holds the group maxima of SPL rows (scatter_max), computes
      // their scales and reciprocals (one IEEE division per lane, not per
      // row), and the group's lanes fetch them back row by row.
      constexpr int GL = GROUP / 4;
      constexpr int SPL = RPT / GL > 0 ? RPT / GL : 1;
      const int li = lane % GL;
      float m[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        asm("max.f32 %0, %1, %2, %3;" : "=f"(m[j]) : "f"(fabsf(h[j].x)), "f"(fabsf(h[j].y)),
            "f"(fmaxf(fabsf(h[j].z), fabsf(h[j].w))));
      scatter_max<GL / 2, RPT, SPL>(m, li);
      // s = amax / 127 (0 for an all-zero group, whose values are all +-0 and
      // give code 0 with any finite reciprocal); r = RN(1 / s), 1 for an
      // all-zero group and +inf where amax / 127 underflows to 0
      float s_own[SPL], r_own[SPL];
      bool tiny = false;
#pragma unroll
      for (int i = 0; i < SPL; ++i) {
        s_own[i] = int8_scale(m[i]);
        r_own[i] = s_own[i] > 0.0f ? __frcp_rn(s_own[i]) : (m[i] > 0.0f ? __int_as_float(0x7f800000) : 1.0f);
        tiny |= m[i] > 0.0f && s_own[i] < 0x1p-100f;
      }
      // A scale below 2^-100 (or one that underflowed) takes the scalar
      // codec's steps: the pre-scaled quotient and the clamp, which such a
      // scale needs since its relative rounding error is not bounded by
      // 2^-24.  Every other row divides directly, and |x| / s < 127 + 2^-16
      // makes its clamp the identity (int8_round4).
      const bool any_tiny = __any_sync(0xffffffffu, tiny);
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int src = (lane & ~(GL - 1)) | scatter_owner<GL / 2, RPT, SPL>(j);
        const float sj = __shfl_sync(0xffffffffu, s_own[j % SPL], src);
        const float rj = __shfl_sync(0xffffffffu, r_own[j % SPL], src);
        uint64_t q01, q23;
        if (!any_tiny) {
          const uint64_t rr = f2_pack(rj, rj), ns = f2_pack(-sj, -sj);
          const uint64_t x01 = f2_pack(h[j].x, h[j].y), x23 = f2_pack(h[j].z, h[j].w);
          q01 = f2_mul(x01, rr);
          q23 = f2_mul(x23, rr);
          q01 = f2_fma(f2_fma(q01, ns, x01), rr, q01);
          q23 = f2_fma(f2_fma(q23, ns, x23), rr, q23);
        } else {
          ScaleRecip sr;
          sr.s = sj;
          sr.pre = sj < 0x1p-100f ? 0x1p64f : 1.0f;
          sr.s2 = __fmul_rn(sj, sr.pre);
          sr.r = sr.pre == 1.0f ? rj : __frcp_rn(sr.s2);
          float q[4];
          div_by_scale2(h[j].x, h[j].y, sr, q[0], q[1]);
          div_by_scale2(h[j].z, h[j].w, sr, q[2], q[3]);
          const bool zero_row = sj == 0.0f && rj == 1.0f;
#pragma unroll
          for (int e = 0; e < 4; ++e) q[e] = zero_row ? 0.0f : fminf(fmaxf(q[e], -127.0f), 127.0f);
          q01 = f2_pack(q[0], q[1]);
          q23 = f2_pack(q[2], q[3]);
        }
        float4 c;
        cw[j] = int8_round4(q01, q23, c);
        if (!PACKED) h[j] = mul4(c, sj);
        if (PACKED && (col % GROUP) == 0)
          sr.scales[(rg + 16 * j) * (DV / GROUP) + col / GROUP] = sj;
      }
    } else if (QK == kQdqFp8Tile) {
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(h[j].x), fabsf(h[j].y)), fmaxf(fabsf(h[j].z), fabsf(h[j].w))));
      m = group_max<32>(m);
      if (lane == 0) red[warp] = m;
      __syncthreads();
      m = red[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
      if (m == 0.0f) {
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          cw[j] = 0u;
        }
      } else {
        const ScaleRecip s = make_scale(fp8_scale(m));
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          // the quotients in packed pairs (the scalar codec's roundings)
          float q0, q1, q2, q3;
          div_by_scale2(h[j].x, h[j].y, s, q0, q1);
          div_by_scale2(h[j].z, h[j].w, s, q2, q3);
          const unsigned short lo = (unsigned short)__nv_cvt_float2_to_fp8x2(
              make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
          const unsigned short hi = (unsigned short)__nv_cvt_float2_to_fp8x2(
              make_float2(q2, q3), __NV_SATFINITE, __NV_E4M3);
          if (PACKED) {
            cw[j] = (uint32_t)lo | ((uint32_t)hi << 16);
          } else {
            const float2 a = e4m3_pair_to_f2(lo), b = e4m3_pair_to_f2(hi);
            h[j] = mul4(make_float4(a.x, a.y, b.x, b.y), s.s);
          }
        }
      }
      if (PACKED && rg == 0 && (col % 64) == 0) sr.scales[col / 64] = m == 0.0f ? 0.0f : fp8_scale(m);
    }
    if (!PACKED) {
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        __stcs(reinterpret_cast<float4 *>(sr.vals + (rg + 16 * j) * DV + col), h[j]);
    } else {
#pragma unroll
      for (int j = 0; j < RPT; ++j)
        __stcs(reinterpret_cast<unsigned int *>(sr.codes + (rg + 16 * j) * DV + col), cw[j]);
    }
  }
};

// The token update of one slab once its state (h), k, q, the decays and v
// are staged: decay, the key-axis reductions, the output, the delta update,
// the QDQ and the store.  Shared by both decode kernels, so the fp32 and the
// packed storage run the same arithmetic.
// Key-indexed vectors (k, q, the per-key decay) are staged in shared memory
// permuted, row r at (r % 16) * (d_k / 16) + r / 16, so that the d_k / 16
// rows rg, rg + 16, ... of a thread are contiguous and arrive in 128-bit loads.
template <int DK>
__host__ __device__ constexpr int key_slot(int r) {
  return (r % 16) * (DK / 16) + r / 16;
}
template <int RPT>
__device__ __forceinline__ void load_rows(const float *s, int rg, float (&x)[RPT]) {
#pragma unroll
  for (int j = 0; j < RPT; j += 4) {
    const float4 v = *reinterpret_cast<const float4 *>(s + rg * RPT + j);
    x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
  }
}

template <typename Tin, int DK, int DV, bool PER_KEY, int QK, int GROUP, bool PACKED>
__device__ __forceinline__ void decode_slab(float4 (&h)[DK / 16], const float *s_k,
                                            const float *s_q, const float *s_al, float a_scalar,
                                            float bt, float4 v4, float4 (*red_a)[16],
                                            float4 (*red_b)[16], float *red_m, float *s_kq,
                                            const StateRef &sr, Tin *__restrict__ o_row, int col,
                                            float scale) {
  using IO = StateIO<DK, DV, QK, GROUP, PACKED>;
  constexpr int RPT = IO::RPT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 15, rg = tid >> 4;

  // Decay and the partial key-axis reductions a = Ht^T k, b = Ht^T q.
  // (fp32 pairs in packed f32x2 arithmetic: each lane rounds as the scalar
  // instruction)
  float kv[RPT], qv[RPT], av[RPT];
  load_rows<RPT>(s_k, rg, kv);
  load_rows<RPT>(s_q, rg, qv);
  if (PER_KEY) load_rows<RPT>(s_al, rg, av);
  uint64_t pa01 = 0, pa23 = 0, pb01 = 0, pb23 = 0;  // +0.0 pairs
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const float al = PER_KEY ? av[j] : a_scalar, kr = kv[j], qr = qv[j];
    const uint64_t al2 = f2_pack(al, al), kr2 = f2_pack(kr, kr), qr2 = f2_pack(qr, qr);
    const uint64_t h01 = f2_mul(f2_pack(h[j].x, h[j].y), al2);
    const uint64_t h23 = f2_mul(f2_pack(h[j].z, h[j].w), al2);
    f2_unpack(h01, h[j].x, h[j].y);
    f2_unpack(h23, h[j].z, h[j].w);
    pa01 = f2_fma(h01, kr2, pa01); pa23 = f2_fma(h23, kr2, pa23);
    pb01 = f2_fma(h01, qr2, pb01); pb23 = f2_fma(h23, qr2, pb23);
  }
  float pa[4], pb[4];
  f2_unpack(pa01, pa[0], pa[1]); f2_unpack(pa23, pa[2], pa[3]);
  f2_unpack(pb01, pb[0], pb[1]); f2_unpack(pb23, pb[2], pb[3]);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    pa[e] += __shfl_xor_sync(0xffffffffu, pa[e], 16);
    pb[e] += __shfl_xor_sync(0xffffffffu, pb[e], 16);
  }
  if (lane < 16) {
    red_a[warp][cq] = make_float4(pa[0], pa[1], pa[2], pa[3]);
    red_b[warp][cq] = make_float4(pb[0], pb[1], pb[2], pb[3]);
  }
  __syncthreads();
  // the 8 warps' partial sums, in warp order (packed pairs, the scalar
  // additions' roundings), formed once per column by warp 0 (lanes 0-15: a,
  // 16-31: b) into row 0 and read back by every thread; warp 1 forms k^T q
  if (warp == 1) {
    float kq = 0.0f;
#pragma unroll
    for (int r = lane; r < DK; r += 32) kq += s_k[key_slot<DK>(r)] * s_q[key_slot<DK>(r)];
    kq = warp_sum(kq);
    if (lane == 0) *s_kq = kq;
  }
  if (warp == 0) {
    float4(*red)[16] = lane < 16 ? red_a : red_b;
    const int c = lane & 15;
    uint64_t s01 = 0, s23 = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float4 x = red[w][c];
      s01 = f2_add(s01, f2_pack(x.x, x.y));
      s23 = f2_add(s23, f2_pack(x.z, x.w));
    }
    float4 r;
    f2_unpack(s01, r.x, r.y);
    f2_unpack(s23, r.z, r.w);
    red[0][c] = r;
  }
  __syncthreads();
  const float4 sa = red_a[0][cq], sb = red_b[0][cq];
  const uint64_t a01 = f2_pack(sa.x, sa.y), a23 = f2_pack(sa.z, sa.w);
  const uint64_t b01 = f2_pack(sb.x, sb.y), b23 = f2_pack(sb.z, sb.w);
  float a[4], b[4], u[4];
  f2_unpack(a01, a[0], a[1]); f2_unpack(a23, a[2], a[3]);
  f2_unpack(b01, b[0], b[1]); f2_unpack(b23, b[2], b[3]);
  {
    const uint64_t bt2 = f2_pack(bt, bt);
    f2_unpack(f2_mul(bt2, f2_add(f2_pack(v4.x, v4.y), f2_pack(-a[0], -a[1]))), u[0], u[1]);
    f2_unpack(f2_mul(bt2, f2_add(f2_pack(v4.z, v4.w), f2_pack(-a[2], -a[3]))), u[2], u[3]);
  }
  if (rg == 0) {
    const float kq = *s_kq;
    store4(o_row + col, scale * fmaf(kq, u[0], b[0]), scale * fmaf(kq, u[1], b[1]),
           scale * fmaf(kq, u[2], b[2]), scale * fmaf(kq, u[3], b[3]));
  }

  // Delta update H = Ht + k u^T.
  const uint64_t u01 = f2_pack(u[0], u[1]), u23 = f2_pack(u[2], u[3]);
  load_rows<RPT>(s_k, rg, kv);
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const float kr = kv[j];
    const uint64_t kr2 = f2_pack(kr, kr);
    f2_unpack(f2_fma(kr2, u01, f2_pack(h[j].x, h[j].y)), h[j].x, h[j].y);
    f2_unpack(f2_fma(kr2, u23, f2_pack(h[j].z, h[j].w)), h[j].z, h[j].w);
  }

  // State QDQ and store.
  IO::qdq_store(sr, rg, col, lane, warp, red_m, h);
}

__device__ __forceinline__ StateRef state_ref(float *state, uint8_t *codes, float *scales,
                                              long long unit, int dk_dv, int n_scales) {
  StateRef sr;
  sr.vals = state ? state + unit * (long long)dk_dv : nullptr;
  sr.codes = codes ? codes + unit * (long long)dk_dv : nullptr;
  sr.scales = scales ? scales + unit * (long long)n_scales : nullptr;
  return sr;
}

// One 256-thread CTA per slab.  QK: kQdqNone / kQdqFp8Tile / kQdqInt8;
// GROUP: INT8 group width (16/32/64); PACKED: the state is stored as codes +
// scales (QK != kQdqNone).  k, q and the per-key decays sit in shared memory
// so the state values are the only large register footprint: <= 64
// registers give 4 CTAs per SM (128 KB of fp32 state loads in flight; a few
// spilled bytes in some specialisations cost less than a fourth of the CTA
// slots: 3 CTAs per SM measured 8 % slower on the serving workload).
template <typename Tin, int DK, int DV, bool PER_KEY, int QK, int GROUP, bool PACKED>
__global__ void __launch_bounds__(256, 4)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
              const Tin *__restrict__ v, const float *__restrict__ g,
              const float *__restrict__ beta, float *__restrict__ state,
              uint8_t *__restrict__ codes, float *__restrict__ scales,
              Tin *__restrict__ o, float scale) {
  using IO = StateIO<DK, DV, QK, GROUP, PACKED>;
  constexpr int NSC = QK == kQdqInt8 ? DK * (DV / GROUP) : DV / 64;  // scales per state
  // row-permuted (key_slot), 16-byte aligned for the 128-bit row loads
  __shared__ __align__(16) float s_k[DK];
  __shared__ __align__(16) float s_q[DK];
  __shared__ __align__(16) float s_al[PER_KEY ? DK : 4];
  __shared__ float4 red_a[8][16], red_b[8][16];
  __shared__ float red_m[8];
  __shared__ float s_kq;

  constexpr int nvt = DV / 64;
  const long long unit = blockIdx.x / nvt;  // sequence * H + head
  const int vt = blockIdx.x - (int)(unit * nvt);
  const int tid = threadIdx.x;
  const int col = vt * 64 + (tid & 15) * 4, rg = tid >> 4;

  const StateRef sr = state_ref(state, codes, scales, unit, DK * DV, NSC);
  // Issue the state loads first: they are the only HBM-sized traffic.
  float4 h[IO::RPT];
  IO::load(sr, rg, col, h);

  if (tid < DK) {
    s_k[key_slot<DK>(tid)] = to_f32(k[unit * DK + tid]);
    s_q[key_slot<DK>(tid)] = to_f32(q[unit * DK + tid]);
    if (PER_KEY) s_al[key_slot<DK>(tid)] = expf(__ldg(g + unit * DK + tid));
  }
  const float bt = __ldg(beta + unit);
  const float a_scalar = PER_KEY ? 0.0f : expf(__ldg(g + unit));
  const float4 v4 = load4(v + unit * DV + col);
  __syncthreads();
  decode_slab<Tin, DK, DV, PER_KEY, QK, GROUP, PACKED>(h, s_k, s_q, s_al, a_scalar, bt, v4, red_a,
                                                       red_b, red_m, &s_kq, sr, o + unit * DV, col,
                                                       scale);
}

// Conversion between the two storages of a state batch [n, d_k, d_v]: pack
// applies the QDQ codec to fp32 states and stores codes + scales (the packed
// state then dequantizes to exactly the QDQ'd values); unpack dequantizes.
template <int DK, int DV, int QK, int GROUP, bool TO_PACKED>
__global__ void __launch_bounds__(256, 3)
state_convert_kernel(float *__restrict__ state, uint8_t *__restrict__ codes,
                     float *__restrict__ scales) {
  constexpr int nvt = DV / 64;
  const long long unit = blockIdx.x / nvt;
  const int vt = blockIdx.x - (int)(unit * nvt);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 15, rg = tid >> 4;
  const int col = vt * 64 + cq * 4;
  __shared__ float red_m[8];
  StateRef sr;
  sr.vals = state + unit * (long long)(DK * DV);
  sr.codes = codes + unit * (long long)(DK * DV);
  sr.scales = scales + unit * (long long)(QK == kQdqInt8 ? DK * (DV / GROUP) : DV / 64);
  float4 h[DK / 16];
  if (TO_PACKED) {
    StateIO<DK, DV, QK, GROUP, false>::load(sr, rg, col, h);
    StateIO<DK, DV, QK, GROUP, true>::qdq_store(sr, rg, col, lane, warp, red_m, h);
  } else {
    StateIO<DK, DV, QK, GROUP, true>::load(sr, rg, col, h);
#pragma unroll
    for (int j = 0; j < DK / 16; ++j)
      *reinterpret_cast<float4 *>(sr.vals + (rg + 16 * j) * DV + col) = h[j];
  }
}

}  // namespace gdn
