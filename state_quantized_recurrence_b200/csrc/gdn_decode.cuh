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
// writes every state once (2 * 4 * d_k * d_v bytes per head), so the kernel
// streams the state once with coalesced 128-bit loads and stores, keeps it in
// registers across the two key-axis reductions, and writes it back in place.
//
// Work split: one 256-thread CTA per (sequence, head, 64-column value tile),
// i.e. a d_k x 64 fp32 slab (32 KB at d_k = 128) - exactly one FP8 scale
// tile.  Thread t owns columns 4*(t % 16) .. +3 of rows (t / 16) + 16 j, so a
// warp reads two full 256-byte row segments per load instruction, an INT8
// group of 32 columns lives in 8 consecutive lanes, and the key-axis
// reductions are one xor-16 shuffle plus an 8-warp shared-memory pass.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

// QK: kQdqNone / kQdqFp8Tile / kQdqInt8; GROUP: INT8 group width (16/32/64).
// 256 threads and <= 80 registers per thread give 3 CTAs (96 KB of state
// loads in flight) per SM; k, q and the per-key decays sit in shared memory
// so the 32 state values are the only large register footprint.
template <typename Tin, int DK, int DV, bool PER_KEY, int QK, int GROUP>
__global__ void __launch_bounds__(256, 3)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
              const Tin *__restrict__ v, const float *__restrict__ g,
              const float *__restrict__ beta, float *__restrict__ state,
              Tin *__restrict__ o, float scale) {
  constexpr int RPT = DK / 16;  // state rows per thread
  __shared__ float s_k[DK], s_q[DK], s_al[PER_KEY ? DK : 1];
  __shared__ float4 red_a[8][16], red_b[8][16];
  __shared__ float red_m[8];

  constexpr int nvt = DV / 64;
  const long long unit = blockIdx.x / nvt;  // sequence * H + head
  const int vt = blockIdx.x - (int)(unit * nvt);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 15, rg = tid >> 4;
  const int col = vt * 64 + cq * 4;

  float *S = state + unit * (long long)(DK * DV) + (rg * DV + col);
  // Issue the state loads first: they are the only HBM-sized traffic.
  float4 h[RPT];
#pragma unroll
  for (int j = 0; j < RPT; ++j)
    h[j] = __ldcs(reinterpret_cast<const float4 *>(S + 16 * j * DV));

  if (tid < DK) {
    s_k[tid] = to_f32(k[unit * DK + tid]);
    s_q[tid] = to_f32(q[unit * DK + tid]);
    if (PER_KEY) s_al[tid] = expf(__ldg(g + unit * DK + tid));
  }
  const float bt = __ldg(beta + unit);
  const float a_scalar = PER_KEY ? 0.0f : expf(__ldg(g + unit));
  const float4 v4 = load4(v + unit * DV + col);
  __syncthreads();

  // k^T q, computed redundantly by every warp from shared memory.
  float kq = 0.0f;
#pragma unroll
  for (int r = lane; r < DK; r += 32) kq += s_k[r] * s_q[r];
  kq = warp_sum(kq);

  // Decay and the partial key-axis reductions a = Ht^T k, b = Ht^T q.
  float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const int r = rg + 16 * j;
    const float al = PER_KEY ? s_al[r] : a_scalar, kr = s_k[r], qr = s_q[r];
    h[j].x *= al; h[j].y *= al; h[j].z *= al; h[j].w *= al;
    pa[0] += h[j].x * kr; pa[1] += h[j].y * kr; pa[2] += h[j].z * kr; pa[3] += h[j].w * kr;
    pb[0] += h[j].x * qr; pb[1] += h[j].y * qr; pb[2] += h[j].z * qr; pb[3] += h[j].w * qr;
  }
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
  float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float4 x = red_a[w][cq], y = red_b[w][cq];
    a[0] += x.x; a[1] += x.y; a[2] += x.z; a[3] += x.w;
    b[0] += y.x; b[1] += y.y; b[2] += y.z; b[3] += y.w;
  }
  float u[4];
  u[0] = bt * (v4.x - a[0]); u[1] = bt * (v4.y - a[1]);
  u[2] = bt * (v4.z - a[2]); u[3] = bt * (v4.w - a[3]);
  if (rg == 0)
    store4(o + unit * DV + col, scale * fmaf(kq, u[0], b[0]), scale * fmaf(kq, u[1], b[1]),
           scale * fmaf(kq, u[2], b[2]), scale * fmaf(kq, u[3], b[3]));

  // Delta update H = Ht + k u^T.
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const float kr = s_k[rg + 16 * j];
    h[j].x = fmaf(kr, u[0], h[j].x); h[j].y = fmaf(kr, u[1], h[j].y);
    h[j].z = fmaf(kr, u[2], h[j].z); h[j].w = fmaf(kr, u[3], h[j].w);
  }

  // State QDQ.
  if (QK == kQdqInt8) {
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      float m = fmaxf(fmaxf(fabsf(h[j].x), fabsf(h[j].y)), fmaxf(fabsf(h[j].z), fabsf(h[j].w)));
      m = group_max<GROUP / 4>(m);  // a group spans GROUP / 4 consecutive lanes
      if (m == 0.0f) {
        h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const ScaleRecip sr = make_scale(int8_scale(m));
        h[j].x = qdq_int8(h[j].x, sr); h[j].y = qdq_int8(h[j].y, sr);
        h[j].z = qdq_int8(h[j].z, sr); h[j].w = qdq_int8(h[j].w, sr);
      }
    }
  } else if (QK == kQdqFp8Tile) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < RPT; ++j)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(h[j].x), fabsf(h[j].y)), fmaxf(fabsf(h[j].z), fabsf(h[j].w))));
    m = group_max<32>(m);
    if (lane == 0) red_m[warp] = m;
    __syncthreads();
    m = red_m[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red_m[w]);
    if (m == 0.0f) {
#pragma unroll
      for (int j = 0; j < RPT; ++j) h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const ScaleRecip sr = make_scale(fp8_scale(m));
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const float2 lo = qdq_fp8_2(h[j].x, h[j].y, sr);
        const float2 hi = qdq_fp8_2(h[j].z, h[j].w, sr);
        h[j] = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
    }
  }

#pragma unroll
  for (int j = 0; j < RPT; ++j)
    __stcs(reinterpret_cast<float4 *>(S + 16 * j * DV), h[j]);
}

}  // namespace gdn
