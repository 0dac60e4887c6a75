// Backward pass of the gated delta rule with a fake-quantized state, fp32
// CUDA-core kernel, for training with the state QAT of the pages (PR #2497
// What section: fake quantization of the recurrent state; the QDQ is passed
// straight through in the backward pass).
//
// Forward per token t (H = S^T, [d_k, d_v]):
//   Ht = diag(alpha_t) H_{t-1},  a = Ht^T k_t,  u = beta_t (v_t - a),
//   Hn = Ht + k_t u^T,  o_t = scale Hn^T q_t,  H_t = QDQ(Hn) at a chunk end.
// Reverse, dH the gradient with respect to H_t (QDQ passed straight through):
//   dHn = dH + scale q_t do_t^T;  dq_t = scale Hn do_t
//   du = dHn^T k_t;  dk_t = dHn u - beta_t Ht du;  dbeta_t = du . (v_t - a)
//   dv_t = beta_t du;  dHt = dHn - beta_t k_t du^T
//   dalpha_i = sum_j H_{t-1}[i,j] dHt[i,j];  dg_t = alpha (*) dalpha
//   (summed over i for a scalar gate);  dH_{t-1} = diag(alpha_t) dHt.
//
// One CTA of 256 threads per (sequence, head, 64-column value tile); each
// thread holds rows rg + 16 j (j < d_k / 16) x 4 columns of a state, as the
// decode kernel does.  Phase 1 runs the forward token recurrence with the
// QDQ at every chunk end and keeps each chunk's starting state in the
// workspace; phase 2 walks the chunks backwards: it recomputes the chunk's
// per-token states into the workspace, then runs the reverse recurrence
// over them.  Every thread reads back only the workspace words it wrote.
// Each token's inputs are fetched into registers one token ahead.
// Sums over value columns (dq, dk, dg, dbeta) come from one atomic add per
// tile into zeroed fp32 buffers, so with at most two tiles (d_v <= 128)
// the result does not depend on the order of the adds.
#pragma once

#include "gdn_common.cuh"

namespace gdn {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kChunk = 64;

// Column sums over the 16 row groups: every thread receives the sums of its
// 4 columns.  `red` [8][16] float4 of shared memory; all threads call.
__device__ __forceinline__ float4 sum_rows(float4 p, float4 (*red)[16], int warp, int lane) {
  p.x += __shfl_xor_sync(0xffffffffu, p.x, 16);
  p.y += __shfl_xor_sync(0xffffffffu, p.y, 16);
  p.z += __shfl_xor_sync(0xffffffffu, p.z, 16);
  p.w += __shfl_xor_sync(0xffffffffu, p.w, 16);
  __syncthreads();  // the previous call's results have been read
  if (lane < 16) red[warp][lane] = p;
  __syncthreads();
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float4 x = red[w][lane & 15];
    s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
  }
  return s;
}

// Row sum over the 16 column quads of a half-warp (all 16 lanes receive it).
__device__ __forceinline__ float sum_cols(float x) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Block-wide sum of one float per thread (thread 0 receives it).
__device__ __forceinline__ float sum_block(float x, float *red8, int warp, int lane) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  __syncthreads();
  if (lane == 0) red8[warp] = x;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red8[w];
  return s;
}

// In-register QDQ of the slab (the codec of the forward kernels): INT8
// groups of GROUP columns along a key row (GROUP / 4 lanes), or one FP8
// scale for the CTA's 64-column tile.
template <int RPT, int QK, int GROUP>
__device__ __forceinline__ void qdq_slab(float4 (&h)[RPT], float *red8, int warp, int lane) {
  if (QK == kQdqInt8) {
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      float m = fmaxf(fmaxf(fabsf(h[j].x), fabsf(h[j].y)), fmaxf(fabsf(h[j].z), fabsf(h[j].w)));
      m = group_max<GROUP / 4>(m);
      if (m == 0.0f) {
        h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const ScaleRecip s = make_scale(int8_scale(m));
        h[j].x = qdq_int8(h[j].x, s); h[j].y = qdq_int8(h[j].y, s);
        h[j].z = qdq_int8(h[j].z, s); h[j].w = qdq_int8(h[j].w, s);
      }
    }
  } else if (QK == kQdqFp8Tile) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < RPT; ++j)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(h[j].x), fabsf(h[j].y)), fmaxf(fabsf(h[j].z), fabsf(h[j].w))));
    m = group_max<32>(m);
    __syncthreads();
    if (lane == 0) red8[warp] = m;
    __syncthreads();
    m = red8[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red8[w]);
    if (m == 0.0f) {
#pragma unroll
      for (int j = 0; j < RPT; ++j) h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const ScaleRecip s = make_scale(fp8_scale(m));
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const float2 lo = qdq_fp8_2(h[j].x, h[j].y, s);
        const float2 hi = qdq_fp8_2(h[j].z, h[j].w, s);
        h[j] = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
    }
  }
}

// Workspace words of a thread within one [d_k x 64] state: j-th float4 at
// j * 1024 + 4 * tid (coalesced, and read back by the same thread).
template <int RPT>
__device__ __forceinline__ void ws_store(float *base, int tid, const float4 (&h)[RPT]) {
#pragma unroll
  for (int j = 0; j < RPT; ++j) reinterpret_cast<float4 *>(base + j * 1024)[tid] = h[j];
}
template <int RPT>
__device__ __forceinline__ void ws_load(const float *base, int tid, float4 (&h)[RPT]) {
#pragma unroll
  for (int j = 0; j < RPT; ++j) h[j] = reinterpret_cast<const float4 *>(base + j * 1024)[tid];
}

template <typename Tin, int DK, bool PER_KEY, int QK, int GROUP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_backward_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                        const Tin *__restrict__ v, const float *__restrict__ g,
                        const float *__restrict__ beta, const float *__restrict__ state_in,
                        const int *__restrict__ cu_seqlens, int T, int H, int DV, float scale,
                        const Tin *__restrict__ dout, const float *__restrict__ dstate_out,
                        float *__restrict__ ws_chunk, float *__restrict__ ws_tok,
                        float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                        float *__restrict__ dg, float *__restrict__ dbeta,
                        float *__restrict__ dstate_in, unsigned *__restrict__ err) {
  constexpr int RPT = DK / 16;
  constexpr int TILE = DK * 64;
  __shared__ float s_k[DK], s_q[DK], s_al[PER_KEY ? DK : 1];
  __shared__ float4 red4[8][16];
  __shared__ float red8[8];

  const int nvt = DV >> 6;
  const int vt = blockIdx.x % nvt;
  const int h = (blockIdx.x / nvt) % H;
  const int s = (blockIdx.x / nvt) / H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 15, rg = tid >> 4;
  const int col = vt * 64 + cq * 4;

  long long t0, t1, slot0;
  const long long chunks_dense = ((long long)T + kChunk - 1) / kChunk;
  if (cu_seqlens) {
    t0 = cu_seqlens[s];
    t1 = cu_seqlens[s + 1];
    const int n_seq = gridDim.x / (H * nvt);
    if (t0 < 0 || t1 < t0 || t1 > T || (s == 0 && t0 != 0) || (s == n_seq - 1 && t1 != T)) {
      if (tid == 0) atomicOr(err, kErrBadSeqlens);
      return;
    }
    slot0 = s + t0 / kChunk;  // sequences' chunk slots never overlap
  } else {
    t0 = (long long)s * T;
    t1 = t0 + T;
    slot0 = (long long)s * chunks_dense;
  }
  const long long L = t1 - t0;
  const int n_chunks = (int)((L + kChunk - 1) / kChunk);
  const long long st_off = ((long long)s * H + h) * DK * DV;
  auto chunk_ws = [&](int c) { return ws_chunk + (((slot0 + c) * H + h) * nvt + vt) * (long long)TILE; };
  float *tok_ws = ws_tok + (long long)blockIdx.x * kChunk * TILE;

  // Inputs of one token, fetched into registers one token ahead and then
  // committed: k, q and the per-key decays to shared memory, the rest to
  // registers.
  struct Raw {
    float kf, qf, gf, gs, bt;
    float4 v4, do4;
  };
  auto fetch = [&](long long tok, bool with_do, Raw &r) {
    if (tid < DK) {
      r.kf = to_f32(k[(tok * H + h) * DK + tid]);
      r.qf = to_f32(q[(tok * H + h) * DK + tid]);
      if (PER_KEY) r.gf = __ldg(g + (tok * H + h) * DK + tid);
    }
    if (!PER_KEY) r.gs = __ldg(g + tok * H + h);
    r.bt = __ldg(beta + tok * H + h);
    r.v4 = load4(v + (tok * H + h) * DV + col);
    if (with_do) r.do4 = load4(dout + (tok * H + h) * DV + col);
  };
  float al_s = 1.0f, bt = 0.0f;
  float4 v4, do4;
  auto commit = [&](const Raw &r) {
    __syncthreads();  // the previous token's shared inputs have been read
    if (tid < DK) {
      s_k[tid] = r.kf;
      s_q[tid] = r.qf;
      if (PER_KEY) s_al[tid] = expf(r.gf);
    }
    if (!PER_KEY) al_s = expf(r.gs);
    bt = r.bt;
    v4 = r.v4;
    do4 = r.do4;
    __syncthreads();
  };
  // forward token step on the slab: h <- diag(alpha) h + k u^T; returns a
  // (this thread's 4 columns) and leaves the decayed state in ht
  auto fwd_step = [&](float4 (&hs)[RPT], float4 (&ht)[RPT]) -> float4 {
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      const int r = rg + 16 * j;
      const float al = PER_KEY ? s_al[r] : al_s, kr = s_k[r];
      ht[j] = make_float4(al * hs[j].x, al * hs[j].y, al * hs[j].z, al * hs[j].w);
      pa.x += ht[j].x * kr; pa.y += ht[j].y * kr; pa.z += ht[j].z * kr; pa.w += ht[j].w * kr;
    }
    const float4 a = sum_rows(pa, red4, warp, lane);
    const float4 u = make_float4(bt * (v4.x - a.x), bt * (v4.y - a.y), bt * (v4.z - a.z),
                                 bt * (v4.w - a.w));
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      const float kr = s_k[rg + 16 * j];
      hs[j] = make_float4(fmaf(kr, u.x, ht[j].x), fmaf(kr, u.y, ht[j].y), fmaf(kr, u.z, ht[j].z),
                          fmaf(kr, u.w, ht[j].w));
    }
    return a;
  };

  float4 hst[RPT], htd[RPT];
  Raw cur, nxt;
  cur.do4 = nxt.do4 = make_float4(0.f, 0.f, 0.f, 0.f);
  // ---- phase 1: forward with the chunk-end QDQ; chunk-start states kept ----
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    hst[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) hst[j] = *reinterpret_cast<const float4 *>(state_in + st_off + (rg + 16 * j) * DV + col);
  }
  if (L > 0) fetch(t0, false, cur);
  for (long long t = 0; t < L; ++t) {
    if (t % kChunk == 0) ws_store<RPT>(chunk_ws((int)(t / kChunk)), tid, hst);
    commit(cur);
    if (t + 1 < L) fetch(t0 + t + 1, false, nxt);
    (void)fwd_step(hst, htd);
    if (t % kChunk == kChunk - 1 || t == L - 1) qdq_slab<RPT, QK, GROUP>(hst, red8, warp, lane);
    cur = nxt;
  }

  // ---- phase 2: chunks in reverse ----
  float4 dH[RPT];
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    dH[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (dstate_out) dH[j] = *reinterpret_cast<const float4 *>(dstate_out + st_off + (rg + 16 * j) * DV + col);
  }
  for (int c = n_chunks - 1; c >= 0; --c) {
    const int n = (int)min((long long)kChunk, L - (long long)c * kChunk);
    const long long tb = t0 + (long long)c * kChunk;
    ws_load<RPT>(chunk_ws(c), tid, hst);
    fetch(tb, false, cur);
    for (int t = 0; t < n; ++t) {  // per-token states H_{t-1}
      ws_store<RPT>(tok_ws + (long long)t * TILE, tid, hst);
      commit(cur);
      if (t + 1 < n) fetch(tb + t + 1, false, nxt);
      (void)fwd_step(hst, htd);
      cur = nxt;
    }
    fetch(tb + n - 1, true, cur);
    for (int t = n - 1; t >= 0; --t) {
      const long long tok = tb + t;
      float4 hp[RPT];
      ws_load<RPT>(tok_ws + (long long)t * TILE, tid, hp);
      commit(cur);
      if (t > 0) fetch(tok - 1, true, nxt);
#pragma unroll
      for (int j = 0; j < RPT; ++j) hst[j] = hp[j];
      const float4 a = fwd_step(hst, htd);  // hst = Hn, htd = Ht
      const float4 u = make_float4(bt * (v4.x - a.x), bt * (v4.y - a.y), bt * (v4.z - a.z),
                                   bt * (v4.w - a.w));
      // dHn = dH + scale q do^T (in dH); dq_t = scale Hn do_t
      float4 pdu = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int r = rg + 16 * j;
        const float qr = scale * s_q[r], kr = s_k[r];
        dH[j].x = fmaf(qr, do4.x, dH[j].x); dH[j].y = fmaf(qr, do4.y, dH[j].y);
        dH[j].z = fmaf(qr, do4.z, dH[j].z); dH[j].w = fmaf(qr, do4.w, dH[j].w);
        const float dqr = sum_cols(hst[j].x * do4.x + hst[j].y * do4.y + hst[j].z * do4.z +
                                   hst[j].w * do4.w);
        if (cq == 0) atomicAdd(dq + (tok * H + h) * DK + r, scale * dqr);
        pdu.x += dH[j].x * kr; pdu.y += dH[j].y * kr; pdu.z += dH[j].z * kr; pdu.w += dH[j].w * kr;
      }
      const float4 du = sum_rows(pdu, red4, warp, lane);
      // du, a and v are the same in every row group: row group 0 writes dv,
      // and dbeta_t's sum over the tile's columns takes one half-warp
      const float db = sum_cols(du.x * (v4.x - a.x) + du.y * (v4.y - a.y) +
                                du.z * (v4.z - a.z) + du.w * (v4.w - a.w));
      if (rg == 0)
        *reinterpret_cast<float4 *>(dv + (tok * H + h) * DV + col) =
            make_float4(bt * du.x, bt * du.y, bt * du.z, bt * du.w);
      if (tid == 0) atomicAdd(dbeta + tok * H + h, db);
      float galpha = 0.0f;
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int r = rg + 16 * j;
        const float kr = s_k[r];
        // dk_t = dHn u - beta Ht du
        const float dkr = sum_cols(dH[j].x * u.x + dH[j].y * u.y + dH[j].z * u.z + dH[j].w * u.w -
                                   bt * (htd[j].x * du.x + htd[j].y * du.y + htd[j].z * du.z +
                                         htd[j].w * du.w));
        if (cq == 0) atomicAdd(dk + (tok * H + h) * DK + r, dkr);
        // dHt = dHn - beta k du^T
        const float bk = bt * kr;
        dH[j].x = fmaf(-bk, du.x, dH[j].x); dH[j].y = fmaf(-bk, du.y, dH[j].y);
        dH[j].z = fmaf(-bk, du.z, dH[j].z); dH[j].w = fmaf(-bk, du.w, dH[j].w);
        // dalpha_r = sum_c H_{t-1} dHt; dH_{t-1} = alpha dHt
        const float dar = hp[j].x * dH[j].x + hp[j].y * dH[j].y + hp[j].z * dH[j].z + hp[j].w * dH[j].w;
        const float al = PER_KEY ? s_al[r] : al_s;
        if (PER_KEY) {
          const float dgr = sum_cols(dar);
          if (cq == 0) atomicAdd(dg + (tok * H + h) * DK + r, al * dgr);
        } else {
          galpha += dar;
        }
        dH[j].x *= al; dH[j].y *= al; dH[j].z *= al; dH[j].w *= al;
      }
      if (!PER_KEY) {
        const float tot = sum_block(galpha, red8, warp, lane);
        if (tid == 0) atomicAdd(dg + tok * H + h, al_s * tot);
      }
      cur = nxt;
    }
  }
#pragma unroll
  for (int j = 0; j < RPT; ++j)
    *reinterpret_cast<float4 *>(dstate_in + st_off + (rg + 16 * j) * DV + col) = dH[j];
}

}  // namespace bwd
}  // namespace gdn
