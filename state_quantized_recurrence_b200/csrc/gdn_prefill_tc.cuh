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
// key axis): [K;Q] K^T, H0^T [K;Q]^T, R^T T^T, Vn^T Aqk^T and K^T (dVn).  The
// A operands R^T and Vn^T go to TMEM (their epilogue thread already owns the
// row); the rest are fp16 in 128-byte-swizzled shared-memory tiles.  q/k
// arrive by TMA (bf16, swizzled) into a double buffer; [K;Q] K^T reads the
// raw bf16 tile, which is then converted to fp16 in place for the state
// products (exact for |x| in the fp16 range).  Non-exact fp32 operands
// (H0, R, T, dVn) are split into hi + lo fp16 pairs (about 22 significant
// bits); with FP8 QDQ the state after the first boundary is exactly
// E4M3 code x tile scale, so H0 enters as one exact fp16 term and the scale
// is applied to the product.  Output-only terms use the hi part.
//
// Schedule of one chunk c (256 threads, warpgroups WG0 = warps 0-3 and
// WG1 = warps 4-7, both covering TMEM lanes 0-127):
//   MMA2(c)                       [thread 0]
//   all: A, Aqk from MMA1(c)
//   WG0: triangular solve, levels 16 and 32
//   WG1: R = beta (V - gamma P) -> TMEM; next gates; MMA1(c+1) on the next
//        chunk's raw bf16 tile
//   all: the solve's last level and T hi/lo
//   MMA3(c): Vn^T = R^T T^T       [thread 0]; meanwhile half of the next
//        tile's in-place fp16 conversion (once MMA1(c+1) has read it)
//   all: Vn^T -> TMEM, dVn^T hi/lo -> shared memory
//   MMA4(c): (Aqk Vn)^T, MMA5(c): H += K^T dVn   [thread 0]; meanwhile the
//        other half of the conversion
//   all: outputs (a whole chunk's through a swizzled tile and TMA stores),
//        state QDQ (each warpgroup one 64-column tile), H0 operands;
//        prefetch chunk c+2 into the buffer chunk c released
// Every mbarrier wait is bounded; on a timeout the CTA records kErrTimeout,
// stops, lets its in-flight TMA loads land, releases its TMEM and returns.
#pragma once

#include "gdn_tc_util.cuh"

namespace gdn {
namespace tc {

using namespace tcu;

constexpr int kThreads = 256;
constexpr int kC = 64;      // chunk length
constexpr int kD = 128;     // d_k = d_v
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded waits give up after 2 s

// Shared-memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_KQ = 0;          // 2 buffers x [K;Q]: 2 blocks x [128 rows x 128 B]
constexpr uint32_t OFF_H = 65536;       // H0 hi (2 blocks), lo (2 blocks): [k][v]
constexpr uint32_t OFF_X = 131072;      // 32 KB, reused within a chunk (below)
constexpr uint32_t OFF_AQK = 163840;    // Aqk fp16 [64 x 64]
constexpr uint32_t OFF_V = 172032;      // V staging (TMA, bf16): 2 x [64 tok x 64 v]
constexpr int LDT = 68;                 // fp32 row stride of the solve's matrices
constexpr uint32_t OFF_P = 188416;      // solve partial products fp32 [32 x LDT]
constexpr uint32_t OFF_T = OFF_P + 32 * LDT * 4;  // solve T fp32 [64 x LDT]
constexpr uint32_t OFF_SMALL = OFF_T + 64 * LDT * 4;  // gates, flags, barriers
// Output tile of a whole chunk, bf16 [v half][64 t][64 v], 128B-swizzled, for
// the TMA store: it borrows the solve's scratch (P, T), which is idle from
// epilogue 4 until the next chunk's solve.
constexpr uint32_t OFF_O = OFF_P;
static_assert(OFF_O % 1024 == 0 && OFF_O + 16384 <= OFF_SMALL, "output tile");
constexpr int kStoreTid = 224;
constexpr uint32_t kSmemBytes = OFF_SMALL + 4096 + 1024;  // + alignment slack
// Region X: first half of a chunk: A fp32 [64 x LDT] at [0, 17408) (its last
// row overlaps T hi, which is written only after the solve has read A), T hi
// at [16K,24K), T lo at [24K,32K); second half: dVn^T hi [0,16K), lo [16K,32K).
constexpr uint32_t X_A = 0, X_THI = 16384, X_TLO = 24576, X_DVHI = 0, X_DVLO = 16384;
// TMEM columns.
constexpr uint32_t TM_D1 = 0;     // [K;Q] K^T               128 x 64 fp32
constexpr uint32_t TM_D2 = 64;    // P^T | O^T accumulator    128 x 128 fp32
constexpr uint32_t TM_D3 = 192;   // Vn^T                     128 x 64 fp32
constexpr uint32_t TM_D4 = 256;   // H [k][v]                 128 x 128 fp32
constexpr uint32_t TM_RHI = 384;  // R^T hi as A operand      128 x 64 fp16
constexpr uint32_t TM_RLO = 416;  // R^T lo
constexpr uint32_t TM_D5 = 384;   // (Aqk Vn)^T, after MMA 3  128 x 64 fp32
constexpr uint32_t TM_VN = 448;   // Vn^T hi as A operand     128 x 64 fp16
constexpr uint32_t TM_COLS = 512;

struct Small {
  Gates gt[2];      // gates of the current and the next chunk
  float red[2][4];  // FP8 tile amax partials per warpgroup
  float hs[2];      // FP8 tile scales of H0 when `exact`
  int exact;        // H0 operand holds exact codes (FP8, after a boundary)
  int abort;
  int qk_pend[2], v_pend;  // 1 + parity of an issued, unconsumed TMA phase
  uint32_t tmem;
  uint64_t wait_ns;  // limit of the bounded waits (the drains keep kWaitNs)
  uint64_t bar_qk[2], bar_v, bar_m1, bar_m2, bar_m3, bar_m4, bar_drain[2];
};
static_assert(sizeof(Small) <= 4096, "small-state block overflows its slot");
static_assert(sizeof(Gates) % 16 == 0 && OFF_SMALL % 16 == 0, "gate arrays must stay 16-byte aligned");
static_assert(OFF_P % 16 == 0 && OFF_T % 16 == 0 && (LDT * 4) % 16 == 0, "float4 rows");

// Bounded wait by every calling thread; a timeout marks the CTA aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Small *sm,
                                              unsigned *err) {
  if (!sm100::mbar_wait(bar, parity, sm->wait_ns)) {
    sm->abort = 1;
    atomicOr(err, kErrTimeout);
    return false;
  }
  return true;
}

template <int QK, int GROUP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const float *__restrict__ g,
                  const float *__restrict__ beta, const float *__restrict__ state_in,
                  const int *__restrict__ cu_seqlens, int T, int H, float scale,
                  __nv_bfloat16 *__restrict__ o, float *__restrict__ state_out,
                  unsigned *__restrict__ err, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw_addr);
  Small *sm = reinterpret_cast<Small *>(gbase + OFF_SMALL);
  float *sA = reinterpret_cast<float *>(gbase + OFF_X + X_A);
  float *sP = reinterpret_cast<float *>(gbase + OFF_P);
  float *sT = reinterpret_cast<float *>(gbase + OFF_T);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wg = warp >> 2;                // warpgroup
  const int row = 32 * (warp & 3) + lane;  // TMEM lane = accumulator row
  const int h = blockIdx.x % H;
  int s = blockIdx.x / H;
  if (cu_seqlens && (int)gridDim.x / H <= kThreads)  // packed: longest sequences first
    s = seq_of_rank(cu_seqlens, (int)gridDim.x / H, s);
  const int unit = s * H + h;  // (sequence, head)

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
    sm100::mbar_init(&sm->bar_qk[0], 1);
    sm100::mbar_init(&sm->bar_qk[1], 1);
    sm100::mbar_init(&sm->bar_v, 1);
    sm100::mbar_init(&sm->bar_m1, 1);
    sm100::mbar_init(&sm->bar_m2, 1);
    sm100::mbar_init(&sm->bar_m3, 1);
    sm100::mbar_init(&sm->bar_m4, 1);
    sm100::mbar_init(&sm->bar_drain[0], 1);
    sm100::mbar_init(&sm->bar_drain[1], 1);
    sm100::fence_mbar_init();
    sm->abort = 0;
    sm->wait_ns = wait_ns;
    sm->exact = 0;
    sm->qk_pend[0] = sm->qk_pend[1] = sm->v_pend = 0;
  }
  if (warp == 0) {
    sm100::tmem_alloc(&sm->tmem, TM_COLS);
    sm100::tmem_relinquish();
  }
  if (warp == 7) load_gates(&sm->gt[0], g, beta, t0, (int)min((long long)kC, L), H, h, lane);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sm->tmem;
  const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;  // this warp's TMEM lanes

  // TMA: chunk j's q/k into [K;Q] buffer j % 2 (K rows 0-63, Q rows 64-127 of
  // each 64-column block, 128B-swizzled), v into the staging slot.
  auto issue_qk = [&](long long tb, int j) {
    const int b = j & 1;
    uint8_t *dst = gbase + OFF_KQ + b * 32768;
    sm100::mbar_arrive_expect_tx(&sm->bar_qk[b], 4 * 8192);
    sm100::tma_load_3d(dst + 0, &tm_k, &sm->bar_qk[b], 0, h, (int)tb);
    sm100::tma_load_3d(dst + 8192, &tm_q, &sm->bar_qk[b], 0, h, (int)tb);
    sm100::tma_load_3d(dst + 16384, &tm_k, &sm->bar_qk[b], 64, h, (int)tb);
    sm100::tma_load_3d(dst + 24576, &tm_q, &sm->bar_qk[b], 64, h, (int)tb);
    sm->qk_pend[b] = 1 + ((j >> 1) & 1);
  };
  auto issue_v = [&](long long tb, int j) {
    sm100::mbar_arrive_expect_tx(&sm->bar_v, 2 * 8192);
    sm100::tma_load_3d(gbase + OFF_V, &tm_v, &sm->bar_v, 0, h, (int)tb);
    sm100::tma_load_3d(gbase + OFF_V + 8192, &tm_v, &sm->bar_v, 64, h, (int)tb);
    sm->v_pend = 1 + (j & 1);
  };

  // [K;Q] K^T on the raw bf16 tile (exact products), before its conversion
  const uint32_t ID_KQ = sm100::idesc_f16_f32(128, 64, 0, 0) | (1u << 7) | (1u << 10);
  const uint32_t ID_H2 = sm100::idesc_f16_f32(128, 128, 1, 0);
  const uint32_t ID_H2LO = sm100::idesc_f16_f32(128, 64, 1, 0);
  const uint32_t ID_64 = sm100::idesc_f16_f32(128, 64, 0, 0);
  const uint32_t ID_KV = sm100::idesc_f16_f32(128, 128, 1, 0);
  // MMAs are issued by one elected lane of a whole, converged warp (the
  // descriptors stay warp-uniform and no sibling lane spins meanwhile).
  auto issue_mma1 = [&](int b) {  // D1 = [K;Q] K^T
    const uint32_t kqb = base + OFF_KQ + (uint32_t)b * 32768u;
    if (sm100::elect_one()) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a = kqb + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
        sm100::mma_f16_ss(tmem + TM_D1, kdesc(a), kdesc(a), ID_KQ, ks > 0);
      }
      sm100::mma_commit(&sm->bar_m1);
    }
    __syncwarp();
  };

  const int n_chunks = (int)((L + kC - 1) / kC);
  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    issue_qk(t0, 0);
    issue_v(t0, 0);
    if (n_chunks > 1) issue_qk(t0 + kC, 1);
  }

  // ---- initial state: TMEM D4 = gamma_n * H0 (fp32) and H0 hi/lo tiles;
  //      each warp: 32 key rows x 64 value columns (warpgroup half) ----
  {
    const float gnx = sm->gt[0].gn_exp;
#pragma unroll 1
    for (int p = 0; p < 2; ++p) {
      const int c0 = 64 * wg + 32 * p;
      float x[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (state_in) v4 = *reinterpret_cast<const float4 *>(state_in + st_off + row * kD + c0 + i);
        x[i] = v4.x; x[i + 1] = v4.y; x[i + 2] = v4.z; x[i + 3] = v4.w;
      }
      store32_hl(base + OFF_H + 16384u * wg, base + OFF_H + 32768u + 16384u * wg, row, 4 * p, x);
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] *= gnx;
      sm100::tmem_st32(tmem + lane_off + TM_D4 + c0, x);
    }
  }
  // ---- chunk 0's [K;Q]: wait, MMA1 on the raw tile, then convert it for
  //      MMAs 2 and 5 (later chunks' during the previous chunk) ----
  if (wait_or_abort(&sm->bar_qk[0], 0, sm, err) && tid == 0) sm->qk_pend[0] = 0;
  __syncthreads();
  if (warp == 0 && !sm->abort) {
    sm100::tc_fence_after();
    issue_mma1(0);
  }
  wait_or_abort(&sm->bar_m1, 0, sm, err);
  convert_kq_half(gbase + OFF_KQ, (int)min((long long)kC, L), tid, 0);
  convert_kq_half(gbase + OFF_KQ, (int)min((long long)kC, L), tid, 1);
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();

  // Outputs of a partial chunk (only a sequence's last can be one) are
  // computed in its last epilogue and stored after the loop, directly: 32
  // tokens x this thread's value row, packed as bf16 pairs.  Whole chunks
  // leave through the output tile and TMA stores instead.
  uint32_t opk[16];
  __nv_bfloat16 *op_dst = nullptr;  // token 0 of the pending block, or null
  int op_cnt = 0;                   // valid tokens in it
  const long long op_ts = (long long)H * kD;
  auto flush_outputs = [&]() {
    if (op_dst) {
#pragma unroll
      for (int t = 0; t < 32; t += 2) {
        const uint32_t w = opk[t >> 1];
        if (t < op_cnt) op_dst[t * op_ts] = __ushort_as_bfloat16((unsigned short)(w & 0xffffu));
        if (t + 1 < op_cnt) op_dst[(t + 1) * op_ts] = __ushort_as_bfloat16((unsigned short)(w >> 16));
      }
      op_dst = nullptr;
    }
  };

  int it = 0;
  for (long long c0 = 0; c0 < L; c0 += kC, ++it) {  // left only at the checks after barriers
    const int n = (int)min((long long)kC, L - c0);
    const long long tb = t0 + c0;
    const bool last = it == n_chunks - 1;
    const uint32_t par = (uint32_t)(it & 1);
    const int kb = it & 1;
    const uint32_t kq = base + OFF_KQ + (uint32_t)kb * 32768u;
    const Gates *gt = &sm->gt[it & 1];
    Gates *gt_next = &sm->gt[(it + 1) & 1];
    const bool exact = sm->exact != 0;
    // H0's FP8 tile scale for this thread's value row (read before epilogue 4
    // overwrites it with the next chunk's scales)
    const float hsv = exact ? sm->hs[row >> 6] : 1.0f;
    // the next chunk's raw gates, loaded now so that their latency is hidden
    // behind this chunk's first phases (finished by warp 7 in epilogue 2)
    GateRaw graw{};
    if (warp == 7 && !last)
      graw = load_gates_raw(g, beta, tb + kC, (int)min((long long)kC, L - c0 - kC), H, h, lane);

    // ---- MMA 2: D2 = H0^T [K;Q]^T (hi, or exact codes), + H0lo^T K^T ----
    if (warp == 0) {
      sm100::tc_fence_after();
      if (sm100::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t b = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          sm100::mma_f16_ss(tmem + TM_D2, mndesc(base + OFF_H + (uint32_t)ks * 2048u, 16384),
                            kdesc(b), ID_H2, ks > 0);
        }
        if (!exact) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t b = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
            sm100::mma_f16_ss(tmem + TM_D2,
                              mndesc(base + OFF_H + 32768u + (uint32_t)ks * 2048u, 16384),
                              kdesc(b), ID_H2LO, 1);
          }
        }
        sm100::mma_commit(&sm->bar_m2);
      }
      __syncwarp();
    }


    // ---- epilogue 1 (all warps; warps w and w + 4 split D1's 64 columns):
    //      rows 0-63 -> A (fp32, for the solve), rows 64-127 -> Aqk (fp16) ----
    {
      wait_or_abort(&sm->bar_m1, par, sm, err);
      sm100::tc_fence_after();
      const int r = row & 63, i0 = 32 * wg;
      float v[32];
      sm100::tmem_ld32(tmem + lane_off + TM_D1 + i0, v);
      if (gt->direct) {
        const float Gr = gt->G[r];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= expf(Gr - gt->G[i0 + i]);
      } else {
        const float epr = gt->ep[r];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 e4 = *reinterpret_cast<const float4 *>(gt->em + i0 + i);
          v[i] *= epr * e4.x; v[i + 1] *= epr * e4.y; v[i + 2] *= epr * e4.z; v[i + 3] *= epr * e4.w;
        }
      }
      if (row < 64) {
        const float br = gt->beta[r];
        float *arow = sA + r * LDT + i0;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(arow + i) =
              make_float4(i0 + i < r ? br * v[i] : 0.f, i0 + i + 1 < r ? br * v[i + 1] : 0.f,
                          i0 + i + 2 < r ? br * v[i + 2] : 0.f, i0 + i + 3 < r ? br * v[i + 3] : 0.f);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = i0 + 8 * c + e <= r ? v[8 * c + e] : 0.f;
          st_shared_v4(sw128(base + OFF_AQK, r, 4 * wg + c), pack_h2(y[0], y[1]),
                       pack_h2(y[2], y[3]), pack_h2(y[4], y[5]), pack_h2(y[6], y[7]));
        }
      }
    }
    sm100::fence_proxy_async();
    // the previous chunk's output tile (in the solve's scratch) has been read
    if (tid == kStoreTid) sm100::bulk_wait_read_all();
    __syncthreads();
    if (sm->abort) break;

    if (wg == 0) {
      // ---- WG0: triangular solve T = (I + A)^-1 in three levels ----
      // Level 0: the 16x16 diagonal blocks by column substitution (warps 0-1,
      // one thread per column); warps 2-3 zero the blocks (0,1) and (2,3)
      // above the diagonal that the 32x32 level reads.
      if (tid < 64) {
        // right-looking: once x[m] is final it updates every later row, so
        // the dependent chain is 16 steps long instead of 120
        const int b = tid >> 4, jj = tid & 15, j0 = 16 * b;
        const float *ablk = sA + j0 * LDT + j0;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) x[rr] = rr == jj ? 1.0f : 0.0f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
#pragma unroll
          for (int rr = m + 1; rr < 16; ++rr) x[rr] -= ablk[rr * LDT + m] * x[m];
        }
        float *tcol = sT + j0 * LDT + j0 + jj;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) tcol[rr * LDT] = x[rr];
      } else {
        const int e = tid - 64;  // 64 threads x 8 values
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int idx = e * 8 + i, b = idx >> 8, rr = (idx >> 4) & 15, cc = idx & 15;
          sT[(32 * b + rr) * LDT + 32 * b + 16 + cc] = 0.0f;
        }
      }
      asm volatile("bar.sync 3, 128;" ::: "memory");
      // Level 1: blocks (1,0) and (3,2): T_ij = -T_ii (A_ij T_jj).
      {
        const int blk = tid >> 6, idx = tid & 63, rr = idx >> 2, cc = (idx & 3) * 4;
        const int r0 = 16 + 32 * blk, c0b = 32 * blk;
        const float *arow = sA + (r0 + rr) * LDT + c0b;
        const float *tcol = sT + c0b * LDT + c0b + cc;
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float a = arow[m];
          const float4 t4 = *reinterpret_cast<const float4 *>(tcol + m * LDT);
          p.x += a * t4.x; p.y += a * t4.y; p.z += a * t4.z; p.w += a * t4.w;
        }
        *reinterpret_cast<float4 *>(sP + (16 * blk + rr) * LDT + cc) = p;
        asm volatile("bar.sync 3, 128;" ::: "memory");
        const float *trow = sT + (r0 + rr) * LDT + r0;
        const float *pcol = sP + 16 * blk * LDT + cc;
        float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float t = trow[m];
          const float4 p4 = *reinterpret_cast<const float4 *>(pcol + m * LDT);
          q.x += t * p4.x; q.y += t * p4.y; q.z += t * p4.z; q.w += t * p4.w;
        }
        *reinterpret_cast<float4 *>(sT + (r0 + rr) * LDT + c0b + cc) =
            make_float4(-q.x, -q.y, -q.z, -q.w);
      }
    } else {
      // ---- WG1, epilogue 2: R = diag(beta) (V - diag(gamma) P) -> TMEM as
      //      the A operand of MMA 3; then the next chunk's gates (warp 7) ----
      if (wait_or_abort(&sm->bar_v, par, sm, err) && tid == 128) sm->v_pend = 0;
      wait_or_abort(&sm->bar_m2, par, sm, err);
      sm100::tc_fence_after();
      if (n < kC) {  // a partial last chunk: rows past n read as zero
        for (int e = tid - 128; e < 2 * 64 * 8; e += 128) {
          const int blk = e >> 9, rw = (e >> 3) & 63, ch = e & 7;
          if (rw >= n) st_shared_v4(base + OFF_V + blk * 8192 + rw * 128 + ch * 16, 0u, 0u, 0u, 0u);
        }
        asm volatile("bar.sync 4, 128;" ::: "memory");
      }
      const uint8_t *stgv = gbase + OFF_V + (row >> 6) * 8192 + (row & 63) * 2;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float x[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D2 + 32 * half, x);
        uint32_t whi[16], wlo[16];
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const int tok = 32 * half + t;
          const float4 b4 = *reinterpret_cast<const float4 *>(gt->beta + tok);
          const float4 g4 = *reinterpret_cast<const float4 *>(gt->gam + tok);
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w}, gg[4] = {g4.x, g4.y, g4.z, g4.w};
          float r4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float vt =
                __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(stgv + (tok + e) * 128));
            // past n: beta, v and P (K rows zeroed) are all zero, so R is 0
            r4[e] = bb[e] * (vt - (gg[e] * hsv) * x[t + e]);
          }
          split_h2(r4[0], r4[1], whi[t >> 1], wlo[t >> 1]);
          split_h2(r4[2], r4[3], whi[(t >> 1) + 1], wlo[(t >> 1) + 1]);
        }
        sm100::tmem_st16(tmem + lane_off + TM_RHI + 16 * half, whi);
        sm100::tmem_st16(tmem + lane_off + TM_RLO + 16 * half, wlo);
      }
      if (warp == 7 && !last) finish_gates(gt_next, graw, (int)min((long long)kC, L - c0 - kC), lane);
      if (!last && warp == 4) {
        // the next chunk's MMA 1 on its raw tile (landed by TMA a chunk ago;
        // D1 was read by epilogue 1 already); the tile is converted later
        const int nb = kb ^ 1;
        const bool ok = __all_sync(
            0xffffffffu,
            wait_or_abort(&sm->bar_qk[nb], (uint32_t)(((it + 1) >> 1) & 1), sm, err));
        if (ok && lane == 0) sm->qk_pend[nb] = 0;
        sm100::tc_fence_after();
        if (__all_sync(0xffffffffu, ok && !sm->abort)) issue_mma1(nb);
      }
    }
    __syncthreads();  // T11, T22 and the level-0 blocks final; R in TMEM
    // Level 2 (all warps): the lower-left 32x32 block T_21 = -T_22 (A_21 T_11),
    // each thread 4 entries of P = A_21 T_11, then of T_21 = -T_22 P
    {
      const int rr = tid >> 3, cc = (tid & 7) * 4;
      const float *arow = sA + (32 + rr) * LDT;
      const float *tcol = sT + cc;
      float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const float a = arow[m];
        const float4 t4 = *reinterpret_cast<const float4 *>(tcol + m * LDT);
        p.x += a * t4.x; p.y += a * t4.y; p.z += a * t4.z; p.w += a * t4.w;
      }
      *reinterpret_cast<float4 *>(sP + rr * LDT + cc) = p;
      __syncthreads();
      const float *trow = sT + (32 + rr) * LDT + 32;
      const float *pcol = sP + cc;
      float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const float t = trow[m];
        const float4 p4 = *reinterpret_cast<const float4 *>(pcol + m * LDT);
        q.x += t * p4.x; q.y += t * p4.y; q.z += t * p4.z; q.w += t * p4.w;
      }
      *reinterpret_cast<float4 *>(sT + (32 + rr) * LDT + cc) = make_float4(-q.x, -q.y, -q.z, -q.w);
    }
    __syncthreads();
    // T -> hi/lo fp16 tiles [tok][tok'] (upper triangle zero), all warps:
    // row tid / 4, columns 16 (tid % 4) .. + 15
    {
      const int r = tid >> 2, cpart = (tid & 3) * 16;
      const float *trow = sT + r * LDT + cpart;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        const float4 t4 = *reinterpret_cast<const float4 *>(trow + i);
        x[i] = cpart + i <= r ? t4.x : 0.f;
        x[i + 1] = cpart + i + 1 <= r ? t4.y : 0.f;
        x[i + 2] = cpart + i + 2 <= r ? t4.z : 0.f;
        x[i + 3] = cpart + i + 3 <= r ? t4.w : 0.f;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        split_h2(x[8 * c], x[8 * c + 1], h0, l0);
        split_h2(x[8 * c + 2], x[8 * c + 3], h1, l1);
        split_h2(x[8 * c + 4], x[8 * c + 5], h2, l2);
        split_h2(x[8 * c + 6], x[8 * c + 7], h3, l3);
        st_shared_v4(sw128(base + OFF_X + X_THI, r, (cpart >> 3) + c), h0, h1, h2, h3);
        st_shared_v4(sw128(base + OFF_X + X_TLO, r, (cpart >> 3) + c), l0, l1, l2, l3);
      }
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (sm->abort) break;
    // the next chunk's V goes to the staging slot epilogue 2 just read (issued
    // by a warp that has no MMA to issue next)
    if (tid == 224 && !last) issue_v(tb + kC, it + 1);

    // ---- MMA 3: Vn^T = R^T T^T (hi*hi + hi*lo + lo*hi), R^T from TMEM ----
    if (warp == 0) {
      sm100::tc_fence_after();
      if (sm100::elect_one()) {
        const uint32_t rA[3] = {TM_RHI, TM_RHI, TM_RLO}, tB[3] = {X_THI, X_TLO, X_THI};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            sm100::mma_f16_ts(tmem + TM_D3, tmem + rA[pass] + 8u * ks,
                              kdesc(base + OFF_X + tB[pass] + 32u * ks), ID_64, pass + ks > 0);
        sm100::mma_commit(&sm->bar_m3);
      }
      __syncwarp();
    }
    // while MMA 3 runs: once the next chunk's MMA 1 has read its raw tile,
    // the first half of the tile's conversion (for its MMAs 2 and 5)
    if (!last) {
      wait_or_abort(&sm->bar_m1, (uint32_t)((it + 1) & 1), sm, err);
      convert_kq_half(gbase + OFF_KQ + (kb ^ 1) * 32768, (int)min((long long)kC, L - c0 - kC),
                      tid, 0);
    }

    // ---- epilogue 3: Vn^T hi -> TMEM (A of MMA 4); decayed dVn^T hi/lo -> smem ----
    {
      wait_or_abort(&sm->bar_m3, par, sm, err);
      sm100::tc_fence_after();
      const int vv = row, t0h = 32 * wg;
      float x[32];
      sm100::tmem_ld32(tmem + lane_off + TM_D3 + t0h, x);
      uint32_t w[16];
#pragma unroll
      for (int t = 0; t < 32; t += 2) w[t >> 1] = pack_h2(x[t], x[t + 1]);
      sm100::tmem_st16(tmem + lane_off + TM_VN + 16 * wg, w);
#pragma unroll
      for (int t = 0; t < 32; ++t) x[t] *= gt->dec[t0h + t];
      store32_hl(base + OFF_X + X_DVHI, base + OFF_X + X_DVLO, vv, 4 * wg, x);
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (sm->abort) break;

    // ---- MMA 4: D5 = Vn^T Aqk^T (Vn^T from TMEM);  MMA 5: H += K^T dVn ----
    if (warp == 0) {
      sm100::tc_fence_after();
      if (sm100::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          sm100::mma_f16_ts(tmem + TM_D5, tmem + TM_VN + 8u * ks,
                            kdesc(base + OFF_AQK + 32u * ks), ID_64, ks > 0);
#pragma unroll
        for (int pass = 0; pass < 2; ++pass)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            sm100::mma_f16_ss(tmem + TM_D4, mndesc(kq + (uint32_t)ks * 2048u, 16384),
                              kdesc(base + OFF_X + (pass ? X_DVLO : X_DVHI) + 32u * ks), ID_KV, 1);
        sm100::mma_commit(&sm->bar_m4);
      }
      __syncwarp();
    }
    // while MMAs 4 and 5 run: the second half of the conversion
    if (!last)
      convert_kq_half(gbase + OFF_KQ + (kb ^ 1) * 32768, (int)min((long long)kC, L - c0 - kC),
                      tid, 1);

    // ---- epilogue 4 ----
    wait_or_abort(&sm->bar_m4, par, sm, err);
    sm100::tc_fence_after();
    // the buffer MMA 5 just released takes the chunk after next
    if (tid == 128 && !last && it + 2 < n_chunks && !sm->abort) issue_qk(tb + 2 * kC, it + 2);
    {
      // O^T[v][t] = scale (gamma_t (Q H0)^T[v][t] + (Aqk Vn)^T[v][t]) ->
      // o[t][h][v]: warpgroup wg writes tokens 32 wg .. + 31
      if (n == kC) {
        // a whole chunk: fragments of 16 value rows x 32 tokens, packed to
        // bf16 token pairs and stored transposed into the output tile; the TMA
        // store is issued after the barrier that ends this chunk
        const int c = lane & 3;
        const float sh = scale * hsv;
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
          const int L = 32 * (warp & 3) + 16 * hl;  // first value row of the block
          const uint32_t lsel = (uint32_t)L << 16;
          uint32_t qh[16], av[16];
          sm100::tmem_ld16x256b_x4(tmem + lsel + TM_D2 + 64 + 32 * wg, qh);
          sm100::tmem_ld16x256b_x4(tmem + lsel + TM_D5 + 32 * wg, av);
          uint32_t pk[8];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const float2 g2 = *reinterpret_cast<const float2 *>(gt->gam + 32 * wg + 8 * kk + 2 * c);
            const float s0 = sh * g2.x, s1 = sh * g2.y;
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {  // value rows L + lane / 4 and L + 8 + lane / 4
              const int e = 4 * kk + 2 * hv;
              const float o0 = fmaf(s0, __uint_as_float(qh[e]), scale * __uint_as_float(av[e]));
              const float o1 = fmaf(s1, __uint_as_float(qh[e + 1]), scale * __uint_as_float(av[e + 1]));
              __nv_bfloat162 p2 = __floats2bfloat162_rn(o0, o1);
              pk[2 * kk + hv] = *reinterpret_cast<uint32_t *>(&p2);
            }
          }
#pragma unroll
          for (int k0 = 0; k0 < 4; k0 += 2) {
            const int m = lane >> 3, rr = lane & 7;
            const int t = 32 * wg + 8 * (k0 + (m >> 1)) + rr;
            const int v0 = L + 8 * (m & 1);
            const uint32_t addr = base + OFF_O + (uint32_t)(v0 >> 6) * 8192u + (uint32_t)t * 128u +
                                  ((uint32_t)(((v0 & 63) >> 3) ^ (t & 7)) << 4);
            sm100::stmatrix_x4_trans(addr, pk[2 * k0], pk[2 * k0 + 1], pk[2 * k0 + 2],
                                     pk[2 * k0 + 3]);
          }
        }
        op_dst = nullptr;
      } else {  // a partial last chunk: stored directly after the loop
        float qh[32], av[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D2 + 64 + 32 * wg, qh);
        sm100::tmem_ld32(tmem + lane_off + TM_D5 + 32 * wg, av);
        const float sh = scale * hsv;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const float4 g4 = *reinterpret_cast<const float4 *>(gt->gam + 32 * wg + t);
          qh[t] = fmaf(sh * g4.x, qh[t], scale * av[t]);
          qh[t + 1] = fmaf(sh * g4.y, qh[t + 1], scale * av[t + 1]);
          qh[t + 2] = fmaf(sh * g4.z, qh[t + 2], scale * av[t + 2]);
          qh[t + 3] = fmaf(sh * g4.w, qh[t + 3], scale * av[t + 3]);
        }
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          __nv_bfloat162 p2 = __floats2bfloat162_rn(qh[t], qh[t + 1]);
          opk[t >> 1] = *reinterpret_cast<uint32_t *>(&p2);
        }
        op_cnt = n - 32 * wg;
        op_dst = op_cnt > 0 ? o + ((tb + 32 * wg) * H + h) * kD + row : nullptr;
      }
      // H: key row `row`, value columns 64 wg .. + 63 (one FP8 tile per
      // warpgroup).  Pass 1 (FP8 tiles, INT8 groups of 64): amax of the 64
      // columns, for FP8 reduced over the warpgroup's 128 rows.
      float mh = 0.f;
      if (QK == kQdqFp8Tile || (QK == kQdqInt8 && GROUP == 64)) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          float y[32];
          sm100::tmem_ld32(tmem + lane_off + TM_D4 + 64 * wg + 32 * p, y);
#pragma unroll
          for (int i = 0; i < 32; i += 2) mh = max_abs2(mh, y[i], y[i + 1]);
        }
      }
      if (QK == kQdqFp8Tile) {
        mh = group_max<32>(mh);
        if (lane == 0) sm->red[wg][warp & 3] = mh;
        asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory");
        mh = fmaxf(fmaxf(sm->red[wg][0], sm->red[wg][1]), fmaxf(sm->red[wg][2], sm->red[wg][3]));
      }
      const float gn_next = last ? 1.0f : sm->gt[(it + 1) & 1].gn_exp;
      const ScaleRecip sr_tile = make_scale(fp8_scale(QK == kQdqFp8Tile && mh > 0.f ? mh : 1.0f));
      // FP8: the dequantized codes go straight into the next carry's accumulator
      // (code x (s gamma_n), one rounding); the last chunk's are the state itself
      const float sdq = last ? sr_tile.s : sr_tile.s * gn_next;
      // Pass 2: quantize; H0 operand tiles (exact codes for FP8, hi/lo
      // otherwise); gamma_n(next) * H into TMEM as the next carry's
      // accumulator; state_out after the last chunk.
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int c0v = 64 * wg + 32 * p;
        float y[32];
        sm100::tmem_ld32(tmem + lane_off + TM_D4 + c0v, y);
        if (QK == kQdqFp8Tile) {
          uint32_t code[16];
          if (mh == 0.0f) {  // zero tile: codes and values 0
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) code[i] = 0u;
          } else if (sr_tile.pre == 1.0f) {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              code[i >> 1] = fp8_code_pair(y[i], y[i + 1], sr_tile.s, sr_tile.r, y[i], y[i + 1], sdq);
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              code[i >> 1] = fp8_code_pair(y[i] * sr_tile.pre, y[i + 1] * sr_tile.pre, sr_tile.s2,
                                           sr_tile.r, y[i], y[i + 1], sdq);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(sw128(base + OFF_H + 16384u * wg, row, 4 * p + c), code[4 * c],
                         code[4 * c + 1], code[4 * c + 2], code[4 * c + 3]);
        } else {
          if (QK == kQdqInt8) {
            constexpr int GW = GROUP < 32 ? GROUP : 32;  // group width inside this piece
#pragma unroll
            for (int g0 = 0; g0 < 32; g0 += GW) {
              float m = 0.f;
              if (GROUP == 64) {
                m = mh;
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
          }
          store32_hl(base + OFF_H + 16384u * wg, base + OFF_H + 32768u + 16384u * wg, row,
                     4 * p, y);
        }
        if (last) {
          float *dst = state_out + st_off + row * kD + c0v;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(dst + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
        } else {
          if (QK != kQdqFp8Tile) scale32(y, gn_next);
          sm100::tmem_st32(tmem + lane_off + TM_D4 + c0v, y);
        }
      }
      if (QK == kQdqFp8Tile && (tid & 127) == 0) sm->hs[wg] = mh == 0.0f ? 0.0f : sr_tile.s;
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    if (tid == kStoreTid && n == kC) {
      sm100::tma_store_3d(&tm_o, gbase + OFF_O, 0, h, (int)tb);
      sm100::tma_store_3d(&tm_o, gbase + OFF_O + 8192, 64, h, (int)tb);
      sm100::bulk_commit();
    }
    if (tid == 0) sm->exact = QK == kQdqFp8Tile ? 1 : 0;
    __syncthreads();
  }

  flush_outputs();  // a partial last chunk's outputs
  if (tid == kStoreTid) sm100::bulk_wait_all();

  // An aborted CTA lets its outstanding TMA loads land and its MMAs (issued
  // by warps 0 and 4) finish, again bounded, before its shared memory and
  // TMEM are released.
  if (tid == 0 && sm->abort) {
    for (int b = 0; b < 2; ++b)
      if (sm->qk_pend[b])
        (void)sm100::mbar_wait(&sm->bar_qk[b], (uint32_t)(sm->qk_pend[b] - 1), kWaitNs);
    if (sm->v_pend) (void)sm100::mbar_wait(&sm->bar_v, (uint32_t)(sm->v_pend - 1), kWaitNs);
  }
  if (sm->abort && (warp == 0 || warp == 4)) drain_mmas(&sm->bar_drain[warp >> 2]);
  __syncthreads();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace tc
}  // namespace gdn
