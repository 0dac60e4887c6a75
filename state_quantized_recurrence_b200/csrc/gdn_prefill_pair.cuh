// Chunked prefix of the gated delta rule (GDN, scalar gate) with a QDQ state
// on the sm_100a tensor cores, split over a pair of CTAs (a thread-block
// cluster of two, one (sequence, head) per pair, d_k = d_v = 128).
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
// A, Aqk and T depend only on the chunk's inputs; the rest is the state
// chain, sequential across chunks.  The pair divides them:
//
//   rank 0 (chain)     the state chain of every chunk, as one CTA: MMA 2
//                      (H0^T [K;Q]^T), R -> TMEM, MMA 3 (Vn^T = R^T T^T),
//                      Vn^T -> TMEM / dVn^T hi,lo -> smem, MMA 4/5, QDQ;
//   rank 1 (producer)  for each chunk, one ahead of the chain: [K;Q] K^T on
//                      the raw bf16 tile (exact products), the A / Aqk
//                      epilogue, the triangular solve, T hi/lo; then one bulk
//                      copy of T hi, T lo and Aqk (24 KB) into the chain CTA's
//                      receive buffer (distributed shared memory, no
//                      multicast).  The next chunk's [K;Q] K^T is issued
//                      right after an epilogue and runs during the solve.
//
// Off the chain CTA's critical path, in the windows where its warps would
// wait for the tensor cores: the in-place fp16 conversion of the next [K;Q]
// tile (one half while MMA 2 runs, one with the next chunk's gates while
// MMA 3 runs), and the previous chunk's outputs (while MMAs 4 and 5 run).
// Outputs leave by TMA stores of a staged 64-token tile.
//
// Hand-off: the copy completes its bytes on the chain CTA's `rx_full`
// mbarrier (armed by the chain CTA for each chunk); once MMAs 3 and 4 of a
// chunk have read the buffer the chain CTA arrives on the producer's
// `rx_free`.  Every wait is bounded (2 s); on a timeout a CTA records
// kErrTimeout and stops, and both CTAs meet at the cluster barrier before
// either exits, so no copy or remote arrival targets a CTA that has left.
#pragma once

#include "gdn_tc_util.cuh"

namespace gdn {
namespace pair {

using namespace tcu;

constexpr int kThreads = 256;
constexpr int kC = 64;
constexpr int kD = 128;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kRxBytes = 3 * 8192;  // T hi, T lo, Aqk

// ---- chain CTA shared memory (byte offsets from a 1024-byte aligned base)
constexpr uint32_t C_KQ = 0;           // 2 x [K;Q] fp16 (in place of the bf16 TMA tiles)
constexpr uint32_t C_H = 65536;        // H0 hi (2 blocks), lo (2 blocks)
constexpr uint32_t C_DV = 131072;      // dVn^T hi [0,16K), lo [16K,32K)
constexpr uint32_t C_V = 163840;       // V staging (bf16) 2 x [64 tok x 64 v]
constexpr uint32_t C_RX = 180224;      // received: T hi, T lo, Aqk [64 x 64] fp16 each
constexpr uint32_t C_O = C_RX + kRxBytes;  // output tile, bf16 [2 halves of v][64 t][64 v]
constexpr uint32_t C_SMALL = C_O + 16384;
// ---- producer CTA shared memory
constexpr int LDT = 68;
constexpr uint32_t P_KQ = 0;           // 2 x [K;Q] bf16 (TMA)
constexpr uint32_t P_SA = 65536;       // A fp32 [64 x LDT]
constexpr uint32_t P_SP = P_SA + 64 * LDT * 4;  // partial products [32 x LDT]
constexpr uint32_t P_ST = P_SP + 32 * LDT * 4;  // T fp32 [64 x LDT]
// staging for the copy, two slots (chunk j uses slot j % 2): T hi, T lo, Aqk.
// A copy into another CTA's shared memory signals completion only on the
// receiver's mbarrier, so the producer learns that slot j % 2 has been read
// from the release of chunk j - 2, which it waits for before copying chunk
// j - 1; two slots therefore need no further wait.
constexpr uint32_t P_STG = 109568;
constexpr uint32_t P_SMALL = P_STG + 2 * kRxBytes;
// both roles run the same kernel: the larger map decides the allocation, and
// the two Small blocks sit at distinct offsets, so each CTA can address the
// peer's barriers by offset
constexpr uint32_t kSmallBytes = 8192;
static_assert(P_SMALL + kSmallBytes <= C_SMALL || C_SMALL + kSmallBytes <= P_SMALL,
              "the two roles' small blocks must not overlap");
static_assert(P_ST + 64 * LDT * 4 <= P_STG && P_STG % 1024 == 0 && C_RX % 1024 == 0,
              "producer map");
constexpr uint32_t kSmemBytes = C_SMALL + kSmallBytes + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");

// TMEM columns of the chain CTA (the producer uses 64 columns for [K;Q] K^T).
// Chunk j uses region 128 (j % 2): its first 64 columns hold P^T, then
// Vn^T (MMA 3, after P has been read), then (Aqk Vn)^T (MMA 4, after Vn^T
// has been read); the next 64 hold (Q H0)^T.  The output epilogue of chunk j
// runs during chunk j+1, which works in the other region.
constexpr uint32_t TM_REG = 128;  // region stride
constexpr uint32_t TM_QH = 64;    // (Q H0)^T within a region  128 x 64 fp32
constexpr uint32_t TM_D4 = 256;   // H [k][v]                  128 x 128 fp32
constexpr uint32_t TM_R = 384;    // R^T as A operand, fp16: tokens 32 w .. + 31 hi at
                                  // R + 32 w, lo at R + 32 w + 16 (w = 0, 1)
constexpr uint32_t TM_VN = 448;   // Vn^T hi as A operand      128 x 32 (fp16 pairs)
constexpr uint32_t TM_COLS_C = 512, TM_COLS_P = 64;

struct SmallC {
  Gates gt[3];  // chunk j's gates in slot j % 3 (the output epilogue of j runs in j+1)
  float red[2][4];
  float hs[2];
  int exact, abort;
  int qk_pend[2], v_pend;
  int rx_pend;  // 1 + parity of an armed transfer not yet waited for
  uint32_t tmem;
  uint64_t wait_ns;  // limit of the bounded waits (the drains keep kWaitNs)
  uint64_t bar_qk[2], bar_v, bar_m2, bar_m3, bar_m4, rx_full, bar_drain[2];
};
struct SmallP {
  Gates gt;
  int abort;
  int qk_pend[2];
  uint32_t tmem;
  uint64_t wait_ns;
  uint64_t bar_qk[2], bar_m1, rx_free, bar_drain[2];
};
static_assert(sizeof(SmallC) <= kSmallBytes && sizeof(SmallP) <= kSmallBytes, "small blocks");

template <class S>
__device__ __forceinline__ bool wait_local(uint64_t *bar, uint32_t parity, S *sm, unsigned *err) {
  if (!sm100::mbar_wait(bar, parity, sm->wait_ns)) {
    sm->abort = 1;
    atomicOr(err, kErrTimeout);
    return false;
  }
  return true;
}
template <class S>
__device__ __forceinline__ bool wait_cluster(uint64_t *bar, uint32_t parity, S *sm, unsigned *err) {
  if (!sm100::mbar_wait_cluster(bar, parity, sm->wait_ns)) {
    sm->abort = 1;
    atomicOr(err, kErrTimeout);
    return false;
  }
  return true;
}

template <int QK, int GROUP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
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
  const uint32_t rank = sm100::cluster_ctarank();

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wg = warp >> 2;
  const int row = 32 * (warp & 3) + lane;  // TMEM lane = accumulator row
  const int pair_id = blockIdx.x >> 1;
  const int n_units = gridDim.x >> 1;
  const int h = pair_id % H;
  int s = pair_id / H;
  if (cu_seqlens && n_units / H <= kThreads)  // packed: longest sequences first
    s = seq_of_rank(cu_seqlens, n_units / H, s);
  const int unit = s * H + h;

  long long t0, t1;
  bool valid = true;
  if (cu_seqlens) {
    t0 = cu_seqlens[s];
    t1 = cu_seqlens[s + 1];
    const int n_seq = n_units / H;
    if (t0 < 0 || t1 < t0 || t1 > T || (s == 0 && t0 != 0) || (s == n_seq - 1 && t1 != T)) {
      if (tid == 0 && rank == 0) atomicOr(err, kErrBadSeqlens);
      valid = false;
    }
  } else {
    t0 = (long long)s * T;
    t1 = t0 + T;
  }
  const long long L = valid ? t1 - t0 : 0;
  const long long st_off = (long long)unit * kD * kD;

  if (!valid || L == 0) {  // no token: the state passes through unchanged
    if (valid && rank == 0) {
      for (int i = tid; i < kD * kD / 4; i += kThreads) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (state_in) x = reinterpret_cast<const float4 *>(state_in + st_off)[i];
        reinterpret_cast<float4 *>(state_out + st_off)[i] = x;
      }
    }
    sm100::cluster_sync();
    return;
  }
  const int n_chunks = (int)((L + kC - 1) / kC);
  auto chunk_len = [&](int j) { return (int)min((long long)kC, L - (long long)j * kC); };

  SmallC *smc = reinterpret_cast<SmallC *>(gbase + C_SMALL);
  SmallP *smp = reinterpret_cast<SmallP *>(gbase + P_SMALL);
  // the peer's barriers, by offset (same shared-memory map in both CTAs)
  const uint32_t rx_full_remote = sm100::mapa(sm100::smem_u32(&smc->rx_full), 0);
  const uint32_t rx_free_remote = sm100::mapa(sm100::smem_u32(&smp->rx_free), 1);
  const uint32_t rx_buf_remote = sm100::mapa(base + C_RX, 0);

  // ---------------------------------------------------------------- setup
  if (rank == 0) {
    if (tid == 0) {
      sm100::mbar_init(&smc->bar_qk[0], 1);
      sm100::mbar_init(&smc->bar_qk[1], 1);
      sm100::mbar_init(&smc->bar_v, 1);
      sm100::mbar_init(&smc->bar_m2, 1);
      sm100::mbar_init(&smc->bar_m3, 1);
      sm100::mbar_init(&smc->bar_m4, 1);
      sm100::mbar_init(&smc->rx_full, 1);
      sm100::mbar_init(&smc->bar_drain[0], 1);
      sm100::mbar_init(&smc->bar_drain[1], 1);
      sm100::fence_mbar_init();
      smc->abort = 0;
      smc->wait_ns = wait_ns;
      smc->exact = 0;
      smc->qk_pend[0] = smc->qk_pend[1] = smc->v_pend = 0;
      // chunk 0's transfer (issued only after the cluster barrier below)
      sm100::mbar_arrive_expect_tx(&smc->rx_full, kRxBytes);
      smc->rx_pend = 1;
    }
    if (warp == 0) {
      sm100::tmem_alloc(&smc->tmem, TM_COLS_C);
      sm100::tmem_relinquish();
    }
    if (warp == 7) load_gates(&smc->gt[0], g, beta, t0, chunk_len(0), H, h, lane);
  } else {
    if (tid == 0) {
      sm100::mbar_init(&smp->bar_qk[0], 1);
      sm100::mbar_init(&smp->bar_qk[1], 1);
      sm100::mbar_init(&smp->bar_m1, 1);
      sm100::mbar_init(&smp->rx_free, 1);
      sm100::mbar_init(&smp->bar_drain[0], 1);
      sm100::mbar_init(&smp->bar_drain[1], 1);
      sm100::fence_mbar_init();
      smp->abort = 0;
      smp->wait_ns = wait_ns;
      smp->qk_pend[0] = smp->qk_pend[1] = 0;
    }
    if (warp == 0) {
      sm100::tmem_alloc(&smp->tmem, TM_COLS_P);
      sm100::tmem_relinquish();
    }
  }
  sm100::tc_fence_before();
  sm100::cluster_sync();  // both CTAs' barriers initialised before any remote use
  sm100::tc_fence_after();
  const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;

  if (rank == 1) {
    // ======================= producer: A, Aqk, T for every chunk ==========
    SmallP *sm = smp;
    const uint32_t tmem = sm->tmem;
    float *sA = reinterpret_cast<float *>(gbase + P_SA);
    float *sP = reinterpret_cast<float *>(gbase + P_SP);
    float *sT = reinterpret_cast<float *>(gbase + P_ST);
    const uint32_t ID_KQ = sm100::idesc_f16_f32(128, 64, 0, 0) | (1u << 7) | (1u << 10);  // bf16
    auto issue_qk = [&](int j) {
      const long long tb = t0 + (long long)j * kC;
      const int b = j & 1;
      uint8_t *dst = gbase + P_KQ + b * 32768;
      sm100::mbar_arrive_expect_tx(&sm->bar_qk[b], 4 * 8192);
      sm100::tma_load_3d(dst + 0, &tm_k, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 8192, &tm_q, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 16384, &tm_k, &sm->bar_qk[b], 64, h, (int)tb);
      sm100::tma_load_3d(dst + 24576, &tm_q, &sm->bar_qk[b], 64, h, (int)tb);
      sm->qk_pend[b] = 1 + ((j >> 1) & 1);
    };
    // D1 = [K;Q] K^T on the raw bf16 tile (exact products); one elected lane
    // of a converged warp issues, the warp stays together
    auto issue_mma1 = [&](int j) {
      const uint32_t kqb = base + P_KQ + (uint32_t)(j & 1) * 32768u;
      if (sm100::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = kqb + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          sm100::mma_f16_ss(tmem, kdesc(a), kdesc(a), ID_KQ, ks > 0);
        }
        sm100::mma_commit(&sm->bar_m1);
      }
      __syncwarp();
    };
    if (tid == 0) {
      sm100::prefetch_tmap(&tm_q);
      sm100::prefetch_tmap(&tm_k);
      issue_qk(0);
      if (n_chunks > 1) issue_qk(1);
    }
    GateRaw graw{};
    if (warp == 7) graw = load_gates_raw(g, beta, t0, chunk_len(0), H, h, lane);
    // chunk 0's MMA 1 (each later chunk's is issued during the previous solve)
    if (warp == 0) {
      const bool ok = __all_sync(0xffffffffu, wait_local(&sm->bar_qk[0], 0, sm, err));
      if (ok && lane == 0) sm->qk_pend[0] = 0;
      sm100::tc_fence_after();
      if (ok) issue_mma1(0);
    }
    for (int j = 0; j < n_chunks; ++j) {  // left only at the checks after barriers
      const int n = chunk_len(j);
      const int b = j & 1;
      const uint32_t stg = base + P_STG + (uint32_t)b * kRxBytes;
      const Gates *gt = &sm->gt;
      // this chunk's gates (the previous chunk's were last read by its
      // epilogue), and the raw gates of the next one
      if (warp == 7) {
        finish_gates(&sm->gt, graw, n, lane);
        if (j + 1 < n_chunks)
          graw = load_gates_raw(g, beta, t0 + (long long)(j + 1) * kC, chunk_len(j + 1), H, h, lane);
      }
      wait_local(&sm->bar_m1, (uint32_t)(j & 1), sm, err);
      sm100::tc_fence_after();
      // the tile is free again: chunk j+2 goes into it
      if (tid == 0 && j + 2 < n_chunks && !sm->abort) issue_qk(j + 2);
      __syncthreads();
      if (sm->abort) break;
      // ---- epilogue: rows 0-63 -> A (fp32, for the solve), rows 64-127 ->
      //      Aqk (fp16, staging); warps w and w+4 split the 64 columns ----
      {
        const int r = row & 63, i0 = 32 * wg;
        float v[32];
        sm100::tmem_ld32(tmem + lane_off + i0, v);
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
            st_shared_v4(sw128(stg + 16384u, r, 4 * wg + c), pack_h2(y[0], y[1]),
                         pack_h2(y[2], y[3]), pack_h2(y[4], y[5]), pack_h2(y[6], y[7]));
          }
        }
      }
      sm100::tc_fence_before();
      __syncthreads();
      // the next chunk's MMA 1 runs during this chunk's solve (D1 has been read)
      if (warp == 4 && j + 1 < n_chunks) {
        const int nbuf = (j + 1) & 1;
        const bool ok = __all_sync(
            0xffffffffu, wait_local(&sm->bar_qk[nbuf], (uint32_t)(((j + 1) >> 1) & 1), sm, err));
        if (ok && lane == 0) sm->qk_pend[nbuf] = 0;
        sm100::tc_fence_after();
        if (ok) issue_mma1(j + 1);
      }
      // ---- triangular solve T = (I + A)^-1 in three levels (warpgroup 0) ----
      if (wg == 0) {
        if (tid < 64) {
          // level 0: 16x16 diagonal blocks by right-looking column substitution
          const int bb = tid >> 4, jj = tid & 15, j0 = 16 * bb;
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
          const int e = tid - 64;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int idx = e * 8 + i, bb = idx >> 8, rr = (idx >> 4) & 15, cc = idx & 15;
            sT[(32 * bb + rr) * LDT + 32 * bb + 16 + cc] = 0.0f;
          }
        }
        asm volatile("bar.sync 3, 128;" ::: "memory");
        // level 1: blocks (1,0) and (3,2): T_ij = -T_ii (A_ij T_jj)
        {
          const int blk = tid >> 6, idx = tid & 63, rr = idx >> 2, cc = (idx & 3) * 4;
          const int r0 = 16 + 32 * blk, c0b = 32 * blk;
          const float *arow = sA + (r0 + rr) * LDT + c0b;
          const float *tcol = sT + c0b * LDT + c0b + cc;
          float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
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
#pragma unroll 4
          for (int m = 0; m < 16; ++m) {
            const float t = trow[m];
            const float4 p4 = *reinterpret_cast<const float4 *>(pcol + m * LDT);
            q.x += t * p4.x; q.y += t * p4.y; q.z += t * p4.z; q.w += t * p4.w;
          }
          *reinterpret_cast<float4 *>(sT + (r0 + rr) * LDT + c0b + cc) = make_float4(-q.x, -q.y, -q.z, -q.w);
        }
        asm volatile("bar.sync 3, 128;" ::: "memory");
        // level 2: the lower-left 32x32 block: T_21 = -T_22 (A_21 T_11).
        // The products of levels 1 and 2 are unrolled by 4 only: fully
        // unrolled, the producer's code grew large enough that instruction
        // fetch, which neighbouring SMs share, slowed pairs by up to 20 %
        // depending on where they ran
        {
          const int rr = tid >> 2, cc = (tid & 3) * 8;
          const float *arow = sA + (32 + rr) * LDT;
          const float *tcol = sT + cc;
          float p[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
          for (int m = 0; m < 32; ++m) {
            const float a = arow[m];
            const float4 t0v = *reinterpret_cast<const float4 *>(tcol + m * LDT);
            const float4 t1v = *reinterpret_cast<const float4 *>(tcol + m * LDT + 4);
            p[0] += a * t0v.x; p[1] += a * t0v.y; p[2] += a * t0v.z; p[3] += a * t0v.w;
            p[4] += a * t1v.x; p[5] += a * t1v.y; p[6] += a * t1v.z; p[7] += a * t1v.w;
          }
          *reinterpret_cast<float4 *>(sP + rr * LDT + cc) = make_float4(p[0], p[1], p[2], p[3]);
          *reinterpret_cast<float4 *>(sP + rr * LDT + cc + 4) = make_float4(p[4], p[5], p[6], p[7]);
          asm volatile("bar.sync 3, 128;" ::: "memory");
          const float *trow = sT + (32 + rr) * LDT + 32;
          const float *pcol = sP + cc;
          float q[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
          for (int m = 0; m < 32; ++m) {
            const float t = trow[m];
            const float4 p0v = *reinterpret_cast<const float4 *>(pcol + m * LDT);
            const float4 p1v = *reinterpret_cast<const float4 *>(pcol + m * LDT + 4);
            q[0] += t * p0v.x; q[1] += t * p0v.y; q[2] += t * p0v.z; q[3] += t * p0v.w;
            q[4] += t * p1v.x; q[5] += t * p1v.y; q[6] += t * p1v.z; q[7] += t * p1v.w;
          }
          float *tout = sT + (32 + rr) * LDT + cc;
          *reinterpret_cast<float4 *>(tout) = make_float4(-q[0], -q[1], -q[2], -q[3]);
          *reinterpret_cast<float4 *>(tout + 4) = make_float4(-q[4], -q[5], -q[6], -q[7]);
        }
        asm volatile("bar.sync 3, 128;" ::: "memory");
        // T -> hi/lo fp16 tiles [tok][tok'] (upper triangle zero), staging
        {
          const int r = tid >> 1, cpart = (tid & 1) * 32;
          const float *trow = sT + r * LDT + cpart;
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(trow + i);
            x[i] = cpart + i <= r ? t4.x : 0.f;
            x[i + 1] = cpart + i + 1 <= r ? t4.y : 0.f;
            x[i + 2] = cpart + i + 2 <= r ? t4.z : 0.f;
            x[i + 3] = cpart + i + 3 <= r ? t4.w : 0.f;
          }
          store32_hl(stg, stg + 8192u, r, cpart >> 3, x);
        }
      }
      sm100::fence_proxy_async();  // staging written by this CTA's threads -> bulk copy reads it
      __syncthreads();
      // ---- hand T hi, T lo, Aqk to the chain CTA once it has released the
      //      previous chunk's ----
      if (tid == 0) {
        bool ok = true;
        if (j > 0) ok = wait_cluster(&sm->rx_free, (uint32_t)((j - 1) & 1), sm, err);
        if (ok && !sm->abort)
          sm100::bulk_copy_to_cluster(rx_buf_remote, stg, kRxBytes, rx_full_remote);
      }
      __syncthreads();
    }
    // an aborted producer lets its TMA loads land before leaving
    if (tid == 0 && sm->abort) {
      for (int bb = 0; bb < 2; ++bb)
        if (sm->qk_pend[bb])
          (void)sm100::mbar_wait(&sm->bar_qk[bb], (uint32_t)(sm->qk_pend[bb] - 1), kWaitNs);
    }
  } else {
    // ============================ chain CTA ==============================
    SmallC *sm = smc;
    const uint32_t tmem = sm->tmem;
    auto issue_qk = [&](long long tb, int j) {
      const int b = j & 1;
      uint8_t *dst = gbase + C_KQ + b * 32768;
      sm100::mbar_arrive_expect_tx(&sm->bar_qk[b], 4 * 8192);
      sm100::tma_load_3d(dst + 0, &tm_k, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 8192, &tm_q, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 16384, &tm_k, &sm->bar_qk[b], 64, h, (int)tb);
      sm100::tma_load_3d(dst + 24576, &tm_q, &sm->bar_qk[b], 64, h, (int)tb);
      sm->qk_pend[b] = 1 + ((j >> 1) & 1);
    };
    auto issue_v = [&](long long tb, int j) {
      sm100::mbar_arrive_expect_tx(&sm->bar_v, 2 * 8192);
      sm100::tma_load_3d(gbase + C_V, &tm_v, &sm->bar_v, 0, h, (int)tb);
      sm100::tma_load_3d(gbase + C_V + 8192, &tm_v, &sm->bar_v, 64, h, (int)tb);
      sm->v_pend = 1 + (j & 1);
    };
    const uint32_t ID_H2 = sm100::idesc_f16_f32(128, 128, 1, 0);
    const uint32_t ID_N64 = sm100::idesc_f16_f32(128, 64, 1, 0);
    const uint32_t ID_64 = sm100::idesc_f16_f32(128, 64, 0, 0);
    const uint32_t ID_KV = sm100::idesc_f16_f32(128, 128, 1, 0);

    if (tid == 0) {
      sm100::prefetch_tmap(&tm_q);
      sm100::prefetch_tmap(&tm_k);
      sm100::prefetch_tmap(&tm_v);
      issue_qk(t0, 0);
      issue_v(t0, 0);
      if (n_chunks > 1) issue_qk(t0 + kC, 1);
    }
    // initial state: TMEM D4 = gamma_n * H0 and H0 hi/lo tiles
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
        store32_hl(base + C_H + 16384u * wg, base + C_H + 32768u + 16384u * wg, row, 4 * p, x);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] *= gnx;
        sm100::tmem_st32(tmem + lane_off + TM_D4 + c0, x);
      }
    }
    // chunk 0's [K;Q]: wait, convert (later chunks' during the previous chunk)
    if (wait_local(&sm->bar_qk[0], 0, sm, err) && tid == 0) sm->qk_pend[0] = 0;
    convert_kq_half(gbase + C_KQ, chunk_len(0), tid, 0);
    convert_kq_half(gbase + C_KQ, chunk_len(0), tid, 1);
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();

    // Outputs of chunk j: O^T[v][t] = scale (gamma_t hs_j (Q H0)^T[v][t] +
    // (Aqk Vn)^T[v][t]) -> o[t][h][v].  Run during chunk j+1's MMAs 4 and 5,
    // off the state chain; warpgroup wg covers tokens 32 wg .. + 31.  A whole chunk
    // goes through a shared-memory tile and two TMA stores issued by thread
    // 224; a partial chunk (the last of a sequence) is stored directly, so
    // that no row of the neighbouring sequence is written.
    constexpr int kStoreTid = 224;
    auto out_epilogue = [&](int j, long long tbj, int nj, float hs_j) {
      const Gates *gj = &sm->gt[j % 3];
      const uint32_t reg = (uint32_t)(j & 1) * TM_REG;
      const float sh = scale * hs_j;
      if (nj == kC) {
        // Fragments of 16 value rows x 32 tokens (two per warp), combined,
        // packed to bf16 token pairs and stored transposed into the tile
        // [v half][t][64 v] (128-byte rows, 16-byte chunks swizzled by t % 8).
        const int c = lane & 3, gq = lane >> 2;
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
          const int L = 32 * (warp & 3) + 16 * hl;  // first value row of the block
          const uint32_t lsel = (uint32_t)L << 16;
          uint32_t qh[16], av[16];
          sm100::tmem_ld16x256b_x4(tmem + lsel + reg + TM_QH + 32 * wg, qh);
          sm100::tmem_ld16x256b_x4(tmem + lsel + reg + 32 * wg, av);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 g2 = *reinterpret_cast<const float2 *>(gj->gam + 32 * wg + 8 * k + 2 * c);
            const float s0 = sh * g2.x, s1 = sh * g2.y;
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {  // value rows L + gq and L + 8 + gq
              const int e = 4 * k + 2 * hv;
              const float o0 = fmaf(s0, __uint_as_float(qh[e]), scale * __uint_as_float(av[e]));
              const float o1 = fmaf(s1, __uint_as_float(qh[e + 1]), scale * __uint_as_float(av[e + 1]));
              __nv_bfloat162 p2 = __floats2bfloat162_rn(o0, o1);
              pk[2 * k + hv] = *reinterpret_cast<uint32_t *>(&p2);
            }
          }
          // matrix m of an instruction: tokens 32 wg + 8 (k0 + m / 2) .. + 7,
          // values L + 8 (m % 2) .. + 7; this thread addresses row lane % 8 of
          // matrix lane / 8
#pragma unroll
          for (int k0 = 0; k0 < 4; k0 += 2) {
            const int m = lane >> 3, rr = lane & 7;
            const int t = 32 * wg + 8 * (k0 + (m >> 1)) + rr;
            const int v0 = L + 8 * (m & 1);
            const uint32_t addr = base + C_O + (uint32_t)(v0 >> 6) * 8192u + (uint32_t)t * 128u +
                                  ((uint32_t)(((v0 & 63) >> 3) ^ (t & 7)) << 4);
            sm100::stmatrix_x4_trans(addr, pk[2 * k0], pk[2 * k0 + 1], pk[2 * k0 + 2],
                                     pk[2 * k0 + 3]);
          }
        }
        sm100::fence_proxy_async();
        asm volatile("bar.sync 5, 256;" ::: "memory");
        if (tid == kStoreTid) {
          sm100::tma_store_3d(&tm_o, gbase + C_O, 0, h, (int)tbj);
          sm100::tma_store_3d(&tm_o, gbase + C_O + 8192, 64, h, (int)tbj);
          sm100::bulk_commit();
        }
      } else {
        float qh[32], av[32];
        sm100::tmem_ld32(tmem + lane_off + reg + TM_QH + 32 * wg, qh);
        sm100::tmem_ld32(tmem + lane_off + reg + 32 * wg, av);
        const int cnt = nj - 32 * wg;
        __nv_bfloat16 *dst = o + ((tbj + 32 * wg) * H + h) * kD + row;
        const long long ts = (long long)H * kD;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float ot = fmaf(sh * gj->gam[32 * wg + t], qh[t], scale * av[t]);
          if (t < cnt) dst[t * ts] = __float2bfloat16_rn(ot);
        }
      }
    };

    long long tb_prev = 0;
    int n_prev = 0;
    float hs_prev = 1.0f;
    for (int it = 0; it < n_chunks; ++it) {  // left only at the checks after barriers
      const long long c0 = (long long)it * kC;
      const int n = chunk_len(it);
      const long long tb = t0 + c0;
      const bool last = it == n_chunks - 1;
      const uint32_t par = (uint32_t)(it & 1);
      const int kb = it & 1, nb = kb ^ 1;
      const uint32_t kq = base + C_KQ + (uint32_t)kb * 32768u;
      const Gates *gt = &sm->gt[it % 3];
      Gates *gt_next = &sm->gt[(it + 1) % 3];
      const bool exact = sm->exact != 0;
      const float hsv = exact ? sm->hs[row >> 6] : 1.0f;
      GateRaw graw{};
      if (warp == 7 && !last) graw = load_gates_raw(g, beta, tb + kC, chunk_len(it + 1), H, h, lane);

      // ---- MMA 2: [P | Q H0]^T = H0^T [K;Q]^T (hi, or exact codes), + H0lo^T K^T,
      //      into this chunk's region ----
      const uint32_t reg = (uint32_t)kb * TM_REG;
      if (warp == 0) {
        sm100::tc_fence_after();
        if (sm100::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t bq = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
            sm100::mma_f16_ss(tmem + reg, mndesc(base + C_H + (uint32_t)ks * 2048u, 16384),
                              kdesc(bq), ID_H2, ks > 0);
          }
          if (!exact) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t bq = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
              sm100::mma_f16_ss(tmem + reg,
                                mndesc(base + C_H + 32768u + (uint32_t)ks * 2048u, 16384),
                                kdesc(bq), ID_N64, 1);
            }
          }
          sm100::mma_commit(&sm->bar_m2);
        }
        __syncwarp();
      }
      // while MMA 2 runs: the first half of the next chunk's [K;Q] conversion
      if (!last) {
        if (wait_local(&sm->bar_qk[nb], (uint32_t)(((it + 1) >> 1) & 1), sm, err) && tid == 0)
          sm->qk_pend[nb] = 0;
        convert_kq_half(gbase + C_KQ + nb * 32768, chunk_len(it + 1), tid, 0);
      }

      // ---- R = diag(beta) (V - diag(gamma) P) -> TMEM (all warps; warpgroup
      //      wg: tokens 32 wg .. + 31, hi at R + 32 wg, lo at R + 32 wg + 16) ----
      {
        if (wait_local(&sm->bar_v, par, sm, err) && tid == 128) sm->v_pend = 0;
        wait_local(&sm->bar_m2, par, sm, err);
        sm100::tc_fence_after();
        const uint8_t *stgv = gbase + C_V + (row >> 6) * 8192 + (row & 63) * 2;
        float x[32];
        sm100::tmem_ld32(tmem + lane_off + reg + 32 * wg, x);
        uint32_t whi[16], wlo[16];
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const int tok = 32 * wg + t;
          const float4 b4 = *reinterpret_cast<const float4 *>(gt->beta + tok);
          const float4 g4 = *reinterpret_cast<const float4 *>(gt->gam + tok);
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w}, gg[4] = {g4.x, g4.y, g4.z, g4.w};
          float r4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float vt =
                __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(stgv + (tok + e) * 128));
            // tokens past n (a partial last chunk): the staged rows belong to
            // another sequence or lie past the tensor; R is zero there
            r4[e] = tok + e < n ? bb[e] * (vt - (gg[e] * hsv) * x[t + e]) : 0.0f;
          }
          split_h2(r4[0], r4[1], whi[t >> 1], wlo[t >> 1]);
          split_h2(r4[2], r4[3], whi[(t >> 1) + 1], wlo[(t >> 1) + 1]);
        }
        sm100::tmem_st16(tmem + lane_off + TM_R + 32 * wg, whi);
        sm100::tmem_st16(tmem + lane_off + TM_R + 32 * wg + 16, wlo);
      }
      sm100::tc_fence_before();
      __syncthreads();
      if (sm->abort) break;
      if (tid == 224 && !last) issue_v(tb + kC, it + 1);

      // ---- MMA 3: Vn^T = R^T T^T (hi*hi + hi*lo + lo*hi), T from the
      //      producer's transfer ----
      if (warp == 0) {
        const bool got = __all_sync(0xffffffffu, wait_cluster(&sm->rx_full, par, sm, err));
        if (got && lane == 0) sm->rx_pend = 0;
        sm100::tc_fence_after();
        if (got && sm100::elect_one()) {
          const uint32_t tB[3] = {0u, 8192u, 0u}, lo[3] = {0u, 0u, 16u};
#pragma unroll
          for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              sm100::mma_f16_ts(tmem + reg,
                                tmem + TM_R + 32u * (ks >> 1) + 8u * (ks & 1) + lo[pass],
                                kdesc(base + C_RX + tB[pass] + 32u * ks), ID_64, pass + ks > 0);
          sm100::mma_commit(&sm->bar_m3);
        }
        __syncwarp();
      }
      // while MMA 3 runs: the next chunk's gates (slot (it+1) % 3 was last
      // read by the output epilogue of chunk it-2), visible to epilogue 4
      // after the barrier that follows epilogue 3, and the second half of
      // the next chunk's conversion
      if (warp == 7 && !last) finish_gates(gt_next, graw, chunk_len(it + 1), lane);
      if (!last) convert_kq_half(gbase + C_KQ + nb * 32768, chunk_len(it + 1), tid, 1);

      // ---- epilogue 3: Vn^T hi -> TMEM (A of MMA 4); decayed dVn^T hi/lo -> smem ----
      {
        wait_local(&sm->bar_m3, par, sm, err);
        sm100::tc_fence_after();
        const int vv = row, t0h = 32 * wg;
        float x[32];
        sm100::tmem_ld32(tmem + lane_off + reg + t0h, x);
        uint32_t w[16];
#pragma unroll
        for (int t = 0; t < 32; t += 2) w[t >> 1] = pack_h2(x[t], x[t + 1]);
        sm100::tmem_st16(tmem + lane_off + TM_VN + 16 * wg, w);
#pragma unroll
        for (int t = 0; t < 32; ++t) x[t] *= gt->dec[t0h + t];
        store32_hl(base + C_DV, base + C_DV + 16384u, vv, 4 * wg, x);
      }
      sm100::fence_proxy_async();
      sm100::tc_fence_before();
      __syncthreads();
      if (sm->abort) break;

      // ---- MMA 4: D5 = Vn^T Aqk^T (Aqk from the transfer);  MMA 5: H += K^T dVn ----
      if (warp == 0) {
        sm100::tc_fence_after();
        if (sm100::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            sm100::mma_f16_ts(tmem + reg, tmem + TM_VN + 8u * ks,
                              kdesc(base + C_RX + 16384u + 32u * ks), ID_64, ks > 0);
#pragma unroll
          for (int pass = 0; pass < 2; ++pass)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              sm100::mma_f16_ss(tmem + TM_D4, mndesc(kq + (uint32_t)ks * 2048u, 16384),
                                kdesc(base + C_DV + (pass ? 16384u : 0u) + 32u * ks), ID_KV, 1);
          sm100::mma_commit(&sm->bar_m4);
        }
        __syncwarp();
      }
      // while MMAs 4 and 5 run: the previous chunk's outputs (its MMA 4 wrote
      // the other TMEM region; its output tile was read out a chunk ago)
      if (it > 0) out_epilogue(it - 1, tb_prev, n_prev, hs_prev);

      // ---- epilogue 4 ----
      wait_local(&sm->bar_m4, par, sm, err);
      sm100::tc_fence_after();
      if (tid == 0 && !sm->abort) {
        // MMAs 3 and 4 have read the received tiles: arm the next chunk's
        // transfer, then release the buffer to the producer.  A relaxed
        // arrive: what the producer must not overtake are the tensor-core
        // reads of the buffer, which the commit barrier this thread has
        // waited for already orders; no thread of this CTA writes the buffer
        // (a release arrive would also wait for this thread's outstanding
        // stores of the previous chunk's outputs).
        if (!last) {
          sm100::mbar_arrive_expect_tx(&sm->rx_full, kRxBytes);
          sm->rx_pend = 1 + ((it + 1) & 1);
        }
        sm100::mbar_arrive_cluster_relaxed(rx_free_remote);
      }
      // the buffer MMA 5 just released takes the chunk after next
      if (tid == 128 && !last && it + 2 < n_chunks && !sm->abort) issue_qk(tb + 2 * kC, it + 2);
      {
        // H: key row `row`, value columns 64 wg .. + 63 (one FP8 tile per warpgroup)
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
        const float gn_next = last ? 1.0f : gt_next->gn_exp;
        const ScaleRecip sr_tile = make_scale(fp8_scale(QK == kQdqFp8Tile && mh > 0.f ? mh : 1.0f));
        // FP8: the dequantized codes go straight into the next carry's accumulator
        // (code x (s gamma_n), one rounding); the last chunk's are the state itself
        const float sdq = last ? sr_tile.s : sr_tile.s * gn_next;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const int c0v = 64 * wg + 32 * p;
          float y[32];
          sm100::tmem_ld32(tmem + lane_off + TM_D4 + c0v, y);
          if (QK == kQdqFp8Tile) {
            uint32_t code[16];
            if (mh == 0.0f) {
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
              st_shared_v4(sw128(base + C_H + 16384u * wg, row, 4 * p + c), code[4 * c],
                           code[4 * c + 1], code[4 * c + 2], code[4 * c + 3]);
          } else {
            if (QK == kQdqInt8) {
              constexpr int GW = GROUP < 32 ? GROUP : 32;
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
            store32_hl(base + C_H + 16384u * wg, base + C_H + 32768u + 16384u * wg, row, 4 * p, y);
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
      tb_prev = tb;
      n_prev = n;
      hs_prev = hsv;
      if (tid == kStoreTid) sm100::bulk_wait_read_all();  // the output tile is free again
      sm100::fence_proxy_async();
      sm100::tc_fence_before();
      __syncthreads();
      if (tid == 0) sm->exact = QK == kQdqFp8Tile ? 1 : 0;
      __syncthreads();
      if (last) out_epilogue(it, tb, n, hsv);  // the last chunk's outputs
    }
    if (tid == kStoreTid) sm100::bulk_wait_all();
    if (tid == 0 && sm->abort) {
      for (int bb = 0; bb < 2; ++bb)
        if (sm->qk_pend[bb])
          (void)sm100::mbar_wait(&sm->bar_qk[bb], (uint32_t)(sm->qk_pend[bb] - 1), kWaitNs);
      if (sm->v_pend) (void)sm100::mbar_wait(&sm->bar_v, (uint32_t)(sm->v_pend - 1), kWaitNs);
      // and the producer's transfer into the receive buffer, if one is armed
      if (sm->rx_pend)
        (void)sm100::mbar_wait_cluster(&sm->rx_full, (uint32_t)(sm->rx_pend - 1), kWaitNs);
    }
  }

  // ---- teardown: an aborted CTA lets the MMAs of its issuing warps (0 and
  //      4) finish; neither CTA leaves while the peer may still copy into or
  //      arrive on its shared memory ----
  {
    const int ab = rank == 0 ? smc->abort : smp->abort;
    uint64_t *bd = rank == 0 ? smc->bar_drain : smp->bar_drain;
    if (ab && (warp == 0 || warp == 4)) drain_mmas(&bd[warp >> 2]);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(rank == 0 ? smc->tmem : smp->tmem, rank == 0 ? TM_COLS_C : TM_COLS_P);
  }
}

}  // namespace pair
}  // namespace gdn
