// Chunked prefix of the gated delta rule (GDN, scalar gate) with an FP8 E4M3
// tile QDQ state, in the WY form proper, on a pair of CTAs (a thread-block
// cluster of two per (sequence, head), d_k = d_v = 128).
//
// Algebra per 64-token chunk (PR #2497 What section: 64-token chunks, the
// WY-transformed W; PR #2507 What section: exact triangular solve), with G_t
// the within-chunk cumulative log gate, gamma_t = exp(G_t), dec_t =
// exp(G_{n-1} - G_t), S0 the chunk-start state as the pages write it
// ([d_v, d_k], the transpose of the stored H):
//
//   A   = strict_lower(diag(beta) (K K^T) * exp(G_r - G_i))
//   Aqk = lower((Q K^T) * exp(G_r - G_i))
//   T   = (I + A)^-1                                 (exact substitution)
//   W   = T diag(beta gamma) K,   U = T diag(beta) V
//   Vn  = U - W S0^T
//   O   = scale (diag(gamma) Q S0^T + Aqk Vn)
//   S   = gamma_n S0 + Vn^T diag(dec) K,   then S = QDQ(S)
//
// Division of the work:
//
//   rank 1 (producer)  one or two chunks ahead of the chain: [K;Q] K^T on the
//                      raw bf16 tile, the A / Aqk epilogue, the solve, then
//                      W^T = K^T (T diag(beta gamma))^T on the tensor cores;
//                      hands W (hi, lo), T diag(beta) (hi, lo) and Aqk (56 KB)
//                      to the chain CTA's receive slot (distributed shared
//                      memory, no multicast); two slots, so a copy has a whole
//                      chunk to land.
//   rank 0 (chain)     per chunk: U^T = V^T (T diag(beta))^T (issued a chunk
//                      early), X = S0c W^T, Vn^T = U^T - s0 X, Vn^T and
//                      dec * Vn^T (hi, lo) back into TMEM, O^T = S0c (gamma Q)^T
//                      + Vn^T Aqk^T, S += (dec Vn)^T K, the QDQ.
//
// The chain keeps S in TMEM with one value column per lane (S[v][k], lanes =
// v), so one FP8 tile (all keys x 64 value columns) is 64 lanes and every
// thread has a single scale.  The QDQ writes the tile's E4M3 codes (exact in
// fp16) straight back into TMEM as the A operand of the next chunk's products
// (S0 = s0 * codes; the scale is applied in the epilogues), so no operand of
// the state path passes through shared memory: A operands come from TMEM,
// B operands (W, K, Q, Aqk) from shared memory.  The chain's critical path
// per chunk is X -> Vn epilogue -> (O part 2, S update) -> QDQ.
//
// Every wait is bounded (2 s): on a timeout a CTA records kErrTimeout and
// stops, lets its own asynchronous copies land, and both CTAs meet at the
// cluster barrier before either exits.
#pragma once

#include "gdn_tc_util.cuh"

namespace gdn {
namespace wy {

using namespace tcu;

constexpr int kThreads = 256;
constexpr int kC = 64;
constexpr int kD = 128;
constexpr uint64_t kWaitNs = 2000000000ull;

// ---- one hand-off slot (byte offsets; every tile 1024-byte aligned)
constexpr uint32_t H_WHI = 0;       // W hi  [k][t] fp16, 128 rows x 128 B (B of X, MN-major)
constexpr uint32_t H_WLO = 16384;   // W lo
constexpr uint32_t H_THI = 32768;   // (T diag(beta)) hi [t][t'] (B of U, K-major)
constexpr uint32_t H_TLO = 40960;   // (T diag(beta)) lo
constexpr uint32_t H_AQK = 49152;   // Aqk [t][t'] fp16 (B of O part 2, K-major)
constexpr uint32_t kRxBytes = 57344;
// With the FP8 QDQ of W: the W area holds the E4M3 codes of W, K-major
// [t][k] (two 64-key halves 8 KB apart; B of X), and the 64 row scales at
// H_WLO; 16,640 bytes of it are handed over.
constexpr uint32_t H_WSC = H_WLO;
constexpr uint32_t kWqBytes = 16384 + 256;
constexpr uint32_t kRxBytesWq = kWqBytes + (kRxBytes - H_THI);
constexpr int LDW = 129;  // row stride (floats) of W staged as fp32 [t][k] for the row amax

// ---- chain CTA shared memory
constexpr uint32_t C_KQ = 0;        // 2 x [K | gamma Q] fp16 (K h0 | Q h0 | K h1 | Q h1, 8 KB each)
constexpr uint32_t C_V = 65536;     // 2 x V fp16 [t][v] (v halves 8 KB apart)
constexpr uint32_t C_RX = 98304;    // 2 receive slots
constexpr uint32_t C_SMALL = C_RX + 2 * kRxBytes;
// ---- producer CTA shared memory
constexpr int LDT = 68;
constexpr uint32_t P_KQ = 0;        // 2 x [K;Q] bf16 (TMA); K converted to fp16 in place after MMA 1
constexpr uint32_t P_SA = 65536;    // A fp32 [64 x LDT]
constexpr uint32_t P_SP = P_SA + 64 * LDT * 4;  // partial products [32 x LDT]
constexpr uint32_t P_ST = P_SP + 32 * LDT * 4;  // T fp32 [64 x LDT]
constexpr uint32_t P_STG = 109568;  // 2 staging slots (chunk j: slot j % 2); T diag(beta gamma)
                                    // hi/lo sit in the W area until the W product has read it
constexpr uint32_t P_SMALL = P_STG + 2 * kRxBytes;
constexpr uint32_t kSmallBytes = 4096;
static_assert(C_SMALL + kSmallBytes <= P_SMALL, "the two roles' small blocks must not overlap");
static_assert(P_ST + 64 * LDT * 4 <= P_STG && P_STG % 1024 == 0 && C_RX % 1024 == 0 &&
                  kRxBytes % 1024 == 0,
              "shared-memory maps");
constexpr uint32_t kSmemBytes = P_SMALL + kSmallBytes + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");

// ---- chain TMEM columns (lanes = value columns v)
constexpr uint32_t TM_S = 0;      // S [v][k] fp32 accumulator                     128
constexpr uint32_t TM_S0C = 128;  // S0 codes (or hi) fp16 [v][k], A operand         64
constexpr uint32_t TM_X = 192;    // X = S0c [W hi | W lo]^T [v][t a | t b]          128
                                  // then dVn hi (t 32 w .. +31) at X + 32 w, lo at + 16
constexpr uint32_t TM_U = 320;    // U^T [v][t]; then Vn hi at U + 32 w               64
constexpr uint32_t TM_O1 = 384;   // S0c (gamma Q)^T [v][t]                           64
constexpr uint32_t TM_O2 = 448;   // Vn^T Aqk^T [v][t]; S0 lo before chunk 0's X      64
constexpr uint32_t TM_COLS_C = 512;
// ---- producer TMEM (lanes = rows of [K;Q] for MMA 1, keys k for W^T)
constexpr uint32_t TP_D1 = 0;     // [K;Q] K^T                                        64
constexpr uint32_t TP_W = 64;     // W^T [k][t hi part | t lo part]                  128
constexpr uint32_t TM_COLS_P = 256;

struct ChainGates {
  float gam[64], dec[64];
  float gn;  // exp(G_{n-1})
  float pad[3];
};
struct SmallC {
  ChainGates gt[3];  // chunk j in slot j % 3
  float red[2][4];   // FP8 tile amax of the 4 warps of each tile
  int abort;
  int qk_pend[2], v_pend[2], rx_pend[2];  // 1 + parity of a transfer not yet waited for
  uint32_t tmem;
  uint64_t wait_ns;  // limit of the bounded waits (the drains keep kWaitNs)
  uint64_t bar_qk[2], bar_v[2], bar_x, bar_o2, bar_m5, bar_u, rx_full[2], bar_drain[2];
};
struct SmallP {
  Gates gt;
  int abort;
  int qk_pend[2];
  uint32_t tmem;
  uint64_t wait_ns;
  uint64_t bar_qk[2], bar_m1, bar_w, rx_free[2], bar_drain[2];
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

// The chain's gates of one chunk (one warp): gamma, dec and gamma_n from the
// raw log gates (rows past n are zero-gated, so gamma stays finite).
__device__ __forceinline__ void finish_chain_gates(ChainGates *gt, GateRaw r, int n, int lane) {
  float x0 = r.g0, x1 = r.g1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
    const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
    if (lane >= off) { x0 += y0; x1 += y1; }
  }
  x1 += __shfl_sync(0xffffffffu, x0, 31);
  const float gn = __shfl_sync(0xffffffffu, (n - 1) < 32 ? x0 : x1, (n - 1) & 31);
  gt->gam[lane] = expf(x0);
  gt->gam[lane + 32] = expf(x1);
  gt->dec[lane] = expf(gn - x0);
  gt->dec[lane + 32] = expf(gn - x1);
  if (lane == 0) gt->gn = expf(gn);
}

// In-place bf16 -> fp16 conversion of the 64-row half `part` of a 16 KB
// tile pair at `buf` + part * 8192 (V: value halves) by 256 threads; rows
// past n are zeroed.
__device__ __forceinline__ void convert_v_half(uint8_t *buf, int n, int t, int part) {
  uint4 x[2];
  uint8_t *ad[2];
  bool live[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = u * 256 + t;  // < 512 chunks of 16 B
    const int rw = e >> 3, ch = e & 7;
    ad[u] = buf + part * 8192 + rw * 128 + ch * 16;
    live[u] = rw < n;
    x[u] = *reinterpret_cast<const uint4 *>(ad[u]);
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
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

// In-place conversion of half `part` (key columns 64 part .. + 63) of one
// [K | Q] buffer: K rows (0-63) to fp16, Q rows (64-127, token r - 64) to
// fp16(gamma_t q); rows of tokens past n are zeroed.
__device__ __forceinline__ void convert_kq_gamma_half(uint8_t *buf, int n, int t, int part,
                                                      const float *gam) {
  uint4 x[4];
  uint8_t *ad[4];
  int rw[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int e = u * 256 + t;  // < 1024
    rw[u] = e >> 3;
    ad[u] = buf + part * 16384 + rw[u] * 128 + (e & 7) * 16;
    x[u] = *reinterpret_cast<const uint4 *>(ad[u]);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int tok = rw[u] & 63;
    const float sc = rw[u] < 64 ? 1.0f : gam[tok];
    const uint32_t in[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (tok < n) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = pack_h2(sc * __uint_as_float(in[j] << 16), sc * __uint_as_float(in[j] & 0xffff0000u));
    }
    *reinterpret_cast<uint4 *>(ad[u]) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// E4M3 codes of x0 / s and x1 / s as an exact fp16 pair (correctly rounded
// quotients from r = RN(1/s2) and Markstein's correction; `pre` scaling only
// for tiny scales, see make_scale).
__device__ __forceinline__ uint32_t fp8_codes(float x0, float x1, const ScaleRecip &sr) {
  uint64_t x = f2_pack(x0, x1);
  if (sr.pre != 1.0f) x = f2_mul(x, f2_pack(sr.pre, sr.pre));
  const uint64_t rr = f2_pack(sr.r, sr.r);
  const uint64_t q = f2_mul(x, rr);
  const uint64_t t = f2_fma(f2_fma(q, f2_pack(-sr.s2, -sr.s2), x), rr, q);
  float t0, t1;
  f2_unpack(t, t0, t1);
  const __nv_fp8x2_storage_t f8 =
      __nv_cvt_float2_to_fp8x2(make_float2(t0, t1), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(f8, __NV_E4M3);
  return *reinterpret_cast<const uint32_t *>(&hr);
}

// code pair (fp16) * c -> two fp32 values.
__device__ __forceinline__ void dequant2(uint32_t code, float c, float &y0, float &y1) {
  float a, b;
  h2_to_f32(code, a, b);
  y0 = a * c;
  y1 = b * c;
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <bool WQ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
prefill_wy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
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
  const int row = 32 * (warp & 3) + lane;  // TMEM lane
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
  // the peer's barriers and buffers, by offset (same map in both CTAs)
  uint32_t rx_full_remote[2], rx_free_remote[2], rx_buf_remote[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    rx_full_remote[b] = sm100::mapa(sm100::smem_u32(&smc->rx_full[b]), 0);
    rx_free_remote[b] = sm100::mapa(sm100::smem_u32(&smp->rx_free[b]), 1);
    rx_buf_remote[b] = sm100::mapa(base + C_RX + (uint32_t)b * kRxBytes, 0);
  }

  // ---------------------------------------------------------------- setup
  if (rank == 0) {
    if (tid == 0) {
      for (int b = 0; b < 2; ++b) {
        sm100::mbar_init(&smc->bar_qk[b], 1);
        sm100::mbar_init(&smc->bar_v[b], 1);
        sm100::mbar_init(&smc->rx_full[b], 1);
      }
      sm100::mbar_init(&smc->bar_x, 1);
      sm100::mbar_init(&smc->bar_o2, 1);
      sm100::mbar_init(&smc->bar_m5, 1);
      sm100::mbar_init(&smc->bar_u, 1);
      sm100::mbar_init(&smc->bar_drain[0], 1);
      sm100::mbar_init(&smc->bar_drain[1], 1);
      sm100::fence_mbar_init();
      smc->abort = 0;
      smc->wait_ns = wait_ns;
      for (int b = 0; b < 2; ++b) smc->qk_pend[b] = smc->v_pend[b] = smc->rx_pend[b] = 0;
      // chunks 0 and 1: both receive slots armed before the producer may copy
      for (int b = 0; b < 2 && b < n_chunks; ++b) {
        sm100::mbar_arrive_expect_tx(&smc->rx_full[b], WQ ? kRxBytesWq : kRxBytes);
        smc->rx_pend[b] = 1;
      }
    }
    if (warp == 0) {
      sm100::tmem_alloc(&smc->tmem, TM_COLS_C);
      sm100::tmem_relinquish();
    }
    if (warp == 7) {
      finish_chain_gates(&smc->gt[0], load_gates_raw(g, beta, t0, chunk_len(0), H, h, lane),
                         chunk_len(0), lane);
      if (n_chunks > 1)
        finish_chain_gates(&smc->gt[1],
                           load_gates_raw(g, beta, t0 + kC, chunk_len(1), H, h, lane),
                           chunk_len(1), lane);
    }
  } else {
    if (tid == 0) {
      sm100::mbar_init(&smp->bar_qk[0], 1);
      sm100::mbar_init(&smp->bar_qk[1], 1);
      sm100::mbar_init(&smp->bar_m1, 1);
      sm100::mbar_init(&smp->bar_w, 1);
      sm100::mbar_init(&smp->rx_free[0], 1);
      sm100::mbar_init(&smp->rx_free[1], 1);
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
    // =================== producer: A, Aqk, T, W for every chunk ===========
    SmallP *sm = smp;
    const uint32_t tmem = sm->tmem;
    float *sA = reinterpret_cast<float *>(gbase + P_SA);
    float *sP = reinterpret_cast<float *>(gbase + P_SP);
    float *sT = reinterpret_cast<float *>(gbase + P_ST);
    const uint32_t ID_KQ = sm100::idesc_f16_f32(128, 64, 0, 0) | (1u << 7) | (1u << 10);  // bf16
    const uint32_t ID_W = sm100::idesc_f16_f32(128, 128, 1, 0);
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
    // D1 = [K;Q] K^T on the raw bf16 tile (exact products)
    auto issue_mma1 = [&](int j) {
      const uint32_t kqb = base + P_KQ + (uint32_t)(j & 1) * 32768u;
      if (sm100::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = kqb + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          sm100::mma_f16_ss(tmem + TP_D1, kdesc(a), kdesc(a), ID_KQ, ks > 0);
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
      const uint32_t kbuf = base + P_KQ + (uint32_t)b * 32768u;
      const Gates *gt = &sm->gt;
      if (warp == 7) {
        finish_gates(&sm->gt, graw, n, lane);
        if (j + 1 < n_chunks)
          graw = load_gates_raw(g, beta, t0 + (long long)(j + 1) * kC, chunk_len(j + 1), H, h, lane);
      }
      // staging slot b (and the chain's receive slot b) free again: released
      // by the chain after its chunk j - 2
      if (tid == 0 && j >= 2) wait_cluster(&sm->rx_free[b], (uint32_t)(((j - 2) >> 1) & 1), sm, err);
      wait_local(&sm->bar_m1, (uint32_t)(j & 1), sm, err);
      sm100::tc_fence_after();
      __syncthreads();
      if (sm->abort) break;
      // ---- epilogue 1: rows 0-63 -> A (fp32, for the solve), rows 64-127 ->
      //      Aqk (fp16, staging); warps w and w+4 split the 64 columns ----
      {
        const int r = row & 63, i0 = 32 * wg;
        float v[32];
        sm100::tmem_ld32(tmem + lane_off + TP_D1 + i0, v);
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
            st_shared_v4(sw128(stg + H_AQK, r, 4 * wg + c), pack_h2(y[0], y[1]),
                         pack_h2(y[2], y[3]), pack_h2(y[4], y[5]), pack_h2(y[6], y[7]));
          }
        }
      }
      // K of this chunk -> fp16 in place (A operand of the W product); MMA 1
      // has read the bf16 tile
      convert_kq_half(gbase + P_KQ + b * 32768, n, tid, 0);
      convert_kq_half(gbase + P_KQ + b * 32768, n, tid, 1);
      sm100::fence_proxy_async();
      sm100::tc_fence_before();
      __syncthreads();
      // the hand-off leaves in three pieces as they are ready (Aqk now, T
      // diag(beta) after the solve, W last), all counted on the chain's
      // receive barrier of this slot
      if (tid == 0 && !sm->abort)
        sm100::bulk_copy_to_cluster(rx_buf_remote[b] + H_AQK, stg + H_AQK, kRxBytes - H_AQK,
                                    rx_full_remote[b]);
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
          // level 0: 16x16 diagonal blocks by column substitution
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
          *reinterpret_cast<float4 *>(sT + (r0 + rr) * LDT + c0b + cc) = make_float4(-q.x, -q.y, -q.z, -q.w);
        }
      }
      __syncthreads();
      // level 2 (all 256 threads): the lower-left 32x32 block,
      // T_21 = -T_22 (A_21 T_11); thread: row rr, columns cc .. cc + 3
      {
        const int rr = tid >> 3, cc = (tid & 7) * 4;
        float a[32];  // the thread's row of A_21, then of T_22
#pragma unroll
        for (int m = 0; m < 32; m += 4) {
          const float4 a4 = *reinterpret_cast<const float4 *>(sA + (32 + rr) * LDT + m);
          a[m] = a4.x; a[m + 1] = a4.y; a[m + 2] = a4.z; a[m + 3] = a4.w;
        }
        const float *tcol = sT + cc;
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f), p2 = p;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
          const float4 t4 = *reinterpret_cast<const float4 *>(tcol + m * LDT);
          const float4 u4 = *reinterpret_cast<const float4 *>(tcol + (m + 1) * LDT);
          p.x += a[m] * t4.x; p.y += a[m] * t4.y; p.z += a[m] * t4.z; p.w += a[m] * t4.w;
          p2.x += a[m + 1] * u4.x; p2.y += a[m + 1] * u4.y; p2.z += a[m + 1] * u4.z; p2.w += a[m + 1] * u4.w;
        }
        *reinterpret_cast<float4 *>(sP + rr * LDT + cc) =
            make_float4(p.x + p2.x, p.y + p2.y, p.z + p2.z, p.w + p2.w);
#pragma unroll
        for (int m = 0; m < 32; m += 4) {
          const float4 a4 = *reinterpret_cast<const float4 *>(sT + (32 + rr) * LDT + 32 + m);
          a[m] = a4.x; a[m + 1] = a4.y; a[m + 2] = a4.z; a[m + 3] = a4.w;
        }
        __syncthreads();
        const float *pcol = sP + cc;
        float4 q = make_float4(0.f, 0.f, 0.f, 0.f), q2 = q;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
          const float4 p4 = *reinterpret_cast<const float4 *>(pcol + m * LDT);
          const float4 v4 = *reinterpret_cast<const float4 *>(pcol + (m + 1) * LDT);
          q.x += a[m] * p4.x; q.y += a[m] * p4.y; q.z += a[m] * p4.z; q.w += a[m] * p4.w;
          q2.x += a[m + 1] * v4.x; q2.y += a[m + 1] * v4.y; q2.z += a[m + 1] * v4.z; q2.w += a[m + 1] * v4.w;
        }
        *reinterpret_cast<float4 *>(sT + (32 + rr) * LDT + cc) =
            make_float4(-(q.x + q2.x), -(q.y + q2.y), -(q.z + q2.z), -(q.w + q2.w));
      }
      __syncthreads();
      // ---- T diag(beta gamma) -> hi/lo (B of the W product, in the W area)
      //      and T diag(beta) -> hi/lo (handed over); [t][t'] rows, upper
      //      triangle zero; thread: row tid / 4, 16 columns ----
      {
        const int r = tid >> 2, c0 = (tid & 3) * 16;
        const float *trow = sT + r * LDT + c0;
        float xw[16], xu[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 t4 = *reinterpret_cast<const float4 *>(trow + i);
          const float4 b4 = *reinterpret_cast<const float4 *>(gt->beta + c0 + i);
          const float4 g4 = *reinterpret_cast<const float4 *>(gt->gam + c0 + i);
          const float tt[4] = {t4.x, t4.y, t4.z, t4.w}, bb[4] = {b4.x, b4.y, b4.z, b4.w},
                      gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float tv = c0 + i + e <= r ? tt[e] : 0.f;
            xu[i + e] = tv * bb[e];
            xw[i + e] = xu[i + e] * gg[e];
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t hw[4], lw[4], hu[4], lu[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            split_h2(xw[8 * c + 2 * e], xw[8 * c + 2 * e + 1], hw[e], lw[e]);
            split_h2(xu[8 * c + 2 * e], xu[8 * c + 2 * e + 1], hu[e], lu[e]);
          }
          const int ch = (c0 >> 3) + c;
          st_shared_v4(sw128(stg + H_WHI, r, ch), hw[0], hw[1], hw[2], hw[3]);
          st_shared_v4(sw128(stg + H_WHI + 8192u, r, ch), lw[0], lw[1], lw[2], lw[3]);
          st_shared_v4(sw128(stg + H_THI, r, ch), hu[0], hu[1], hu[2], hu[3]);
          st_shared_v4(sw128(stg + H_TLO, r, ch), lu[0], lu[1], lu[2], lu[3]);
        }
      }
      sm100::fence_proxy_async();
      sm100::tc_fence_before();
      __syncthreads();
      if (tid == 0 && !sm->abort)
        sm100::bulk_copy_to_cluster(rx_buf_remote[b] + H_THI, stg + H_THI, H_AQK - H_THI,
                                    rx_full_remote[b]);
      // ---- W^T [k][t hi part | t lo part] = K^T (T diag(beta gamma))^T ----
      if (warp == 0) {
        sm100::tc_fence_after();
        if (sm100::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            sm100::mma_f16_ss(tmem + TP_W, mndesc(kbuf + (uint32_t)ks * 2048u, 16384),
                              kdesc(stg + H_WHI + 32u * ks), ID_W, ks > 0);
          sm100::mma_commit(&sm->bar_w);
        }
        __syncwarp();
      }
      wait_local(&sm->bar_w, (uint32_t)(j & 1), sm, err);
      sm100::tc_fence_after();
      // K has been read: the buffer takes chunk j + 2
      if (tid == 0 && j + 2 < n_chunks && !sm->abort) issue_qk(j + 2);
      // ---- W = sum of the two parts; thread: key row `row`, tokens 32 wg .. + 31 ----
      if (!WQ) {
        // -> hi/lo [k][t] (B of the chain's X)
        float wa[32], wb[32];
        sm100::tmem_ld32(tmem + lane_off + TP_W + 32 * wg, wa);
        sm100::tmem_ld32(tmem + lane_off + TP_W + 64 + 32 * wg, wb);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          f2_unpack(f2_add(f2_pack(wa[i], wa[i + 1]), f2_pack(wb[i], wb[i + 1])), wa[i], wa[i + 1]);
        store32_hl(stg + H_WHI, stg + H_WLO, row, 4 * wg, wa);
      } else {
        // FP8 QDQ of W, one scale per row (token) over the keys: W^T goes
        // through the solve's scratch as fp32 [t][k] (stride LDW), each row
        // is reduced by four threads (keys 32 q .. + 31), then coded
        float *sW = reinterpret_cast<float *>(gbase + P_SA);
        float *sRed = reinterpret_cast<float *>(gbase + P_SA) + 64 * LDW;
        {
          float wa[32], wb[32];
          sm100::tmem_ld32(tmem + lane_off + TP_W + 32 * wg, wa);
          sm100::tmem_ld32(tmem + lane_off + TP_W + 64 + 32 * wg, wb);
#pragma unroll
          for (int i = 0; i < 32; ++i) sW[(32 * wg + i) * LDW + row] = wa[i] + wb[i];
        }
        __syncthreads();
        const int t = tid & 63, qk = tid >> 6;  // row t, keys 32 qk .. + 31
        float w[32];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          w[i] = sW[t * LDW + 32 * qk + i];
          m = fmaxf(m, fabsf(w[i]));
        }
        sRed[qk * 64 + t] = m;
        __syncthreads();
        m = fmaxf(fmaxf(sRed[t], sRed[64 + t]), fmaxf(sRed[128 + t], sRed[192 + t]));
        const ScaleRecip sr = make_scale(fp8_scale(m > 0.f ? m : 1.0f));
        uint32_t c[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) c[i] = m > 0.f ? fp8_codes(w[2 * i], w[2 * i + 1], sr) : 0u;
        const uint32_t half = stg + H_WHI + (uint32_t)(qk >> 1) * 8192u;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared_v4(sw128(half, t, 4 * (qk & 1) + cc), c[4 * cc], c[4 * cc + 1], c[4 * cc + 2],
                       c[4 * cc + 3]);
        if (qk == 0) reinterpret_cast<float *>(gbase + P_STG + b * kRxBytes + H_WSC)[t] = m > 0.f ? sr.s : 0.f;
      }
      sm100::fence_proxy_async();  // staging written by this CTA's threads -> bulk copy reads it
      sm100::tc_fence_before();
      __syncthreads();
      if (tid == 0 && !sm->abort)
        sm100::bulk_copy_to_cluster(rx_buf_remote[b] + H_WHI, stg + H_WHI,
                                    WQ ? kWqBytes : H_THI - H_WHI, rx_full_remote[b]);
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
    auto issue_qk = [&](int j) {
      const long long tb = t0 + (long long)j * kC;
      const int b = j & 1;
      uint8_t *dst = gbase + C_KQ + b * 32768;
      sm100::mbar_arrive_expect_tx(&sm->bar_qk[b], 4 * 8192);
      sm100::tma_load_3d(dst + 0, &tm_k, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 8192, &tm_q, &sm->bar_qk[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 16384, &tm_k, &sm->bar_qk[b], 64, h, (int)tb);
      sm100::tma_load_3d(dst + 24576, &tm_q, &sm->bar_qk[b], 64, h, (int)tb);
      sm->qk_pend[b] = 1 + ((j >> 1) & 1);
    };
    auto issue_v = [&](int j) {
      const long long tb = t0 + (long long)j * kC;
      const int b = j & 1;
      uint8_t *dst = gbase + C_V + b * 16384;
      sm100::mbar_arrive_expect_tx(&sm->bar_v[b], 2 * 8192);
      sm100::tma_load_3d(dst, &tm_v, &sm->bar_v[b], 0, h, (int)tb);
      sm100::tma_load_3d(dst + 8192, &tm_v, &sm->bar_v[b], 64, h, (int)tb);
      sm->v_pend[b] = 1 + ((j >> 1) & 1);
    };
    const uint32_t ID_X = sm100::idesc_f16_f32(128, 128, 0, 1);    // A tmem, B MN-major
    const uint32_t ID_X64 = sm100::idesc_f16_f32(128, 64, 0, 1);
    const uint32_t ID_O = sm100::idesc_f16_f32(128, 64, 0, 0);     // B K-major
    const uint32_t ID_U = sm100::idesc_f16_f32(128, 64, 1, 0);     // A MN-major smem
    // U^T(j) = V(j)^T (T diag(beta))^T(j), hi and lo parts into one accumulator
    auto issue_u = [&](int j) {
      const uint32_t vb = base + C_V + (uint32_t)(j & 1) * 16384u;
      const uint32_t rx = base + C_RX + (uint32_t)(j & 1) * kRxBytes;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          sm100::mma_f16_ss(tmem + TM_U, mndesc(vb + (uint32_t)ks * 2048u, 8192),
                            kdesc(rx + (pass ? H_TLO : H_THI) + 32u * ks), ID_U, pass + ks > 0);
      sm100::mma_commit(&sm->bar_u);
    };

    if (tid == 0) {
      sm100::prefetch_tmap(&tm_q);
      sm100::prefetch_tmap(&tm_k);
      sm100::prefetch_tmap(&tm_v);
    }
    if (tid == 224) {
      issue_qk(0);
      issue_v(0);
      if (n_chunks > 1) {
        issue_qk(1);
        issue_v(1);
      }
    }
    // ---- the initial state: thread (lane v, warpgroup wg) holds S0[v][k]
    //      for k in 64 wg .. + 63.  A zero state is exact (codes 0); a given
    //      one enters as fp16 hi (codes region) + lo (O2 region), scale 1 ----
    const bool exact0 = state_in == nullptr;
    float s0 = exact0 ? 0.0f : 1.0f;  // scale of the chunk-start state of this lane's tile
    uint32_t code[32];                // chunk-start codes (exact fp16 pairs), k = 64 wg + 2i
    {
      float x[64];
#pragma unroll
      for (int i = 0; i < 64; ++i)
        x[i] = exact0 ? 0.0f : __ldg(state_in + st_off + (long long)(64 * wg + i) * kD + row);
      uint32_t lo[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) split_h2(x[2 * i], x[2 * i + 1], code[i], lo[i]);
      tmem_st32u(tmem + lane_off + TM_S0C + 32 * wg, code);
      if (!exact0) tmem_st32u(tmem + lane_off + TM_O2 + 32 * wg, lo);
      const float gn0 = sm->gt[0].gn;
      float y[32];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] = gn0 * x[32 * p + i];
        sm100::tmem_st32(tmem + lane_off + TM_S + 64 * wg + 32 * p, y);
      }
    }
    // chunk 0's tiles: wait, convert (later chunks' during the previous chunk)
    {
      const bool ok = wait_local(&sm->bar_qk[0], 0, sm, err) & wait_local(&sm->bar_v[0], 0, sm, err);
      if (ok && tid == 0) sm->qk_pend[0] = sm->v_pend[0] = 0;
      convert_kq_gamma_half(gbase + C_KQ, chunk_len(0), tid, 0, sm->gt[0].gam);
      convert_kq_gamma_half(gbase + C_KQ, chunk_len(0), tid, 1, sm->gt[0].gam);
      convert_v_half(gbase + C_V, chunk_len(0), tid, 0);
      convert_v_half(gbase + C_V, chunk_len(0), tid, 1);
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    __syncthreads();
    GateRaw graw{};
    bool exact = exact0;
    bool u_done = false;  // (warp 0) the current chunk's U has been issued
    for (int it = 0; it < n_chunks; ++it) {  // left only at the checks after barriers
      const int n = chunk_len(it);
      const long long tb = t0 + (long long)it * kC;
      const bool last = it == n_chunks - 1;
      const int kb = it & 1;
      const uint32_t kq = base + C_KQ + (uint32_t)kb * 32768u;
      const uint32_t rx = base + C_RX + (uint32_t)kb * kRxBytes;
      const ChainGates *gt = &sm->gt[it % 3];

      // ---- (A) X = S0c [W hi | W lo]^T, (+ S0lo W hi^T before the first
      //      boundary of a given state); O part 1 = S0c (gamma Q)^T ----
      if (warp == 0) {
        bool got = true;
        if (!u_done) {  // this chunk's hand-off had not landed at the previous step (D)
          got = __all_sync(0xffffffffu,
                           wait_cluster(&sm->rx_full[kb], (uint32_t)((it >> 1) & 1), sm, err));
          if (got && lane == 0) sm->rx_pend[kb] = 0;
        }
        sm100::tc_fence_after();
        if (got && sm100::elect_one()) {
          if (!u_done) issue_u(it);
          if (!WQ) {
#pragma unroll 1
            for (int ks = 0; ks < 8; ++ks)
              sm100::mma_f16_ts(tmem + TM_X, tmem + TM_S0C + 8u * ks,
                                mndesc(rx + H_WHI + (uint32_t)ks * 2048u, 16384), ID_X, ks > 0);
            if (!exact) {
#pragma unroll 1
              for (int ks = 0; ks < 8; ++ks)
                sm100::mma_f16_ts(tmem + TM_X, tmem + TM_O2 + 8u * ks,
                                  mndesc(rx + H_WHI + (uint32_t)ks * 2048u, 16384), ID_X64, 1);
            }
          } else {
            // X = S0c Wc^T with the E4M3 codes of W (exact in fp16): one pass
#pragma unroll 1
            for (int ks = 0; ks < 8; ++ks)
              sm100::mma_f16_ts(tmem + TM_X, tmem + TM_S0C + 8u * ks,
                                kdesc(rx + H_WHI + (uint32_t)(ks >> 2) * 8192u + (uint32_t)(ks & 3) * 32u),
                                ID_O, ks > 0);
            if (!exact) {
#pragma unroll 1
              for (int ks = 0; ks < 8; ++ks)
                sm100::mma_f16_ts(tmem + TM_X, tmem + TM_O2 + 8u * ks,
                                  kdesc(rx + H_WHI + (uint32_t)(ks >> 2) * 8192u + (uint32_t)(ks & 3) * 32u),
                                  ID_O, 1);
            }
          }
          sm100::mma_commit(&sm->bar_x);
#pragma unroll 1
          for (int ks = 0; ks < 8; ++ks)
            sm100::mma_f16_ts(tmem + TM_O1, tmem + TM_S0C + 8u * ks,
                              kdesc(kq + 8192u + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u),
                              ID_O, ks > 0);
        }
        __syncwarp();
      }
      // ---- (B) while X runs: S = gamma_n S0 into the accumulator (from the
      //      codes), the next chunk's K / gamma Q / V conversion, the raw
      //      gates of the chunk after it ----
      if (it > 0) {
        const float c = gt->gn * s0;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          float y[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) dequant2(code[16 * p + i], c, y[2 * i], y[2 * i + 1]);
          sm100::tmem_st32(tmem + lane_off + TM_S + 64 * wg + 32 * p, y);
        }
      }
      if (!last) {
        const int nb = kb ^ 1, n1 = chunk_len(it + 1);
        const uint32_t ph = (uint32_t)(((it + 1) >> 1) & 1);
        const bool ok = wait_local(&sm->bar_qk[nb], ph, sm, err) & wait_local(&sm->bar_v[nb], ph, sm, err);
        if (ok && tid == 0) sm->qk_pend[nb] = sm->v_pend[nb] = 0;
        const float *gam1 = sm->gt[(it + 1) % 3].gam;
        convert_kq_gamma_half(gbase + C_KQ + nb * 32768, n1, tid, 0, gam1);
        convert_kq_gamma_half(gbase + C_KQ + nb * 32768, n1, tid, 1, gam1);
        convert_v_half(gbase + C_V + nb * 16384, n1, tid, 0);
        convert_v_half(gbase + C_V + nb * 16384, n1, tid, 1);
        sm100::fence_proxy_async();  // read by the tensor cores after the barrier below
      }
      if (warp == 7 && it + 2 < n_chunks)
        graw = load_gates_raw(g, beta, tb + 2 * kC, chunk_len(it + 2), H, h, lane);

      // ---- (C) Vn^T = U^T - s0 (X a + X b); Vn hi -> TMEM (A of O part 2);
      //      dec * Vn^T hi/lo -> TMEM (A of the S update).  Warpgroup wg:
      //      tokens 32 wg .. + 31 ----
      {
        wait_local(&sm->bar_x, (uint32_t)(it & 1), sm, err);
        wait_local(&sm->bar_u, (uint32_t)(it & 1), sm, err);
        sm100::tc_fence_after();
        float xa[32], xb[32], u[32];
        sm100::tmem_ld32(tmem + lane_off + TM_X + 32 * wg, xa);
        if (!WQ) {
          sm100::tmem_ld32(tmem + lane_off + TM_X + 64 + 32 * wg, xb);
        } else {
          // the row scales of W: X a[t] * s_t, X b = 0
          const float *wsc = reinterpret_cast<const float *>(gbase + C_RX + kb * kRxBytes + H_WSC) + 32 * wg;
#pragma unroll
          for (int t = 0; t < 32; t += 4) {
            const float4 s4 = *reinterpret_cast<const float4 *>(wsc + t);
            xa[t] *= s4.x; xa[t + 1] *= s4.y; xa[t + 2] *= s4.z; xa[t + 3] *= s4.w;
            xb[t] = xb[t + 1] = xb[t + 2] = xb[t + 3] = 0.0f;
          }
        }
        sm100::tmem_ld32(tmem + lane_off + TM_U + 32 * wg, u);
        const uint64_t ms = f2_pack(-s0, -s0);
        uint32_t vh[16], dh[16], dl[16];
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const float4 d4 = *reinterpret_cast<const float4 *>(gt->dec + 32 * wg + t);
          float vv[4];
          f2_unpack(f2_fma(ms, f2_add(f2_pack(xa[t], xa[t + 1]), f2_pack(xb[t], xb[t + 1])),
                           f2_pack(u[t], u[t + 1])), vv[0], vv[1]);
          f2_unpack(f2_fma(ms, f2_add(f2_pack(xa[t + 2], xa[t + 3]), f2_pack(xb[t + 2], xb[t + 3])),
                           f2_pack(u[t + 2], u[t + 3])), vv[2], vv[3]);
          vh[t >> 1] = pack_h2(vv[0], vv[1]);
          vh[(t >> 1) + 1] = pack_h2(vv[2], vv[3]);
          float dd[4];
          f2_unpack(f2_mul(f2_pack(vv[0], vv[1]), f2_pack(d4.x, d4.y)), dd[0], dd[1]);
          f2_unpack(f2_mul(f2_pack(vv[2], vv[3]), f2_pack(d4.z, d4.w)), dd[2], dd[3]);
          split_h2(dd[0], dd[1], dh[t >> 1], dl[t >> 1]);
          split_h2(dd[2], dd[3], dh[(t >> 1) + 1], dl[(t >> 1) + 1]);
        }
        sm100::tmem_st16(tmem + lane_off + TM_U + 32 * wg, vh);
        sm100::tmem_st16(tmem + lane_off + TM_X + 32 * wg, dh);
        sm100::tmem_st16(tmem + lane_off + TM_X + 32 * wg + 16, dl);
      }
      sm100::tc_fence_before();
      __syncthreads();
      if (sm->abort) break;

      // ---- (D) O part 2 += Vn^T Aqk^T; S += (dec Vn)^T K (hi, lo); then the
      //      next chunk's U ----
      if (warp == 0) {
        sm100::tc_fence_after();
        if (sm100::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            sm100::mma_f16_ts(tmem + TM_O2, tmem + TM_U + 32u * (ks >> 1) + 8u * (ks & 1),
                              kdesc(rx + H_AQK + 32u * ks), ID_O, ks > 0);
          sm100::mma_commit(&sm->bar_o2);
#pragma unroll
          for (int pass = 0; pass < 2; ++pass)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              sm100::mma_f16_ts(tmem + TM_S,
                                tmem + TM_X + 16u * pass + 32u * (ks >> 1) + 8u * (ks & 1),
                                mndesc(kq + (uint32_t)ks * 2048u, 16384), ID_X, 1);
          sm100::mma_commit(&sm->bar_m5);
        }
        __syncwarp();
        // the next chunk's U as soon as its hand-off has landed (tested, not
        // waited for: the S update above is on the critical path; otherwise
        // step (A) of the next chunk waits and issues it)
        u_done = false;
        if (!last) {
          const int nb = kb ^ 1;
          const bool ready = __shfl_sync(
              0xffffffffu,
              lane == 0 ? sm100::mbar_try_wait_cluster(&sm->rx_full[nb], (uint32_t)(((it + 1) >> 1) & 1)) : false,
              0);
          if (ready) {
            if (lane == 0) sm->rx_pend[nb] = 0;
            sm100::tc_fence_after();
            if (sm100::elect_one()) issue_u(it + 1);
            __syncwarp();
            u_done = true;
          }
        }
      }
      // ---- (E) while the S update runs: this chunk's outputs,
      //      o[t][v] = scale (s0 O1 + O2), straight to global ----
      {
        wait_local(&sm->bar_o2, (uint32_t)(it & 1), sm, err);
        sm100::tc_fence_after();
        if (tid == 0 && !sm->abort) {
          // the receive slot has been read (W by X, T diag(beta) by U, Aqk by
          // O part 2; this thread has seen those MMAs complete): arm it for
          // chunk it + 2, then hand it back to the producer
          if (it + 2 < n_chunks) {
            sm100::mbar_arrive_expect_tx(&sm->rx_full[kb], WQ ? kRxBytesWq : kRxBytes);
            sm->rx_pend[kb] = 1 + (((it + 2) >> 1) & 1);
          }
          sm100::mbar_arrive_cluster_relaxed(rx_free_remote[kb]);
        }
        float o1[32], o2[32];
        sm100::tmem_ld32(tmem + lane_off + TM_O1 + 32 * wg, o1);
        sm100::tmem_ld32(tmem + lane_off + TM_O2 + 32 * wg, o2);
        const int cnt = n - 32 * wg;
        unsigned short *dst =
            reinterpret_cast<unsigned short *>(o + ((tb + 32 * wg) * H + h) * kD + row);
        const long long ts = (long long)H * kD;
        const float ss = scale * s0;
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const __nv_bfloat162 p2 =
              __floats2bfloat162_rn(fmaf(ss, o1[t], scale * o2[t]), fmaf(ss, o1[t + 1], scale * o2[t + 1]));
          const uint32_t w = *reinterpret_cast<const uint32_t *>(&p2);
          if (t < cnt) dst[t * ts] = (unsigned short)(w & 0xffffu);
          if (t + 1 < cnt) dst[(t + 1) * ts] = (unsigned short)(w >> 16);
        }
      }
      if (warp == 7 && it + 2 < n_chunks)
        finish_chain_gates(&sm->gt[(it + 2) % 3], graw, chunk_len(it + 2), lane);
      // U of this chunk has read V: the buffer takes chunk it + 2
      if (tid == 224 && it + 2 < n_chunks && !sm->abort) issue_v(it + 2);

      // ---- (F) the QDQ ----
      wait_local(&sm->bar_m5, (uint32_t)(it & 1), sm, err);
      sm100::tc_fence_after();
      // the S update has read K: the buffer takes chunk it + 2
      if (tid == 224 && it + 2 < n_chunks && !sm->abort) issue_qk(it + 2);
      {
        float y[64];
        sm100::tmem_ld32(tmem + lane_off + TM_S + 64 * wg, *reinterpret_cast<float(*)[32]>(y));
        sm100::tmem_ld32(tmem + lane_off + TM_S + 64 * wg + 32, *reinterpret_cast<float(*)[32]>(y + 32));
        float mh = 0.f;
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          asm("max.f32 %0, %1, %2, %3;" : "=f"(mh) : "f"(mh), "f"(fabsf(y[i])), "f"(fabsf(y[i + 1])));
        }
        mh = group_max<32>(mh);
        // one FP8 tile = value columns 64 tile .. + 63 = warps (2 tile, 2 tile + 1)
        // of both warpgroups
        const int tile = (warp & 3) >> 1;
        if (lane == 0) sm->red[tile][(warp & 1) + 2 * wg] = mh;
        asm volatile("bar.sync %0, 128;" ::"r"(1 + tile) : "memory");
        mh = fmaxf(fmaxf(sm->red[tile][0], sm->red[tile][1]), fmaxf(sm->red[tile][2], sm->red[tile][3]));
        const ScaleRecip sr = make_scale(fp8_scale(mh > 0.f ? mh : 1.0f));
        if (mh == 0.0f) {
#pragma unroll
          for (int i = 0; i < 32; ++i) code[i] = 0u;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) code[i] = fp8_codes(y[2 * i], y[2 * i + 1], sr);
        }
        s0 = mh == 0.0f ? 0.0f : sr.s;
        if (last) {
          // state_out[k][v] = s * code; a warp writes 128 contiguous bytes per key
          float *dst = state_out + st_off + (long long)(64 * wg) * kD + row;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float y0, y1;
            dequant2(code[i], s0, y0, y1);
            dst[(2 * i) * kD] = y0;
            dst[(2 * i + 1) * kD] = y1;
          }
        } else {
          tmem_st32u(tmem + lane_off + TM_S0C + 32 * wg, code);
        }
      }
      exact = true;
      sm100::tc_fence_before();
      __syncthreads();
    }
    if (tid == 0 && sm->abort) {
      for (int bb = 0; bb < 2; ++bb) {
        if (sm->qk_pend[bb])
          (void)sm100::mbar_wait(&sm->bar_qk[bb], (uint32_t)(sm->qk_pend[bb] - 1), kWaitNs);
        if (sm->v_pend[bb])
          (void)sm100::mbar_wait(&sm->bar_v[bb], (uint32_t)(sm->v_pend[bb] - 1), kWaitNs);
        // and the producer's transfers into the receive slots, if armed
        if (sm->rx_pend[bb])
          (void)sm100::mbar_wait_cluster(&sm->rx_full[bb], (uint32_t)(sm->rx_pend[bb] - 1), kWaitNs);
      }
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

}  // namespace wy
}  // namespace gdn
