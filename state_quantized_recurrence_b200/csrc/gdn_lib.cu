// C ABI of the gated-delta-rule library (declared in include/gdn_qdq.h):
// argument validation on the host, kernel selection, and the per-device
// error word.  Nothing here computes the method; every arithmetic step runs
// in the kernels included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "gdn_qdq.h"
#include "gdn_common.cuh"
#include "gdn_backward.cuh"
#include "gdn_decode.cuh"
#include "gdn_prefill_simt.cuh"
#include "gdn_prefill_pair.cuh"
#include "gdn_prefill_wy.cuh"
#include "gdn_prefill_tc.cuh"
#include <stdlib.h>

namespace {

// Per-device error word (bits gdn::kErrBadSeqlens / kErrTimeout), set by
// kernels with atomicOr and read-and-cleared by gdn_last_error().
__device__ unsigned g_err_word;

constexpr int kMaxDevices = 64;
unsigned *g_err_ptr[kMaxDevices];  // device address of g_err_word per device

gdn_status err_word(unsigned **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  if (!g_err_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return GDN_ERR_CUDA;
    g_err_ptr[dev] = static_cast<unsigned *>(p);
  }
  *out = g_err_ptr[dev];
  return GDN_OK;
}

// Limit of the tensor-core kernels' bounded waits: 2 s, or the value of
// GDN_WAIT_LIMIT_NS (nanoseconds, read at every launch; 0 gives up at the
// first wait that is not already complete).  A shorter limit exists to
// exercise the kernels' timeout path: the kernel records GDN_ERR_TIMEOUT
// in the error word and exits cleanly.
uint64_t wait_limit_ns() {
  const char *e = getenv("GDN_WAIT_LIMIT_NS");
  if (!e || !*e) return 2000000000ull;
  char *end = nullptr;
  const unsigned long long v = strtoull(e, &end, 10);
  return (end && *end == 0) ? (uint64_t)v : 2000000000ull;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool qdq_params(gdn_qdq_mode m, int d_v, int *kind, int *group) {
  switch (m) {
    case GDN_QDQ_NONE: *kind = gdn::kQdqNone; *group = 32; return true;
    case GDN_QDQ_FP8_E4M3_TILE64: *kind = gdn::kQdqFp8Tile; *group = 64; return d_v % 64 == 0;
    case GDN_QDQ_INT8_GROUP16: *kind = gdn::kQdqInt8; *group = 16; return true;
    case GDN_QDQ_INT8_GROUP32: *kind = gdn::kQdqInt8; *group = 32; return true;
    case GDN_QDQ_INT8_GROUP64: *kind = gdn::kQdqInt8; *group = 64; return true;
  }
  return false;
}

// Shared checks; returns GDN_OK or the status to report.
// `tokens` is the number of token rows the call reads (0: the token
// pointers are not used and may be NULL).
gdn_status check_common(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const void *o, int n_seq, int H, int d_k,
                        int d_v, gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                        long long tokens) {
  if (n_seq < 0 || H <= 0 || d_k <= 0 || d_v <= 0) return GDN_ERR_INVALID_ARG;
  if (dt != GDN_DTYPE_BF16 && dt != GDN_DTYPE_F32) return GDN_ERR_UNSUPPORTED;
  if (gk != GDN_GATE_SCALAR && gk != GDN_GATE_PER_KEY) return GDN_ERR_UNSUPPORTED;
  if ((unsigned)qdq > (unsigned)GDN_QDQ_INT8_GROUP64) return GDN_ERR_UNSUPPORTED;
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return GDN_ERR_UNSUPPORTED;
  if (n_seq == 0 || tokens == 0) return GDN_OK;
  if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(g, 4) || !aligned(beta, 4))
    return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

// State storage of a decode call: fp32 values, or packed codes + scales.
struct StateArgs {
  float *vals;
  uint8_t *codes;
  float *scales;
  bool packed;
};

template <typename Tin, int DK, int DV, bool PK, int QK, int GR>
void decode_launch_one(dim3 grid, cudaStream_t st, const Tin *q, const Tin *k, const Tin *v,
                       const float *g, const float *beta, const StateArgs &sa, Tin *o,
                       float scale) {
  if (sa.packed) {
    if constexpr (QK != gdn::kQdqNone)
      gdn::decode_kernel<Tin, DK, DV, PK, QK, GR, true><<<grid, 256, 0, st>>>(
          q, k, v, g, beta, nullptr, sa.codes, sa.scales, o, scale);
  } else {
    gdn::decode_kernel<Tin, DK, DV, PK, QK, GR, false><<<grid, 256, 0, st>>>(
        q, k, v, g, beta, sa.vals, nullptr, nullptr, o, scale);
  }
}

template <typename Tin, int DK, int DV, bool PK>
void decode_dispatch(dim3 grid, cudaStream_t st, const Tin *q, const Tin *k, const Tin *v,
                     const float *g, const float *beta, const StateArgs &sa, Tin *o, float scale,
                     int kind, int group) {
#define GDN_DEC(QK, GR) decode_launch_one<Tin, DK, DV, PK, QK, GR>(grid, st, q, k, v, g, beta, sa, o, scale)
  if (kind == gdn::kQdqNone) GDN_DEC(gdn::kQdqNone, 32);
  else if (kind == gdn::kQdqFp8Tile) GDN_DEC(gdn::kQdqFp8Tile, 32);
  else if (group == 16) GDN_DEC(gdn::kQdqInt8, 16);
  else if (group == 64) GDN_DEC(gdn::kQdqInt8, 64);
  else GDN_DEC(gdn::kQdqInt8, 32);
#undef GDN_DEC
}

template <typename Tin, int DK, int DV>
void decode_dispatch_gate(bool per_key, dim3 grid, cudaStream_t st, const Tin *q, const Tin *k,
                          const Tin *v, const float *g, const float *beta, const StateArgs &sa,
                          Tin *o, float scale, int kind, int group) {
  if (per_key) decode_dispatch<Tin, DK, DV, true>(grid, st, q, k, v, g, beta, sa, o, scale, kind, group);
  else decode_dispatch<Tin, DK, DV, false>(grid, st, q, k, v, g, beta, sa, o, scale, kind, group);
}

template <typename Tin>
gdn_status launch_decode(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const StateArgs &state, int n_seq, int H, int d_k,
                         int d_v, bool per_key, int kind, int group, void *o,
                         cudaStream_t st) {
  const long long blocks = (long long)n_seq * H * (d_v / 64);
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  const float scale = (float)(1.0 / sqrt((double)d_k));
  const Tin *qq = static_cast<const Tin *>(q), *kk = static_cast<const Tin *>(k),
            *vv = static_cast<const Tin *>(v);
  Tin *oo = static_cast<Tin *>(o);
  dim3 grid((unsigned)blocks);
#define GDN_DECG(DK, DV) \
  decode_dispatch_gate<Tin, DK, DV>(per_key, grid, st, qq, kk, vv, g, beta, state, oo, scale, kind, group)
  if (d_k == 128) { if (d_v == 128) GDN_DECG(128, 128); else GDN_DECG(128, 64); }
  else            { if (d_v == 128) GDN_DECG(64, 128);  else GDN_DECG(64, 64); }
#undef GDN_DECG
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin, int DK, bool PK, bool NEU>
gdn_status launch_simt_neu(const Tin *q, const Tin *k, const Tin *v, const float *g,
                           const float *beta, const float *state_in, const int32_t *cu,
                           int T, int H, int d_v, float scale, int kind, int group, Tin *o,
                           float *state_out, unsigned *err, unsigned blocks, int neu_m,
                           cudaStream_t st) {
  using L = gdn::simt::Smem<DK, NEU>;
  auto kern = gdn::simt::prefill_simt_kernel<Tin, DK, PK, NEU>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  kern<<<blocks, gdn::simt::kThreads, L::kBytes, st>>>(q, k, v, g, beta, state_in, cu, T, H, d_v,
                                                       scale, kind, group, o, state_out, err,
                                                       neu_m);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// neu_m = 0: exact solve; neu_m >= 1: Neumann degree 2^neu_m - 1.
template <typename Tin, int DK, bool PK>
gdn_status launch_simt_one(const Tin *q, const Tin *k, const Tin *v, const float *g,
                           const float *beta, const float *state_in, const int32_t *cu,
                           int T, int H, int d_v, float scale, int kind, int group, Tin *o,
                           float *state_out, unsigned *err, unsigned blocks, int neu_m,
                           cudaStream_t st) {
  if (neu_m > 0)
    return launch_simt_neu<Tin, DK, PK, true>(q, k, v, g, beta, state_in, cu, T, H, d_v, scale,
                                              kind, group, o, state_out, err, blocks, neu_m, st);
  return launch_simt_neu<Tin, DK, PK, false>(q, k, v, g, beta, state_in, cu, T, H, d_v, scale,
                                             kind, group, o, state_out, err, blocks, 0, st);
}

template <int DK, int DV, bool TO>
void convert_dispatch(dim3 grid, cudaStream_t st, float *vals, uint8_t *codes, float *scales,
                      int kind, int group) {
#define GDN_CV(QK, GR) gdn::state_convert_kernel<DK, DV, QK, GR, TO><<<grid, 256, 0, st>>>(vals, codes, scales)
  if (kind == gdn::kQdqFp8Tile) GDN_CV(gdn::kQdqFp8Tile, 32);
  else if (group == 16) GDN_CV(gdn::kQdqInt8, 16);
  else if (group == 64) GDN_CV(gdn::kQdqInt8, 64);
  else GDN_CV(gdn::kQdqInt8, 32);
#undef GDN_CV
}

gdn_status launch_convert(float *vals, uint8_t *codes, float *scales, int n, int H, int d_k,
                          int d_v, int kind, int group, bool to_packed, cudaStream_t st) {
  const long long blocks = (long long)n * H * (d_v / 64);
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  dim3 grid((unsigned)blocks);
#define GDN_CVD(DK, DV) \
  (to_packed ? convert_dispatch<DK, DV, true>(grid, st, vals, codes, scales, kind, group) \
             : convert_dispatch<DK, DV, false>(grid, st, vals, codes, scales, kind, group))
  if (d_k == 128) { if (d_v == 128) GDN_CVD(128, 128); else GDN_CVD(128, 64); }
  else            { if (d_v == 128) GDN_CVD(64, 128);  else GDN_CVD(64, 64); }
#undef GDN_CVD
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin>
gdn_status launch_prefill_simt(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *state_in, const int32_t *cu,
                               int n_seq, int T, int H, int d_k, int d_v, bool per_key,
                               int kind, int group, void *o, float *state_out, unsigned *err,
                               int neu_m, cudaStream_t st) {
  const long long blocks = (long long)n_seq * H * (d_v / 64);
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  const float scale = (float)(1.0 / sqrt((double)d_k));
  const Tin *qq = static_cast<const Tin *>(q), *kk = static_cast<const Tin *>(k),
            *vv = static_cast<const Tin *>(v);
  Tin *oo = static_cast<Tin *>(o);
  const unsigned nb = (unsigned)blocks;
#define GDN_PF(DK, PK) \
  launch_simt_one<Tin, DK, PK>(qq, kk, vv, g, beta, state_in, cu, T, H, d_v, scale, kind, group, oo, state_out, err, nb, neu_m, st)
  if (d_k == 128) return per_key ? GDN_PF(128, true) : GDN_PF(128, false);
  return per_key ? GDN_PF(64, true) : GDN_PF(64, false);
#undef GDN_PF
}

// ---- tensor-core prefill: TMA descriptors and launch -----------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

gdn_status encode_fn() {
  if (g_encode_tiled) return GDN_OK;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return GDN_ERR_CUDA;
  g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return GDN_OK;
}

// [rows, H, 128] bf16 viewed as a 3-D tensor; box = 64 columns x 1 head x 64
// token rows (128-byte rows, optionally 128B-swizzled into the layout the
// tensor cores read).  Rows past the end of the tensor read as zero.
gdn_status make_token_map(CUtensorMap *m, const void *ptr, int H, long long rows, bool swizzle) {
  memset(m, 0, sizeof(*m));
  if (rows <= 0) return GDN_OK;  // no chunk is processed, the map is never used
  cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr),
                              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GDN_OK : GDN_ERR_CUDA;
}

template <int QK, int GR>
gdn_status launch_tc_one(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                         const CUtensorMap &mo, const float *g, const float *beta,
                         const float *state_in,
                         const int32_t *cu, int T, int H, float scale, __nv_bfloat16 *o,
                         float *state_out, unsigned *err, unsigned blocks, cudaStream_t st) {
  auto kern = gdn::tc::prefill_tc_kernel<QK, GR>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gdn::tc::kSmemBytes) != cudaSuccess)
    return GDN_ERR_CUDA;
  kern<<<blocks, gdn::tc::kThreads, gdn::tc::kSmemBytes, st>>>(mq, mk, mv, mo, g, beta, state_in,
                                                               cu, T, H, scale, o, state_out, err,
                                                               wait_limit_ns());
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// The same chunk algebra split over a CTA pair (one thread-block cluster of
// two per (sequence, head)): the producer CTA computes A, Aqk and T a chunk
// ahead, the chain CTA carries the state.
template <int QK, int GR>
gdn_status launch_pair_one(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                           const CUtensorMap &mo, const float *g, const float *beta,
                           const float *state_in,
                           const int32_t *cu, int T, int H, float scale, __nv_bfloat16 *o,
                           float *state_out, unsigned *err, unsigned units, cudaStream_t st) {
  auto kern = gdn::pair::prefill_pair_kernel<QK, GR>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gdn::pair::kSmemBytes) != cudaSuccess)
    return GDN_ERR_CUDA;
  kern<<<2 * units, gdn::pair::kThreads, gdn::pair::kSmemBytes, st>>>(
      mq, mk, mv, mo, g, beta, state_in, cu, T, H, scale, o, state_out, err, wait_limit_ns());
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// The WY-form pair (FP8 tiles): the producer CTA also forms W and hands it
// over; the chain CTA keeps the state transposed in TMEM.
template <bool WQ>
gdn_status launch_wy_one(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv_sw,
                         const float *g, const float *beta, const float *state_in,
                         const int32_t *cu, int T, int H, float scale, __nv_bfloat16 *o,
                         float *state_out, unsigned *err, unsigned units, cudaStream_t st) {
  auto kern = gdn::wy::prefill_wy_kernel<WQ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gdn::wy::kSmemBytes) != cudaSuccess)
    return GDN_ERR_CUDA;
  kern<<<2 * units, gdn::wy::kThreads, gdn::wy::kSmemBytes, st>>>(
      mq, mk, mv_sw, g, beta, state_in, cu, T, H, scale, o, state_out, err, wait_limit_ns());
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// How many CTA pairs of the tensor-core prefill can be resident at once on
// the current device (0 if the pair kernel cannot run), cached per device.
int g_pair_slots[kMaxDevices];
bool g_pair_slots_known[kMaxDevices];

int pair_slots() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (!g_pair_slots_known[dev]) {
    auto kern = gdn::pair::prefill_pair_kernel<gdn::kQdqFp8Tile, 32>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)gdn::pair::kSmemBytes) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(gdn::pair::kThreads, 1, 1);
      cfg.dynamicSmemBytes = gdn::pair::kSmemBytes;
      if (cudaOccupancyMaxActiveClusters(&n, (void *)kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a refused query leaves no sticky error behind
    g_pair_slots[dev] = n;
    g_pair_slots_known[dev] = true;
  }
  return g_pair_slots[dev];
}

// Schedule of the bf16 d = 128 GDN prefill.  A pair finishes a (sequence,
// head) faster than one CTA but takes two SMs, so pairs pay when every unit
// gets its pair at once (one wave); with more units than pair slots the
// single-CTA kernel keeps more units in flight.  GDN_PREFILL_CTA_PAIR=1 or 0
// in the environment forces the pair or the single-CTA kernel.
bool use_pair(long long units) {
  const char *e = getenv("GDN_PREFILL_CTA_PAIR");
  if (e && e[0] == '0' && e[1] == 0) return false;
  const int slots = pair_slots();
  if (slots <= 0) return false;
  if (e && e[0] == '1' && e[1] == 0) return true;
  return units <= slots;
}

// Among the pair kernels, FP8-tile codecs take the WY-form pair when
// GDN_PREFILL_WY=1 in the environment (read at every call); otherwise the
// delta-form pair.
bool use_wy(int kind) {
  if (kind != gdn::kQdqFp8Tile) return false;
  const char *e = getenv("GDN_PREFILL_WY");
  return e && e[0] == '1' && e[1] == 0;
}

// bf16 GDN at d_k = d_v = 128 runs on the tensor cores; fp32 inputs (whose
// 1e-5 tolerance the fp16 operand splits cannot promise), per-key (KDA)
// gates and d = 64 run on the CUDA-core kernel.
bool tc_path(gdn_dtype dt, gdn_gate_kind gk, int d_k, int d_v) {
  return dt == GDN_DTYPE_BF16 && gk == GDN_GATE_SCALAR && d_k == 128 && d_v == 128;
}

gdn_status launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *state_in, const int32_t *cu,
                             int n_seq, int T, int H, int kind, int group, void *o,
                             float *state_out, unsigned *err, cudaStream_t st, bool w_qdq) {
  const long long blocks = (long long)n_seq * H;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  const long long rows = cu ? (long long)T : (long long)n_seq * T;
  if (rows > 0x7fffffffLL - 64) return GDN_ERR_UNSUPPORTED;
  gdn_status s = encode_fn();
  if (s != GDN_OK) return s;
  CUtensorMap mq, mk, mv;
  if ((s = make_token_map(&mq, q, H, rows, true)) != GDN_OK) return s;
  if ((s = make_token_map(&mk, k, H, rows, true)) != GDN_OK) return s;
  if ((s = make_token_map(&mv, v, H, rows, false)) != GDN_OK) return s;
  const float scale = (float)(1.0 / sqrt(128.0));
  __nv_bfloat16 *oo = static_cast<__nv_bfloat16 *>(o);
  const unsigned nb = (unsigned)blocks;
  CUtensorMap mo;  // outputs [rows, H, 128] bf16, stored by whole 64-token chunks
  if ((s = make_token_map(&mo, o, H, rows, true)) != GDN_OK) return s;
  if (w_qdq || use_pair(blocks)) {
    if (blocks > 0x3fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (w_qdq || use_wy(kind)) {
      CUtensorMap mvs;  // V tiles 128B-swizzled: the A operand of U^T = V^T (T diag(beta))^T
      if ((s = make_token_map(&mvs, v, H, rows, true)) != GDN_OK) return s;
      if (w_qdq)
        return launch_wy_one<true>(mq, mk, mvs, g, beta, state_in, cu, T, H, scale, oo, state_out,
                                   err, nb, st);
      return launch_wy_one<false>(mq, mk, mvs, g, beta, state_in, cu, T, H, scale, oo, state_out,
                                  err, nb, st);
    }
#define GDN_TP(QK, GR) \
  launch_pair_one<QK, GR>(mq, mk, mv, mo, g, beta, state_in, cu, T, H, scale, oo, state_out, err, nb, st)
    if (kind == gdn::kQdqNone) return GDN_TP(gdn::kQdqNone, 32);
    if (kind == gdn::kQdqFp8Tile) return GDN_TP(gdn::kQdqFp8Tile, 32);
    if (group == 16) return GDN_TP(gdn::kQdqInt8, 16);
    if (group == 64) return GDN_TP(gdn::kQdqInt8, 64);
    return GDN_TP(gdn::kQdqInt8, 32);
#undef GDN_TP
  }
#define GDN_TC(QK, GR) \
  launch_tc_one<QK, GR>(mq, mk, mv, mo, g, beta, state_in, cu, T, H, scale, oo, state_out, err, nb, st)
  if (kind == gdn::kQdqNone) return GDN_TC(gdn::kQdqNone, 32);
  if (kind == gdn::kQdqFp8Tile) return GDN_TC(gdn::kQdqFp8Tile, 32);
  if (group == 16) return GDN_TC(gdn::kQdqInt8, 16);
  if (group == 64) return GDN_TC(gdn::kQdqInt8, 64);
  return GDN_TC(gdn::kQdqInt8, 32);
#undef GDN_TC
}

// ---- backward (CUDA cores) ------------------------------------------------
// Workspace: every chunk's starting state per (slot, head, value tile), plus
// one chunk of per-token states per CTA.  Packed sequences take chunk slots
// s + cu[s] / 64 onwards, at most n_seq + T / 64 in all.
long long backward_ws_floats(int n_seq, long long T, int H, int d_k, int d_v, bool packed,
                             long long *chunk_floats) {
  const long long nvt = d_v / 64, tile = (long long)d_k * 64;
  const long long slots = packed ? n_seq + T / 64 : (long long)n_seq * ((T + 63) / 64);
  const long long ctas = (long long)n_seq * H * nvt;
  *chunk_floats = slots * H * nvt * tile;
  return *chunk_floats + ctas * 64 * tile;
}

template <typename Tin, int DK, bool PK, int QK, int GR>
gdn_status launch_bwd_one(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *state_in, const int32_t *cu, int T,
                          int H, int d_v, const void *d_o, const float *dstate_out, float *ws,
                          long long chunk_floats, float *dq, float *dk, float *dv, float *dg,
                          float *dbeta, float *dstate_in, unsigned *err, unsigned blocks,
                          cudaStream_t st) {
  const float scale = (float)(1.0 / sqrt((double)DK));
  gdn::bwd::prefill_backward_kernel<Tin, DK, PK, QK, GR><<<blocks, gdn::bwd::kThreads, 0, st>>>(
      static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v), g,
      beta, state_in, cu, T, H, d_v, scale, static_cast<const Tin *>(d_o), dstate_out, ws,
      ws + chunk_floats, dq, dk, dv, dg, dbeta, dstate_in, err);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin, int DK, bool PK>
gdn_status launch_bwd_qdq(int kind, int group, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *state_in,
                          const int32_t *cu, int T, int H, int d_v, const void *d_o,
                          const float *dstate_out, float *ws, long long chunk_floats, float *dq,
                          float *dk, float *dv, float *dg, float *dbeta, float *dstate_in,
                          unsigned *err, unsigned blocks, cudaStream_t st) {
#define GDN_BW(QK, GR)                                                                            \
  launch_bwd_one<Tin, DK, PK, QK, GR>(q, k, v, g, beta, state_in, cu, T, H, d_v, d_o, dstate_out, \
                                      ws, chunk_floats, dq, dk, dv, dg, dbeta, dstate_in, err,     \
                                      blocks, st)
  if (kind == gdn::kQdqNone) return GDN_BW(gdn::kQdqNone, 32);
  if (kind == gdn::kQdqFp8Tile) return GDN_BW(gdn::kQdqFp8Tile, 32);
  if (group == 16) return GDN_BW(gdn::kQdqInt8, 16);
  if (group == 64) return GDN_BW(gdn::kQdqInt8, 64);
  return GDN_BW(gdn::kQdqInt8, 32);
#undef GDN_BW
}

// Validation and kernel choice shared by gdn_prefill and gdn_prefill_neumann
// (neu_m = 0: exact solve; >= 1: Neumann degree 2^neu_m - 1).
gdn_status prefill_impl(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *state_in, const int32_t *cu_seqlens,
                        int n_seq, int T, int H, int d_k, int d_v, gdn_dtype dt,
                        gdn_gate_kind gk, gdn_qdq_mode qdq, int neu_m, void *o,
                        float *state_out, void *cuda_stream,
                        gdn_w_qdq_mode w_qdq = GDN_W_QDQ_NONE) {
  if (T < 0) return GDN_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)n_seq * T;
  gdn_status s = check_common(q, k, v, g, beta, o, n_seq, H, d_k, d_v, dt, gk, qdq, rows);
  if (s != GDN_OK) return s;
  int kind = 0, group = 32;
  if (!qdq_params(qdq, d_v, &kind, &group)) return GDN_ERR_UNSUPPORTED;
  if (w_qdq != GDN_W_QDQ_NONE && w_qdq != GDN_W_QDQ_FP8_E4M3_ROW) return GDN_ERR_UNSUPPORTED;
  // the W codec is built on the WY-form pair: bf16 GDN at d = 128 with FP8 state tiles
  if (w_qdq != GDN_W_QDQ_NONE &&
      (neu_m != 0 || !tc_path(dt, gk, d_k, d_v) || kind != gdn::kQdqFp8Tile))
    return GDN_ERR_UNSUPPORTED;
  if (n_seq == 0) return GDN_OK;
  if (!state_out || !aligned(state_out, 16)) return GDN_ERR_INVALID_ARG;
  if (state_in && !aligned(state_in, 16)) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
  // Total token rows must index within 64-bit element offsets comfortably.
  if (rows * H * 128 > (1LL << 46)) return GDN_ERR_UNSUPPORTED;
  unsigned *err = nullptr;
  if ((s = err_word(&err)) != GDN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bool pk = gk == GDN_GATE_PER_KEY;
  // Kernel choice by specialisation (tc_path); the Neumann solve runs on the
  // CUDA-core kernel for every dtype.  Both compute the same chunked algebra.
  if (neu_m == 0 && tc_path(dt, gk, d_k, d_v))
    return launch_prefill_tc(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, kind, group, o,
                             state_out, err, st, w_qdq != GDN_W_QDQ_NONE);
  if (dt == GDN_DTYPE_BF16)
    return launch_prefill_simt<__nv_bfloat16>(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T,
                                              H, d_k, d_v, pk, kind, group, o, state_out, err,
                                              neu_m, st);
  return launch_prefill_simt<float>(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, d_k,
                                    d_v, pk, kind, group, o, state_out, err, neu_m, st);
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
  }
  return "GDN_ERR_UNKNOWN";
}

int gdn_version(void) { return 100; }

gdn_status gdn_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state_inout, int n_seq, int H, int d_k,
                      int d_v, gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq, void *o,
                      void *cuda_stream) {
  gdn_status s = check_common(q, k, v, g, beta, o, n_seq, H, d_k, d_v, dt, gk, qdq, n_seq);
  if (s != GDN_OK) return s;
  int kind = 0, group = 32;
  if (!qdq_params(qdq, d_v, &kind, &group)) return GDN_ERR_UNSUPPORTED;
  if (n_seq == 0) return GDN_OK;
  if (!state_inout || !aligned(state_inout, 16)) return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bool pk = gk == GDN_GATE_PER_KEY;
  const StateArgs sa{state_inout, nullptr, nullptr, false};
  if (dt == GDN_DTYPE_BF16)
    return launch_decode<__nv_bfloat16>(q, k, v, g, beta, sa, n_seq, H, d_k, d_v, pk, kind,
                                        group, o, st);
  return launch_decode<float>(q, k, v, g, beta, sa, n_seq, H, d_k, d_v, pk, kind, group, o, st);
}

gdn_status gdn_decode_packed(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, void *codes, float *scales, int n_seq, int H,
                             int d_k, int d_v, gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                             void *o, void *cuda_stream) {
  gdn_status s = check_common(q, k, v, g, beta, o, n_seq, H, d_k, d_v, dt, gk, qdq, n_seq);
  if (s != GDN_OK) return s;
  int kind = 0, group = 32;
  if (!qdq_params(qdq, d_v, &kind, &group) || kind == gdn::kQdqNone) return GDN_ERR_UNSUPPORTED;
  if (n_seq == 0) return GDN_OK;
  if (!codes || !scales || !aligned(codes, 4) || !aligned(scales, 4)) return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bool pk = gk == GDN_GATE_PER_KEY;
  const StateArgs sa{nullptr, static_cast<uint8_t *>(codes), scales, true};
  if (dt == GDN_DTYPE_BF16)
    return launch_decode<__nv_bfloat16>(q, k, v, g, beta, sa, n_seq, H, d_k, d_v, pk, kind,
                                        group, o, st);
  return launch_decode<float>(q, k, v, g, beta, sa, n_seq, H, d_k, d_v, pk, kind, group, o, st);
}

static gdn_status state_convert(float *state, void *codes, float *scales, int n, int H, int d_k,
                                int d_v, gdn_qdq_mode qdq, bool to_packed, void *cuda_stream) {
  if (n < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return GDN_ERR_UNSUPPORTED;
  if ((unsigned)qdq > (unsigned)GDN_QDQ_INT8_GROUP64) return GDN_ERR_UNSUPPORTED;
  int kind = 0, group = 32;
  if (!qdq_params(qdq, d_v, &kind, &group) || kind == gdn::kQdqNone) return GDN_ERR_UNSUPPORTED;
  if (n == 0) return GDN_OK;
  if (!state || !codes || !scales || !aligned(state, 16) || !aligned(codes, 4) ||
      !aligned(scales, 4))
    return GDN_ERR_INVALID_ARG;
  return launch_convert(state, static_cast<uint8_t *>(codes), scales, n, H, d_k, d_v, kind, group,
                        to_packed, static_cast<cudaStream_t>(cuda_stream));
}

gdn_status gdn_state_pack(const float *state, void *codes, float *scales, int n, int H, int d_k,
                          int d_v, gdn_qdq_mode qdq, void *cuda_stream) {
  return state_convert(const_cast<float *>(state), codes, scales, n, H, d_k, d_v, qdq, true,
                       cuda_stream);
}

gdn_status gdn_state_unpack(const void *codes, const float *scales, float *state, int n, int H,
                            int d_k, int d_v, gdn_qdq_mode qdq, void *cuda_stream) {
  return state_convert(state, const_cast<void *>(codes), const_cast<float *>(scales), n, H, d_k,
                       d_v, qdq, false, cuda_stream);
}

gdn_status gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *state_in, const int32_t *cu_seqlens,
                       int n_seq, int T, int H, int d_k, int d_v, gdn_dtype dt,
                       gdn_gate_kind gk, gdn_qdq_mode qdq, void *o, float *state_out,
                       void *cuda_stream) {
  return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, d_k, d_v, dt, gk, qdq,
                      0, o, state_out, cuda_stream);
}

gdn_status gdn_prefill_w_qdq(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *state_in, const int32_t *cu_seqlens,
                             int n_seq, int T, int H, int d_k, int d_v, gdn_dtype dt,
                             gdn_gate_kind gk, gdn_qdq_mode qdq, gdn_w_qdq_mode w_qdq, void *o,
                             float *state_out, void *cuda_stream) {
  return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, d_k, d_v, dt, gk, qdq,
                      0, o, state_out, cuda_stream, w_qdq);
}

gdn_status gdn_prefill_neumann(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *state_in,
                               const int32_t *cu_seqlens, int n_seq, int T, int H, int d_k,
                               int d_v, gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                               int degree, void *o, float *state_out, void *cuda_stream) {
  int m = 0;
  while (m < 6 && degree != (1 << (m + 1)) - 1) ++m;
  if (m == 6) return GDN_ERR_INVALID_ARG;  // degree not in {1, 3, 7, 15, 31, 63}
  return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, d_k, d_v, dt, gk, qdq,
                      m + 1, o, state_out, cuda_stream);
}

size_t gdn_prefill_backward_workspace_bytes(int n_seq, int T, int H, int d_k, int d_v,
                                            int packed) {
  if (n_seq < 0 || T < 0 || H <= 0) return 0;
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return 0;
  long long chunk_floats = 0;
  return (size_t)backward_ws_floats(n_seq, T, H, d_k, d_v, packed != 0, &chunk_floats) *
         sizeof(float);
}

gdn_status gdn_prefill_backward(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *state_in,
                                const int32_t *cu_seqlens, int n_seq, int T, int H, int d_k,
                                int d_v, gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                                const void *d_o, const float *dstate_out, void *workspace,
                                size_t workspace_bytes, float *dq, float *dk, float *dv,
                                float *dg, float *dbeta, float *dstate_in, void *cuda_stream) {
  if (T < 0) return GDN_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)n_seq * T;
  gdn_status s = check_common(q, k, v, g, beta, d_o, n_seq, H, d_k, d_v, dt, gk, qdq, rows);
  if (s != GDN_OK) return s;
  int kind = 0, group = 32;
  if (!qdq_params(qdq, d_v, &kind, &group)) return GDN_ERR_UNSUPPORTED;
  if (n_seq == 0) return GDN_OK;
  if (!dstate_in || !aligned(dstate_in, 16)) return GDN_ERR_INVALID_ARG;
  if (state_in && !aligned(state_in, 16)) return GDN_ERR_INVALID_ARG;
  if (dstate_out && !aligned(dstate_out, 16)) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
  if (rows > 0 && (!dq || !dk || !dv || !dg || !dbeta)) return GDN_ERR_INVALID_ARG;
  if (!aligned(dq, 4) || !aligned(dk, 4) || !aligned(dv, 16) || !aligned(dg, 4) ||
      !aligned(dbeta, 4))
    return GDN_ERR_INVALID_ARG;
  if (rows * H * 128 > (1LL << 46)) return GDN_ERR_UNSUPPORTED;
  long long chunk_floats = 0;
  const long long need = backward_ws_floats(n_seq, T, H, d_k, d_v, cu_seqlens != nullptr,
                                            &chunk_floats);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < (size_t)need * sizeof(float))
    return GDN_ERR_INVALID_ARG;
  const long long blocks = (long long)n_seq * H * (d_v / 64);
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  unsigned *err = nullptr;
  if ((s = err_word(&err)) != GDN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bool pk = gk == GDN_GATE_PER_KEY;
  // sums over value tiles are accumulated with atomic adds
  if (rows > 0) {
    const size_t kb = (size_t)rows * H * d_k * sizeof(float);
    if (cudaMemsetAsync(dq, 0, kb, st) != cudaSuccess ||
        cudaMemsetAsync(dk, 0, kb, st) != cudaSuccess ||
        cudaMemsetAsync(dg, 0, pk ? kb : (size_t)rows * H * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(dbeta, 0, (size_t)rows * H * sizeof(float), st) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  float *ws = static_cast<float *>(workspace);
  const unsigned nb = (unsigned)blocks;
#define GDN_BQ(TIN, DK, PK)                                                                       \
  launch_bwd_qdq<TIN, DK, PK>(kind, group, q, k, v, g, beta, state_in, cu_seqlens, T, H, d_v, d_o, \
                              dstate_out, ws, chunk_floats, dq, dk, dv, dg, dbeta, dstate_in, err, \
                              nb, st)
  if (dt == GDN_DTYPE_BF16) {
    if (d_k == 128) return pk ? GDN_BQ(__nv_bfloat16, 128, true) : GDN_BQ(__nv_bfloat16, 128, false);
    return pk ? GDN_BQ(__nv_bfloat16, 64, true) : GDN_BQ(__nv_bfloat16, 64, false);
  }
  if (d_k == 128) return pk ? GDN_BQ(float, 128, true) : GDN_BQ(float, 128, false);
  return pk ? GDN_BQ(float, 64, true) : GDN_BQ(float, 64, false);
#undef GDN_BQ
}

}  // extern "C"

namespace {
// Scratch of gdn_prefill_backward_static: the library's own device memory,
// reserved with the module on each device that loads it (no per-call
// allocation).  Every word is written before it is read, so nothing in it
// needs to start at zero.  Calls that overlap on one device (two streams or
// host threads) share it and race.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];
void *g_bwd_scratch_ptr[kMaxDevices];  // its address per device, looked up once
}  // namespace

extern "C" {

// For callers that must not allocate device memory while they run (a step
// whose memory budget is fixed after start-up, where an allocation could
// fail or stall on the caching allocator): the workspace comes from the
// static array above instead of the caller.
gdn_status gdn_prefill_backward_static(const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, const float *state_in,
                                       const int32_t *cu_seqlens, int n_seq, int T, int H,
                                       int d_k, int d_v, gdn_dtype dt, gdn_gate_kind gk,
                                       gdn_qdq_mode qdq, const void *d_o,
                                       const float *dstate_out, float *dq, float *dk, float *dv,
                                       float *dg, float *dbeta, float *dstate_in,
                                       void *cuda_stream) {
  const size_t need = gdn_prefill_backward_workspace_bytes(n_seq, T, H, d_k, d_v,
                                                           cu_seqlens != nullptr);
  if (need > kStaticScratchBytes) return GDN_ERR_UNSUPPORTED;
  void *ws = nullptr;
  if (need > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    if (!g_bwd_scratch_ptr[dev]) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
      g_bwd_scratch_ptr[dev] = p;
    }
    ws = g_bwd_scratch_ptr[dev];
  }
  return gdn_prefill_backward(q, k, v, g, beta, state_in, cu_seqlens, n_seq, T, H, d_k, d_v, dt,
                              gk, qdq, d_o, dstate_out, ws, ws ? kStaticScratchBytes : 0, dq, dk,
                              dv, dg, dbeta, dstate_in, cuda_stream);
}

int gdn_prefill_schedule(int n_seq, int H, int d_k, int d_v, gdn_dtype dt, gdn_gate_kind gk,
                         gdn_qdq_mode qdq) {
  if (n_seq < 0 || H <= 0) return -1;
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return -1;
  if (dt != GDN_DTYPE_BF16 && dt != GDN_DTYPE_F32) return -1;
  if (gk != GDN_GATE_SCALAR && gk != GDN_GATE_PER_KEY) return -1;
  int kind = 0, group = 32;
  if ((unsigned)qdq > (unsigned)GDN_QDQ_INT8_GROUP64 || !qdq_params(qdq, d_v, &kind, &group))
    return -1;
  if (!tc_path(dt, gk, d_k, d_v)) return GDN_PREFILL_CUDA_CORES;
  const long long units = (long long)n_seq * H;
  if (!use_pair(units)) return GDN_PREFILL_TC_ONE_CTA;
  return use_wy(kind) ? GDN_PREFILL_TC_WY_PAIR : GDN_PREFILL_TC_CTA_PAIR;
}

gdn_status gdn_last_error(void *cuda_stream) {
  unsigned *err = nullptr;
  gdn_status s = err_word(&err);
  if (s != GDN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  unsigned host = 0;
  if (cudaMemcpyAsync(&host, err, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaMemsetAsync(err, 0, sizeof(unsigned), st) != cudaSuccess) return GDN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
  if (host & gdn::kErrTimeout) return GDN_ERR_TIMEOUT;
  if (host & gdn::kErrBadSeqlens) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

}  // extern "C"
