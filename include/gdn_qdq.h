/*
 * gdn_qdq.h - C ABI of the B200 (sm_100a) gated-delta-rule library with a
 * fake-quantized (QDQ) recurrent state.
 *
 * The operations follow the GatedDeltaNet / KDA state-QAT pages (the
 * "linear_attention" QAT series of NVIDIA Model-Optimizer):
 *   - prefix ("chunked prefix", PR #2519 What section; "64-token chunks" and
 *     the "WY-transformed W", PR #2497 What section): the sequence is cut into
 *     64-token chunks, each chunk is solved in the WY form with an exact
 *     triangular solve (PR #2507 What section: "exact triangular solve
 *     remains the default"), and the state is carried chunk to chunk;
 *   - suffix ("recurrent suffix", recurrent_decode, PR #2519 What section):
 *       S_t = S_{t-1} diag(alpha_t);  u_t = beta_t (v_t - S_t k_t);
 *       S_t += u_t k_t^T;  o_t = S_t q_t / sqrt(d_k);
 *   - state QDQ at every 64-token chunk boundary of the prefix and after every
 *     decode token: dynamic FP8 E4M3 with one scale per (all d_k keys x 64
 *     value columns) tile per sequence and head, scale = amax / 448 with a
 *     zero guard (PR #2497 What section); or dynamic INT8 with groups of 32
 *     along the last axis, scale = amax / 127, round half to even, clamp to
 *     [-127, 127] (PR #2519 commit notes, recipe
 *     linear_attention_state_int8_block32_dynamic); groups of 16 and 64 are
 *     offered as well;
 *   - fp32 working values for the state and the gates, bf16 or fp32 q/k/v
 *     promoted to fp32 (PR #2519 commit notes).
 *
 * Layouts (all row-major, contiguous):
 *   state  fp32 [n_seq, H, d_k, d_v]: the transpose H = S^T of the pages'
 *          state, row = key, column = value, so the FP8 tile is d_k rows x
 *          64 columns and INT8 groups run along d_v (the last axis).
 *   q, k   [.., H, d_k]; v, o [.., H, d_v] in the dtype `dt`;
 *   g      fp32 natural-log gates (alpha = exp(g) in (0, 1]): [.., H] for
 *          GDN (GDN_GATE_SCALAR) or [.., H, d_k] for KDA (GDN_GATE_PER_KEY);
 *   beta   fp32 [.., H].
 *
 * Ownership: every pointer is caller-owned memory; no call allocates memory
 * and none keeps a reference after it returns.  The library's own device
 * memory is a per-device error word and the 64 MiB scratch array of
 * gdn_prefill_backward_static, both reserved when its module is loaded.
 * Pointers are device pointers unless a function says otherwise.
 *
 * Asynchrony and errors: argument errors are detected on the host and
 * returned before anything is launched (nothing is written).  Compute calls
 * are asynchronous on `cuda_stream` (a cudaStream_t; NULL = the legacy
 * default stream).  Errors found on the device (a malformed cu_seqlens, a
 * bounded wait that ran out) are recorded in a per-device error word that
 * gdn_last_error() reports.  There is no fallback of any kind: an
 * unsupported combination returns GDN_ERR_UNSUPPORTED.
 *
 * Supported: d_k, d_v in {64, 128}; dt in {bf16, f32}; q, k, v, o and the
 * states 16-byte aligned, g and beta 4-byte aligned.
 */
#ifndef GDN_QDQ_H_
#define GDN_QDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or cu_seqlens */
    GDN_ERR_UNSUPPORTED = 2,  /* valid but unsupported combination */
    GDN_ERR_CUDA = 3,         /* a CUDA runtime call failed */
    GDN_ERR_TIMEOUT = 4       /* a bounded device-side wait ran out */
} gdn_status;

typedef enum {
    GDN_QDQ_NONE = 0,
    GDN_QDQ_FP8_E4M3_TILE64 = 1, /* one scale per (d_k x 64 value columns) */
    GDN_QDQ_INT8_GROUP32 = 2,    /* groups of 32 along d_v */
    GDN_QDQ_INT8_GROUP16 = 3,    /* groups of 16 along d_v */
    GDN_QDQ_INT8_GROUP64 = 4     /* groups of 64 along d_v */
} gdn_qdq_mode;

typedef enum { GDN_DTYPE_BF16 = 0, GDN_DTYPE_F32 = 1 } gdn_dtype;

typedef enum {
    GDN_GATE_SCALAR = 0,   /* GDN: one log-gate per token and head */
    GDN_GATE_PER_KEY = 1   /* KDA: one log-gate per token, head, key channel */
} gdn_gate_kind;

/*
 * gdn_prefill - chunked prefix over n_seq sequences.
 *
 * Dense layout (cu_seqlens == NULL): q, k, v, o are [n_seq, T, H, d], g is
 * [n_seq, T, H(, d_k)], beta [n_seq, T, H]; every sequence has T tokens.
 * Packed layout (cu_seqlens != NULL, int32 device array [n_seq + 1]): the
 * tensors are [1, T, H, d] with T the total token count; sequence s owns
 * tokens [cu_seqlens[s], cu_seqlens[s+1]).  cu_seqlens must start at 0, be
 * non-decreasing and end at T; a violation found on the device skips that
 * sequence and is reported by gdn_last_error() as GDN_ERR_INVALID_ARG.
 *
 * state_in: fp32 [n_seq, H, d_k, d_v] initial states, or NULL for zeros; it
 *   is used as given (not quantized).  state_out: same shape, receives the
 *   state after each sequence's last token (QDQ'd unless qdq is NONE or the
 *   sequence is empty); it may alias state_in exactly (in-place update).
 * o: [.., H, d_v] in dtype dt; o_t uses the state before that token's QDQ.
 * The state QDQ runs after tokens 64, 128, ... of each sequence (counted from
 * its own start) and after its last token.
 *
 * Kernel choice (results agree within the documented tolerances; they can
 * differ in the last bits of o): bf16 GDN at d_k = d_v = 128 runs on the
 * tensor cores, with either one CTA per (sequence, head) or a CTA pair (a
 * thread-block cluster of two: one CTA computes each chunk's A, Aqk and
 * triangular solve a chunk ahead, the other carries the state).  Pairs are
 * used when every (sequence, head) gets its pair in one wave on the current
 * device; the environment variable GDN_PREFILL_CTA_PAIR=0 or =1, read at
 * every call, forces one CTA or the pair.  Every other combination (fp32
 * q/k/v, KDA gates, d_k or d_v = 64) runs a CUDA-core kernel with one CTA
 * per (sequence, head, 64-column value tile) computing the same chunked
 * form in fp32.  gdn_prefill_schedule() reports which kernel a shape gets.
 *
 * Returns GDN_OK after a successful launch (or when there is no work).
 */
gdn_status gdn_prefill(const void *q, const void *k, const void *v,
                       const float *g, const float *beta,
                       const float *state_in, const int32_t *cu_seqlens,
                       int n_seq, int T, int H, int d_k, int d_v,
                       gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                       void *o, float *state_out, void *cuda_stream);

/*
 * gdn_decode - one decode token for each of n_seq sequences.
 *
 * q, k: [n_seq, H, d_k]; v, o: [n_seq, H, d_v] in dtype dt; g: fp32
 * [n_seq, H] or [n_seq, H, d_k]; beta fp32 [n_seq, H]; state_inout: fp32
 * [n_seq, H, d_k, d_v], advanced by one token and QDQ'd in place.  o is
 * computed from the state before its QDQ.
 */
gdn_status gdn_decode(const void *q, const void *k, const void *v,
                      const float *g, const float *beta, float *state_inout,
                      int n_seq, int H, int d_k, int d_v, gdn_dtype dt,
                      gdn_gate_kind gk, gdn_qdq_mode qdq, void *o,
                      void *cuda_stream);

/*
 * Packed state storage.  The pages keep the QDQ'd state as fp32 values and
 * say that compressed state storage is not part of their change (PR #2497
 * What section); these three calls add it as a storage format of the same
 * state.  A QDQ'd state is exactly code * scale, so a packed state holds:
 *   codes   one byte per element, [n, H, d_k, d_v] (same order as the fp32
 *           state): int8 codes in [-127, 127] for the INT8 modes, E4M3 bytes
 *           (bias 7, no infinities) for GDN_QDQ_FP8_E4M3_TILE64;
 *   scales  fp32: INT8 group G: [n, H, d_k, d_v / G] (one per key row and
 *           group of G value columns); FP8 tile: [n, H, d_v / 64] (one per
 *           d_k x 64 tile).  A zero group or tile has scale 0 and codes 0.
 * Decoding a packed state gives bit-identical outputs and states to
 * gdn_decode on the fp32 state it dequantizes to, while moving 1 + 4/G
 * bytes per element (INT8) or 1 + 4/(64 d_k) (FP8) instead of 4.
 * qdq must be an FP8 or INT8 mode (GDN_QDQ_NONE: GDN_ERR_UNSUPPORTED);
 * codes and scales must be 4-byte aligned, the fp32 state 16-byte aligned.
 *
 * gdn_state_pack   - apply the state QDQ codec of `qdq` to fp32 states and
 *                    store the codes and scales (the packed state then
 *                    dequantizes to exactly QDQ(state)).
 * gdn_state_unpack - dequantize: state = code * scale, element by element.
 * gdn_decode_packed - gdn_decode with the state read and written packed, in
 *                    place; the arguments are those of gdn_decode with
 *                    state_inout replaced by (codes, scales).
 * All three are asynchronous on cuda_stream; argument errors are returned
 * before any launch.
 */
gdn_status gdn_state_pack(const float *state, void *codes, float *scales,
                          int n, int H, int d_k, int d_v, gdn_qdq_mode qdq,
                          void *cuda_stream);
gdn_status gdn_state_unpack(const void *codes, const float *scales,
                            float *state, int n, int H, int d_k, int d_v,
                            gdn_qdq_mode qdq, void *cuda_stream);
gdn_status gdn_decode_packed(const void *q, const void *k, const void *v,
                             const float *g, const float *beta, void *codes,
                             float *scales, int n_seq, int H, int d_k, int d_v,
                             gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                             void *o, void *cuda_stream);

/*
 * gdn_last_error - synchronize cuda_stream, then read and clear the current
 * device's error word.  Returns GDN_OK if no device-side error was recorded
 * since the last call, GDN_ERR_INVALID_ARG for a malformed cu_seqlens,
 * GDN_ERR_TIMEOUT for a bounded wait that ran out, GDN_ERR_CUDA if the
 * synchronization itself failed.
 */
gdn_status gdn_last_error(void *cuda_stream);

/*
 * gdn_prefill_neumann - gdn_prefill with the approximate triangular solve of
 * the approximate-inverse PR (#2507, What section: an explicit Neumann
 * polynomial degree, no silent change of degree, no fallback): every chunk's
 * (I + A)^-1 is replaced by T_d = sum_{n=0}^{d} (-A)^n, evaluated as
 * prod_{i<m} (I + (-A)^(2^i)) for d = 2^m - 1.
 *
 * degree: one of 1, 3, 7, 15, 31, 63, else GDN_ERR_INVALID_ARG (nothing is
 *   launched).  A chunk of n tokens has A^n = 0, so degree >= n - 1 gives
 *   the exact solve for it; 63 is exact for every chunk.
 * All other arguments, layouts, ownership and errors as gdn_prefill.  Runs
 * on the CUDA-core (FFMA) kernel for every dtype, gate kind and shape.
 */
gdn_status gdn_prefill_neumann(const void *q, const void *k, const void *v,
                               const float *g, const float *beta,
                               const float *state_in, const int32_t *cu_seqlens,
                               int n_seq, int T, int H, int d_k, int d_v,
                               gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                               int degree, void *o, float *state_out,
                               void *cuda_stream);

/*
 * gdn_prefill_backward - gradients of one gdn_prefill call (the same
 * inputs, layout and qdq mode) for training with the state QAT of the
 * pages (PR #2497, What section: fake quantization of the recurrent state;
 * the QDQ is passed straight through in the backward pass, STE).
 *
 * d_o: upstream gradient of o, dtype dt, shaped like o.  dstate_out: fp32
 *   gradient of state_out [n_seq, H, d_k, d_v], or NULL for zero.
 * Outputs (fp32, caller-owned device memory, shaped like the matching input):
 *   dq, dk [.., H, d_k]; dv [.., H, d_v]; dg [.., H] or [.., H, d_k]; dbeta
 *   [.., H]; dstate_in [n_seq, H, d_k, d_v] (the gradient of state_in; of
 *   the zero state when state_in is NULL).  dq, dk, dg and dbeta are zeroed
 *   on the stream and accumulated.
 * workspace: caller-owned device memory of at least
 *   gdn_prefill_backward_workspace_bytes(n_seq, T, H, d_k, d_v,
 *   cu_seqlens != NULL) bytes, 16-byte aligned; its contents are scratch.
 *   The forward recurrence is recomputed from state_in (in fp32, with the
 *   QDQ at every chunk end), so no forward activations are needed.
 * Errors: as gdn_prefill; a missing, misaligned or short workspace, or a
 *   missing output, is GDN_ERR_INVALID_ARG.  Runs on the CUDA cores for
 *   every dtype, gate kind and shape.
 */
size_t gdn_prefill_backward_workspace_bytes(int n_seq, int T, int H, int d_k,
                                            int d_v, int packed);
gdn_status gdn_prefill_backward(const void *q, const void *k, const void *v,
                                const float *g, const float *beta,
                                const float *state_in, const int32_t *cu_seqlens,
                                int n_seq, int T, int H, int d_k, int d_v,
                                gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                                const void *d_o, const float *dstate_out,
                                void *workspace, size_t workspace_bytes,
                                float *dq, float *dk, float *dv, float *dg,
                                float *dbeta, float *dstate_in, void *cuda_stream);

/*
 * gdn_prefill_backward_static - gdn_prefill_backward with its workspace in
 * the library's own static device array (64 MiB per device, reserved when
 * the library's module is loaded) instead of caller memory; it allocates
 * nothing.  For callers that must not allocate device memory while they
 * run.  The methods described on the pages have no counterpart: this is an
 * interface choice.
 *
 * Arguments, layouts, outputs and errors as gdn_prefill_backward, without
 * the workspace.  A call whose workspace would exceed 64 MiB
 * (gdn_prefill_backward_workspace_bytes) returns GDN_ERR_UNSUPPORTED before
 * touching the device.  The first call on a device looks up the array's
 * address (cudaGetSymbolAddress) and fails with GDN_ERR_CUDA if it cannot;
 * make that first call outside any stream capture.  Calls that overlap on
 * one device (two streams, or two host threads) share the array and race:
 * order them.
 */
gdn_status gdn_prefill_backward_static(const void *q, const void *k, const void *v,
                                       const float *g, const float *beta,
                                       const float *state_in, const int32_t *cu_seqlens,
                                       int n_seq, int T, int H, int d_k, int d_v,
                                       gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                                       const void *d_o, const float *dstate_out,
                                       float *dq, float *dk, float *dv, float *dg,
                                       float *dbeta, float *dstate_in, void *cuda_stream);

/*
 * gdn_prefill_w_qdq - gdn_prefill with the second, independent QDQ site of
 * the pages: dynamic FP8 E4M3 fake quantization of the WY-transformed W
 * activations (PR #2497 "GDN state/W QAT foundation", What section: "independent
 * dynamic FP8 fake QDQ to WY-transformed W activations"; Usage section: the W
 * quantizer keeps axes (0, 1, 2), i.e. batch, token and head).
 *
 * In every 64-token chunk, W = T diag(beta gamma) K ([chunk tokens, d_k])
 * is replaced by its QDQ before V_new = U - W H0 is formed: one scale per
 * row of W (one token of one head), s = amax over the d_k keys / 448 in
 * fp32, with a zero guard; code = E4M3(x / s) rounded to nearest even and
 * saturated at +-448; value = code * s.  Everything else is gdn_prefill.
 *
 * w_qdq = GDN_W_QDQ_NONE is exactly gdn_prefill.  GDN_W_QDQ_FP8_E4M3_ROW is
 * supported for bf16 q/k/v, scalar (GDN) gates, d_k = d_v = 128 and
 * qdq = GDN_QDQ_FP8_E4M3_TILE64, and always runs the WY-form CTA pair
 * kernel; other combinations return GDN_ERR_UNSUPPORTED before any launch.
 * Arguments, layouts, ownership and errors as for gdn_prefill.
 */
typedef enum {
    GDN_W_QDQ_NONE = 0,
    GDN_W_QDQ_FP8_E4M3_ROW = 1   /* one scale per row of W (token, head) */
} gdn_w_qdq_mode;
gdn_status gdn_prefill_w_qdq(const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             const float *state_in, const int32_t *cu_seqlens,
                             int n_seq, int T, int H, int d_k, int d_v,
                             gdn_dtype dt, gdn_gate_kind gk, gdn_qdq_mode qdq,
                             gdn_w_qdq_mode w_qdq, void *o, float *state_out,
                             void *cuda_stream);

/*
 * gdn_prefill_schedule - which prefill kernel gdn_prefill launches for these
 * shapes and this codec on the current device, under the current
 * GDN_PREFILL_CTA_PAIR and GDN_PREFILL_WY settings (the same selection code).
 * Host-only; it may query the device's cluster occupancy once.  Returns a
 * gdn_prefill_kernel value, or -1 for arguments gdn_prefill would reject as
 * invalid or unsupported.  This has no counterpart in the method's
 * description: it reports an implementation choice.
 */
typedef enum {
    GDN_PREFILL_CUDA_CORES = 0,   /* fp32, KDA or d = 64: FFMA kernel */
    GDN_PREFILL_TC_ONE_CTA = 1,   /* tensor cores, one CTA per (sequence, head) */
    GDN_PREFILL_TC_CTA_PAIR = 2,  /* tensor cores, a CTA pair per (sequence, head) */
    GDN_PREFILL_TC_WY_PAIR = 3    /* tensor cores, a CTA pair in the WY form (FP8 tiles) */
} gdn_prefill_kernel;
int gdn_prefill_schedule(int n_seq, int H, int d_k, int d_v, gdn_dtype dt, gdn_gate_kind gk,
                         gdn_qdq_mode qdq);

/* gdn_status_string - static, human-readable name of a status code. */
const char *gdn_status_string(gdn_status s);

/* gdn_version - library version as 10000*major + 100*minor + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_QDQ_H_ */
