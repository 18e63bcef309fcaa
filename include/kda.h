/*
 * kda.h — C ABI of libkda.so: the Kimi Delta Attention (KDA) forward pass on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed.  Per head, the gated delta rule of the Kimi K3 technical
 * report digest (discuss.pytorch.kr, "Kimi K3 model weights and technical
 * report"), section "Kimi Delta Attention: delta rule with a per-channel
 * forget gate", state-update equation:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                    (the read uses the updated state)
 *
 * q_t, k_t in R^dk; v_t, o_t in R^dv; S_t in R^{dk x dv}; alpha_t in (0,1)^dk
 * scales row i (key channel i) of S; beta_t in (0,1).  The caller passes the
 * log-decay g_t = log(alpha_t) ("log_alpha"), as in the digest's section
 * "Bounded decay: diagonal tiles back on the tensor cores" (alpha = exp(g),
 * g bounded below by g_min = -5).  No 1/sqrt(dk) scale is applied to q; q and
 * k are expected L2-normalised by the caller (the model does this before the
 * recurrence) but nothing relies on it.
 *
 * Precondition (documented, not checked): every g value is finite and <= 0
 * (alpha <= 1, a decay).  The model's range is [-5, 0]; the kernels do not
 * rely on that lower bound (every decay factor they form is at most 1 for
 * any g <= 0; the parity tests cover g down to -20).  Results for g > 0 are
 * not covered by the accuracy contract.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller allocates and owns every buffer.  The library
 *     never allocates, frees or synchronises device memory or streams.
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and the call returns at once.
 *     The only errors returned synchronously are argument validation
 *     failures and launch failures (KDA_ERR_CUDA).  Device-side timeouts of
 *     bounded waits are recorded in the workspace status word and read back
 *     with kda_workspace_status().
 *   - Layout: all tensors are dense, contiguous, row-major, token-major:
 *     q, k, log_alpha [B, T, H, dk]; v, out [B, T, H, dv]; beta [B, T, H];
 *     states [N, H, dk, dv] (key index major: element (i, j) of a head's
 *     state at i*dv + j; each head's state is one contiguous block, as in the
 *     digest's serving section, "unified cache layout", where a head is the
 *     unit of transfer).
 *   - Alignment: every pointer must be 16-byte aligned (KDA_ERR_INVALID_ARG).
 *   - Sizes: dk, dv in {16, 32, 64, 128} (else KDA_ERR_UNSUPPORTED).
 *   - The total token count (B*T, or T when packed) must be below 2^31
 *     (else KDA_ERR_UNSUPPORTED).
 *   - Aliasing: out must not overlap any input.  final_state may alias
 *     init_state exactly (in-place chaining).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or offsets */
    KDA_ERR_UNSUPPORTED = 2,  /* dk/dv/dtype combination not built */
    KDA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    KDA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up */
    KDA_ERR_RANGE = 6         /* a tensor-core operand exceeded fp16 range (see kda_fwd) */
} kda_status_t;

/* Element type of q, k, v and out.  log_alpha, beta and states are always
 * fp32.  KDA_F32 inputs are computed in fp32 on CUDA cores, without rounding
 * operands to TF32 or bf16.  KDA_BF16 inputs with dk = dv = 128 run on the
 * tensor cores with fp16 operands (10-bit mantissa), fp32 accumulation and an
 * fp32 state; other bf16 shapes run in fp32 on CUDA cores. */
typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/*
 * Bytes of device workspace kda_fwd needs for these sizes: a 256-byte
 * status word plus, for packed batches, N int32 slots of scratch in which
 * the longest-first order of the sequences is built.  With cu_seqlens, pass
 * B = N (number of sequences) and T = total packed tokens.
 */
KDA_API size_t kda_fwd_workspace_size(int B, int64_t T, int H, int dk, int dv, kda_dtype_t dt);

/*
 * Prefill / training-style forward over whole sequences (chunked form; the
 * digest's "Kimi Delta Attention" section, chunkwise-parallel equation, and
 * "KDA algorithm-system co-design", FlashKDA paragraph).
 *
 *   q, k       [B, T, H, dk]  dtype dt, device
 *   v          [B, T, H, dv]  dtype dt, device
 *   log_alpha  [B, T, H, dk]  fp32, device; g = log(alpha) <= 0
 *   beta       [B, T, H]      fp32, device
 *   init_state [N, H, dk, dv] fp32, device, or NULL for a zero start
 *   out        [B, T, H, dv]  dtype dt, device, written (rounded to nearest
 *                             even when dt is bf16)
 *   final_state[N, H, dk, dv] fp32, device, or NULL (not written)
 *   cu_seqlens NULL: B independent sequences of T tokens each (N = B).
 *              non-NULL: device int32[N+1] with cu[0] = 0, non-decreasing,
 *              cu[N] = T; tensors are packed [1, T, H, *] and B = N.
 *              Zero-length sequences are allowed (final = init).
 *              The offsets are not validated on the host (they live on the
 *              device); invalid offsets give undefined results.
 *   stream     cudaStream_t as void*
 *   workspace  device scratch of at least kda_fwd_workspace_size(...) bytes,
 *              16-byte aligned; its contents on entry do not matter.  It must
 *              not be shared by calls that may run concurrently.
 * Range (tensor-core path): v, the state and the intermediate values W, U,
 * Delta are rounded to fp16 operands, so their magnitudes must stay below
 * 6e4 (|v| and |S| of order 1e3 or less are safe).  A value beyond that is
 * reported as KDA_ERR_RANGE through kda_workspace_status(); outputs are then
 * not meaningful.
 */
KDA_API kda_status_t kda_fwd(const void *q, const void *k, const void *v,
                     const float *log_alpha, const float *beta,
                     const float *init_state, void *out, float *final_state,
                     int B, int64_t T, int H, int dk, int dv,
                     const int32_t *cu_seqlens, void *stream, kda_dtype_t dt,
                     void *workspace, size_t workspace_bytes);

/*
 * kda_fwd for callers that cannot allocate device memory (for example a
 * hosting runtime that owns all device memory, or a serving loop that must
 * not call cudaMalloc/cudaFree because they can synchronize the device).
 * The pages describe no such interface; it exists for callers of this
 * library.
 *
 * Same arguments and results as kda_fwd, without the workspace: the call
 * uses a fixed device array owned by the library (256 bytes plus 4 bytes per
 * sequence, for at most KDA_NOALLOC_MAX_SEQUENCES sequences; every GPU that
 * loads the library holds it until the process exits) and allocates nothing.
 *   - B (the number of sequences) above KDA_NOALLOC_MAX_SEQUENCES returns
 *     KDA_ERR_WORKSPACE before any device work.
 *   - The first call on each device looks up the array's device address
 *     (with that device current); make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array.  Calls that may overlap on
 *     the GPU (different streams, or other host threads) race on it; issue
 *     them in order on one stream.
 *   - The device status word lives in that array, so device-side errors
 *     (KDA_ERR_TIMEOUT, KDA_ERR_RANGE) of this entry point cannot be read
 *     back; use kda_fwd with a workspace when they must be checked.
 */
#define KDA_NOALLOC_MAX_SEQUENCES 8192
KDA_API kda_status_t kda_fwd_noalloc(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     const float *init_state, void *out, float *final_state,
                                     int B, int64_t T, int H, int dk, int dv,
                                     const int32_t *cu_seqlens, void *stream, kda_dtype_t dt);

/*
 * One decode step: one new token per sequence, state updated in place (the
 * digest's serving section, "speculative decoding and KDA state rewind":
 * the recurrent state is updated in place at every decode step).
 *
 *   q, k       [B, H, dk]      dtype dt, device
 *   v          [B, H, dv]      dtype dt, device
 *   log_alpha  [B, H, dk]      fp32, device
 *   beta       [B, H]          fp32, device
 *   state      [B, H, dk, dv]  fp32, device, read and overwritten in place
 *   out        [B, H, dv]      dtype dt, device
 * No workspace.  B = 0 is a no-op.
 */
KDA_API kda_status_t kda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             float *state, void *out, int B, int H, int dk, int dv,
                             void *stream, kda_dtype_t dt);

/*
 * Read back the device status word of a workspace used by kda_fwd.
 * Synchronises `stream` (it is the one call that does) and returns KDA_OK or
 * the first device-side error recorded since the workspace was last passed
 * to kda_fwd (KDA_ERR_TIMEOUT when a bounded wait expired, KDA_ERR_RANGE
 * when an fp16 operand overflowed).
 */
KDA_API kda_status_t kda_workspace_status(const void *workspace, void *stream);

/* Static, human-readable name of a status code. */
KDA_API const char *kda_status_string(kda_status_t s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
KDA_API int kda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
