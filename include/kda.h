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
 *   - The device status word lives in that array: read device-side errors
 *     (KDA_ERR_TIMEOUT, KDA_ERR_RANGE) of the last call on the current
 *     device with kda_fwd_noalloc_status().
 *   - The array's address is cached per device together with the id of the
 *     device's context; after cudaDeviceReset the next call looks it up
 *     again.
 */
#define KDA_NOALLOC_MAX_SEQUENCES 8192
KDA_API kda_status_t kda_fwd_noalloc(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     const float *init_state, void *out, float *final_state,
                                     int B, int64_t T, int H, int dk, int dv,
                                     const int32_t *cu_seqlens, void *stream, kda_dtype_t dt);

/*
 * Device status of the last kda_fwd_noalloc call on the current device, read
 * from the library's fixed array: synchronises `stream` (pass the stream the
 * call ran on) and returns KDA_OK, KDA_ERR_TIMEOUT or KDA_ERR_RANGE as
 * kda_workspace_status does for a caller workspace.  Allocates nothing.
 */
KDA_API kda_status_t kda_fwd_noalloc_status(void *stream);

/*
 * The tensors of one kda_fwd call, as a set of pointers (all on the host, or
 * all on the device).  init_state, cu_seqlens and final_state may be NULL with
 * the meaning they have in kda_fwd.
 */
typedef struct kda_fwd_tensors {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *init_state;
    const int32_t *cu_seqlens;
    void *out;
    float *final_state;
} kda_fwd_tensors_t;

/*
 * kda_fwd on host buffers: enqueues the host-to-device copies of every input
 * in `host` (q, k, v, log_alpha, beta, and init_state / cu_seqlens when set)
 * into the caller's device buffers `dev`, the forward on `dev`, and the
 * device-to-host copies of out (and final_state when both `host` and `dev`
 * set it).  Sizes and the other arguments are those of kda_fwd; `host` and
 * `dev` must set the same optional tensors.  Host buffers should be
 * page-locked (the copies are then asynchronous and overlap).
 *
 * Batched calls (no cu_seqlens) are split into up to 16 pieces — groups of
 * whole sequences when B > 1, else token slices of the one sequence starting
 * on 64-token chunk boundaries, carried through dev->final_state (which must
 * then be set; without it the call runs in one piece) — and the pieces'
 * copies in, forwards and copies out are overlapped: copies in on one
 * internal stream, forwards on `stream`, copies out on another internal
 * stream, ordered by events.  The results are the bits of one kda_fwd call.
 * Packed batches run in one piece on `stream`.  The internal streams and
 * events are made on the first pipelined call on a device and kept; calls
 * from several host threads are serialised while they enqueue.  `stream`
 * waits for everything the call enqueued: the call returns at once, and
 * synchronising `stream` makes the host outputs readable.  A failure while
 * enqueueing returns KDA_ERR_CUDA (work already enqueued still runs).
 * This is the end-to-end path a serving process without its own device
 * staging logic would call.
 */
KDA_API kda_status_t kda_fwd_host(const kda_fwd_tensors_t *host, const kda_fwd_tensors_t *dev,
                                  int B, int64_t T, int H, int dk, int dv, void *stream,
                                  kda_dtype_t dt, void *workspace, size_t workspace_bytes);

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
 * kda_fwd with the model's input prologue fused in (the digest's "Kimi Delta
 * Attention" section: q and k are L2-normalised, and the decay logits z get a
 * per-head scale; "Bounded decay" section: g = g_min * sigmoid(exp(A_h) * z),
 * alpha = exp(g), with g_min = -5 in the model's configuration):
 *   q, k       [B, T, H, dk]  dtype dt, NOT normalised: the kernel uses
 *              x / sqrt(|x|^2 + 1e-6) per (token, head), in fp32, folded into
 *              its operand scaling (no normalised copy is written)
 *   z          [B, T, H, dk]  dtype dt: the decay logits, in place of log_alpha
 *   A_log      [H] fp32, device: the per-head log scale A_h
 *   g_min      the lower bound of the log decay
 * Everything else as kda_fwd (same workspace).  HBM traffic per token-head
 * drops from 1540 to 1284 bytes for bf16 (z is bf16 where log_alpha is fp32).
 */
KDA_API kda_status_t kda_fwd_gated(const void *q, const void *k, const void *v, const void *z,
                                   const float *A_log, float g_min, const float *beta,
                                   const float *init_state, void *out, float *final_state,
                                   int B, int64_t T, int H, int dk, int dv,
                                   const int32_t *cu_seqlens, void *stream, kda_dtype_t dt,
                                   void *workspace, size_t workspace_bytes);

/*
 * Interval checkpoints for prefix caching (the digest's serving section,
 * "decoupling hash granularity from storage granularity": the KDA state is
 * stored only at a sparse subset of the 512-token hash boundaries, so that a
 * later request whose prefix matches up to such a boundary resumes prefill
 * there instead of recomputing it).
 *
 * Same arguments and results as kda_fwd, plus
 *   checkpoints [capacity, H, dk, dv] fp32, device: the state of every
 *              sequence after each whole multiple of `interval` tokens from
 *              its start (positions interval, 2 interval, ... <= its length;
 *              a sequence whose length is a multiple of `interval` also gets
 *              its final state as its last checkpoint).  Sequence n's
 *              checkpoints are consecutive slots starting at
 *              sum_{m<n} floor(L_m / interval).
 *   interval   a positive multiple of 64 tokens (the chunk length), else
 *              KDA_ERR_UNSUPPORTED.  The pages' hash block is 512.
 *   capacity   number of slots in `checkpoints`.  Batched inputs need
 *              B * floor(T / interval) slots (checked on the host); for packed
 *              batches a slot beyond it is skipped and reported as
 *              KDA_ERR_INVALID_ARG through kda_workspace_status().
 *   workspace  at least kda_fwd_checkpoints_workspace_size(...) bytes.
 * Extra HBM traffic: dk * dv * 4 bytes per head per checkpoint.
 */
KDA_API size_t kda_fwd_checkpoints_workspace_size(int B, int64_t T, int H, int dk, int dv, kda_dtype_t dt);
KDA_API kda_status_t kda_fwd_checkpoints(const void *q, const void *k, const void *v,
                                         const float *log_alpha, const float *beta,
                                         const float *init_state, void *out, float *final_state,
                                         int B, int64_t T, int H, int dk, int dv,
                                         const int32_t *cu_seqlens, void *stream, kda_dtype_t dt,
                                         float *checkpoints, int interval, int64_t capacity,
                                         void *workspace, size_t workspace_bytes);

/*
 * Segment pieces (the digest's "KDA algorithm-system co-design" section,
 * KCP paragraph: with M_t = (I - beta_t k_t k_t^T) Diag(alpha_t) the state
 * after a segment is S~ + M S_in, where the transition M and the zero-start
 * state S~ depend only on the segment's own tokens).  Every sequence of the
 * batch is one segment; for each (sequence, head) this computes
 *   out_zero   [B, T, H, dv] fp32: the outputs from a zero initial state
 *   state_zero [N, H, dk, dv] fp32: the state after the segment from zero (S~)
 *   qhat       [B, T, H, dk] fp32: qhat_t = M_{t<-first}^T q_t, the transition
 *              from the segment start through token t applied to q_t, so that
 *              the output from an initial state S_in is out_zero_t + S_in^T qhat_t
 *   transition [N, H, dk, dk] fp32: M, the product of the segment's M_t
 * Requires dk == dv (else KDA_ERR_UNSUPPORTED).  Other arguments, layouts
 * and the workspace are those of kda_fwd (kda_fwd_workspace_size).
 * Cost: two forward passes over the segment (the second with values taken as
 * zero and an identity start), both with fp32 outputs.
 */
KDA_API kda_status_t kda_segment_fwd(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     float *out_zero, float *state_zero, float *qhat, float *transition,
                                     int B, int64_t T, int H, int dk, int dv,
                                     const int32_t *cu_seqlens, void *stream, kda_dtype_t dt,
                                     void *workspace, size_t workspace_bytes);

/*
 * Prefix composition of segment pieces (same paragraph: the rank-level
 * updates compose associatively, so every segment's incoming state follows
 * from a prefix scan).  N sequences, each cut into R consecutive pieces
 * r = 0..R-1; piece (m, r) is at index m*R + r (rank_major = 0) or r*N + m
 * (rank_major = 1, the layout of an all-gather over R ranks).
 *   transition [R*N, H, dk, dk], state_zero [R*N, H, dk, dv]  (from
 *              kda_segment_fwd of every piece), fp32, device
 *   init_state [N, H, dk, dv] or NULL (zeros): the state before piece 0
 *   state_in   [R*N, H, dk, dv] or NULL: the state entering each piece,
 *              S_in(m, 0) = init, S_in(m, r+1) = S~(m, r) + M(m, r) S_in(m, r)
 *   final_state[N, H, dk, dv] or NULL: the state after the last piece
 * fp32 arithmetic on CUDA cores.  Asynchronous on `stream`; no workspace.
 */
KDA_API kda_status_t kda_state_compose(const float *transition, const float *state_zero,
                                       const float *init_state, float *state_in, float *final_state,
                                       int R, int N, int H, int dk, int dv, int rank_major, void *stream);

/*
 * Outputs of segments whose incoming states are known:
 *   out_t = out_zero_t + S_in^T qhat_t   (rounded once to dtype dt)
 * with out_zero and qhat from kda_segment_fwd and S_in = state_in[n] for the
 * sequence n that holds token t (cu_seqlens as in kda_fwd).
 *   state_in [N, H, dk, dv] fp32; out [B, T, H, dv] in dtype dt.
 * The product runs on the warp-level tensor path with tf32 operands
 * (rounded to nearest) and fp32 accumulation.  No workspace.
 */
KDA_API kda_status_t kda_output_correct(const float *out_zero, const float *qhat, const float *state_in,
                                        void *out, int B, int64_t T, int H, int dk, int dv,
                                        const int32_t *cu_seqlens, void *stream, kda_dtype_t dt);

/*
 * Intra-device context parallelism (the digest's co-design section, the
 * intra-device context-parallel paragraph: under tensor parallelism a rank
 * holds few heads, so a long prefill leaves most SMs idle; the sequence is
 * split over the SMs of one device, the segment transitions are evaluated in
 * parallel and merged to recover each segment's exact initial state, with no
 * inter-device traffic).
 *
 * Same arguments and results as kda_fwd, plus n_seg: every sequence is cut
 * into n_seg segments of near-equal length (at tokens start + floor(L r /
 * n_seg), anywhere inside a 64-token chunk).  Three steps on `stream`:
 *   1. a state pass over all segments at once: the first segment of each
 *      sequence runs from its initial state, every middle segment as a
 *      zero-start run (S~) and a transition run (M), the last segment not at
 *      all; no outputs are written;
 *   2. the composition S_in(r+1) = S~_r + M_r S_in(r) (kda_state_compose's
 *      kernel) gives every segment's incoming state;
 *   3. the ordinary forward (kda_fwd's kernel) over all segments from those
 *      states, writing `out` and the final state.
 * So the serial depth falls from L to about 2 L / n_seg tokens, at the price
 * of about three times the forward work on the middle segments.
 * Requires dk == dv.  n_seg = 1 is the plain forward.
 *   workspace  at least kda_fwd_cp_workspace_size(B, T_total, ..., n_seg)
 *              bytes: four fp32 states per (segment, head) and the segment
 *              offsets (T_total, the token count, is not needed for the size).
 * Worth it when the chains are few: kda_cp_segments(N, L, H, sm_count) gives
 * the largest n_seg whose passes fit one wave of blocks (1 when none does).
 */
KDA_API size_t kda_fwd_cp_workspace_size(int B, int64_t T_total, int H, int dk, int dv, kda_dtype_t dt,
                                         int n_seg);
KDA_API int kda_cp_segments(int N, int64_t tokens_per_sequence, int H, int sm_count);
KDA_API kda_status_t kda_fwd_cp(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *init_state, void *out, float *final_state,
                                int B, int64_t T, int H, int dk, int dv,
                                const int32_t *cu_seqlens, void *stream, kda_dtype_t dt, int n_seg,
                                void *workspace, size_t workspace_bytes);

/*
 * The decode step with the model's input prologue fused in (the digest's KDA
 * section: q and k are L2-normalised, the decay logits get a per-head
 * scale; "Bounded decay" section: g = g_min * sigmoid(exp(A_h) * z)):
 *   q, k       [B, H, dk]  dtype dt, NOT normalised; the kernel uses
 *              x / sqrt(|x|^2 + 1e-6) per (sequence, head)
 *   z          [B, H, dk]  dtype dt: the decay logits
 *   A_log      [H] fp32: the per-head log scale A_h
 *   g_min      the lower bound of the log decay (-5 in the model)
 * Everything else as kda_decode_step.
 */
KDA_API kda_status_t kda_decode_step_gated(const void *q, const void *k, const void *v, const void *z,
                                           const float *A_log, float g_min, const float *beta,
                                           float *state, void *out, int B, int H, int dk, int dv,
                                           void *stream, kda_dtype_t dt);

/*
 * Speculative-decode verification with state replay (the digest's serving
 * section, "speculative decoding and KDA state rewind": the state after the
 * accepted draft prefix is fully determined by the drafts' projected inputs,
 * which are much smaller than the state; so only those inputs are kept, the
 * accepted tokens' states are rebuilt on chip, and only the committed state
 * is written back).
 *
 * One call per decode step, for B sequences:
 *   *_prev     [B, Wp, H, d]: the previous call's window (its projected
 *              inputs, kept by the caller); may be NULL when Wp = 0
 *   n_accepted [B] int32, device: how many of those Wp draft tokens
 *              verification accepted (clamped to [0, Wp])
 *   q, k, v, log_alpha, beta  [B, W, H, d]: the new window; token 0 is the
 *              bonus token (certain), tokens 1..W-1 the next drafts
 *   state      [B, H, dk, dv] fp32: the committed state, read once, and
 *              overwritten once with the state after the accepted tokens and
 *              the bonus token
 *   out        [B, W, H, dv]: the outputs of the W new tokens (each read with
 *              the state after that token)
 * The rejected drafts of the previous window are never applied; the new
 * drafts' states stay on chip.  The replayed and new tokens are taken as one
 * chunk (the chunkwise form of the recurrence, fp32), so the state is read
 * once and written once whatever the window (all Wp + W rows of both windows
 * are read, the rejected drafts' too, so that no load waits for n_accepted;
 * every pointer must be 16-byte aligned).  Wp + W <= KDA_SPEC_MAX_TOKENS
 * (else KDA_ERR_UNSUPPORTED).  W = 0 only replays (and keeps the state after
 * the accepted drafts).  No workspace.
 */
#define KDA_SPEC_MAX_TOKENS 16
KDA_API kda_status_t kda_decode_spec(const void *q_prev, const void *k_prev, const void *v_prev,
                                     const float *log_alpha_prev, const float *beta_prev,
                                     const int32_t *n_accepted,
                                     const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     float *state, void *out, int B, int Wp, int W, int H, int dk, int dv,
                                     void *stream, kda_dtype_t dt);

/*
 * kda_decode_spec with the input prologue fused in, as kda_decode_step_gated:
 * z_prev / z are the decay logits (dtype dt) in place of the log-decays, and
 * q, k are normalised by the kernel; A_log [H] and g_min as there.
 */
KDA_API kda_status_t kda_decode_spec_gated(const void *q_prev, const void *k_prev, const void *v_prev,
                                           const void *z_prev, const float *beta_prev,
                                           const int32_t *n_accepted,
                                           const void *q, const void *k, const void *v, const void *z,
                                           const float *beta, const float *A_log, float g_min,
                                           float *state, void *out, int B, int Wp, int W, int H, int dk, int dv,
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
