/*
 * kda_testing.h — test hooks exported by libkda.so.  Not part of the stable
 * ABI in kda.h; used by the library's own tests to look inside a forward
 * call.  These hooks compute nothing the public entry points do not.
 */
#ifndef KDA_TESTING_H_
#define KDA_TESTING_H_

#include "kda.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Number of floats kda_testing_fwd writes to debug_out. */
KDA_API int kda_testing_debug_floats(void);

/*
 * Same as kda_fwd, plus the hooks below.  A call that sets debug_out or
 * inject_stuck runs the instrumented build of the tensor-core kernel (same
 * source, with the dumps, timestamps and injection compiled in); other calls
 * run the production build, which has none of them.
 *   debug_out  device fp32 buffer of kda_testing_debug_floats() floats or
 *              NULL.  When set (tensor-core path only, else
 *              KDA_ERR_UNSUPPORTED), the block of chain 0 (sequence 0, head 0)
 *              writes the intermediates of its first chunk, row-major fp32
 *              at these float offsets: P [64][64] at 0, A [64][64] at 4096
 *              (strictly lower part), T' [64][64] at 8192, W' [64][128] at
 *              12288 (W' = W Diag(exp(-G_C)), the chunk-end-referenced
 *              pseudo-keys, on chunks whose total decay keeps the
 *              end-referenced operands in fp16 range; W' = W on the others,
 *              which are referenced to the chunk start), U [64][128] at
 *              20480, Delta [64][128] at 28672, O [64][128] at 36864, the
 *              state after the chunk [128][128] at 45056, the chunk-total
 *              log-decay G_C [128] at 61440; and, as
 *              int64 from float offset 61568, [64 chunks][32 events] of SM
 *              clock cycles since the block started: phase boundaries of
 *              the first 64 chunks (events 0-7 and 26: front group, with
 *              29 and 30 inside the Gram of strongly decaying chunks; 16-23
 *              and 25: back group; 8-15, 24, 27, 28: scan group).
 *   wait_ns    bound for every device-side wait in nanoseconds (kda_fwd
 *              uses 2e9).
 *   inject_stuck  when nonzero (tensor-core path), the scan warps of every
 *              block first wait on a barrier that nothing ever signals.  The
 *              wait gives up after wait_ns, records KDA_ERR_TIMEOUT in the
 *              workspace status word and the block unwinds: it drains its own
 *              copies and tensor-core work and releases its tensor memory, so
 *              the GPU context stays usable.  Nothing faults or hangs.
 */
KDA_API kda_status_t kda_testing_fwd(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *init_state, void *out, float *final_state,
                             int B, int64_t T, int H, int dk, int dv,
                             const int32_t *cu_seqlens, void *stream, kda_dtype_t dt,
                             void *workspace, size_t workspace_bytes,
                             float *debug_out, uint64_t wait_ns, int inject_stuck);

/* 1 when kda_fwd uses the tensor-core kernel for this shape, else 0. */
KDA_API int kda_testing_fwd_path(int dk, int dv, kda_dtype_t dt);

#ifdef __cplusplus
}
#endif
#endif /* KDA_TESTING_H_ */
