// C ABI of libkda.so (declared in include/kda.h): host-side validation,
// workspace layout and kernel dispatch.  No entry point allocates, frees or
// synchronises, except kda_workspace_status which reads back a status word.
#include <cstdint>
#include <cstring>

#include "../../include/kda.h"
#include "../../include/kda_testing.h"
#include "kda_internal.cuh"

namespace kda {
cudaError_t launch_fwd_tc_impl(const FwdArgs& a, cudaStream_t s, uint64_t wait_ns, int inject_stuck,
                               int32_t* order_ws);
int fwd_tc_debug_floats();
}  // namespace kda

namespace {

constexpr size_t kStatusBytes = 256;  // DeviceStatus + reserve

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

kda_status_t validate_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          const float* init, const void* out, const float* fin, int B, int64_t T, int H, int dk,
                          int dv, kda_dtype_t dt) {
  if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (T > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  // Token tensors may be NULL only when there are no tokens at all.
  const void* req[] = {q, k, v, g, beta, out};
  for (const void* p : req)
    if ((!p && T > 0 && B > 0) || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (init && !aligned16(init)) return KDA_ERR_INVALID_ARG;
  if (fin && !aligned16(fin)) return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

}  // namespace

extern "C" {

int kda_version(void) { return 100; }

const char* kda_status_string(kda_status_t s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null or misaligned pointer, or bad size";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: dk/dv/dtype combination not built";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or kernel launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a device-side bounded wait gave up";
    case KDA_ERR_RANGE: return "KDA_ERR_RANGE: a tensor-core operand exceeded fp16 range";
  }
  return "KDA_ERR_UNKNOWN";
}

size_t kda_fwd_workspace_size(int B, int64_t T, int H, int dk, int dv, kda_dtype_t dt) {
  (void)T; (void)H; (void)dk; (void)dv; (void)dt;
  const size_t order = B > 0 ? (size_t)B * sizeof(int32_t) : 0;
  return kStatusBytes + ((order + 255) / 256) * 256;
}

static kda_status_t fwd_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                             const float* beta, const float* init_state, void* out, float* final_state, int B,
                             int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, void* stream,
                             kda_dtype_t dt, void* workspace, size_t workspace_bytes, float* dbg,
                             uint64_t wait_ns, int inject_stuck) {
  kda_status_t st = validate_fwd(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, dt);
  if (st != KDA_OK) return st;
  if (cu_seqlens && !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < kda_fwd_workspace_size(B, T, H, dk, dv, dt))
    return KDA_ERR_WORKSPACE;
  // Token coordinates are 32-bit in the kernels (TMA tile coordinates).
  if ((cu_seqlens ? T : (int64_t)B * T) > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  kda::DeviceStatus* status = reinterpret_cast<kda::DeviceStatus*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(kda::DeviceStatus), s) != cudaSuccess) return KDA_ERR_CUDA;
  if (B == 0) return KDA_OK;
  kda::FwdArgs a{q, k, v, log_alpha, beta, init_state, out, final_state, cu_seqlens, B, T, H, dk, dv, status, dbg};
  const bool bf16 = dt == KDA_BF16;
  cudaError_t e;
  const int64_t tokens = cu_seqlens ? T : (int64_t)B * T;
  if (kda::fwd_tc_supported(dk, dv, bf16) && tokens > 0)
    e = kda::launch_fwd_tc_impl(a, s, wait_ns, inject_stuck,
                                reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes));
  else if (dbg || inject_stuck)
    return KDA_ERR_UNSUPPORTED;
  else
    e = kda::launch_fwd_simt(a, bf16, s);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_fwd(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                     const float* init_state, void* out, float* final_state, int B, int64_t T, int H, int dk,
                     int dv, const int32_t* cu_seqlens, void* stream, kda_dtype_t dt, void* workspace,
                     size_t workspace_bytes) {
  return fwd_impl(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, cu_seqlens, stream,
                  dt, workspace, workspace_bytes, nullptr, 2000000000ull, 0);
}

kda_status_t kda_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                             const float* beta, float* state, void* out, int B, int H, int dk, int dv,
                             void* stream, kda_dtype_t dt) {
  if (B < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const void* req[] = {q, k, v, log_alpha, beta, state, out};
  for (const void* p : req)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if ((int64_t)B * H > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  cudaError_t e = kda::launch_decode(q, k, v, log_alpha, beta, state, out, B, H, dk, dv, dt == KDA_BF16,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_workspace_status(const void* workspace, void* stream) {
  if (!workspace || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  kda::DeviceStatus h{};
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  return static_cast<kda_status_t>(h.code);
}

// ---- test hooks (include/kda_testing.h) ----
int kda_testing_debug_floats(void) { return kda::fwd_tc_debug_floats(); }

kda_status_t kda_testing_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                             const float* beta, const float* init_state, void* out, float* final_state, int B,
                             int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, void* stream,
                             kda_dtype_t dt, void* workspace, size_t workspace_bytes, float* debug_out,
                             uint64_t wait_ns, int inject_stuck) {
  return fwd_impl(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, cu_seqlens, stream,
                  dt, workspace, workspace_bytes, debug_out, wait_ns, inject_stuck);
}

int kda_testing_fwd_path(int dk, int dv, kda_dtype_t dt) {
  return kda::fwd_tc_supported(dk, dv, dt == KDA_BF16) ? 1 : 0;
}

}  // extern "C"
