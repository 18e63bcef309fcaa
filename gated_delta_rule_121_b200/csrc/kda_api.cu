// C ABI of libkda.so (declared in include/kda.h): host-side validation,
// workspace layout and kernel dispatch.  No entry point allocates device
// memory, frees or synchronises, except kda_workspace_status which reads back
// a status word; kda_fwd_host makes two streams and a few events per device
// on its first pipelined call and keeps them.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/kda.h"
#include "../../include/kda_testing.h"
#include "kda_internal.cuh"

namespace kda {
cudaError_t launch_fwd_tc_impl(const FwdArgs& a, cudaStream_t s, uint64_t wait_ns, int inject_stuck,
                               int32_t* order_ws, const ModeArgs& ma);
cudaError_t launch_ckpt_base(const int32_t* cu, int N, int interval, int32_t* base, cudaStream_t s);
cudaError_t launch_compose(const float* trans, const float* s0, const float* init, float* state_in, float* fin,
                           int R, int N, int H, int dk, int dv, int rank_major, int first_from_init, int apply_last,
                           cudaStream_t s);
cudaError_t launch_correct(const float* o32, const float* qhat, const float* s_in, void* out, const int32_t* cu,
                           int P, int64_t Tper, int64_t Ttot, int H, int dk, int dv, bool bf16, int skip_every,
                           cudaStream_t s);
cudaError_t launch_segment_cu(const int32_t* cu, int64_t Tper, int N, int R, int32_t* seg_cu, cudaStream_t s);
int fwd_tc_debug_floats();
}  // namespace kda

namespace {

constexpr size_t kStatusBytes = 256;  // DeviceStatus + reserve
constexpr uint64_t kWaitNs = 2000000000ull;  // limit of every in-kernel wait (2 s)

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
                             uint64_t wait_ns, int inject_stuck, const kda::ModeArgs& ma = kda::ModeArgs(),
                             bool reset_status = true) {
  // Segment runs write fp32 outputs to their own buffers (out may be NULL).
  const void* out_chk = ma.mode == kda::MODE_SEG ? (const void*)(ma.o32 ? ma.o32 : final_state) : out;
  kda_status_t st = validate_fwd(q, k, v, log_alpha, beta, init_state, out_chk, final_state, B, T, H, dk, dv, dt);
  if (st != KDA_OK) return st;
  if (cu_seqlens && !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < kda_fwd_workspace_size(B, T, H, dk, dv, dt))
    return KDA_ERR_WORKSPACE;
  // Token coordinates are 32-bit in the kernels (TMA tile coordinates).
  if ((cu_seqlens ? T : (int64_t)B * T) > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  kda::DeviceStatus* status = reinterpret_cast<kda::DeviceStatus*>(workspace);
  if (reset_status && cudaMemsetAsync(status, 0, sizeof(kda::DeviceStatus), s) != cudaSuccess) return KDA_ERR_CUDA;
  if (B == 0) return KDA_OK;
  kda::FwdArgs a{q, k, v, log_alpha, beta, init_state, out, final_state, cu_seqlens, B, T, H, dk, dv, status, dbg};
  const bool bf16 = dt == KDA_BF16;
  cudaError_t e;
  const int64_t tokens = cu_seqlens ? T : (int64_t)B * T;
  if (kda::fwd_tc_supported(dk, dv, bf16) && tokens > 0)
    e = kda::launch_fwd_tc_impl(a, s, wait_ns, inject_stuck,
                                reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes), ma);
  else if (dbg || inject_stuck)
    return KDA_ERR_UNSUPPORTED;
  else
    e = kda::launch_fwd_simt(a, bf16, s, ma);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_fwd(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                     const float* init_state, void* out, float* final_state, int B, int64_t T, int H, int dk,
                     int dv, const int32_t* cu_seqlens, void* stream, kda_dtype_t dt, void* workspace,
                     size_t workspace_bytes) {
  return fwd_impl(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, cu_seqlens, stream,
                  dt, workspace, workspace_bytes, nullptr, kWaitNs, 0);
}

namespace {

constexpr int kHostPieces = 16;  // pieces of a pipelined kda_fwd_host call, at most

// Streams and events of the pipelined host path, one set per device, made on
// first use and kept for the life of the process.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr, ev_in[kHostPieces], ev_comp[kHostPieces];
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];
bool g_pipe_ready[64];

HostPipe* host_pipe(int dev) {  // call with g_pipe_mu held
  if (dev < 0 || dev >= 64) return nullptr;
  HostPipe& p = g_pipe[dev];
  if (g_pipe_ready[dev]) return &p;
  bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; ok && i < kHostPieces; ++i)
    ok = cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.ev_comp[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) return nullptr;
  g_pipe_ready[dev] = true;
  return &p;
}

// Pieces of a batched (no cu_seqlens) kda_fwd_host call: whole sequences
// [b0, b1) when B > 1, else token slices [t0, t1) of the one sequence whose
// starts are multiples of the 64-token chunk (so every piece's chunks are the
// unsliced call's chunks and the results are the same bits).
struct Piece {
  int b0, b1;
  int64_t t0, t1;
};
int plan_pieces(int B, int64_t T, Piece* pc) {
  if (B > 1) {
    const int n = B < kHostPieces ? B : kHostPieces;
    for (int i = 0; i < n; ++i) pc[i] = {(int)((int64_t)B * i / n), (int)((int64_t)B * (i + 1) / n), 0, T};
    return n;
  }
  const int64_t chunks = (T + 63) / 64;
  const int n = (int)(chunks < kHostPieces ? chunks : kHostPieces);
  if (n <= 1) {
    pc[0] = {0, B, 0, T};
    return 1;
  }
  for (int i = 0; i < n; ++i) {
    const int64_t c0 = chunks * i / n, c1 = chunks * (i + 1) / n;
    pc[i] = {0, 1, 64 * c0, c1 == chunks ? T : 64 * c1};
  }
  return n;
}

}  // namespace

kda_status_t kda_fwd_host(const kda_fwd_tensors_t* host, const kda_fwd_tensors_t* dev, int B, int64_t T, int H,
                          int dk, int dv, void* stream, kda_dtype_t dt, void* workspace, size_t workspace_bytes) {
  if (!host || !dev) return KDA_ERR_INVALID_ARG;
  if ((host->init_state == nullptr) != (dev->init_state == nullptr) ||
      (host->cu_seqlens == nullptr) != (dev->cu_seqlens == nullptr))
    return KDA_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H <= 0 || (dt != KDA_F32 && dt != KDA_BF16)) return KDA_ERR_INVALID_ARG;
  kda_status_t st = validate_fwd(dev->q, dev->k, dev->v, dev->log_alpha, dev->beta, dev->init_state, dev->out,
                                 dev->final_state, B, T, H, dk, dv, dt);
  if (st != KDA_OK) return st;
  const bool packed = dev->cu_seqlens != nullptr;
  const int64_t tokens = packed ? T : (int64_t)B * T;
  const size_t esz = dt == KDA_BF16 ? 2 : 4;
  const size_t th = (size_t)tokens * H;
  const size_t state1 = (size_t)H * dk * dv * sizeof(float);  // one sequence's state
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void* hin[] = {host->q, host->k, host->v, host->log_alpha, host->beta};
  for (const void* p : hin)
    if (th > 0 && !p) return KDA_ERR_INVALID_ARG;
  Piece pc[kHostPieces];
  // One piece (every copy, the forward, the copies back, in order on `stream`)
  // for packed batches and where a token-sliced sequence has no final-state
  // buffer to carry its state; otherwise pieces whose copies in, forward and
  // copies out overlap across three streams.
  int np = (packed || tokens == 0 || (B == 1 && !dev->final_state)) ? 1 : plan_pieces(B, T, pc);
  for (int i = 0; i < np; ++i)  // beta rows are H floats: a piece must start on a 16-byte boundary
    if ((((int64_t)pc[i].b0 * T + pc[i].t0) * H * 4) % 16 != 0) np = 1;
  if (np == 1) pc[0] = {0, B, 0, T};
  // Token tensors of a piece: rows [t0, t1) of sequences [b0, b1), one 2-D copy
  // (a row per sequence) per tensor.
  const size_t wq = (size_t)H * dk * esz, wv = (size_t)H * dv * esz, wg = (size_t)H * dk * 4, wb = (size_t)H * 4;
  auto copy_tokens = [&](const Piece& p, cudaStream_t cs, bool in) -> bool {
    const int64_t rows = packed ? 1 : p.b1 - p.b0;
    const int64_t len = packed ? T : p.t1 - p.t0;
    if (rows == 0 || len == 0) return true;
    const int64_t first = packed ? 0 : (int64_t)p.b0 * T + p.t0;  // first token of the piece
    struct C {
      void* d;
      const void* h;
      size_t w;
    };
    if (in) {
      const C cs_in[] = {{const_cast<void*>(dev->q), host->q, wq},
                         {const_cast<void*>(dev->k), host->k, wq},
                         {const_cast<void*>(dev->v), host->v, wv},
                         {const_cast<float*>(dev->log_alpha), host->log_alpha, wg},
                         {const_cast<float*>(dev->beta), host->beta, wb}};
      for (const C& c : cs_in) {
        char* d = static_cast<char*>(c.d) + first * c.w;
        const char* h = static_cast<const char*>(c.h) + first * c.w;
        if (cudaMemcpy2DAsync(d, T * c.w, h, T * c.w, len * c.w, rows, cudaMemcpyHostToDevice, cs) != cudaSuccess)
          return false;
      }
    } else if (host->out) {
      char* h = static_cast<char*>(host->out) + first * wv;
      const char* d = static_cast<const char*>(dev->out) + first * wv;
      if (cudaMemcpy2DAsync(h, T * wv, d, T * wv, len * wv, rows, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return false;
    }
    return true;
  };
  const size_t states = (size_t)B * state1;  // B sequences (packed: B = N)
  if (np == 1) {  // everything in order on the caller's stream
    if (!copy_tokens(pc[0], s, true)) return KDA_ERR_CUDA;
    if (dev->init_state && states > 0 &&
        cudaMemcpyAsync(const_cast<float*>(dev->init_state), host->init_state, states, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
      return KDA_ERR_CUDA;
    if (packed && cudaMemcpyAsync(const_cast<int32_t*>(dev->cu_seqlens), host->cu_seqlens,
                                  (size_t)(B + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, s) != cudaSuccess)
      return KDA_ERR_CUDA;
    st = kda_fwd(dev->q, dev->k, dev->v, dev->log_alpha, dev->beta, dev->init_state, dev->out, dev->final_state, B,
                 T, H, dk, dv, dev->cu_seqlens, stream, dt, workspace, workspace_bytes);
    if (st != KDA_OK) return st;
    if (th > 0 && !copy_tokens(pc[0], s, false)) return KDA_ERR_CUDA;
    if (host->final_state && dev->final_state && states > 0 &&
        cudaMemcpyAsync(host->final_state, dev->final_state, states, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return KDA_ERR_CUDA;
    return KDA_OK;
  }
  if (!workspace || !aligned16(workspace) || workspace_bytes < kda_fwd_workspace_size(B, T, H, dk, dv, dt))
    return KDA_ERR_WORKSPACE;
  int devid = 0;
  if (cudaGetDevice(&devid) != cudaSuccess) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = host_pipe(devid);
  if (!hp) return KDA_ERR_CUDA;
  // The copy streams start after the work already on `stream` (which may
  // still read the device buffers), and `stream` ends after the last copy out.
  if (cudaEventRecord(hp->start, s) != cudaSuccess || cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (dev->init_state && cudaMemcpyAsync(const_cast<float*>(dev->init_state), host->init_state, (size_t)B * state1,
                                         cudaMemcpyHostToDevice, hp->in) != cudaSuccess)
    return KDA_ERR_CUDA;
  for (int i = 0; i < np; ++i) {
    const Piece& p = pc[i];
    if (!copy_tokens(p, hp->in, true) || cudaEventRecord(hp->ev_in[i], hp->in) != cudaSuccess ||
        cudaStreamWaitEvent(s, hp->ev_in[i], 0) != cudaSuccess)
      return KDA_ERR_CUDA;
    const int Bp = p.b1 - p.b0;
    const int64_t Tp = p.t1 - p.t0, first = (int64_t)p.b0 * T + p.t0;
    // A token slice after the first continues from the state the previous
    // slice left in final_state (read and overwritten in place).
    const float* init = B == 1 ? (i == 0 ? dev->init_state : dev->final_state)
                               : (dev->init_state ? dev->init_state + (size_t)p.b0 * state1 / 4 : nullptr);
    float* fin = dev->final_state ? dev->final_state + (size_t)p.b0 * state1 / 4 : nullptr;
    st = fwd_impl(static_cast<const char*>(dev->q) + first * wq, static_cast<const char*>(dev->k) + first * wq,
                  static_cast<const char*>(dev->v) + first * wv, dev->log_alpha + first * H * dk,
                  dev->beta + first * H, init, static_cast<char*>(dev->out) + first * wv, fin, Bp, Tp, H, dk, dv,
                  nullptr, stream, dt, workspace, workspace_bytes, nullptr, kWaitNs, 0, kda::ModeArgs(), i == 0);
    if (st != KDA_OK) return st;
    if (cudaEventRecord(hp->ev_comp[i], s) != cudaSuccess || cudaStreamWaitEvent(hp->out, hp->ev_comp[i], 0) != cudaSuccess ||
        !copy_tokens(p, hp->out, false))
      return KDA_ERR_CUDA;
  }
  if (host->final_state && dev->final_state &&
      cudaMemcpyAsync(host->final_state, dev->final_state, (size_t)B * state1, cudaMemcpyDeviceToHost, hp->out) !=
          cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaEventRecord(hp->done, hp->out) != cudaSuccess || cudaStreamWaitEvent(s, hp->done, 0) != cudaSuccess)
    return KDA_ERR_CUDA;
  return KDA_OK;
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

kda_status_t kda_decode_step_gated(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                                   float g_min, const float* beta, float* state, void* out, int B, int H, int dk,
                                   int dv, void* stream, kda_dtype_t dt) {
  if (B < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const void* req[] = {q, k, v, z, A_log, beta, state, out};
  for (const void* p : req)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if ((int64_t)B * H > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  cudaError_t e = kda::launch_decode_gated(q, k, v, z, A_log, g_min, beta, state, out, B, H, dk, dv,
                                           dt == KDA_BF16, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

static kda_status_t spec_impl(const void* qp, const void* kp, const void* vp, const void* gp, const float* bp,
                              const int32_t* n_accepted, const void* q, const void* k, const void* v, const void* g,
                              const float* beta, const float* A_log, float g_min, float* state, void* out, int B,
                              int Wp, int W, int H, int dk, int dv, void* stream, kda_dtype_t dt) {
  if (B < 0 || H <= 0 || Wp < 0 || W < 0) return KDA_ERR_INVALID_ARG;
  if (Wp + W > KDA_SPEC_MAX_TOKENS) return KDA_ERR_UNSUPPORTED;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (!state || !aligned16(state)) return KDA_ERR_INVALID_ARG;
  if (W > 0) {
    const void* req[] = {q, k, v, g, beta, out};
    for (const void* p : req)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  }
  if (Wp > 0) {
    const void* req[] = {qp, kp, vp, gp, bp, n_accepted};
    for (const void* p : req)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  }
  if ((int64_t)B * H > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  cudaError_t e = kda::launch_spec(qp, kp, vp, gp, bp, Wp > 0 ? n_accepted : nullptr, q, k, v, g, beta, state, out,
                                   B, Wp, W, H, dk, dv, dt == KDA_BF16, A_log, g_min,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_decode_spec(const void* q_prev, const void* k_prev, const void* v_prev, const float* log_alpha_prev,
                             const float* beta_prev, const int32_t* n_accepted, const void* q, const void* k,
                             const void* v, const float* log_alpha, const float* beta, float* state, void* out,
                             int B, int Wp, int W, int H, int dk, int dv, void* stream, kda_dtype_t dt) {
  return spec_impl(q_prev, k_prev, v_prev, log_alpha_prev, beta_prev, n_accepted, q, k, v, log_alpha, beta, nullptr,
                   0.f, state, out, B, Wp, W, H, dk, dv, stream, dt);
}

kda_status_t kda_decode_spec_gated(const void* q_prev, const void* k_prev, const void* v_prev, const void* z_prev,
                                   const float* beta_prev, const int32_t* n_accepted, const void* q, const void* k,
                                   const void* v, const void* z, const float* beta, const float* A_log, float g_min,
                                   float* state, void* out, int B, int Wp, int W, int H, int dk, int dv,
                                   void* stream, kda_dtype_t dt) {
  if (!A_log || !aligned16(A_log)) return KDA_ERR_INVALID_ARG;
  return spec_impl(q_prev, k_prev, v_prev, z_prev, beta_prev, n_accepted, q, k, v, z, beta, A_log, g_min, state,
                   out, B, Wp, W, H, dk, dv, stream, dt);
}

kda_status_t kda_workspace_status(const void* workspace, void* stream) {
  if (!workspace || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  kda::DeviceStatus h{};
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  return static_cast<kda_status_t>(h.code);
}

// ---- the model's input prologue fused into the prefill ----
kda_status_t kda_fwd_gated(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                           float g_min, const float* beta, const float* init_state, void* out, float* final_state,
                           int B, int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, void* stream,
                           kda_dtype_t dt, void* workspace, size_t workspace_bytes) {
  if (!A_log || !aligned16(A_log)) return KDA_ERR_INVALID_ARG;
  kda::ModeArgs ma;
  ma.mode = kda::MODE_GATED;
  ma.A_log = A_log;
  ma.g_min = g_min;
  // The decay logits travel in the log-decay slot; validation checks them
  // as one more token tensor.
  return fwd_impl(q, k, v, static_cast<const float*>(z), beta, init_state, out, final_state, B, T, H, dk, dv,
                  cu_seqlens, stream, dt, workspace, workspace_bytes, nullptr, kWaitNs, 0, ma);
}

// ---- interval checkpoints (prefix-cache states) ----
static size_t order_bytes(int N) { return ((size_t)(N > 0 ? N : 0) * sizeof(int32_t) + 255) / 256 * 256; }

size_t kda_fwd_checkpoints_workspace_size(int B, int64_t T, int H, int dk, int dv, kda_dtype_t dt) {
  return kda_fwd_workspace_size(B, T, H, dk, dv, dt) + order_bytes(B);
}

kda_status_t kda_fwd_checkpoints(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const float* beta, const float* init_state, void* out, float* final_state, int B,
                                 int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, void* stream,
                                 kda_dtype_t dt, float* checkpoints, int interval, int64_t capacity,
                                 void* workspace, size_t workspace_bytes) {
  if (interval <= 0 || interval % 64 != 0) return KDA_ERR_UNSUPPORTED;
  if (capacity < 0 || (capacity > 0 && (!checkpoints || !aligned16(checkpoints)))) return KDA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < kda_fwd_checkpoints_workspace_size(B, T, H, dk, dv, dt))
    return KDA_ERR_WORKSPACE;
  if (!cu_seqlens && B > 0 && (int64_t)B * (T / interval) > capacity) return KDA_ERR_INVALID_ARG;
  kda::ModeArgs ma;
  ma.mode = kda::MODE_CKPT;
  ma.ckpt = checkpoints;
  ma.ckpt_interval = interval;
  ma.ckpt_every = interval / 64;
  ma.ckpt_capacity = capacity;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cu_seqlens && B > 0) {
    if (!aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    int32_t* base = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                               kda_fwd_workspace_size(B, T, H, dk, dv, dt));
    if (kda::launch_ckpt_base(cu_seqlens, B, interval, base, s) != cudaSuccess) return KDA_ERR_CUDA;
    ma.ckpt_base = base;
  }
  return fwd_impl(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, cu_seqlens, stream, dt,
                  workspace, workspace_bytes, nullptr, kWaitNs, 0, ma);
}

// ---- segment pieces, composition, correction (context parallelism) ----
kda_status_t kda_segment_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                             const float* beta, float* out_zero, float* state_zero, float* qhat,
                             float* transition, int B, int64_t T, int H, int dk, int dv,
                             const int32_t* cu_seqlens, void* stream, kda_dtype_t dt, void* workspace,
                             size_t workspace_bytes) {
  if (dk != dv) return KDA_ERR_UNSUPPORTED;
  // out_zero and qhat are both set, or both NULL (states only)
  if ((out_zero == nullptr) != (qhat == nullptr)) return KDA_ERR_INVALID_ARG;
  if (B > 0 && (!state_zero || !transition)) return KDA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)out_zero, (const void*)qhat, (const void*)state_zero, (const void*)transition})
    if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
  kda::ModeArgs ma;
  ma.mode = kda::MODE_SEG;
  ma.o32 = out_zero;
  ma.qhat32 = qhat;
  ma.trans = transition;
  return fwd_impl(q, k, v, log_alpha, beta, nullptr, nullptr, state_zero, B, T, H, dk, dv, cu_seqlens, stream, dt,
                  workspace, workspace_bytes, nullptr, kWaitNs, 0, ma);
}

kda_status_t kda_state_compose(const float* transition, const float* state_zero, const float* init_state,
                               float* state_in, float* final_state, int R, int N, int H, int dk, int dv,
                               int rank_major, void* stream) {
  if (R < 0 || N < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (R > 0 && N > 0 && (!transition || !state_zero)) return KDA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)transition, (const void*)state_zero, (const void*)init_state,
                        (const void*)state_in, (const void*)final_state})
    if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (N == 0) return KDA_OK;
  cudaError_t e = kda::launch_compose(transition, state_zero, init_state, state_in, final_state, R, N, H, dk, dv,
                                      rank_major ? 1 : 0, 0, 1, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_output_correct(const float* out_zero, const float* qhat, const float* state_in, void* out, int B,
                                int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, void* stream,
                                kda_dtype_t dt) {
  if (B < 0 || T < 0 || H <= 0 || (dt != KDA_F32 && dt != KDA_BF16)) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const int64_t tokens = cu_seqlens ? T : (int64_t)B * T;
  if (tokens > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (tokens > 0 && (!out_zero || !qhat || !state_in || !out)) return KDA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)out_zero, (const void*)qhat, (const void*)state_in, (const void*)out,
                        (const void*)cu_seqlens})
    if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (tokens == 0 || B == 0) return KDA_OK;
  cudaError_t e = kda::launch_correct(out_zero, qhat, state_in, out, cu_seqlens, B, cu_seqlens ? 0 : T, tokens, H,
                                      dk, dv, dt == KDA_BF16, 0, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---- intra-device context parallelism ----
namespace {
struct CpLayout {
  size_t seg_cu, order, s0, trans, s_in, fin, total;
};
CpLayout cp_layout(int B, int H, int dk, int dv, int n_seg) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t P = (size_t)(B > 0 ? B : 0) * (size_t)(n_seg > 0 ? n_seg : 1);
  const size_t st = P * H * (size_t)dk * dv * sizeof(float);
  CpLayout L;
  size_t off = kStatusBytes;
  L.seg_cu = off; off += up((P + 1) * sizeof(int32_t));
  L.order = off; off += up(P * sizeof(int32_t));
  L.s0 = off; off += up(st);
  L.trans = off; off += up(P * H * (size_t)dk * dk * sizeof(float));
  L.s_in = off; off += up(st);
  L.fin = off; off += up(st);
  L.total = off;
  return L;
}
}  // namespace

size_t kda_fwd_cp_workspace_size(int B, int64_t T, int H, int dk, int dv, kda_dtype_t dt, int n_seg) {
  (void)T; (void)dt;
  return cp_layout(B, H, dk, dv, n_seg).total;
}

int kda_cp_segments(int N, int64_t tokens_per_sequence, int H, int sm_count) {
  // The state pass runs 2 n_seg - 3 blocks per (sequence, head) for n_seg >= 2
  // (the first segment from its initial state, the middle ones as zero-start
  // and transition runs, the last one not at all) and the output pass n_seg;
  // both must fit one wave of blocks on the SMs.  A segment keeps at least
  // eight 64-token chunks, and the split must shorten the serial depth:
  // two passes of L / n_seg each against one of L.
  const int64_t chains = (int64_t)N * H;
  if (chains <= 0 || sm_count <= 0) return 1;
  int best = 1;
  for (int r = 3; r <= 64; ++r) {
    if (chains * (2 * r - 3) > sm_count || chains * r > sm_count) break;
    if (tokens_per_sequence / r < 8 * 64) break;
    best = r;
  }
  return best;
}

kda_status_t kda_fwd_cp(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                        const float* init_state, void* out, float* final_state, int B, int64_t T, int H, int dk,
                        int dv, const int32_t* cu_seqlens, void* stream, kda_dtype_t dt, int n_seg,
                        void* workspace, size_t workspace_bytes) {
  if (n_seg < 1 || n_seg > 4096) return KDA_ERR_INVALID_ARG;
  if (dk != dv) return KDA_ERR_UNSUPPORTED;
  kda_status_t st = validate_fwd(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, dt);
  if (st != KDA_OK) return st;
  if (cu_seqlens && !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARG;
  const int64_t tokens = cu_seqlens ? T : (int64_t)B * T;
  if (tokens > (int64_t)INT32_MAX || (int64_t)B * n_seg > (int64_t)INT32_MAX / 4) return KDA_ERR_UNSUPPORTED;
  const CpLayout L = cp_layout(B, H, dk, dv, n_seg);
  if (!workspace || !aligned16(workspace) || workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(kda::DeviceStatus), s) != cudaSuccess) return KDA_ERR_CUDA;
  if (B == 0) return KDA_OK;
  const int P = B * n_seg;
  int32_t* seg_cu = reinterpret_cast<int32_t*>(ws + L.seg_cu);
  int32_t* order = reinterpret_cast<int32_t*>(ws + L.order);
  float* s0 = reinterpret_cast<float*>(ws + L.s0);
  float* tr = reinterpret_cast<float*>(ws + L.trans);
  float* s_in = reinterpret_cast<float*>(ws + L.s_in);
  float* fin_seg = reinterpret_cast<float*>(ws + L.fin);
  kda::DeviceStatus* status = reinterpret_cast<kda::DeviceStatus*>(ws);
  const bool tc = kda::fwd_tc_supported(dk, dv, dt == KDA_BF16) && tokens > 0;
  const bool bf16 = dt == KDA_BF16;
  if (kda::launch_segment_cu(cu_seqlens, cu_seqlens ? 0 : T, B, n_seg, seg_cu, s) != cudaSuccess)
    return KDA_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  // Pass 1 (states only): the first segment of every sequence from its
  // initial state, the middle ones as zero-start and transition runs; the
  // segments form a packed batch of P sequences over the same token tensors.
  if (n_seg > 1) {
    kda::ModeArgs ma;
    ma.mode = kda::MODE_SEG;
    ma.seg_per_seq = n_seg;
    ma.trans = tr;
    kda::FwdArgs a{q, k, v, log_alpha, beta, init_state, nullptr, s0, seg_cu, P, tokens, H, dk, dv, status, nullptr};
    e = tc ? kda::launch_fwd_tc_impl(a, s, kWaitNs, 0, order, ma) : kda::launch_fwd_simt(a, bf16, s, ma);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
  }
  // Every segment's incoming state: S_in(0) = init, S_in(1) = the first
  // segment's state, S_in(r+1) = S~_r + M_r S_in(r).
  e = kda::launch_compose(tr, s0, init_state, s_in, nullptr, n_seg, B, H, dk, dv, 0, 1, 0, s);
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  // Pass 2: the ordinary forward over all segments from their incoming states.
  kda::FwdArgs a2{q, k, v, log_alpha, beta, s_in, out, final_state ? fin_seg : nullptr, seg_cu, P, tokens, H, dk, dv,
                  status, nullptr};
  e = tc ? kda::launch_fwd_tc_impl(a2, s, kWaitNs, 0, order, kda::ModeArgs())
         : kda::launch_fwd_simt(a2, bf16, s);
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  // The final state of each sequence is the one after its last segment.
  if (final_state) {
    const size_t head_states = (size_t)H * dk * dv * sizeof(float);
    if (cudaMemcpy2DAsync(final_state, head_states, fin_seg + (size_t)(n_seg - 1) * H * dk * dv,
                          head_states * n_seg, head_states, B, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return KDA_ERR_CUDA;
  }
  return KDA_OK;
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
