// Internal declarations shared by the KDA CUDA sources (not part of the ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/kda.h"

namespace kda {

// Status word at the start of every kda_fwd workspace.  Kernels record the
// first device-side failure here (atomicCAS from KDA_OK).
struct DeviceStatus {
  int code;
  int where;  // which wait gave up (kernel-specific id), for diagnostics
  int pad[2];
};

__device__ __forceinline__ void record_error(DeviceStatus* st, int code, int where) {
  if (st && atomicCAS(&st->code, KDA_OK, code) == KDA_OK) st->where = where;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Arguments of one forward call after host-side validation.
struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  const float* init;
  void* out;
  float* fin;
  const int32_t* cu;  // device offsets or nullptr
  int N;              // number of sequences
  int64_t T;          // tokens per sequence (cu == nullptr) or total tokens
  int H, dk, dv;
  DeviceStatus* status;
  void* dbg;          // optional debug dump (test hook), may be nullptr
};

// What a forward launch produces besides out / final state.
enum FwdMode {
  MODE_PLAIN = 0,  // out and final state
  MODE_CKPT = 1,   // plus the state every `ckpt_every` chunks of each sequence
  MODE_GATED = 3,  // the model's input prologue in the kernel: `g` holds the decay
                   // logits z (dtype of q), g = g_min sigmoid(exp(A_h) z), and q, k
                   // are L2-normalised per token and head
  MODE_SEG = 2,    // segment pieces: two runs per (sequence, head), both with
                   // fp32 outputs and no init state: the zero-start run
                   // (outputs o32, final state fin) and the transition run
                   // (values taken as zero, identity start: outputs qhat32,
                   // final state = the transition, written to trans)
};

struct ModeArgs {
  int mode = MODE_PLAIN;
  // MODE_CKPT
  float* ckpt = nullptr;              // [capacity][H][dk][dv]
  const int32_t* ckpt_base = nullptr; // first checkpoint slot of each sequence (packed batches)
  int ckpt_every = 0;                 // interval in 64-token chunks (tensor-core path) ...
  int ckpt_interval = 0;              // ... and in tokens
  int64_t ckpt_capacity = 0;
  // MODE_SEG
  float* o32 = nullptr;     // [T_total][H][dv]
  float* qhat32 = nullptr;  // [T_total][H][dk]
  float* trans = nullptr;   // [N][H][dk][dk]
  int seg_per_seq = 0;      // > 0: the batch is N/seg_per_seq sequences cut into that many
                            // consecutive segments; the first segment of each runs from the
                            // sequence's initial state and has no transition run, and the
                            // last segment of each is skipped (its pieces are not needed)
                            // Outputs of MODE_SEG runs are written only when o32 / qhat32 are
                            // set (kda_fwd_cp needs states only).
  // MODE_GATED
  const float* A_log = nullptr;  // [H] per-head log scale of the decay logits
  float g_min = -5.0f;           // lower bound of the log decay
};

// Launchers (return a CUDA error code; launches are asynchronous).
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state, void* out, int B, int H, int dk, int dv, bool bf16, cudaStream_t s);
cudaError_t launch_decode_gated(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                                float g_min, const float* beta, float* state, void* out, int B, int H, int dk,
                                int dv, bool bf16, cudaStream_t s);
cudaError_t launch_spec(const void* qp, const void* kp, const void* vp, const void* gp, const float* bp,
                        const int32_t* n_accepted, const void* q, const void* k, const void* v, const void* g,
                        const float* beta, float* state, void* out, int B, int Wp, int W, int H, int dk, int dv,
                        bool bf16, const float* A_log, float g_min, cudaStream_t s);
cudaError_t launch_fwd_simt(const FwdArgs& a, bool bf16, cudaStream_t s, const ModeArgs& m = ModeArgs());
bool fwd_tc_supported(int dk, int dv, bool bf16);
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t s);

}  // namespace kda
