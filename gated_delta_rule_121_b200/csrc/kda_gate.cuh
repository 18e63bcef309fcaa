// The model's input prologue around the recurrence (Kimi K3 digest, "Kimi
// Delta Attention" section: q and k are L2-normalised, the decay logits z
// get a per-head scale; "Bounded decay" section: the log-decay is the scaled
// sigmoid g = g_min * sigmoid(exp(A_h) * z), in (g_min, 0), with g_min = -5
// in the model's configuration).
#pragma once
#include <cuda_runtime.h>

namespace kda {

// Epsilon under the square root of the L2 normalisation, x / sqrt(|x|^2 + eps);
// it only matters for vectors of norm ~1e-3 or below.
constexpr float L2NORM_EPS = 1e-6f;

__device__ __forceinline__ float l2norm_scale(float sumsq) { return rsqrtf(sumsq + L2NORM_EPS); }

// g = g_min * sigmoid(exp(A) * z) = g_min / (1 + exp(-exp(A) z)).
__device__ __forceinline__ float gate_log_decay(float z, float A, float g_min) {
  return g_min / (1.f + __expf(-__expf(A) * z));
}

}  // namespace kda
