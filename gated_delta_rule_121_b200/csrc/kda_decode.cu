// Single-token KDA decode: the recurrence step applied once per (sequence,
// head), with the fp32 state updated in place (Kimi K3 digest, serving
// section, "speculative decoding and KDA state rewind": at decode time the
// cost is managing the in-place-updated recurrent state).
//
// Per head, with S the dk x dv state (row i = key channel i):
//   S'    = Diag(exp g) S                      (forget)
//   u     = S'^T k,   p = S'^T q
//   delta = beta (v - u)
//   o     = S''^T q = p + (q.k) delta          (read uses the updated state)
//   S''   = S' + k delta^T                      (erase + write), stored back
//
// The state is streamed from HBM exactly once and written once: each thread
// keeps ROWS x 4 state values in registers between the read and the write.
// A warp covers whole rows (128 contiguous fp32 = 512 B per load for dv=128),
// loads and stores use streaming cache hints, and the two cross-row
// reductions go through shared memory.  The path is bound by HBM bandwidth:
// 2 * dk * dv * 4 bytes of state traffic per head.
//
// GATED: the token's inputs are those of the model's prologue (q and k
// L2-normalised here; the decay from the decay logits, g = g_min *
// sigmoid(exp(A_h) z), see kda_gate.cuh).
#include "kda_gate.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct DecodeShape {
  static constexpr int COLQ = DV / 4;                                    // float4 column groups
  static constexpr int RG = (256 / COLQ) < DK ? (256 / COLQ) : DK;       // row groups
  static constexpr int ROWS = DK / RG;                                   // rows per thread
  static constexpr int NT = COLQ * RG;                                   // threads per block
};

template <int DK, int DV, typename IO, bool GATED>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
    kda_decode_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                      const void* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                      IO* __restrict__ out, const float* __restrict__ A_log, float g_min, int H) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int COLQ = Sh::COLQ, RG = Sh::RG, ROWS = Sh::ROWS, NT = Sh::NT;
  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ float4 s_ru[RG][COLQ], s_rp[RG][COLQ];
  __shared__ float s_qk;

  const int tid = threadIdx.x;
  const int cq = tid % COLQ, rg = tid / COLQ;
  const int64_t bh = blockIdx.x;
  float4* S = reinterpret_cast<float4*>(state + bh * DK * DV);

  // Issue the state loads first; they are in flight while the token is staged.
  float4 s[ROWS];
#pragma unroll
  for (int m = 0; m < ROWS; ++m) s[m] = __ldcs(S + (rg * ROWS + m) * COLQ + cq);

  for (int i = tid; i < DK; i += NT) {
    s_k[i] = to_f32(k[bh * DK + i]);
    s_q[i] = to_f32(q[bh * DK + i]);
    if constexpr (GATED)
      s_a[i] = __expf(gate_log_decay(to_f32(static_cast<const IO*>(g)[bh * DK + i]), A_log[bh % H], g_min));
    else
      s_a[i] = __expf(static_cast<const float*>(g)[bh * DK + i]);
  }
  __syncthreads();
  // q.k, and for GATED the L2 norms of q and k: every warp reduces them itself
  // (no further block barrier); the rows are scaled as they are used.
  float fq = 1.f, fk = 1.f;
  if constexpr (GATED) {
    float qq = 0.f, kk = 0.f, qk = 0.f;
    for (int i = tid & 31; i < DK; i += 32) {
      const float a = s_q[i], b = s_k[i];
      qq += a * a;
      kk += b * b;
      qk += a * b;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      qq += __shfl_xor_sync(0xffffffffu, qq, o);
      kk += __shfl_xor_sync(0xffffffffu, kk, o);
      qk += __shfl_xor_sync(0xffffffffu, qk, o);
    }
    fq = l2norm_scale(qq);
    fk = l2norm_scale(kk);
    if (tid == 0) s_qk = qk * fq * fk;
  } else if (tid < 32) {
    float acc = 0.f;
    for (int i = tid; i < DK; i += 32) acc += s_q[i] * s_k[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (tid == 0) s_qk = acc;
  }

  float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), pp = pu;
#pragma unroll
  for (int m = 0; m < ROWS; ++m) {
    const int i = rg * ROWS + m;
    const float a = s_a[i], ki = s_k[i] * fk, qi = s_q[i] * fq;
    s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
    pu.x += s[m].x * ki; pu.y += s[m].y * ki; pu.z += s[m].z * ki; pu.w += s[m].w * ki;
    pp.x += s[m].x * qi; pp.y += s[m].y * qi; pp.z += s[m].z * qi; pp.w += s[m].w * qi;
  }
  s_ru[rg][cq] = pu;
  s_rp[rg][cq] = pp;
  __syncthreads();
  float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = u;
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    const float4 a = s_ru[r][cq], b = s_rp[r][cq];
    u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
    p.x += b.x; p.y += b.y; p.z += b.z; p.w += b.w;
  }
  const float bt = beta[bh];
  const IO* vv = v + bh * DV + 4 * cq;
  float4 d;
  d.x = bt * (to_f32(vv[0]) - u.x);
  d.y = bt * (to_f32(vv[1]) - u.y);
  d.z = bt * (to_f32(vv[2]) - u.z);
  d.w = bt * (to_f32(vv[3]) - u.w);
#pragma unroll
  for (int m = 0; m < ROWS; ++m) {
    const float ki = s_k[rg * ROWS + m] * fk;
    s[m].x += ki * d.x; s[m].y += ki * d.y; s[m].z += ki * d.z; s[m].w += ki * d.w;
    __stcs(S + (rg * ROWS + m) * COLQ + cq, s[m]);
  }
  if (rg == 0) {
    const float qk = s_qk;
    IO* o = out + bh * DV + 4 * cq;
    o[0] = from_f32<IO>(p.x + qk * d.x);
    o[1] = from_f32<IO>(p.y + qk * d.y);
    o[2] = from_f32<IO>(p.z + qk * d.z);
    o[3] = from_f32<IO>(p.w + qk * d.w);
  }
}

template <int DK, int DV, bool GATED>
cudaError_t launch_dims(const void* q, const void* k, const void* v, const void* g, const float* beta,
                        float* state, void* out, int B, int H, bool bf16, const float* A_log, float g_min,
                        cudaStream_t s) {
  const unsigned blocks = (unsigned)((int64_t)B * H);
  constexpr int NT = DecodeShape<DK, DV>::NT;
  if (bf16) {
    using T = __nv_bfloat16;
    kda_decode_kernel<DK, DV, T, GATED><<<blocks, NT, 0, s>>>((const T*)q, (const T*)k, (const T*)v, g, beta,
                                                             state, (T*)out, A_log, g_min, H);
  } else {
    kda_decode_kernel<DK, DV, float, GATED><<<blocks, NT, 0, s>>>((const float*)q, (const float*)k,
                                                                 (const float*)v, g, beta, state, (float*)out,
                                                                 A_log, g_min, H);
  }
  return cudaGetLastError();
}

template <int DK, bool GATED>
cudaError_t launch_dv(const void* q, const void* k, const void* v, const void* g, const float* beta,
                      float* state, void* out, int B, int H, int dv, bool bf16, const float* A_log, float g_min,
                      cudaStream_t s) {
  switch (dv) {
    case 16: return launch_dims<DK, 16, GATED>(q, k, v, g, beta, state, out, B, H, bf16, A_log, g_min, s);
    case 32: return launch_dims<DK, 32, GATED>(q, k, v, g, beta, state, out, B, H, bf16, A_log, g_min, s);
    case 64: return launch_dims<DK, 64, GATED>(q, k, v, g, beta, state, out, B, H, bf16, A_log, g_min, s);
    case 128: return launch_dims<DK, 128, GATED>(q, k, v, g, beta, state, out, B, H, bf16, A_log, g_min, s);
  }
  return cudaErrorInvalidValue;
}

template <bool GATED>
cudaError_t launch_decode_g(const void* q, const void* k, const void* v, const void* g, const float* beta,
                            float* state, void* out, int B, int H, int dk, int dv, bool bf16, const float* A_log,
                            float g_min, cudaStream_t s) {
  switch (dk) {
    case 16: return launch_dv<16, GATED>(q, k, v, g, beta, state, out, B, H, dv, bf16, A_log, g_min, s);
    case 32: return launch_dv<32, GATED>(q, k, v, g, beta, state, out, B, H, dv, bf16, A_log, g_min, s);
    case 64: return launch_dv<64, GATED>(q, k, v, g, beta, state, out, B, H, dv, bf16, A_log, g_min, s);
    case 128: return launch_dv<128, GATED>(q, k, v, g, beta, state, out, B, H, dv, bf16, A_log, g_min, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state, void* out, int B, int H, int dk, int dv, bool bf16, cudaStream_t s) {
  return launch_decode_g<false>(q, k, v, g, beta, state, out, B, H, dk, dv, bf16, nullptr, 0.f, s);
}

cudaError_t launch_decode_gated(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                                float g_min, const float* beta, float* state, void* out, int B, int H, int dk,
                                int dv, bool bf16, cudaStream_t s) {
  return launch_decode_g<true>(q, k, v, z, beta, state, out, B, H, dk, dv, bf16, A_log, g_min, s);
}

}  // namespace kda
