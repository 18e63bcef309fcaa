// Speculative-decode verification with KDA state replay (Kimi K3 digest,
// serving section, "speculative decoding and KDA state rewind").
//
// The decode state is updated in place, so once verification rejects some
// draft tokens the state has already moved past the last accepted one and
// cannot simply be rolled back; keeping a snapshot per draft position would
// multiply the state traffic.  Instead the projected inputs of the draft
// window are kept (they are far smaller than the state), the accepted
// tokens' states are rebuilt on chip, and only the committed state is
// written back.  Per (sequence, head) one block takes, as ONE chunk of n
// tokens: the first n_accepted[b] tokens of the previous window (replayed:
// no outputs), then the new window, whose token 0 is the bonus token and the
// rest the next drafts (outputs for all of them); the state written back is
// the one after the bonus token.
//
// Chunk form of the recurrence (the digest's KDA section; every decay factor
// is formed between the two tokens it connects, so none exceeds 1), with the
// in-chunk cumulative log-decay G_t = sum_{s<=t} g_s per key channel and the
// incoming state S0:
//   X_t = S0^T (e^{G_t} * k_t),   Y_t = S0^T (e^{G_t} * q_t)
//   A_ts = sum_c k_tc k_sc e^{G_tc - G_sc} (s < t),  P_ts = sum_c q_tc k_sc e^{G_tc - G_sc} (s <= t)
//   delta_t = beta_t (v_t - X_t - sum_{s<t} A_ts delta_s)      (forward substitution)
//   o_t = Y_t + sum_{s<=t} P_ts delta_s
//   S_c = Diag(e^{G_c}) S0 + sum_{s<=c} (k_s * e^{G_c - G_s}) delta_s^T   (c: the bonus token)
// So the state is read once into registers (ROWS x 4 values per thread) and
// written once; what grows with the window is two dot products per token
// against those registers plus an n x n triangular system, with no block
// barrier in the token loop: a column group's RG row groups are lanes of one
// warp, so the reductions over rows are shuffles.
//
// GATED: the inputs are the raw ones of the model's prologue (digest, KDA
// section and "Bounded decay" section): q and k are L2-normalised per token
// and head, and the decay is g = g_min * sigmoid(exp(A_h) * z) from the decay
// logits z.
#include "../../include/kda.h"
#include "kda_gate.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct SpecShape {
  static constexpr int COLQ = DV / 4;                                  // float4 column groups
  static constexpr int RG0 = (256 / COLQ) < DK ? (256 / COLQ) : DK;
  static constexpr int RG = RG0 < 32 ? RG0 : 32;                       // row groups: lanes of one warp
  static constexpr int ROWS = DK / RG;                                 // rows per thread
  static constexpr int NT = COLQ * RG;                                 // threads per block
};

// Shared-memory floats of a block for chunks of up to `n` tokens.
template <int DK, int DV>
constexpr size_t spec_smem_floats(int n) {
  const size_t n4 = (size_t)((n + 3) & ~3);
  return 3 * (size_t)n * DK + 2 * (size_t)n * DV + 2 * (size_t)n * n4 + n4 + DK;
}

struct SpecTok {  // where one token's inputs live
  const void* q;
  const void* k;
  const void* v;
  const void* g;  // fp32 log-decay, or the decay logits (dtype IO) when gated
  const float* beta;
};

template <int DK, int DV, typename IO, bool GATED>
__global__ void __launch_bounds__(SpecShape<DK, DV>::NT)
    kda_spec_kernel(SpecTok prev, SpecTok cur, const int32_t* __restrict__ n_accepted, float* __restrict__ state,
                    IO* __restrict__ out, int Wp, int W, int H, const float* __restrict__ A_log, float g_min) {
  using Sh = SpecShape<DK, DV>;
  constexpr int COLQ = Sh::COLQ, RG = Sh::RG, ROWS = Sh::ROWS, NT = Sh::NT;
  extern __shared__ float ssm[];
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int tid = threadIdx.x, rg = tid % RG, cq = tid / RG, lane = tid & 31, warp = tid >> 5;
  int na = n_accepted ? n_accepted[b] : 0;
  na = na < 0 ? 0 : (na > Wp ? Wp : na);
  const int n = na + W;               // tokens of the chunk
  const int c = W > 0 ? na : na - 1;  // the token after which the state is kept (-1: none, unchanged)
  if (c < 0) return;
  // shared layout (floats; every array starts on a multiple of 4 floats):
  //   s_k, s_q, s_G [n][DK]  k, q, G; then e^G k, e^G q and k_t e^{G_c - G_t}
  //   s_v, s_d [n][DV]       values, delta
  //   s_A, s_P [n][n4]       pair sums;  s_b [n4] beta;  s_gc [DK] e^{G_c}
  const int n4 = (n + 3) & ~3;
  float* s_k = ssm;
  float* s_q = s_k + n * DK;
  float* s_G = s_q + n * DK;
  float* s_v = s_G + n * DK;
  float* s_d = s_v + n * DV;
  float* s_A = s_d + n * DV;
  float* s_P = s_A + n * n4;
  float* s_b = s_P + n * n4;
  float* s_gc = s_b + n4;

  float4* S = reinterpret_cast<float4*>(state + ((int64_t)b * H + h) * DK * DV);
  float4 s[ROWS];  // rows m * RG + rg, columns 4 cq .. 4 cq + 3
#pragma unroll
  for (int m = 0; m < ROWS; ++m) s[m] = __ldcs(S + (m * RG + rg) * COLQ + cq);

  // ---- stage the chunk: the replayed tokens, then the new window.  Every
  // thread issues all of its loads before it uses any (the window is at most
  // KDA_SPEC_MAX_TOKENS tokens), so their latencies overlap each other and
  // the state loads above.
  auto src_row = [&](int t) {
    return t < na ? ((int64_t)b * Wp + t) * H + h : ((int64_t)b * W + (t - na)) * H + h;
  };
  {
    constexpr int PK = (KDA_SPEC_MAX_TOKENS * DK + NT - 1) / NT, PV = (KDA_SPEC_MAX_TOKENS * DV + NT - 1) / NT;
    float rk[PK], rq[PK], rg2[PK], rv[PV];
#pragma unroll
    for (int j = 0; j < PK; ++j) {
      const int e = tid + j * NT;
      if (e < n * DK) {
        const int t = e / DK, i = e % DK;
        const SpecTok& src = t < na ? prev : cur;
        const int64_t o = src_row(t) * DK + i;
        rk[j] = to_f32(static_cast<const IO*>(src.k)[o]);
        rq[j] = to_f32(static_cast<const IO*>(src.q)[o]);
        if constexpr (GATED)
          rg2[j] = to_f32(static_cast<const IO*>(src.g)[o]);
        else
          rg2[j] = static_cast<const float*>(src.g)[o];
      }
    }
#pragma unroll
    for (int j = 0; j < PV; ++j) {
      const int e = tid + j * NT;
      if (e < n * DV) {
        const int t = e / DV, i = e % DV;
        rv[j] = to_f32(static_cast<const IO*>((t < na ? prev : cur).v)[src_row(t) * DV + i]);
      }
    }
    const float bt = tid < n ? (tid < na ? prev : cur).beta[src_row(tid)] : 0.f;
    const float Ah = GATED ? A_log[h] : 0.f;
#pragma unroll
    for (int j = 0; j < PK; ++j) {
      const int e = tid + j * NT;
      if (e < n * DK) {
        s_k[e] = rk[j];
        s_q[e] = rq[j];
        s_G[e] = GATED ? gate_log_decay(rg2[j], Ah, g_min) : rg2[j];
      }
    }
#pragma unroll
    for (int j = 0; j < PV; ++j) {
      const int e = tid + j * NT;
      if (e < n * DV) s_v[e] = rv[j];
    }
    if (tid < n) s_b[tid] = bt;
  }
  __syncthreads();
  if constexpr (GATED) {  // L2-normalise q and k per token, one warp per token
    for (int t = warp; t < n; t += NT / 32) {
      float qq = 0.f, kk = 0.f;
      for (int i = lane; i < DK; i += 32) {
        qq += s_q[t * DK + i] * s_q[t * DK + i];
        kk += s_k[t * DK + i] * s_k[t * DK + i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        qq += __shfl_xor_sync(0xffffffffu, qq, o);
        kk += __shfl_xor_sync(0xffffffffu, kk, o);
      }
      const float fq = l2norm_scale(qq), fk = l2norm_scale(kk);
      for (int i = lane; i < DK; i += 32) {
        s_q[t * DK + i] *= fq;
        s_k[t * DK + i] *= fk;
      }
    }
    __syncthreads();
  }
  // cumulative log-decay over the chunk, one thread per key channel
  for (int i = tid; i < DK; i += NT) {
    float acc = 0.f;
    for (int t = 0; t < n; ++t) {
      acc += s_G[t * DK + i];
      s_G[t * DK + i] = acc;
    }
  }
  __syncthreads();
  // ---- pair sums, one warp per pair (t, s), s <= t
  for (int p = warp; p < n * (n + 1) / 2; p += NT / 32) {
    int t = 0;
    while ((t + 1) * (t + 2) / 2 <= p) ++t;
    const int s2 = p - t * (t + 1) / 2;
    float pa = 0.f, pp = 0.f;
    for (int i = lane; i < DK; i += 32) {
      const float ke = s_k[s2 * DK + i] * __expf(s_G[t * DK + i] - s_G[s2 * DK + i]);  // decay s -> t, <= 1
      pa += s_k[t * DK + i] * ke;
      pp += s_q[t * DK + i] * ke;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pa += __shfl_xor_sync(0xffffffffu, pa, o);
      pp += __shfl_xor_sync(0xffffffffu, pp, o);
    }
    if (lane == 0) {
      s_A[t * n4 + s2] = pa;
      s_P[t * n4 + s2] = pp;
    }
  }
  __syncthreads();
  // ---- per-token operands in place: e^{G_t} k_t, e^{G_t} q_t, k_t e^{G_c - G_t} (t <= c)
  for (int i = tid; i < DK; i += NT) {
    const float gc = s_G[c * DK + i];
    s_gc[i] = __expf(gc);
    for (int t = 0; t < n; ++t) {
      const float G = s_G[t * DK + i], kk = s_k[t * DK + i];
      const float eg = __expf(G);
      s_k[t * DK + i] = eg * kk;
      s_q[t * DK + i] *= eg;
      s_G[t * DK + i] = t <= c ? kk * __expf(gc - G) : 0.f;
    }
  }
  __syncthreads();

  // ---- token loop: X_t, Y_t by row-group shuffles, delta_t by substitution, o_t
  IO* o_base = out + ((int64_t)b * W * H + h) * DV + 4 * cq;
  for (int t = 0; t < n; ++t) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
      const int i = m * RG + rg;
      const float gk = s_k[t * DK + i], gq = s_q[t * DK + i];
      x.x += s[m].x * gk; x.y += s[m].y * gk; x.z += s[m].z * gk; x.w += s[m].w * gk;
      y.x += s[m].x * gq; y.y += s[m].y * gq; y.z += s[m].z * gq; y.w += s[m].w * gq;
    }
#pragma unroll
    for (int o = 1; o < RG; o <<= 1) {
      x.x += __shfl_xor_sync(0xffffffffu, x.x, o); x.y += __shfl_xor_sync(0xffffffffu, x.y, o);
      x.z += __shfl_xor_sync(0xffffffffu, x.z, o); x.w += __shfl_xor_sync(0xffffffffu, x.w, o);
      y.x += __shfl_xor_sync(0xffffffffu, y.x, o); y.y += __shfl_xor_sync(0xffffffffu, y.y, o);
      y.z += __shfl_xor_sync(0xffffffffu, y.z, o); y.w += __shfl_xor_sync(0xffffffffu, y.w, o);
    }
    const float* vv = s_v + t * DV + 4 * cq;
    float4 d = make_float4(vv[0] - x.x, vv[1] - x.y, vv[2] - x.z, vv[3] - x.w);
    for (int s2 = 0; s2 < t; ++s2) {
      const float a = s_A[t * n4 + s2];
      const float4 ds = *reinterpret_cast<const float4*>(s_d + s2 * DV + 4 * cq);
      d.x -= a * ds.x; d.y -= a * ds.y; d.z -= a * ds.z; d.w -= a * ds.w;
    }
    const float bt = s_b[t];
    d.x *= bt; d.y *= bt; d.z *= bt; d.w *= bt;
    if (rg == 0) *reinterpret_cast<float4*>(s_d + t * DV + 4 * cq) = d;
    if (t >= na && rg == RG - 1) {  // another lane of the group writes the output
      float4 o = y;
      for (int s2 = 0; s2 < t; ++s2) {
        const float pq = s_P[t * n4 + s2];
        const float4 ds = *reinterpret_cast<const float4*>(s_d + s2 * DV + 4 * cq);
        o.x += pq * ds.x; o.y += pq * ds.y; o.z += pq * ds.z; o.w += pq * ds.w;
      }
      const float pq = s_P[t * n4 + t];
      o.x += pq * d.x; o.y += pq * d.y; o.z += pq * d.z; o.w += pq * d.w;
      IO* dst = o_base + (int64_t)(t - na) * H * DV;
      dst[0] = from_f32<IO>(o.x);
      dst[1] = from_f32<IO>(o.y);
      dst[2] = from_f32<IO>(o.z);
      dst[3] = from_f32<IO>(o.w);
    }
    __syncwarp();  // delta_t is visible to the group's lanes for the next tokens
  }
  // ---- the kept state: S_c = Diag(e^{G_c}) S0 + sum_{s<=c} (k_s e^{G_c - G_s}) delta_s^T
#pragma unroll
  for (int m = 0; m < ROWS; ++m) {
    const int i = m * RG + rg;
    const float eg = s_gc[i];
    float4 a = make_float4(s[m].x * eg, s[m].y * eg, s[m].z * eg, s[m].w * eg);
    for (int t = 0; t <= c; ++t) {
      const float kc = s_G[t * DK + i];
      const float4 ds = *reinterpret_cast<const float4*>(s_d + t * DV + 4 * cq);
      a.x += kc * ds.x; a.y += kc * ds.y; a.z += kc * ds.z; a.w += kc * ds.w;
    }
    __stcs(S + (m * RG + rg) * COLQ + cq, a);
  }
}

template <int DK, int DV, bool GATED>
cudaError_t launch_spec_t(const SpecTok& prev, const SpecTok& cur, const int32_t* na, float* state, void* out,
                          int B, int Wp, int W, int H, bool bf16, const float* A_log, float g_min, cudaStream_t s) {
  using Sh = SpecShape<DK, DV>;
  const size_t smem = sizeof(float) * spec_smem_floats<DK, DV>(Wp + W);
  const unsigned blocks = (unsigned)((int64_t)B * H);
  if (bf16) {
    auto* kern = kda_spec_kernel<DK, DV, __nv_bfloat16, GATED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<blocks, Sh::NT, smem, s>>>(prev, cur, na, state, (__nv_bfloat16*)out, Wp, W, H, A_log, g_min);
  } else {
    auto* kern = kda_spec_kernel<DK, DV, float, GATED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<blocks, Sh::NT, smem, s>>>(prev, cur, na, state, (float*)out, Wp, W, H, A_log, g_min);
  }
  return cudaGetLastError();
}

template <int DK, bool GATED>
cudaError_t launch_spec_dv(const SpecTok& prev, const SpecTok& cur, const int32_t* na, float* state, void* out,
                           int B, int Wp, int W, int H, int dv, bool bf16, const float* A_log, float g_min,
                           cudaStream_t s) {
  switch (dv) {
    case 16: return launch_spec_t<DK, 16, GATED>(prev, cur, na, state, out, B, Wp, W, H, bf16, A_log, g_min, s);
    case 32: return launch_spec_t<DK, 32, GATED>(prev, cur, na, state, out, B, Wp, W, H, bf16, A_log, g_min, s);
    case 64: return launch_spec_t<DK, 64, GATED>(prev, cur, na, state, out, B, Wp, W, H, bf16, A_log, g_min, s);
    case 128: return launch_spec_t<DK, 128, GATED>(prev, cur, na, state, out, B, Wp, W, H, bf16, A_log, g_min, s);
  }
  return cudaErrorInvalidValue;
}

template <bool GATED>
cudaError_t launch_spec_g(const SpecTok& prev, const SpecTok& cur, const int32_t* na, float* state, void* out,
                          int B, int Wp, int W, int H, int dk, int dv, bool bf16, const float* A_log, float g_min,
                          cudaStream_t s) {
  switch (dk) {
    case 16: return launch_spec_dv<16, GATED>(prev, cur, na, state, out, B, Wp, W, H, dv, bf16, A_log, g_min, s);
    case 32: return launch_spec_dv<32, GATED>(prev, cur, na, state, out, B, Wp, W, H, dv, bf16, A_log, g_min, s);
    case 64: return launch_spec_dv<64, GATED>(prev, cur, na, state, out, B, Wp, W, H, dv, bf16, A_log, g_min, s);
    case 128: return launch_spec_dv<128, GATED>(prev, cur, na, state, out, B, Wp, W, H, dv, bf16, A_log, g_min, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_spec(const void* qp, const void* kp, const void* vp, const void* gp, const float* bp,
                        const int32_t* n_accepted, const void* q, const void* k, const void* v, const void* g,
                        const float* beta, float* state, void* out, int B, int Wp, int W, int H, int dk, int dv,
                        bool bf16, const float* A_log, float g_min, cudaStream_t s) {
  const SpecTok prev{qp, kp, vp, gp, bp}, cur{q, k, v, g, beta};
  return A_log ? launch_spec_g<true>(prev, cur, n_accepted, state, out, B, Wp, W, H, dk, dv, bf16, A_log, g_min, s)
               : launch_spec_g<false>(prev, cur, n_accepted, state, out, B, Wp, W, H, dk, dv, bf16, A_log, g_min, s);
}

}  // namespace kda
