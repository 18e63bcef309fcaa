// Speculative-decode verification with KDA state replay (Kimi K3 digest,
// serving section, "speculative decoding and KDA state rewind").
//
// The decode state is updated in place, so once verification rejects some
// draft tokens the state has already moved past the last accepted one and
// cannot simply be rolled back; keeping a snapshot per draft position would
// multiply the state traffic.  Instead the projected inputs of the draft
// window are kept (they are far smaller than the state), the accepted
// tokens' states are rebuilt on chip, and only the committed state is
// written back.  One kernel runs, per (sequence, head), in one recurrence
// loop:
//   1. replay: the first n_accepted[b] tokens of the previous window (their
//      outputs were produced when they were drafted; only the state moves);
//   2. the new window: token 0 (the bonus token, certain) and the next draft
//      tokens, each with its output;
// and writes the state back once, right after the bonus token.  The draft
// tokens' states live only in registers.
//
// Per token: S' = Diag(e^g) S; u = S'^T k; p = S'^T q; delta = beta (v - u);
// o = p + (q.k) delta; S = S' + k delta^T (the recurrence of the digest's
// KDA section, read with the updated state).  The state is streamed from HBM
// once and written once; each thread keeps ROWS x 4 of it in registers.
//
// GATED: the inputs are the raw ones of the model's prologue (digest, KDA
// section and "Bounded decay" section): q and k are L2-normalised per token
// and head, and the decay is g = g_min * sigmoid(exp(A_h) * z) from the decay
// logits z.
#include "kda_gate.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct SpecShape {
  static constexpr int COLQ = DV / 4;                               // float4 column groups
  static constexpr int RG = (256 / COLQ) < DK ? (256 / COLQ) : DK;  // row groups
  static constexpr int ROWS = DK / RG;
  static constexpr int NT = COLQ * RG;
};

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
  const int tid = threadIdx.x, cq = tid % COLQ, rg = tid / COLQ;
  int na = n_accepted ? n_accepted[b] : 0;
  na = na < 0 ? 0 : (na > Wp ? Wp : na);
  const int nt = na + W;  // tokens run through the recurrence
  // shared layout (floats): per token k, q, alpha [DK] and v [DV] (multiples
  // of 16 floats each), beta and q.k (each padded to a multiple of 4), then
  // the two reduction buffers [2][2][RG][COLQ] of float4, 16-byte aligned.
  const int nt4 = (nt + 3) & ~3;
  float* s_k = ssm;
  float* s_q = s_k + nt * DK;
  float* s_a = s_q + nt * DK;
  float* s_v = s_a + nt * DK;
  float* s_b = s_v + nt * DV;
  float* s_qk = s_b + nt4;
  float4* s_red = reinterpret_cast<float4*>(s_qk + nt4);

  float4* S = reinterpret_cast<float4*>(state + ((int64_t)b * H + h) * DK * DV);
  float4 s[ROWS];
#pragma unroll
  for (int m = 0; m < ROWS; ++m) s[m] = __ldcs(S + (rg * ROWS + m) * COLQ + cq);

  // Stage every token: the replayed ones from the previous window, then the new window.
  for (int t = 0; t < nt; ++t) {
    const bool rep = t < na;
    const SpecTok& src = rep ? prev : cur;
    const int64_t row = ((int64_t)b * (rep ? Wp : W) + (rep ? t : t - na)) * H + h;
    for (int i = tid; i < DK; i += NT) {
      s_k[t * DK + i] = to_f32(static_cast<const IO*>(src.k)[row * DK + i]);
      s_q[t * DK + i] = to_f32(static_cast<const IO*>(src.q)[row * DK + i]);
      if constexpr (GATED)
        s_a[t * DK + i] = __expf(gate_log_decay(to_f32(static_cast<const IO*>(src.g)[row * DK + i]), A_log[h], g_min));
      else
        s_a[t * DK + i] = __expf(static_cast<const float*>(src.g)[row * DK + i]);
    }
    for (int i = tid; i < DV; i += NT) s_v[t * DV + i] = to_f32(static_cast<const IO*>(src.v)[row * DV + i]);
    if (tid == 0) s_b[t] = src.beta[row];
  }
  __syncthreads();
  // Per token: q.k, and (gated) the L2 normalisation of q and k; one warp per token.
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < nt; t += NT / 32) {
      float qq = 0.f, kk = 0.f, qk = 0.f;
      for (int i = lane; i < DK; i += 32) {
        const float a = s_q[t * DK + i], c = s_k[t * DK + i];
        qq += a * a;
        kk += c * c;
        qk += a * c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        qq += __shfl_xor_sync(0xffffffffu, qq, o);
        kk += __shfl_xor_sync(0xffffffffu, kk, o);
        qk += __shfl_xor_sync(0xffffffffu, qk, o);
      }
      if constexpr (GATED) {
        const float rq = l2norm_scale(qq), rk = l2norm_scale(kk);
        for (int i = lane; i < DK; i += 32) {
          s_q[t * DK + i] *= rq;
          s_k[t * DK + i] *= rk;
        }
        qk *= rq * rk;
      }
      if (lane == 0) s_qk[t] = qk;
    }
  }
  __syncthreads();

  IO* o_base = out + ((int64_t)b * W * H + h) * DV + 4 * cq;
  for (int t = 0; t < nt; ++t) {
    const bool emit = t >= na;  // tokens of the new window produce outputs
    float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), pp = pu;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
      const int i = rg * ROWS + m;
      const float a = s_a[t * DK + i], ki = s_k[t * DK + i], qi = s_q[t * DK + i];
      s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
      pu.x += s[m].x * ki; pu.y += s[m].y * ki; pu.z += s[m].z * ki; pu.w += s[m].w * ki;
      pp.x += s[m].x * qi; pp.y += s[m].y * qi; pp.z += s[m].z * qi; pp.w += s[m].w * qi;
    }
    float4* red = s_red + (t & 1) * 2 * RG * COLQ;  // double-buffered: one barrier per token
    red[rg * COLQ + cq] = pu;
    red[(RG + rg) * COLQ + cq] = pp;
    __syncthreads();
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = u;
#pragma unroll 8
    for (int r = 0; r < RG; ++r) {
      const float4 a = red[r * COLQ + cq], c = red[(RG + r) * COLQ + cq];
      u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
      p.x += c.x; p.y += c.y; p.z += c.z; p.w += c.w;
    }
    const float bt = s_b[t];
    const float* vv = s_v + t * DV + 4 * cq;
    const float4 d = make_float4(bt * (vv[0] - u.x), bt * (vv[1] - u.y), bt * (vv[2] - u.z), bt * (vv[3] - u.w));
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
      const float ki = s_k[t * DK + rg * ROWS + m];
      s[m].x += ki * d.x; s[m].y += ki * d.y; s[m].z += ki * d.z; s[m].w += ki * d.w;
    }
    if (emit && rg == 0) {
      const float qk = s_qk[t];
      IO* o = o_base + (int64_t)(t - na) * H * DV;
      o[0] = from_f32<IO>(p.x + qk * d.x);
      o[1] = from_f32<IO>(p.y + qk * d.y);
      o[2] = from_f32<IO>(p.z + qk * d.z);
      o[3] = from_f32<IO>(p.w + qk * d.w);
    }
    if (t == na) {  // the bonus token: the state to keep
#pragma unroll
      for (int m = 0; m < ROWS; ++m) __stcs(S + (rg * ROWS + m) * COLQ + cq, s[m]);
    }
  }
  if (W == 0) {  // nothing new: keep the replayed state
#pragma unroll
    for (int m = 0; m < ROWS; ++m) __stcs(S + (rg * ROWS + m) * COLQ + cq, s[m]);
  }
}

template <int DK, int DV, bool GATED>
cudaError_t launch_spec_t(const SpecTok& prev, const SpecTok& cur, const int32_t* na, float* state, void* out,
                          int B, int Wp, int W, int H, bool bf16, const float* A_log, float g_min, cudaStream_t s) {
  using Sh = SpecShape<DK, DV>;
  const int ntmax = Wp + W;
  const size_t smem = sizeof(float) * ((size_t)ntmax * (3 * DK + DV) + 2 * (size_t)((ntmax + 3) & ~3)) +
                      sizeof(float4) * 4 * Sh::RG * Sh::COLQ;
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
