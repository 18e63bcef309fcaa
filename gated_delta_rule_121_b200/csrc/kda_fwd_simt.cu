// Token-serial KDA forward on CUDA cores, exact fp32 arithmetic.
//
// This path serves fp32 inputs (whose accuracy contract forbids rounding
// operands to TF32 or bf16) and the (dk, dv) shapes that have no tensor-core
// kernel.  It runs the recurrence of the Kimi K3 digest's "Kimi Delta
// Attention" section token by token:
//   S' = Diag(exp g_t) S;  u = S'^T k_t;  S = S' + beta_t k_t (v_t - u)^T;
//   o_t = S^T q_t.
//
// Work split: one block per (sequence, head, 32-column block of dv).  Columns
// of S evolve independently (each v-channel sees the same k, g, beta), so
// the dv split needs no communication.  Within a block, a warp owns 8
// columns; its 32 lanes are 8 columns x 4 row groups, and lane (rg, j) keeps
// rows i = 4m + rg of column j in registers.  Both per-token reductions over
// rows (u and o) are 4-lane shuffles inside the warp, so the token loop has
// no block barrier; barriers appear only when a chunk of TOK tokens is
// staged in shared memory.
#include "kda_gate.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int TOK = 16;  // tokens staged per shared-memory round

// MODE (FwdMode): MODE_CKPT also writes the state every ma.ckpt_interval
// tokens of each sequence; MODE_SEG runs every (sequence, head, column block)
// twice, the second time (blocks from `units` on) as the transition run:
// values taken as zero, identity start, outputs and final state to qhat32
// and trans (dk == dv); MODE_GATED takes the decay logits in `g` (dtype IO)
// and normalises q and k per token (the model's prologue, kda_gate.cuh).
template <int DK, int DVB, typename IO, int MODE>
__global__ void __launch_bounds__(DVB * 4)
    kda_fwd_simt_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                        const float* __restrict__ g, const float* __restrict__ beta,
                        const float* __restrict__ init, IO* __restrict__ out, float* __restrict__ fin,
                        const int32_t* __restrict__ cu, int64_t Tper, int H, int dv, const ModeArgs ma,
                        int units, DeviceStatus* status) {
  constexpr int R = DK / 4;  // rows per lane
  constexpr int NT = DVB * 4;
  __shared__ float s_k[TOK][DK], s_q[TOK][DK], s_a[TOK][DK];
  __shared__ float s_v[TOK][DVB], s_b[TOK], s_o[TOK][DVB];

  const int nblk = dv / DVB;
  int bid = blockIdx.x;
  bool trans = false;
  if constexpr (MODE == MODE_SEG) {
    trans = bid >= units;
    if (trans) bid -= units;
    if (trans) fin = ma.trans;
  }
  const int blk = bid % nblk;
  const int h = (bid / nblk) % H;
  const int n = bid / (nblk * H);
  // MODE_SEG: a sequence's first segment runs from its initial state with
  // ordinary outputs and needs no transition run.
  const bool first = MODE == MODE_SEG && ma.seg_per_seq > 0 && n % ma.seg_per_seq == 0;
  const bool last = MODE == MODE_SEG && ma.seg_per_seq > 0 && n % ma.seg_per_seq == ma.seg_per_seq - 1;
  if ((first && trans) || (last && !first)) return;
  float* const obuf = trans ? ma.qhat32 : ma.o32;  // MODE_SEG: null = states only
  if (MODE == MODE_SEG && !first) init = nullptr;
  int64_t t0, L;
  if (cu) {
    t0 = cu[n];
    L = (int64_t)cu[n + 1] - t0;
  } else {
    t0 = (int64_t)n * Tper;
    L = Tper;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = lane >> 3, jc = lane & 7;
  const int jl = warp * 8 + jc;       // column within the block
  const int j = blk * DVB + jl;       // column of S / v / o
  const int64_t sbase = ((int64_t)n * H + h) * DK * dv;
  const int64_t ibase = first ? ((int64_t)(n / ma.seg_per_seq) * H + h) * DK * dv : sbase;

  float s[R];
#pragma unroll
  for (int m = 0; m < R; ++m) {
    s[m] = init ? init[ibase + (int64_t)(4 * m + rg) * dv + j] : 0.f;
    if (MODE == MODE_SEG && !first) s[m] = (trans && 4 * m + rg == j) ? 1.f : 0.f;
  }
  int64_t ckpt0 = 0;
  if constexpr (MODE == MODE_CKPT)
    ckpt0 = ma.ckpt_base ? ma.ckpt_base[n] : (int64_t)n * (Tper / ma.ckpt_interval);

  for (int64_t c0 = 0; c0 < L; c0 += TOK) {
    const int nt = (int)((L - c0) < TOK ? (L - c0) : TOK);
    __syncthreads();
    for (int e = tid; e < TOK * DK; e += NT) {
      const int r = e / DK, i = e % DK;
      float kk = 0.f, qq = 0.f, aa = 1.f;
      if (r < nt) {
        const int64_t row = ((t0 + c0 + r) * H + h) * DK + i;
        kk = to_f32(k[row]);
        qq = to_f32(q[row]);
        if constexpr (MODE == MODE_GATED)
          aa = __expf(gate_log_decay(to_f32(reinterpret_cast<const IO*>(g)[row]), ma.A_log[h], ma.g_min));
        else
          aa = __expf(g[row]);
      }
      s_k[r][i] = kk; s_q[r][i] = qq; s_a[r][i] = aa;
    }
    for (int e = tid; e < TOK * DVB; e += NT) {
      const int r = e / DVB, c = e % DVB;
      s_v[r][c] = (r < nt && !trans) ? to_f32(v[((t0 + c0 + r) * H + h) * dv + blk * DVB + c]) : 0.f;
    }
    if (tid < TOK) s_b[tid] = tid < nt ? beta[(t0 + c0 + tid) * H + h] : 0.f;
    __syncthreads();
    if constexpr (MODE == MODE_GATED) {  // L2-normalise the staged q and k rows, one warp per token
      for (int r = warp; r < nt; r += NT / 32) {
        float sq = 0.f, sk = 0.f;
        for (int i = lane; i < DK; i += 32) {
          sq += s_q[r][i] * s_q[r][i];
          sk += s_k[r][i] * s_k[r][i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sq += __shfl_xor_sync(0xffffffffu, sq, o);
          sk += __shfl_xor_sync(0xffffffffu, sk, o);
        }
        const float fq = l2norm_scale(sq), fk = l2norm_scale(sk);
        for (int i = lane; i < DK; i += 32) {
          s_q[r][i] *= fq;
          s_k[r][i] *= fk;
        }
      }
      __syncthreads();
    }

    for (int r = 0; r < nt; ++r) {
      float pu = 0.f;
#pragma unroll
      for (int m = 0; m < R; ++m) {
        const int i = 4 * m + rg;
        s[m] *= s_a[r][i];
        pu += s[m] * s_k[r][i];
      }
      pu += __shfl_xor_sync(0xffffffffu, pu, 8);
      pu += __shfl_xor_sync(0xffffffffu, pu, 16);
      const float d = s_b[r] * (s_v[r][jl] - pu);
      float po = 0.f;
#pragma unroll
      for (int m = 0; m < R; ++m) {
        const int i = 4 * m + rg;
        s[m] += s_k[r][i] * d;
        po += s[m] * s_q[r][i];
      }
      po += __shfl_xor_sync(0xffffffffu, po, 8);
      po += __shfl_xor_sync(0xffffffffu, po, 16);
      if (rg == 0) s_o[r][jl] = po;
      if constexpr (MODE == MODE_CKPT) {
        const int64_t done = c0 + r + 1;  // tokens of this sequence processed so far
        if (done % ma.ckpt_interval == 0) {
          const int64_t slot = ckpt0 + done / ma.ckpt_interval - 1;
          if (slot < ma.ckpt_capacity) {
            float* dst = ma.ckpt + (slot * H + h) * DK * dv;
#pragma unroll
            for (int m = 0; m < R; ++m) dst[(int64_t)(4 * m + rg) * dv + j] = s[m];
          } else if (status && rg == 0 && jl == 0) {
            record_error(status, KDA_ERR_INVALID_ARG, 41);
          }
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < nt * DVB; e += NT) {
      const int r = e / DVB, c = e % DVB;
      const int64_t o = ((t0 + c0 + r) * H + h) * dv + blk * DVB + c;
      if (MODE == MODE_SEG) {
        if (obuf) obuf[o] = s_o[r][c];
      } else {
        out[o] = from_f32<IO>(s_o[r][c]);
      }
    }
  }
  if (fin) {
#pragma unroll
    for (int m = 0; m < R; ++m) fin[sbase + (int64_t)(4 * m + rg) * dv + j] = s[m];
  }
}

template <int DK, typename IO, int MODE>
cudaError_t launch_k(const FwdArgs& a, cudaStream_t st, const ModeArgs& ma) {
  const int DVB = a.dv < 32 ? a.dv : 32;
  const int units = (int)((int64_t)a.N * a.H * (a.dv / DVB));
  const unsigned blocks = (unsigned)(MODE == MODE_SEG ? 2 * (int64_t)units : (int64_t)units);
  if (blocks == 0) return cudaSuccess;
  const int64_t Tper = a.cu ? 0 : a.T;
#define KDA_SIMT_LAUNCH(DVB_)                                                                            \
  kda_fwd_simt_kernel<DK, DVB_, IO, MODE><<<blocks, DVB_ * 4, 0, st>>>(                                  \
      (const IO*)a.q, (const IO*)a.k, (const IO*)a.v, a.g, a.beta, a.init, (IO*)a.out, a.fin, a.cu, Tper, \
      a.H, a.dv, ma, units, a.status)
  if (DVB == 16) KDA_SIMT_LAUNCH(16);
  else KDA_SIMT_LAUNCH(32);
#undef KDA_SIMT_LAUNCH
  return cudaGetLastError();
}

template <typename IO, int MODE>
cudaError_t launch_io(const FwdArgs& a, cudaStream_t s, const ModeArgs& ma) {
  switch (a.dk) {
    case 16: return launch_k<16, IO, MODE>(a, s, ma);
    case 32: return launch_k<32, IO, MODE>(a, s, ma);
    case 64: return launch_k<64, IO, MODE>(a, s, ma);
    case 128: return launch_k<128, IO, MODE>(a, s, ma);
  }
  return cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_mode(const FwdArgs& a, bool bf16, cudaStream_t s, const ModeArgs& ma) {
  return bf16 ? launch_io<__nv_bfloat16, MODE>(a, s, ma) : launch_io<float, MODE>(a, s, ma);
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, bool bf16, cudaStream_t s, const ModeArgs& ma) {
  switch (ma.mode) {
    case MODE_CKPT: return launch_mode<MODE_CKPT>(a, bf16, s, ma);
    case MODE_SEG: return launch_mode<MODE_SEG>(a, bf16, s, ma);
    case MODE_GATED: return launch_mode<MODE_GATED>(a, bf16, s, ma);
    default: return launch_mode<MODE_PLAIN>(a, bf16, s, ma);
  }
}

}  // namespace kda
