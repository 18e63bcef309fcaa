// Segment decomposition of the KDA state scan: the kernels that compose
// segment pieces and correct zero-start outputs (Kimi K3 digest, "KDA
// algorithm-system co-design", paragraphs on intra-device context
// parallelism and on KDA context parallelism, KCP).
//
// With the transition form of the recurrence, S_t = M_t S_{t-1} + beta_t
// k_t v_t^T, M_t = (I - beta_t k_t k_t^T) Diag(alpha_t), the state after a
// segment that starts from S_in is
//     S_end = S~ + M S_in,
// where S~ is the segment's state from a zero start and M = M_last ... M_first
// its transition; both depend only on the segment's own tokens.  Inside the
// segment the output of token t is, by the same linearity,
//     o_t = o~_t + S_in^T qhat_t,   qhat_t = M_{t<-first}^T q_t,
// with o~ the zero-start output.  The forward kernels produce (o~, S~) and
// (qhat, M) per segment (MODE_SEG); this file holds
//   - the composition S_in[r+1] = S~_r + M_r S_in[r] over the segments of a
//     sequence (a sequential prefix, fp32 on CUDA cores, one block per
//     (sequence, head, 32 value columns): the columns of S evolve
//     independently), and
//   - the correction o_t = o~_t + S_in^T qhat_t (dense 64-token x dv tiles on
//     the warp-level tensor path with tf32 operands rounded to nearest; the
//     zero-start output o~ stays fp32, so the result is rounded once).  For
//     fp32 outputs, whose contract allows no tf32 rounding, every product is
//     split into three tf32 products (hi*hi + hi*lo + lo*hi), accurate to
//     about fp32.
#include <cstdint>

#include "../../include/kda.h"
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

// ------------------------------------------------------------ composition
// 16-byte asynchronous global->shared copies (zero-filled when src_bytes = 0).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Pieces of sequence m: p = m * R + r (piece-major) or r * N + m (rank-major,
// the order of an all-gather over ranks).  state_in[p] = the state entering
// piece p; final_state[m] = the state after the last piece.  Each step stages
// the piece's transition M_p [DK][DK] in shared memory with asynchronous
// copies, then every thread forms its rows of S~_p + M_p cur for its column.
template <int DK>
__global__ void __launch_bounds__(256)
    compose_kernel(const float* __restrict__ trans, const float* __restrict__ s0, const float* __restrict__ init,
                   float* __restrict__ state_in, float* __restrict__ fin, int R, int N, int H, int dv,
                   int rank_major, int first_from_init, int apply_last) {
  constexpr int RPT = DK / 8;  // rows per thread: warp w holds rows w, w + 8, ...
  extern __shared__ float cm[];
  float* s_m = cm;                        // [DK][DK + 4]
  float* s_cur = cm + DK * (DK + 4);      // [DK][33]
  const int ncb = (dv + 31) / 32;
  const int cb = blockIdx.x % ncb;
  const int h = (blockIdx.x / ncb) % H;
  const int m = blockIdx.x / (ncb * H);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = cb * 32 + lane;
  const bool col = c < dv;
  const int64_t sd = (int64_t)DK * dv, mm = (int64_t)DK * DK;

  float cur[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int i = w + 8 * u;
    cur[u] = (init && col) ? init[((int64_t)m * H + h) * sd + (int64_t)i * dv + c] : 0.f;
  }
  for (int r = 0; r < R; ++r) {
    const int64_t p = rank_major ? (int64_t)r * N + m : (int64_t)m * R + r;
    const int64_t ph = p * H + h;
    // first_from_init: piece 0 already ran from the initial state, so its
    // "zero-start" state is the state after it and it has no transition.
    const bool skip_m = first_from_init && r == 0;
    if (r == R - 1 && !apply_last) {  // the last piece's incoming state is all that is wanted
#pragma unroll
      for (int u = 0; u < RPT; ++u)
        if (col && state_in) state_in[ph * sd + (int64_t)(w + 8 * u) * dv + c] = cur[u];
      break;
    }
    const float* Mp = trans + ph * mm;
    if (!skip_m) {
      for (int e = threadIdx.x; e < DK * DK / 4; e += 256) {
        const int i = e / (DK / 4), k4 = (e % (DK / 4)) * 4;
        cp_async16(s_m + i * (DK + 4) + k4, Mp + (int64_t)i * DK + k4, 16);
      }
    }
    float acc[RPT];
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      const int i = w + 8 * u;
      if (col && state_in) state_in[ph * sd + (int64_t)i * dv + c] = cur[u];
      s_cur[i * 33 + lane] = cur[u];
      acc[u] = col ? __ldg(s0 + ph * sd + (int64_t)i * dv + c) : 0.f;
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < (skip_m ? 0 : DK); ++kk) {
      const float sv = s_cur[kk * 33 + lane];
#pragma unroll
      for (int u = 0; u < RPT; ++u) acc[u] = fmaf(s_m[(w + 8 * u) * (DK + 4) + kk], sv, acc[u]);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < RPT; ++u) cur[u] = acc[u];
  }
  if (fin && col && apply_last) {
#pragma unroll
    for (int u = 0; u < RPT; ++u)
      fin[((int64_t)m * H + h) * sd + (int64_t)(w + 8 * u) * dv + c] = cur[u];
  }
}

// ------------------------------------------------------------ correction
constexpr int CPAD = 4;       // row padding (floats) of the shared tiles: conflict-free fragments

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Piece that holds packed token t: the last p with cu[p] <= t.
__device__ __forceinline__ int piece_of(const int32_t* cu, int P, int64_t t) {
  int lo = 0, hi = P - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Persistent blocks walk 64-token tiles (tile index i = head * ntiles +
// tile; block b takes a contiguous range of them, so consecutive tiles
// usually share the head and the piece), with a two-stage pipeline:
// while a tile is computed, the next tile's qhat rows and zero-start outputs
// are already landing in shared memory (asynchronous copies).  The incoming
// state S_in of a piece is staged once and kept while consecutive tiles stay
// in that piece.  Each of the 4 warps owns 16 tokens of a tile; K = DK in
// steps of 8.  A tile that straddles pieces is computed once per piece, each
// pass writing only its own rows; pieces p with p % skip_every == 0 ran from
// their initial state, so their (fp32) outputs are only rounded to IO.
constexpr int TT = 64;  // tokens per tile

template <int DK, int DV>
__device__ __forceinline__ void stage_tile(float* s_q, float* s_o, const float* qhat, const float* o32, int64_t t0,
                                           int nt, int h, int H) {
  for (int e = threadIdx.x; e < TT * (DK / 4); e += 128) {
    const int r = e / (DK / 4), c4 = (e % (DK / 4)) * 4;
    const int64_t t = t0 + (r < nt ? r : 0);
    cp_async16(s_q + r * (DK + CPAD) + c4, qhat + (t * H + h) * DK + c4, r < nt ? 16u : 0u);
  }
  for (int e = threadIdx.x; e < TT * (DV / 4); e += 128) {
    const int r = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
    const int64_t t = t0 + (r < nt ? r : 0);
    cp_async16(s_o + r * (DV + CPAD) + c4, o32 + (t * H + h) * DV + c4, r < nt ? 16u : 0u);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(128)
    correct_kernel(const float* __restrict__ o32, const float* __restrict__ qhat, const float* __restrict__ s_in,
                   IO* __restrict__ out, const int32_t* __restrict__ cu, int P, int64_t Tper, int64_t Ttot, int H,
                   int skip_every) {
  extern __shared__ float csm[];
  float* s_s = csm;                          // [DK][DV + CPAD]   S_in of the current piece
  float* s_q0 = s_s + DK * (DV + CPAD);      // [2][TT][DK + CPAD]
  float* s_o0 = s_q0 + 2 * TT * (DK + CPAD);  // [2][TT][DV + CPAD]
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, tq = lane & 3;
  const int64_t ntiles = (Ttot + TT - 1) / TT;
  const int64_t total = ntiles * H;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  int64_t i = (int64_t)blockIdx.x * per;
  const int64_t iend = i + per < total ? i + per : total;
  if (i >= iend) return;
  int cur_p = -1, cur_h = -1;  // piece/head whose S_in is staged
  int buf = 0;
  {
    const int h = (int)(i / ntiles);
    const int64_t t0 = (i % ntiles) * TT;
    stage_tile<DK, DV>(s_q0, s_o0, qhat, o32, t0, (int)((Ttot - t0) < TT ? (Ttot - t0) : TT), h, H);
  }
  for (; i < iend; ++i, buf ^= 1) {
    const int h = (int)(i / ntiles);
    const int64_t t0 = (i % ntiles) * TT;
    const int nt = (int)((Ttot - t0) < TT ? (Ttot - t0) : TT);
    float* s_q = s_q0 + buf * TT * (DK + CPAD);
    float* s_o = s_o0 + buf * TT * (DV + CPAD);
    // prefetch the next tile into the other buffer (its previous reader
    // finished at the barrier that ended the last iteration)
    const int64_t inext = i + 1;
    if (inext < iend) {
      const int hn = (int)(inext / ntiles);
      const int64_t tn = (inext % ntiles) * TT;
      stage_tile<DK, DV>(s_q0 + (buf ^ 1) * TT * (DK + CPAD), s_o0 + (buf ^ 1) * TT * (DV + CPAD), qhat, o32, tn,
                         (int)((Ttot - tn) < TT ? (Ttot - tn) : TT), hn, H);
      asm volatile("cp.async.wait_group 1;" ::: "memory");  // this tile's copies have landed
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const int p_first = cu ? piece_of(cu, P, t0) : (int)(t0 / Tper);
    const int p_last = cu ? piece_of(cu, P, t0 + nt - 1) : (int)((t0 + nt - 1) / Tper);
    for (int p = p_first; p <= p_last; ++p) {
      const int64_t lo = cu ? cu[p] : (int64_t)p * Tper, hi = cu ? cu[p + 1] : (int64_t)(p + 1) * Tper;
      if (hi <= lo) continue;  // empty piece
      if (skip_every > 0 && p % skip_every == 0) {  // outputs final: round this piece's rows
        for (int e = tid; e < nt * (DV / 4); e += 128) {
          const int r = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
          const int64_t t = t0 + r;
          if (t < lo || t >= hi) continue;
          const float* zo = s_o + r * (DV + CPAD) + c4;
          const int64_t base = (t * H + h) * DV + c4;
          out[base] = from_f32<IO>(zo[0]);
          out[base + 1] = from_f32<IO>(zo[1]);
          out[base + 2] = from_f32<IO>(zo[2]);
          out[base + 3] = from_f32<IO>(zo[3]);
        }
        continue;
      }
      if (p != cur_p || h != cur_h) {  // stage this piece's S_in (kept for the next tiles)
        __syncthreads();               // every warp is done with the previous S_in
        const float* S = s_in + ((int64_t)p * H + h) * DK * DV;
        for (int e = tid; e < DK * (DV / 4); e += 128) {
          const int r = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
          *reinterpret_cast<float4*>(s_s + r * (DV + CPAD) + c4) = __ldg(reinterpret_cast<const float4*>(S + r * DV + c4));
        }
        __syncthreads();
        cur_p = p;
        cur_h = h;
      }
      if (w * 16 >= nt) continue;
      float d[DV / 8][4];
#pragma unroll
      for (int n = 0; n < DV / 8; ++n) d[n][0] = d[n][1] = d[n][2] = d[n][3] = 0.f;
      const float* qa = s_q + (w * 16) * (DK + CPAD);
      constexpr bool SPLIT = sizeof(IO) == 4;  // fp32 outputs: three-term tf32 products
#pragma unroll 2
      for (int k0 = 0; k0 < DK; k0 += 8) {
        const float af[4] = {qa[g * (DK + CPAD) + k0 + tq], qa[(g + 8) * (DK + CPAD) + k0 + tq],
                             qa[g * (DK + CPAD) + k0 + tq + 4], qa[(g + 8) * (DK + CPAD) + k0 + tq + 4]};
        uint32_t a[4], al[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a[j] = tf32_rna(af[j]);
          if (SPLIT) al[j] = tf32_rna(af[j] - __uint_as_float(a[j]));
        }
#pragma unroll
        for (int n = 0; n < DV / 8; ++n) {
          const float bf[2] = {s_s[(k0 + tq) * (DV + CPAD) + n * 8 + g],
                               s_s[(k0 + tq + 4) * (DV + CPAD) + n * 8 + g]};
          uint32_t bb[2] = {tf32_rna(bf[0]), tf32_rna(bf[1])};
          mma_tf32_16x8x8(d[n], a, bb);
          if (SPLIT) {
            const uint32_t bl[2] = {tf32_rna(bf[0] - __uint_as_float(bb[0])), tf32_rna(bf[1] - __uint_as_float(bb[1]))};
            mma_tf32_16x8x8(d[n], a, bl);
            mma_tf32_16x8x8(d[n], al, bb);
          }
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = w * 16 + g + 8 * half;
        const int64_t t = t0 + r;
        if (r >= nt || t < lo || t >= hi) continue;
        const int64_t base = (t * H + h) * DV;
        const float* zo = s_o + r * (DV + CPAD);
#pragma unroll
        for (int n = 0; n < DV / 8; ++n) {
          const int c = n * 8 + 2 * tq;
          out[base + c] = from_f32<IO>(zo[c] + d[n][2 * half]);
          out[base + c + 1] = from_f32<IO>(zo[c + 1] + d[n][2 * half + 1]);
        }
      }
    }
    __syncthreads();  // the buffer of this tile may be refilled next iteration
  }
  cp_async_wait_all();  // no copy may still be landing when the block leaves
}

// ------------------------------------------------------------ segment layout
// Segment offsets for the intra-device split: sequence m of length L is cut
// into R segments at tokens c0 + floor(L r / R).  seg_cu[m R + r] is the start
// of segment r; seg_cu[N R] = the total token count.
__global__ void segment_cu_kernel(const int32_t* __restrict__ cu, int64_t Tper, int N, int R,
                                  int32_t* __restrict__ seg_cu) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i > (int64_t)N * R) return;
  if (i == (int64_t)N * R) {
    seg_cu[i] = cu ? cu[N] : (int32_t)(Tper * N);
    return;
  }
  const int m = (int)(i / R), r = (int)(i % R);
  const int64_t c0 = cu ? cu[m] : Tper * m;
  const int64_t L = cu ? (int64_t)cu[m + 1] - c0 : Tper;
  seg_cu[i] = (int32_t)(c0 + (L * r) / R);
}

template <int DK>
cudaError_t compose_dk(const float* trans, const float* s0, const float* init, float* state_in, float* fin, int R,
                       int N, int H, int dv, int rank_major, int first_from_init, int apply_last, cudaStream_t s) {
  const int ncb = (dv + 31) / 32;
  const int64_t blocks = (int64_t)N * H * ncb;
  if (blocks == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)DK * (DK + 4) + (size_t)DK * 33);
  cudaError_t e = cudaFuncSetAttribute(compose_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  compose_kernel<DK><<<(unsigned)blocks, 256, smem, s>>>(trans, s0, init, state_in, fin, R, N, H, dv, rank_major,
                                                          first_from_init, apply_last);
  return cudaGetLastError();
}

template <int DK, int DV, typename IO>
cudaError_t correct_t(const float* o32, const float* qhat, const float* s_in, void* out, const int32_t* cu, int P,
                      int64_t Tper, int64_t Ttot, int H, int skip_every, cudaStream_t s) {
  if (Ttot == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)DK * (DV + CPAD) + 2 * (size_t)TT * (DK + CPAD) +
                                       2 * (size_t)TT * (DV + CPAD));
  auto* kern = correct_kernel<DK, DV, IO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (Ttot + TT - 1) / TT * H;
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);  // one persistent block per SM
  kern<<<grid, 128, smem, s>>>(o32, qhat, s_in, (IO*)out, cu, P, Tper, Ttot, H, skip_every);
  return cudaGetLastError();
}

template <int DK, typename IO>
cudaError_t correct_dv(const float* o32, const float* qhat, const float* s_in, void* out, const int32_t* cu, int P,
                       int64_t Tper, int64_t Ttot, int H, int dv, int skip_every, cudaStream_t s) {
  switch (dv) {
    case 16: return correct_t<DK, 16, IO>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, skip_every, s);
    case 32: return correct_t<DK, 32, IO>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, skip_every, s);
    case 64: return correct_t<DK, 64, IO>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, skip_every, s);
    case 128: return correct_t<DK, 128, IO>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, skip_every, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_compose(const float* trans, const float* s0, const float* init, float* state_in, float* fin,
                           int R, int N, int H, int dk, int dv, int rank_major, int first_from_init, int apply_last,
                           cudaStream_t s) {
  switch (dk) {
    case 16: return compose_dk<16>(trans, s0, init, state_in, fin, R, N, H, dv, rank_major, first_from_init, apply_last, s);
    case 32: return compose_dk<32>(trans, s0, init, state_in, fin, R, N, H, dv, rank_major, first_from_init, apply_last, s);
    case 64: return compose_dk<64>(trans, s0, init, state_in, fin, R, N, H, dv, rank_major, first_from_init, apply_last, s);
    case 128: return compose_dk<128>(trans, s0, init, state_in, fin, R, N, H, dv, rank_major, first_from_init, apply_last, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_correct(const float* o32, const float* qhat, const float* s_in, void* out, const int32_t* cu,
                           int P, int64_t Tper, int64_t Ttot, int H, int dk, int dv, bool bf16, int skip_every,
                           cudaStream_t s) {
  switch (dk) {
#define KDA_CORRECT_DK(DK_)                                                                                  \
  case DK_:                                                                                                  \
    return bf16 ? correct_dv<DK_, __nv_bfloat16>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, dv, skip_every, s) \
                : correct_dv<DK_, float>(o32, qhat, s_in, out, cu, P, Tper, Ttot, H, dv, skip_every, s);
    KDA_CORRECT_DK(16)
    KDA_CORRECT_DK(32)
    KDA_CORRECT_DK(64)
    KDA_CORRECT_DK(128)
#undef KDA_CORRECT_DK
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_segment_cu(const int32_t* cu, int64_t Tper, int N, int R, int32_t* seg_cu, cudaStream_t s) {
  const int64_t n = (int64_t)N * R + 1;
  segment_cu_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(cu, Tper, N, R, seg_cu);
  return cudaGetLastError();
}

}  // namespace kda
