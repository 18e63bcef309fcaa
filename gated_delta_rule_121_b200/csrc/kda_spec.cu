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
// written once, with the decode step's thread mapping: a warp holds whole rows
// (for dv = 128, 16 consecutive rows x 128 columns per warp), so every state
// load and store is 512 contiguous bytes per warp.  The products against the
// state (X_t, Y_t) do not depend on delta, so they are formed for all tokens
// together, four at a time, and the row groups' partial sums are added
// through shared memory.  Only the n x n triangular system on dv-vectors
// stays serial in t: one thread per value column, delta in registers.
//
// GATED: the inputs are the raw ones of the model's prologue (digest, KDA
// section and "Bounded decay" section): q and k are L2-normalised per token
// and head, and the decay is g = g_min * sigmoid(exp(A_h) * z) from the decay
// logits z.
#include <type_traits>

#include "../../include/kda.h"
#include "kda_gate.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct SpecShape {
  static constexpr int COLQ = DV / 4;                                  // float4 column groups
  static constexpr int RG = (256 / COLQ) < DK ? (256 / COLQ) : DK;     // row groups
  static constexpr int ROWS = DK / RG;                                 // consecutive rows per thread
  static constexpr int NT = COLQ * RG;                                 // threads per block
  static constexpr int PART = RG * 4 * 2 * DV;                         // floats of partial X, Y sums
};

// Shared-memory floats of a block for chunks of up to `n` tokens (the
// token-major arrays and the partial sums share one region).
template <int DK, int DV>
constexpr size_t spec_smem_floats(int n) {
  const size_t n4 = (size_t)((n + 3) & ~3);
  const size_t tok = 4 * (size_t)n * DK, part = (size_t)SpecShape<DK, DV>::PART;
  return (tok > part ? tok : part) + 2 * (size_t)n * DV + 2 * (size_t)n * n4 + n4 + DK + 3 * n4 * DK +
         2 * (size_t)n * DV;
}

// One token array of both windows in 16-byte pieces (rows of D elements of T;
// every pointer and row is 16-byte aligned): piece j of a thread is piece
// tid + j * NT of the NW rows.
template <typename T, int D, int NT>
struct Pieces {
  static constexpr int PER_ROW = D * (int)sizeof(T) / 16;                      // pieces per token row
  static constexpr int EPP = 16 / (int)sizeof(T);                               // elements per piece
  static constexpr int CNT = (KDA_SPEC_MAX_TOKENS * PER_ROW + NT - 1) / NT;  // pieces per thread, at most
};

template <typename T, int D, int NT>
__device__ __forceinline__ void load_pieces(const void* prev, const void* cur, int NW, int Wp, int W, int b, int H,
                                            int h, uint4 (&r)[Pieces<T, D, NT>::CNT]) {
  using P = Pieces<T, D, NT>;
#pragma unroll
  for (int j = 0; j < P::CNT; ++j) {
    const int pc = threadIdx.x + j * NT;
    if (pc < NW * P::PER_ROW) {
      const int tt = pc / P::PER_ROW, o = pc % P::PER_ROW;
      const int64_t row = tt < Wp ? ((int64_t)b * Wp + tt) * H + h : ((int64_t)b * W + (tt - Wp)) * H + h;
      r[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(tt < Wp ? prev : cur) + row * D) + o);
    }
  }
}

// The pieces as fp32 rows of dst at chunk position pos(tt) (rows with pos < 0
// are dropped), each element passed through f.
template <typename T, int D, int NT, typename Pos, typename F>
__device__ __forceinline__ void store_pieces(const uint4 (&r)[Pieces<T, D, NT>::CNT], float* dst, int NW, Pos pos,
                                             F f) {
  using P = Pieces<T, D, NT>;
#pragma unroll
  for (int j = 0; j < P::CNT; ++j) {
    const int pc = threadIdx.x + j * NT;
    if (pc < NW * P::PER_ROW) {
      const int p = pos(pc / P::PER_ROW), o = pc % P::PER_ROW;
      if (p >= 0) {
        const uint32_t w[4] = {r[j].x, r[j].y, r[j].z, r[j].w};
        float e[P::EPP];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if constexpr (sizeof(T) == 2) {  // bf16 pairs
            e[2 * u] = f(__uint_as_float(w[u] << 16));
            e[2 * u + 1] = f(__uint_as_float(w[u] & 0xffff0000u));
          } else {
            e[u] = f(__uint_as_float(w[u]));
          }
        }
        float4* d4 = reinterpret_cast<float4*>(dst + p * D + o * P::EPP);
#pragma unroll
        for (int u = 0; u < P::EPP / 4; ++u) d4[u] = make_float4(e[4 * u], e[4 * u + 1], e[4 * u + 2], e[4 * u + 3]);
      }
    }
  }
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

struct SpecTok {  // where one token's inputs live
  const void* q;
  const void* k;
  const void* v;
  const void* g;  // fp32 log-decay, or the decay logits (dtype IO) when gated
  const float* beta;
};

template <int DK, int DV, typename IO, bool GATED>
__global__ void __launch_bounds__(SpecShape<DK, DV>::NT, 2)
    kda_spec_kernel(SpecTok prev, SpecTok cur, const int32_t* __restrict__ n_accepted, float* __restrict__ state,
                    IO* __restrict__ out, int Wp, int W, int H, const float* __restrict__ A_log, float g_min) {
  using Sh = SpecShape<DK, DV>;
  constexpr int COLQ = Sh::COLQ, RG = Sh::RG, ROWS = Sh::ROWS, NT = Sh::NT;
  extern __shared__ float ssm[];
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int tid = threadIdx.x, cq = tid % COLQ, rg = tid / COLQ, lane = tid & 31, warp = tid >> 5;

  // ---- token loads first, for both windows whole (Wp + W <= 16 tokens), so
  // that no address waits for n_accepted; the rejected drafts' rows are
  // dropped when the chunk is laid out.  Then the state (ROWS consecutive
  // rows x 4 columns per thread): its 64 KiB stream in while the chunk's own
  // arithmetic runs.
  const int NW = Wp + W;
  using GT = typename std::conditional<GATED, IO, float>::type;  // element type of the decay input
  uint4 pk[Pieces<IO, DK, NT>::CNT], pq[Pieces<IO, DK, NT>::CNT], pg[Pieces<GT, DK, NT>::CNT],
      pv[Pieces<IO, DV, NT>::CNT];
  load_pieces<IO, DK, NT>(prev.k, cur.k, NW, Wp, W, b, H, h, pk);
  load_pieces<IO, DK, NT>(prev.q, cur.q, NW, Wp, W, b, H, h, pq);
  load_pieces<GT, DK, NT>(prev.g, cur.g, NW, Wp, W, b, H, h, pg);
  load_pieces<IO, DV, NT>(prev.v, cur.v, NW, Wp, W, b, H, h, pv);
  const float bt = tid < NW ? (tid < Wp ? prev.beta[((int64_t)b * Wp + tid) * H + h]
                                        : cur.beta[((int64_t)b * W + (tid - Wp)) * H + h])
                            : 0.f;
  int na = n_accepted ? n_accepted[b] : 0;
  na = na < 0 ? 0 : (na > Wp ? Wp : na);
  const int n = na + W;               // tokens of the chunk
  const int c = W > 0 ? na : na - 1;  // the token after which the state is kept (-1: none, unchanged)
  if (c < 0) return;
  // shared layout (floats; every array starts on a multiple of 4 floats):
  //   s_k, s_q, s_G, s_al [n][DK]  k, q, G, e^{g} (later the partial sums)
  //   s_v, s_d [n][DV]       values, delta
  //   s_A, s_P [n][n4]       pair sums;  s_b [n4] beta;  s_gc [DK] e^{G_c}
  //   s_ek, s_eq, s_kc [n4][DK]  e^G k, e^G q, k e^{G_c - G} (0 past the chunk / the kept token)
  //   s_xy [n][2 DV]         X_t, then Y_t
  // (all token-major: a thread's ROWS consecutive rows of one token are contiguous)
  const int n4 = (n + 3) & ~3;
  const int tok = 4 * n * DK > Sh::PART ? 4 * n * DK : Sh::PART;
  float* s_k = ssm;
  float* s_q = s_k + n * DK;
  float* s_G = s_q + n * DK;
  float* s_al = s_G + n * DK;
  float* s_part = ssm;
  float* s_v = ssm + tok;
  float* s_d = s_v + n * DV;
  float* s_A = s_d + n * DV;
  float* s_P = s_A + n * n4;
  float* s_b = s_P + n * n4;
  float* s_gc = s_b + n4;
  float* s_ek = s_gc + DK;
  float* s_eq = s_ek + n4 * DK;
  float* s_kc = s_eq + n4 * DK;
  float* s_xy = s_kc + n4 * DK;

  // ---- lay out the chunk: prev[0, na) at 0 .. na-1, cur[0, W) at na ..
  {
    const float Ah = GATED ? A_log[h] : 0.f;
    auto pos = [&](int tt) { return tt < Wp ? (tt < na ? tt : -1) : na + (tt - Wp); };
    auto same = [](float x) { return x; };
    store_pieces<IO, DK, NT>(pk, s_k, NW, pos, same);
    store_pieces<IO, DK, NT>(pq, s_q, NW, pos, same);
    // the per-token log-decays g (s_G) and decays alpha = e^g (s_al)
    if constexpr (GATED) {
      store_pieces<GT, DK, NT>(pg, s_G, NW, pos, [&](float z) { return gate_log_decay(z, Ah, g_min); });
      store_pieces<GT, DK, NT>(pg, s_al, NW, pos, [&](float z) { return __expf(gate_log_decay(z, Ah, g_min)); });
    } else {
      store_pieces<GT, DK, NT>(pg, s_G, NW, pos, same);
      store_pieces<GT, DK, NT>(pg, s_al, NW, pos, [](float x) { return __expf(x); });
    }
    store_pieces<IO, DV, NT>(pv, s_v, NW, pos, same);
    if (tid < NW && pos(tid) >= 0) s_b[pos(tid)] = bt;
  }
  __syncthreads();
  float4* S = reinterpret_cast<float4*>(state + ((int64_t)b * H + h) * DK * DV);
  float4 s[ROWS];  // rows rg * ROWS + m, columns 4 cq .. 4 cq + 3; first used by the X, Y products
#pragma unroll
  for (int m = 0; m < ROWS; ++m) s[m] = __ldcs(S + (rg * ROWS + m) * COLQ + cq);
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
  // ---- per-token operands, four channels per work item: e^{G_t} k_t,
  // e^{G_t} q_t, k_t e^{G_c - G_t} (t <= c), zero past the chunk (up to n4),
  // and e^{G_c}; each item sums its own cumulative log-decays G_t and G_c
  // over the tokens (at most 16).  Then (no barrier: other arrays) the pair
  // sums.
  for (int w = tid; w < n4 * (DK / 4); w += NT) {
    const int t = w / (DK / 4), i0 = 4 * (w % (DK / 4));
    float4 ek = make_float4(0.f, 0.f, 0.f, 0.f), eq = ek, kc = ek;
    if (t < n) {
      float4 G = make_float4(0.f, 0.f, 0.f, 0.f), Gc = G, acc = G;
      const int last = t > c ? t : c;
      for (int u = 0; u <= last; ++u) {
        acc = add4(acc, *reinterpret_cast<const float4*>(s_G + u * DK + i0));
        if (u == t) G = acc;
        if (u == c) Gc = acc;
      }
      const float4 kk = *reinterpret_cast<const float4*>(s_k + t * DK + i0);
      const float4 qq = *reinterpret_cast<const float4*>(s_q + t * DK + i0);
      const float4 e = make_float4(__expf(G.x), __expf(G.y), __expf(G.z), __expf(G.w));
      ek = make_float4(e.x * kk.x, e.y * kk.y, e.z * kk.z, e.w * kk.w);
      eq = make_float4(e.x * qq.x, e.y * qq.y, e.z * qq.z, e.w * qq.w);
      if (t <= c)
        kc = make_float4(kk.x * __expf(Gc.x - G.x), kk.y * __expf(Gc.y - G.y), kk.z * __expf(Gc.z - G.z),
                         kk.w * __expf(Gc.w - G.w));
      if (t == c) *reinterpret_cast<float4*>(s_gc + i0) = e;
    }
    *reinterpret_cast<float4*>(s_ek + t * DK + i0) = ek;
    *reinterpret_cast<float4*>(s_eq + t * DK + i0) = eq;
    *reinterpret_cast<float4*>(s_kc + t * DK + i0) = kc;
  }
  // Pair sums A_ts (s < t) and P_ts (s <= t), one warp per s (s = warp, then
  // mirrored so that the warps' loads even out), four channels per lane: the
  // decay e^{G_t - G_s} is the running product of alpha over s < u <= t
  // (every factor <= 1).  The lane sums for t in an 8-token half are
  // reduce-scattered over the warp (offsets 8, 4, 2, 1: lane l keeps value
  // l & 15 = 2 (t - t_half) + {0: A, 1: P}), then added across offset 16.
  {
    constexpr int NWARP = NT / 32;
    const bool lane_on = 4 * lane < DK;
    const int i0 = lane_on ? 4 * lane : 0;
    for (int r = 0; r * NWARP < n; ++r) {
      const int s2 = (r & 1) ? (r + 1) * NWARP - 1 - warp : r * NWARP + warp;
      if (s2 >= n) continue;
      const float4 ks = lane_on ? *reinterpret_cast<const float4*>(s_k + s2 * DK + i0) : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 f = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll 1
      for (int th = (s2 / 8) * 8; th < n; th += 8) {  // 8-token halves of t that reach s
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = th + u;
          if (t >= s2 && t < n) {
            if (t > s2) {
              const float4 al = *reinterpret_cast<const float4*>(s_al + t * DK + i0);
              f.x *= al.x; f.y *= al.y; f.z *= al.z; f.w *= al.w;
            }
            const float4 ke = make_float4(ks.x * f.x, ks.y * f.y, ks.z * f.z, ks.w * f.w);
            const float4 kt = *reinterpret_cast<const float4*>(s_k + t * DK + i0);
            const float4 qt = *reinterpret_cast<const float4*>(s_q + t * DK + i0);
            v[2 * u] = (kt.x * ke.x + kt.y * ke.y) + (kt.z * ke.z + kt.w * ke.w);
            v[2 * u + 1] = (qt.x * ke.x + qt.y * ke.y) + (qt.z * ke.z + qt.w * ke.w);
          }
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
          const bool up = lane & o;
#pragma unroll
          for (int j = 0; j < o; ++j)
            v[j] = (up ? v[j + o] : v[j]) + __shfl_xor_sync(0xffffffffu, up ? v[j] : v[j + o], o);
        }
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);
        const int t = th + ((lane & 15) >> 1);
        if (lane < 16 && t < n) {
          if (lane & 1) {
            if (t >= s2) s_P[t * n4 + s2] = v[0];
          } else if (t > s2) {
            s_A[t * n4 + s2] = v[0];
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- X_t = S0^T ek_t for every token and Y_t = S0^T eq_t for the new
  // window's tokens (t >= na; the replayed ones have no outputs): a list of
  // rows, the X rows first, taken eight at a time (two passes of four
  // accumulators; the last one to seven rows in groups of 4, 2 and 1): each
  // thread's share over its state rows, then the row groups' partial sums
  // added through shared memory (the token-major arrays are no longer
  // needed).
  const int nrows = 2 * n - na;
  // row r: its operand (this thread's entries) and where its sums go in s_xy
  const float* s_eq_na = s_eq + rg * ROWS + (na - n) * DK;  // s_eq_na + r DK: token na + r - n
  auto row_op = [&](int r) -> const float* { return r < n ? s_ek + rg * ROWS + r * DK : s_eq_na + r * DK; };
  auto row_dst = [&](int r) { return r < n ? r * 2 * DV : (na + r - n) * 2 * DV + DV; };
  auto xy_rows = [&](auto tb, int r0) {
    constexpr int TB = decltype(tb)::value;  // rows of this group
    constexpr int PB = TB < 4 ? TB : 4;      // rows per pass
#pragma unroll 1
    for (int pb = 0; pb < TB; pb += PB) {
      float acc[PB][4];
#pragma unroll
      for (int u = 0; u < PB; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const float* e = row_op(r0 + pb + u);
        float ev[ROWS];
        if constexpr (ROWS % 4 == 0) {
#pragma unroll
          for (int m = 0; m < ROWS; m += 4) {
            const float4 e4 = *reinterpret_cast<const float4*>(e + m);
            ev[m] = e4.x; ev[m + 1] = e4.y; ev[m + 2] = e4.z; ev[m + 3] = e4.w;
          }
        } else {
#pragma unroll
          for (int m = 0; m < ROWS; ++m) ev[m] = e[m];
        }
#pragma unroll
        for (int m = 0; m < ROWS; ++m) {
          acc[u][0] += s[m].x * ev[m]; acc[u][1] += s[m].y * ev[m];
          acc[u][2] += s[m].z * ev[m]; acc[u][3] += s[m].w * ev[m];
        }
      }
#pragma unroll
      for (int u = 0; u < PB; ++u)
        *reinterpret_cast<float4*>(s_part + (rg * TB + pb + u) * DV + 4 * cq) =
            make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
    for (int e = tid; e < TB * DV; e += NT) {
      const int row = e / DV, col = e % DV;
      float sum = 0.f;
#pragma unroll 8
      for (int r = 0; r < RG; ++r) sum += s_part[(r * TB + row) * DV + col];
      s_xy[row_dst(r0 + row) + col] = sum;
    }
    __syncthreads();  // the partial sums are read before the next group writes them
  };
  int r0 = 0;
  for (; r0 + 8 <= nrows; r0 += 8) xy_rows(std::integral_constant<int, 8>{}, r0);
  if (nrows - r0 >= 4) {
    xy_rows(std::integral_constant<int, 4>{}, r0);
    r0 += 4;
  }
  if (nrows - r0 >= 2) {
    xy_rows(std::integral_constant<int, 2>{}, r0);
    r0 += 2;
  }
  if (r0 < nrows) xy_rows(std::integral_constant<int, 1>{}, r0);

  // ---- delta_t by forward substitution and o_t, one thread per value column
  IO* o_base = out + ((int64_t)b * W * H + h) * DV;
  for (int j = tid; j < DV; j += NT) {
    float dl[KDA_SPEC_MAX_TOKENS];
#pragma unroll
    for (int t = 0; t < KDA_SPEC_MAX_TOKENS; ++t) {
      if (t < n) {
        float d = s_v[t * DV + j] - s_xy[t * 2 * DV + j];
#pragma unroll
        for (int s2 = 0; s2 < t; ++s2) d -= s_A[t * n4 + s2] * dl[s2];
        d *= s_b[t];
        dl[t] = d;
        s_d[t * DV + j] = d;
        if (t >= na) {
          float o = s_xy[t * 2 * DV + DV + j];
#pragma unroll
          for (int s2 = 0; s2 <= t; ++s2) o += s_P[t * n4 + s2] * dl[s2];
          o_base[(int64_t)(t - na) * H * DV + j] = from_f32<IO>(o);
        }
      }
    }
  }
  __syncthreads();

  // ---- the kept state: S_c = Diag(e^{G_c}) S0 + sum_{s<=c} (k_s e^{G_c - G_s}) delta_s^T,
  // updated in the state registers token by token (the thread's ROWS
  // consecutive rows: its k e^{G_c - G} entries are contiguous).
  {
    const float* eg = s_gc + rg * ROWS;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
      const float e = eg[m];
      s[m].x *= e; s[m].y *= e; s[m].z *= e; s[m].w *= e;
    }
    for (int t = 0; t <= c; ++t) {
      const float4 ds = *reinterpret_cast<const float4*>(s_d + t * DV + 4 * cq);
      const float* kc = s_kc + t * DK + rg * ROWS;
      float kv[ROWS];
      if constexpr (ROWS % 4 == 0) {
#pragma unroll
        for (int m = 0; m < ROWS; m += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kc + m);
          kv[m] = k4.x; kv[m + 1] = k4.y; kv[m + 2] = k4.z; kv[m + 3] = k4.w;
        }
      } else {
#pragma unroll
        for (int m = 0; m < ROWS; ++m) kv[m] = kc[m];
      }
#pragma unroll
      for (int m = 0; m < ROWS; ++m) {
        s[m].x += kv[m] * ds.x; s[m].y += kv[m] * ds.y; s[m].z += kv[m] * ds.z; s[m].w += kv[m] * ds.w;
      }
    }
#pragma unroll
    for (int m = 0; m < ROWS; ++m) __stcs(S + (rg * ROWS + m) * COLQ + cq, s[m]);
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
