// Chunked KDA forward on the sm_100a tensor cores (tcgen05 / TMEM / TMA),
// bf16 q, k, v, out with dk = dv = 128, fp32 state, chunk length C = 64.
//
// What it computes (Kimi K3 digest, "Kimi Delta Attention" section, chunkwise
// form: chunk output = inter-chunk term (Gamma ⊙ Q) S + intra-chunk term
// A Ṽ), written out per chunk with in-chunk cumulative log-decay
// G_r = sum_{s<=r} g_s (per key channel):
//   A_rs  = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)   (s < r)       "A_kk"
//   P_rs  = sum_c q_rc k_sc exp(G_rc - G_sc)          (s <= r)
//   T     = (I + A)^-1,  T' = T diag(beta)
//   W     = T' (K ⊙ Γ),   U = T' V                    (WY / UT transform)
//   Δ     = U - W S                                    (Ṽ of the digest)
//   O     = (Q ⊙ Γ) S + P Δ
//   S    <- Diag(Γ_C) S + (K ⊙ exp(G_C - G))^T Δ
// (Γ = exp(G); Γ_C its last row.)  Unrolling the recurrence of the same
// section over a chunk gives exactly these identities.
//
// Bounded decay ("Bounded decay" section: g >= g_min = -5): the pairwise
// decay exp(G_rc - G_sc) is factorised as exp(G_rc) * exp(-G_sc) so that the
// Gram matrices become dense bf16 matmuls.  The factor exp(-G) stays finite
// only while the chunk's total decay is moderate; a chunk whose total
// log-decay in some channel is below -64 takes the general path, which forms
// the two Gram matrices on CUDA cores from the exact differences G_r - G_s.
// Everything after the Gram matrices is shared by both paths.
//
// Layout of the work: one CTA per (sequence, head) chain, chunks in order.
// All UMMAs are M = 128 with the state kept TRANSPOSED in TMEM (lane j =
// value channel, column c = key channel), so the tensor-core "rows" are the
// 128 value channels:
//   G1  [P ; A_raw](lanes r, 64+r)  = [QΓ ; KΓ] · K̃^T       (K̃ = K ⊙ e^{-G})
//   G2  W^T (lane c)                = (KΓ)^T · T'^T
//   G3  U^T (lane j)                = V^T · T'^T
//   D1  O^T = S^T (QΓ)^T,  (WS)^T = S^T W^T
//   D2  S^T += Δ^T K̂,  O^T += Δ^T P^T                    (K̂ = K ⊙ e^{G_C-G})
// Δ^T = U^T - (WS)^T is formed lane-wise in registers.  S^T lives in TMEM
// (fp32) for the whole chain; a bf16 copy in shared memory is the A operand
// of D1.  Q, K, V tiles arrive by TMA with 128-byte swizzle, two chunks
// ahead; Q and K are rescaled in place into QΓ and KΓ.
#include <cuda.h>

#include "kda_internal.cuh"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

constexpr int CH = 64;    // chunk length
constexpr int D = 128;    // dk = dv
constexpr int NTHR = 128;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float FAST_MIN_LOG2 = -92.0f;  // chunk-total decay floor for the factorised Gram (~e^-64)
constexpr uint64_t WAIT_NS = 2000000000ull;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t STAGE_BYTES = 49152;      // [Q;K] 32 KB + V 16 KB
constexpr uint32_t OFF_QK = 0, OFF_V = 32768;
constexpr uint32_t SM_G = 2 * STAGE_BYTES;   // g tile, fp32 [64][128]       32 KB
constexpr uint32_t SM_KT = SM_G + 32768;     // K̃ (bf16) -> A (fp32) -> T'   16 KB
constexpr uint32_t SM_KH = SM_KT + 16384;    // K̂ (bf16)                     16 KB
constexpr uint32_t SM_P = SM_KH + 16384;     // P (bf16)                      8 KB
constexpr uint32_t SM_WD = SM_P + 8192;      // W, then Δ^T (bf16)           16 KB
constexpr uint32_t SM_SB = SM_WD + 16384;    // S^T bf16                     32 KB
constexpr uint32_t SM_MISC = SM_SB + 32768;
constexpr uint32_t MISC_BYTES = 3072;
constexpr uint32_t SMEM_BYTES = SM_MISC + MISC_BYTES + 1024;  // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes each).
constexpr uint32_t TM_S = 0, TM_O = 128, TM_WS = 192, TM_GRAM = 256, TM_W = 320, TM_U = 384;
constexpr uint32_t TMEM_COLS = 512;

// Debug dump offsets (floats) for chain 0, chunk 0.
constexpr int DBG_P = 0, DBG_A = 4096, DBG_T = 8192, DBG_W = 12288, DBG_U = 20480, DBG_DELTA = 28672,
              DBG_O = 36864, DBG_S = 45056, DBG_GC = 61440, DBG_FLOATS = 61568;

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_b16(uint32_t addr, float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(*reinterpret_cast<uint16_t*>(&h)) : "memory");
}
__device__ __forceinline__ float4 ld_bf16x4(uint32_t addr) {
  uint32_t a, b;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(addr));
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  float2 fx = __bfloat1622float2(x), fy = __bfloat1622float2(y);
  return make_float4(fx.x, fx.y, fy.x, fy.y);
}
__device__ __forceinline__ float ld_bf16(uint32_t addr) {
  uint16_t u;
  asm volatile("ld.shared.b16 %0, [%1];" : "=h"(u) : "r"(addr));
  return __bfloat162float(*reinterpret_cast<__nv_bfloat16*>(&u));
}
__device__ __forceinline__ void st_bf16x4(uint32_t addr, float4 v) {
  st_shared_v2(addr, pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}
// Eight consecutive fp32 values -> one 16-byte chunk of bf16.
__device__ __forceinline__ void st_bf16x8(uint32_t addr, const float* v) {
  st_shared_v4(addr, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
               pack_bf16x2(v[6], v[7]));
}
// fp32 [64][64] matrix with 16-byte units XOR-swizzled by row (conflict-free
// row writes and broadcast reads).
__device__ __forceinline__ uint32_t a_off(uint32_t r, uint32_t s) {
  return r * 256u + ((s >> 2) ^ (r & 7u)) * 16u + (s & 3u) * 4u;
}

__global__ void __launch_bounds__(NTHR, 1)
    kda_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                      const float* __restrict__ beta, const float* __restrict__ init,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ fin, const int32_t* __restrict__ cu,
                      int64_t Tper, int H, DeviceStatus* status, float* __restrict__ dbg, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar_stage = reinterpret_cast<uint64_t*>(sm + SM_MISC);  // [2]
  uint64_t* bar_g = bar_stage + 2;
  uint64_t* bar_mma = bar_stage + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + SM_MISC + 64);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + SM_MISC + 68);
  float* s_beta = reinterpret_cast<float*>(sm + SM_MISC + 128);  // [64]
  float* s_gc = reinterpret_cast<float*>(sm + SM_MISC + 384);    // [128] exp(G_C)
  float* s_red = reinterpret_cast<float*>(sm + SM_MISC + 896);   // [4][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chain = blockIdx.x;
  const int n = chain / H, h = chain % H;
  int64_t t0, L;
  if (cu) {
    t0 = cu[n];
    L = (int64_t)cu[n + 1] - t0;
  } else {
    t0 = (int64_t)n * Tper;
    L = Tper;
  }
  const int nchunks = (int)((L + CH - 1) / CH);
  const bool dump = (dbg != nullptr) && chain == 0;

  if (tid == 0) {
    mbar_init(&bar_stage[0], 1);
    mbar_init(&bar_stage[1], 1);
    mbar_init(bar_g, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *s_abort = 0;
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lane quarter

  // Async-op bookkeeping: thread 0 issues every TMA and UMMA; all threads
  // wait on the same phases in the same order, so the waited counts agree.
  int stage_issued[2] = {0, 0}, stage_waited[2] = {0, 0}, g_issued = 0, g_waited = 0;
  int mma_issued = 0, mma_waited = 0;
  auto issue_stage = [&](int c) {
    const int st = c & 1;
    const int tok = (int)(t0 + (int64_t)c * CH);
    uint8_t* dst = sm + st * STAGE_BYTES;
    mbar_arrive_expect_tx(&bar_stage[st], STAGE_BYTES);
    for (int hh = 0; hh < 2; ++hh) {
      tma_load_3d(dst + OFF_QK + hh * 16384, &tm_q, &bar_stage[st], 64 * hh, h, tok);
      tma_load_3d(dst + OFF_QK + hh * 16384 + 8192, &tm_k, &bar_stage[st], 64 * hh, h, tok);
      tma_load_3d(dst + OFF_V + hh * 8192, &tm_v, &bar_stage[st], 64 * hh, h, tok);
    }
    ++stage_issued[st];
  };
  auto issue_g = [&](int c) {
    mbar_arrive_expect_tx(bar_g, 32768);
    tma_load_3d(sm + SM_G, &tm_g, bar_g, 0, h, (int)(t0 + (int64_t)c * CH));
    ++g_issued;
  };
  auto wait_mma = [&](int where) {
    // Only a completed phase counts as waited; the error path drains the rest.
    if (mbar_wait(bar_mma, mma_waited & 1, wait_ns)) {
      ++mma_waited;
    } else {
      record_error(status, KDA_ERR_TIMEOUT, where);
      *s_abort = 1;
    }
    tc_fence_after();
  };
  // Barrier that also reports whether any thread gave up on a wait.
  auto sync_abort = [&]() -> bool {
    __syncthreads();
    return *s_abort != 0;
  };

  if (tid == 0 && nchunks > 0) {
    issue_stage(0);
    issue_g(0);
    if (nchunks > 1) issue_stage(1);
  }

  const int64_t sbase = ((int64_t)n * H + h) * D * D;
  const int j = tid;  // TMEM lane = value channel in the transposed-state phases
  // ---- initial state: S^T into TMEM, bf16 copy into SB.
#pragma unroll
  for (int cb = 0; cb < 4; ++cb) {
    float r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = init ? init[sbase + (int64_t)(cb * 32 + i) * D + j] : 0.f;
    tmem_st32(tl + TM_S + cb * 32, r);
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      const int c = cb * 32 + q8 * 8;
      st_bf16x8(sb + SM_SB + (c >> 6) * 16384 + sw128_off(j, c & 63), r + q8 * 8);
    }
  }
  tmem_wait_st();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  const uint32_t ID_K64 = idesc_bf16_f32(128, 64, 0, 0);
  const uint32_t ID_MN64 = idesc_bf16_f32(128, 64, 1, 0);
  const uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 1);

  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    const uint32_t stg = sb + st * STAGE_BYTES;
    const int64_t tok0 = t0 + (int64_t)c * CH;
    const int valid = (int)((L - (int64_t)c * CH) < CH ? (L - (int64_t)c * CH) : CH);
    const bool dmp = dump && c == 0;

    if (tid < CH) s_beta[tid] = tid < valid ? beta[(tok0 + tid) * H + h] : 0.f;
    if (mbar_wait(bar_g, g_waited & 1, wait_ns)) {
      ++g_waited;
    } else {
      record_error(status, KDA_ERR_TIMEOUT, 1);
      *s_abort = 1;
    }
    if (mbar_wait(&bar_stage[st], stage_waited[st] & 1, wait_ns)) {
      ++stage_waited[st];
    } else {
      record_error(status, KDA_ERR_TIMEOUT, 2);
      *s_abort = 1;
    }

    // ---- (a1) in-chunk cumulative decay, log2 units.  Thread (rq = warp,
    // cq = lane): rows 16 rq .. 16 rq + 15, channels 4 cq .. 4 cq + 3.
    const int rq = warp;
    const int ch0 = 4 * lane, hh = ch0 >> 6, cc = ch0 & 63;
    float4 G[16];
    {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int r = 16 * rq + m;
        float4 gv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < valid) gv = *reinterpret_cast<const float4*>(sm + SM_G + r * 512 + ch0 * 4);
        acc.x += gv.x * LOG2E; acc.y += gv.y * LOG2E; acc.z += gv.z * LOG2E; acc.w += gv.w * LOG2E;
        G[m] = acc;
      }
      *reinterpret_cast<float4*>(s_red + rq * 128 + ch0) = acc;
    }
    if (sync_abort()) break;
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
    {
      float4 off = tot;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(s_red + q * 128 + ch0);
        if (q < rq) { off.x += v.x; off.y += v.y; off.z += v.z; off.w += v.w; }
        tot.x += v.x; tot.y += v.y; tot.z += v.z; tot.w += v.w;
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        G[m].x += off.x; G[m].y += off.y; G[m].z += off.z; G[m].w += off.w;
      }
    }
    const float4 egc = make_float4(ex2(tot.x), ex2(tot.y), ex2(tot.z), ex2(tot.w));
    if (rq == 0) {
      *reinterpret_cast<float4*>(s_gc + ch0) = egc;
      if (dmp) {
        const float LN2 = 0.6931471805599453f;
        dbg[DBG_GC + ch0 + 0] = tot.x * LN2; dbg[DBG_GC + ch0 + 1] = tot.y * LN2;
        dbg[DBG_GC + ch0 + 2] = tot.z * LN2; dbg[DBG_GC + ch0 + 3] = tot.w * LN2;
      }
    }
    const bool ok_fast = fminf(fminf(tot.x, tot.y), fminf(tot.z, tot.w)) >= FAST_MIN_LOG2;
    const bool fast = __syncthreads_and(ok_fast) != 0;

    const uint32_t qb = stg + OFF_QK + hh * 16384;  // Q rows of this thread's channel half
    const uint32_t kb = qb + 8192;                  // K rows
    const uint32_t ktb = sb + SM_KT + hh * 8192;
    const uint32_t khb = sb + SM_KH + hh * 8192;

    if (fast) {
      // ---- (a2, fast) QΓ, KΓ in place; K̃ = K e^{-G}; K̂ = K e^{G_C - G}.
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int r = 16 * rq + m;
        const uint32_t o = sw128_off(r, cc);
        float4 q4 = ld_bf16x4(qb + o), k4 = ld_bf16x4(kb + o);
        if (r >= valid) q4 = k4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 e = make_float4(ex2(G[m].x), ex2(G[m].y), ex2(G[m].z), ex2(G[m].w));
        const float4 ie = make_float4(ex2(-G[m].x), ex2(-G[m].y), ex2(-G[m].z), ex2(-G[m].w));
        st_bf16x4(qb + o, make_float4(q4.x * e.x, q4.y * e.y, q4.z * e.z, q4.w * e.w));
        st_bf16x4(kb + o, make_float4(k4.x * e.x, k4.y * e.y, k4.z * e.z, k4.w * e.w));
        st_bf16x4(ktb + o, make_float4(k4.x * ie.x, k4.y * ie.y, k4.z * ie.z, k4.w * ie.w));
        st_bf16x4(khb + o, make_float4(k4.x * (egc.x * ie.x), k4.y * (egc.y * ie.y), k4.z * (egc.z * ie.z),
                                       k4.w * (egc.w * ie.w)));
      }
      fence_proxy_async_smem();
      if (sync_abort()) break;
      // ---- (a2) G1: [P ; A_raw] = [QΓ ; KΓ] · K̃^T   (M=128, N=64, K=128)
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint64_t da = sdesc_sw128(stg + OFF_QK + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
          const uint64_t db = sdesc_sw128(sb + SM_KT + (i >> 2) * 8192 + (i & 3) * 32, 16, 1024);
          umma_bf16(tmem + TM_GRAM, da, db, ID_K64, i > 0);
        }
        umma_commit(bar_mma);
        ++mma_issued;
      }
      wait_mma(3);
      if (sync_abort()) break;
      {
        float r0[32], r1[32];
        tmem_ld32(tl + TM_GRAM, r0);
        tmem_ld32(tl + TM_GRAM + 32, r1);
        if (tid < CH) {  // lanes 0..63: P row r, lower triangle incl. diagonal
          const int r = tid;
#pragma unroll
          for (int s = 0; s < 32; ++s) {
            if (s > r) r0[s] = 0.f;
            if (s + 32 > r) r1[s] = 0.f;
          }
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8)
            st_bf16x8(sb + SM_P + r * 128 + (((q8 ^ r) & 7) << 4), q8 < 4 ? r0 + q8 * 8 : r1 + (q8 - 4) * 8);
          if (dmp)
#pragma unroll
            for (int s = 0; s < 64; ++s) dbg[DBG_P + r * 64 + s] = s < 32 ? r0[s] : r1[s - 32];
        } else {  // lanes 64..127: A row r = beta_r * (KΓ K̃^T)_rs, strictly lower
          const int r = tid - CH;
          const float b = s_beta[r];
#pragma unroll
          for (int s = 0; s < 32; ++s) {
            r0[s] = s < r ? b * r0[s] : 0.f;
            r1[s] = s + 32 < r ? b * r1[s] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float* v = u < 8 ? r0 + 4 * u : r1 + 4 * (u - 8);
            *reinterpret_cast<float4*>(sm + SM_KT + a_off(r, 4 * u)) = make_float4(v[0], v[1], v[2], v[3]);
          }
          if (dmp)
#pragma unroll
            for (int s = 0; s < 64; ++s) dbg[DBG_A + r * 64 + s] = s < 32 ? r0[s] : r1[s - 32];
        }
      }
    } else {
      // ---- (a2, general) G over the g tile; P and A on CUDA cores from the
      // exact differences G_r - G_s; then QΓ, KΓ in place and K̂.
#pragma unroll
      for (int m = 0; m < 16; ++m)
        *reinterpret_cast<float4*>(sm + SM_G + (16 * rq + m) * 512 + ch0 * 4) = G[m];
      if (sync_abort()) break;
      {
        const int r = tid & 63, s0 = (tid >> 6) * 32;
        const uint32_t qrow = stg + OFF_QK, krow = stg + OFF_QK + 8192;
        const float br = s_beta[r];
        for (int s = s0; s < s0 + 32; ++s) {
          float p = 0.f, a = 0.f;
          if (s <= r && r < valid) {
            for (int ch = 0; ch < D; ++ch) {
              const uint32_t o_r = (ch >> 6) * 16384 + sw128_off(r, ch & 63);
              const uint32_t o_s = (ch >> 6) * 16384 + sw128_off(s, ch & 63);
              const float gr = *reinterpret_cast<const float*>(sm + SM_G + r * 512 + ch * 4);
              const float gs = *reinterpret_cast<const float*>(sm + SM_G + s * 512 + ch * 4);
              const float e = ex2(gr - gs);
              const float ks = ld_bf16(krow + o_s);
              p += ld_bf16(qrow + o_r) * ks * e;
              a += ld_bf16(krow + o_r) * ks * e;
            }
          }
          a = (s < r) ? br * a : 0.f;
          st_shared_b16(sb + SM_P + sw128_off(r, s), p);
          *reinterpret_cast<float*>(sm + SM_KT + a_off(r, s)) = a;
          if (dmp) {
            dbg[DBG_P + r * 64 + s] = p;
            dbg[DBG_A + r * 64 + s] = a;
          }
        }
      }
      if (sync_abort()) break;
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int r = 16 * rq + m;
        const uint32_t o = sw128_off(r, cc);
        float4 q4 = ld_bf16x4(qb + o), k4 = ld_bf16x4(kb + o);
        if (r >= valid) q4 = k4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 e = make_float4(ex2(G[m].x), ex2(G[m].y), ex2(G[m].z), ex2(G[m].w));
        const float4 eh = make_float4(ex2(tot.x - G[m].x), ex2(tot.y - G[m].y), ex2(tot.z - G[m].z),
                                      ex2(tot.w - G[m].w));
        st_bf16x4(qb + o, make_float4(q4.x * e.x, q4.y * e.y, q4.z * e.z, q4.w * e.w));
        st_bf16x4(kb + o, make_float4(k4.x * e.x, k4.y * e.y, k4.z * e.z, k4.w * e.w));
        st_bf16x4(khb + o, make_float4(k4.x * eh.x, k4.y * eh.y, k4.z * eh.z, k4.w * eh.w));
      }
    }
    fence_proxy_async_smem();
    if (sync_abort()) break;

    // ---- (a3) T = (I + A)^-1 by forward substitution, one column per
    // thread (threads 0..63); T' = T diag(beta) stored as bf16 [r][s].
    {
      float x[CH];
      if (tid < CH) {
#pragma unroll
        for (int r = 0; r < CH; ++r) x[r] = 0.f;
#pragma unroll
        for (int r = 0; r < CH; ++r) {
          float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
          for (int u = 0; u < (r + 3) / 4; ++u) {
            const float4 a4 = *reinterpret_cast<const float4*>(sm + SM_KT + a_off(r, 4 * u));
            acc -= a4.x * x[4 * u] + a4.y * x[4 * u + 1] + a4.z * x[4 * u + 2] + a4.w * x[4 * u + 3];
          }
          x[r] = acc;
        }
      }
      __syncthreads();  // every read of A is done before T' overwrites it
      if (tid < CH) {
        const float bj = s_beta[j];
#pragma unroll
        for (int r = 0; r < CH; ++r) {
          st_shared_b16(sb + SM_KT + sw128_off(r, j), x[r] * bj);
          if (dmp) dbg[DBG_T + r * 64 + j] = x[r] * bj;
        }
      }
    }
    fence_proxy_async_smem();
    if (sync_abort()) break;

    // ---- (a4) G2: W^T = (KΓ)^T T'^T;  G3: U^T = V^T T'^T   (M=128, N=64, K=64)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t da = sdesc_sw128(stg + OFF_QK + 8192 + i * 2048, 16384, 1024);
        const uint64_t db = sdesc_sw128(sb + SM_KT + i * 32, 16, 1024);
        umma_bf16(tmem + TM_W, da, db, ID_MN64, i > 0);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t da = sdesc_sw128(stg + OFF_V + i * 2048, 8192, 1024);
        const uint64_t db = sdesc_sw128(sb + SM_KT + i * 32, 16, 1024);
        umma_bf16(tmem + TM_U, da, db, ID_MN64, i > 0);
      }
      umma_commit(bar_mma);
      ++mma_issued;
      if (c + 1 < nchunks) issue_g(c + 1);  // g tile is free: every read of it is behind us
    }
    wait_mma(4);
    if (sync_abort()) break;
    {  // lane c holds W^T[c][r]; store W[r][c] (K-major B operand of D1)
      float w0[32], w1[32];
      tmem_ld32(tl + TM_W, w0);
      tmem_ld32(tl + TM_W + 32, w1);
      const uint32_t wb = sb + SM_WD + (j >> 6) * 8192;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        st_shared_b16(wb + sw128_off(r, j & 63), w0[r]);
        st_shared_b16(wb + sw128_off(r + 32, j & 63), w1[r]);
      }
      if (dmp) {
        float u0[32], u1[32];
        tmem_ld32(tl + TM_U, u0);
        tmem_ld32(tl + TM_U + 32, u1);
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          dbg[DBG_W + r * 128 + j] = r < 32 ? w0[r] : w1[r - 32];
          dbg[DBG_U + r * 128 + j] = r < 32 ? u0[r] : u1[r - 32];
        }
      }
    }
    fence_proxy_async_smem();
    if (sync_abort()) break;

    // ---- (a5/a6) D1: O^T = S^T (QΓ)^T,  (WS)^T = S^T W^T   (M=128, N=64, K=128)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t da = sdesc_sw128(sb + SM_SB + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
        const uint64_t dq = sdesc_sw128(stg + OFF_QK + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
        umma_bf16(tmem + TM_O, da, dq, ID_K64, i > 0);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t da = sdesc_sw128(sb + SM_SB + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
        const uint64_t dw = sdesc_sw128(sb + SM_WD + (i >> 2) * 8192 + (i & 3) * 32, 16, 1024);
        umma_bf16(tmem + TM_WS, da, dw, ID_K64, i > 0);
      }
      umma_commit(bar_mma);
      ++mma_issued;
    }
    wait_mma(5);
    // The stage's QΓ, KΓ and V have all been consumed: prefetch chunk c+2.
    if (tid == 0 && c + 2 < nchunks && !*s_abort) issue_stage(c + 2);
    {
      // Δ^T[j][r] = U^T - (WS)^T, bf16 row j of the K-major A operand of D2.
      float u[32], w[32], d[64];
      tmem_ld32(tl + TM_U, u);
      tmem_ld32(tl + TM_WS, w);
#pragma unroll
      for (int r = 0; r < 32; ++r) d[r] = u[r] - w[r];
      tmem_ld32(tl + TM_U + 32, u);
      tmem_ld32(tl + TM_WS + 32, w);
#pragma unroll
      for (int r = 0; r < 32; ++r) d[32 + r] = u[r] - w[r];
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) st_bf16x8(sb + SM_WD + j * 128 + (((q8 ^ j) & 7) << 4), d + q8 * 8);
      if (dmp)
#pragma unroll
        for (int r = 0; r < 64; ++r) dbg[DBG_DELTA + r * 128 + j] = d[r];
      // S^T <- S^T Diag(Γ_C)  (decay of key channel c = TMEM column c)
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        float s[32];
        tmem_ld32(tl + TM_S + cb * 32, s);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] *= s_gc[cb * 32 + i];
        tmem_st32(tl + TM_S + cb * 32, s);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (sync_abort()) break;

    // ---- (a5/a6) D2: S^T += Δ^T K̂ (N=128);  O^T += Δ^T P^T (N=64);  K=64
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t da = sdesc_sw128(sb + SM_WD + i * 32, 16, 1024);
        const uint64_t dk = sdesc_sw128(sb + SM_KH + i * 2048, 8192, 1024);
        umma_bf16(tmem + TM_S, da, dk, ID_S, 1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t da = sdesc_sw128(sb + SM_WD + i * 32, 16, 1024);
        const uint64_t dp = sdesc_sw128(sb + SM_P + i * 32, 16, 1024);
        umma_bf16(tmem + TM_O, da, dp, ID_K64, 1);
      }
      umma_commit(bar_mma);
      ++mma_issued;
    }
    wait_mma(6);
    if (sync_abort()) break;
    {
      // New S^T -> bf16 copy for the next chunk's D1.
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        float s[32];
        tmem_ld32(tl + TM_S + cb * 32, s);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int ch = cb * 32 + q8 * 8;
          st_bf16x8(sb + SM_SB + (ch >> 6) * 16384 + sw128_off(j, ch & 63), s + q8 * 8);
        }
        if (dmp)
#pragma unroll
          for (int i = 0; i < 32; ++i) dbg[DBG_S + (cb * 32 + i) * 128 + j] = s[i];
      }
      // O^T lane j -> out[token r][h][j]
      float o[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tl + TM_O + half * 32, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = half * 32 + i;
          if (r < valid) out[((tok0 + r) * H + h) * D + j] = __float2bfloat16_rn(o[i]);
          if (dmp) dbg[DBG_O + r * 128 + j] = o[i];
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (sync_abort()) break;
  }

  if (*s_abort) {
    // Error path: let every copy and UMMA this CTA issued finish (bounded)
    // before the tensor memory is released.
    if (tid == 0) {
      for (int st = 0; st < 2; ++st)
        for (; stage_waited[st] < stage_issued[st]; ++stage_waited[st])
          mbar_wait(&bar_stage[st], stage_waited[st] & 1, WAIT_NS);
      for (; g_waited < g_issued; ++g_waited) mbar_wait(bar_g, g_waited & 1, WAIT_NS);
      for (; mma_waited < mma_issued; ++mma_waited) mbar_wait(bar_mma, mma_waited & 1, WAIT_NS);
    }
  } else if (fin) {
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      float s[32];
      tmem_ld32(tl + TM_S + cb * 32, s);
#pragma unroll
      for (int i = 0; i < 32; ++i) fin[sbase + (int64_t)(cb * 32 + i) * D + j] = s[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor [T_total][H][d] as a 3-D map (d innermost), box {box_d, 1, 64 tokens}.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, uint32_t esz, const void* ptr, int d, int H, int64_t Ttot,
              uint32_t box_d, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)Ttot};
  cuuint64_t strides[2] = {(cuuint64_t)d * esz, (cuuint64_t)H * d * esz};
  cuuint32_t box[3] = {box_d, 1, (cuuint32_t)CH};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fwd_tc_supported(int dk, int dv, bool bf16) { return bf16 && dk == D && dv == D; }

cudaError_t launch_fwd_tc_impl(const FwdArgs& a, cudaStream_t s, uint64_t wait_ns) {
  const int64_t Ttot = a.cu ? a.T : (int64_t)a.N * a.T;
  const unsigned blocks = (unsigned)((int64_t)a.N * a.H);
  if (blocks == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mg;
  // A map needs at least one token row; an all-empty batch still runs the
  // kernel (to copy init -> final) with maps that are never read.
  const int64_t Tmap = Ttot > 0 ? Ttot : 1;
  if (!make_map(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, D, a.H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.k, D, a.H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.v, D, a.H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.g, D, a.H, Tmap, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kda_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kda_fwd_tc_kernel<<<blocks, NTHR, SMEM_BYTES, s>>>(mq, mk, mv, mg, a.beta, a.init, (__nv_bfloat16*)a.out,
                                                     a.fin, a.cu, a.cu ? 0 : a.T, a.H, a.status, (float*)a.dbg,
                                                     wait_ns);
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t s) { return launch_fwd_tc_impl(a, s, WAIT_NS); }

int fwd_tc_debug_floats() { return DBG_FLOATS; }

}  // namespace kda
