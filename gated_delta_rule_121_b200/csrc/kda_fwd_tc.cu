// Chunked KDA forward on the sm_100a tensor cores (tcgen05 / TMEM / TMA).
// bf16 q, k, v, out with dk = dv = 128, fp32 decay, beta and state; chunk
// length C = 64.
//
// What it computes (Kimi K3 digest, "Kimi Delta Attention" section: chunk
// output = inter-chunk term (Gamma ⊙ Q) S + intra-chunk term A Ṽ), written
// out per chunk with the in-chunk cumulative log-decay G_r = sum_{s<=r} g_s
// (per key channel) and its chunk total G_C:
//   A_rs = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)    (s < r)
//   P_rs = sum_c q_rc k_sc exp(G_rc - G_sc)           (s <= r)
//   T    = (I + A)^-1,   T' = T diag(beta)
//   S'   = Diag(exp G_C) S                     (state decayed to chunk end)
//   QE   = Q ⊙ exp(G - G_C),  KE = K ⊙ exp(G - G_C),  KH = K ⊙ exp(G_C - G)
//   W'   = T' KE,   U = T' V,   Δ = U - W' S'
//   O    = QE S' + P Δ
//   S   <- S' + KH^T Δ
// which is the same section's recurrence unrolled over a chunk (QE S' =
// (Q ⊙ e^G) S and W' S' = T' (K ⊙ e^G) S).  The factors exp(G - G_C) grow
// up to exp(-G_C): with the digest's bounded decay ("Bounded decay" section,
// g >= -5) every tile is a dense matmul as long as a chunk's total decay is
// moderate.  A chunk whose total decay in some channel is below 2^-10 takes
// the general variant: its Gram matrices P, A come from four tensor-core
// Grams whose decay references sit at block boundaries between the two
// tokens of every pair (so no operand factor exceeds 1) plus the pairs inside
// 4-row groups on CUDA cores, the operands use the chunk START as reference
// (QE = Q e^G, KE = K e^G), and the scan decays S only after D1.
//
// Operands are fp16 (10-bit mantissa) with fp32 accumulation: the fp32
// state and every product stay accurate to well inside the bf16 output's own
// rounding.  Values that would not fit fp16 set KDA_ERR_RANGE: every
// operand overflow (V, S', W', the Gram tiles) reaches Δ as inf or NaN, so
// the range test is made once, on Δ, with a NaN-propagating maximum.
//
// Work split (one CTA of 16 warps per (sequence, head) chain, chunks in
// order), three groups:
//   warps 4-11, "front" group: for chunk c+2 — cumulative decay fused with
//     the operand scaling, the G1 Gram UMMA, and the P / A tiles;
//   warps 12-15, "back" group: for chunk c+1 — the triangular solve (CUDA
//     cores and warp-level tf32 MMAs), G2/G3 UMMAs for W'^T and U^T, and the
//     W'^T store;
//   warps 0-3, "scan" group (SG): for chunk c — the state recurrence:
//     decay S^T, D1 = { O^T = S'^T QE^T ;  Δ^T = U^T - S'^T W'^T }, Δ^T to
//     fp16, D2 = { S^T += Δ^T KH ;  O^T += Δ^T P^T }, output store.
// The state is kept TRANSPOSED in TMEM (lane j = value channel, column c =
// key channel) so that every UMMA has M = 128: the value channels.  S'^T and
// Δ^T are the A operands of D1/D2 straight from TMEM (fp16 pairs per
// column); every other operand is a 128-byte-swizzled fp16 tile in shared
// memory.  Q, K, V arrive by TMA two chunks ahead.  Each group has one
// elected thread that issues its UMMAs; mbarriers carry the hand-offs.
//
// MODE_GATED takes the model's raw prologue inputs instead (Kimi K3 digest,
// "Kimi Delta Attention" section: q, k L2-normalised, decay logits with a
// per-head scale; "Bounded decay" section: g = g_min sigmoid(exp(A_h) z)).
// The front group maps z to g while it forms the decay prefix and folds the
// per-row normalisation factors 1/|q_r|, 1/|k_r| into the operand scaling
// (fp32, before the fp16 rounding), so no normalised copy of q or k exists.
#include <cuda.h>

#include "kda_gate.cuh"
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

constexpr int CH = 64;  // chunk length
constexpr int D = 128;  // dk = dv
constexpr int NTHR = 512;  // scan (4 warps), front (8 warps) and back (4 warps) groups
constexpr float LOG2E = 1.4426950408889634f;
constexpr float FAST_MIN_LOG2 = -10.0f;  // chunk-total decay floor (log2) for the tensor-core Gram
constexpr float F16_SAFE = 60000.0f;     // |x| above this would overflow fp16 operands
constexpr uint64_t WAIT_NS = 2000000000ull;
// Start value of a transition run (MODE_SEG): the identity times 2^12.  The
// run is linear in its start (its values are zero), so its outputs and final
// state are scaled back by 2^-12 exactly; meanwhile the fp16 operand copies
// of the decaying state (entries of the transition, at most 1 in magnitude
// for normalised keys) stay clear of the fp16 subnormal range down to ~1e-8.
constexpr float TRANS_SCALE = 4096.0f;
constexpr float TRANS_UNSCALE = 1.0f / 4096.0f;

// ---- shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t STAGE_BYTES = 49152;  // [Q;K] 32 KB (per 64-channel half: Q rows, then K rows) + V 16 KB
constexpr uint32_t OFF_QK = 0, OFF_V = 32768;
constexpr uint32_t SM_KX = 2 * STAGE_BYTES;  // KH fp16 [s][c], x2          32 KB
constexpr uint32_t SM_P = SM_KX + 32768;     // P fp16 [r][s], x2            16 KB
constexpr uint32_t SM_WT = SM_P + 16384;     // W'^T fp16 [c][r]             16 KB
constexpr uint32_t SM_A = SM_WT + 16384;     // A fp32 [64][64]              16 KB
constexpr uint32_t SM_DG = SM_A + 16384;     // D_0, D_1 fp32 [32][32]        8 KB
constexpr uint32_t SM_X = SM_DG + 8192;      // X fp32 [32][32] (Y before)    4 KB
constexpr uint32_t SM_T10 = SM_X + 4096;     // T_10 fp32 [32][32]            4 KB
constexpr uint32_t SM_TP = SM_X;             // T' fp16 [64][64] over X, T_10  8 KB
constexpr uint32_t SM_OST = SM_T10 + 4096 + 4096;  // O staging bf16 [64][128] 16 KB (1024-aligned)
constexpr uint32_t SM_MISC = SM_OST + 16384;
constexpr uint32_t MISC_BYTES = 8704;
constexpr uint32_t SMEM_BYTES = SM_MISC + MISC_BYTES + 1024;

// misc layout
// Hand-offs: FULL (TMA -> front), GC (front -> scan: decay totals), OPS
// (front -> scan: QE ready), FR (front -> back: A tile and operands), AFREE (back -> front: A tile
// released), PRO (back -> scan: W'^T, U^T), G1 / G23 / D1A / D1 / D2
// (UMMA completions), BUF (stage and KX/P buffers free), DFREE (Δ^T columns free
// for the next U^T), WFREE (W'^T tile free).
enum Bar {
  B_FULL0 = 0, B_FULL1, B_G1, B_G23, B_D1A, B_D1, B_D2, B_GC0, B_GC1, B_OPS0, B_OPS1, B_FR0, B_FR1, B_AFREE,
  B_PRO0, B_PRO1, B_BUF0, B_BUF1, B_DFREE, B_WFREE, B_DRAIN_F, B_DRAIN_B, B_DRAIN_SG, B_NEVER, NUM_BARS
};
constexpr uint32_t MS_TMEM = 192, MS_ABORT = 196, MS_FAST = 200, MS_CNT = 208;  // MS_CNT: int[4]
constexpr uint32_t MS_T0 = 224;  // int64: clock at block start (timing dump)
constexpr uint32_t MS_BETA = 256;    // [2][64] fp32
constexpr uint32_t MS_GC = 768;      // [2][128] fp32: exp(G_C)
constexpr uint32_t MS_RED = 1792;    // [8][128] fp32 log2 sums
constexpr uint32_t MS_PAIRS = 5888;  // [64][8] fp32: P, A of the pairs inside 4-row groups (general chunks)
constexpr uint32_t MS_RQK = 7936;    // [16][8] fp32: 1/|q_r|, 1/|k_r| of each row group's 4 rows (MODE_GATED)
constexpr uint32_t MS_GATE = 8448;   // [2] fp32: -exp(A_h) log2(e), g_min (MODE_GATED)
constexpr uint32_t MS_END = 8464;
static_assert(NUM_BARS * 8 <= MS_TMEM, "barrier area");
static_assert(MS_END <= MISC_BYTES, "misc area");

// ---- TMEM columns
constexpr uint32_t TM_S = 0;        // S^T fp32, 128 cols
constexpr uint32_t TM_O = 128;      // O^T fp32, 2 x 64 cols
constexpr uint32_t TM_DELTA = 256;  // U^T, then Δ^T fp32; then Δ^T fp16 pairs (A operand) in its first 32 cols
constexpr uint32_t TM_G = 320;      // Gram [P ; A_raw], fp32, 64 cols
constexpr uint32_t TM_SB = 384;     // S'^T fp16 pairs (A operand), 64 cols
constexpr uint32_t TM_W = 448;      // W'^T fp32, 64 cols
constexpr uint32_t TMEM_COLS = 512;

// ---- debug dump (floats) for chain 0, chunk 0
constexpr int DBG_P = 0, DBG_A = 4096, DBG_T = 8192, DBG_W = 12288, DBG_U = 20480, DBG_DELTA = 28672,
              DBG_O = 36864, DBG_S = 45056, DBG_GC = 61440, DBG_TIME = 61568, DBG_FLOATS = 65664;
// DBG_TIME: int64 [64 chunks][32 events] of SM clock cycles since block start
// (events 0-7, 26, 29, 30 front group, 16-23 and 25 back group, 8-15, 24, 27, 28 scan group),
// chain 0 only.
constexpr int TIME_CHUNKS = 64;

// ------------------------------------------------------------------ helpers
// Shared-memory accesses are plain C++ through pointers derived from the
// shared array (so they compile to shared loads/stores and the compiler may
// schedule them freely between barriers).
// Four bf16 (two packed words, element 0 in the low half) to fp32: a bf16 is
// the upper half of the fp32 with the same value.
__device__ __forceinline__ float4 bf16x4_to_f32(uint2 u) {
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ void st_f16x4(uint8_t* p, float4 v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_f16x2(v.x, v.y), pack_f16x2(v.z, v.w));
}
__device__ __forceinline__ void st_f16x8(uint8_t* p, const float* v) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]),
                                            pack_f16x2(v[6], v[7]));
}
// Elementwise float4 arithmetic on the paired fp32 pipe (two lanes per instruction).
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  const float2 lo = __fmul2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
  const float2 hi = __fmul2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
  const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 sub4(float4 a, float4 b) {
  return add4(a, make_float4(-b.x, -b.y, -b.z, -b.w));
}
// max(|m|, |x|), propagating NaN (the sign of the result is not meaningful):
// the fp16 range test of a tensor-core operand, one instruction per element.
__device__ __forceinline__ float amax_nan(float m, float x) {
  float r;
  asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(x));
  return r;
}
__device__ __forceinline__ float4 ex2_4(float4 a) { return make_float4(ex2(a.x), ex2(a.y), ex2(a.z), ex2(a.w)); }
// Eight consecutive channels of one row (the front group's unit of work).
struct F8 {
  float4 a, b;
};
__device__ __forceinline__ F8 f8(float v) { return {make_float4(v, v, v, v), make_float4(v, v, v, v)}; }
__device__ __forceinline__ F8 add8(F8 x, F8 y) { return {add4(x.a, y.a), add4(x.b, y.b)}; }
__device__ __forceinline__ F8 sub8(F8 x, F8 y) { return {sub4(x.a, y.a), sub4(x.b, y.b)}; }
__device__ __forceinline__ F8 mul8(F8 x, F8 y) { return {mul4(x.a, y.a), mul4(x.b, y.b)}; }
__device__ __forceinline__ F8 ex2_8(F8 x) { return {ex2_4(x.a), ex2_4(x.b)}; }
__device__ __forceinline__ F8 bf16x8_to_f32(uint4 u) {
  return {bf16x4_to_f32(make_uint2(u.x, u.y)), bf16x4_to_f32(make_uint2(u.z, u.w))};
}
__device__ __forceinline__ void st_f16x8(uint8_t* p, F8 v) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_f16x2(v.a.x, v.a.y), pack_f16x2(v.a.z, v.a.w),
                                            pack_f16x2(v.b.x, v.b.y), pack_f16x2(v.b.z, v.b.w));
}
__device__ __forceinline__ float min8(F8 x) {
  return fminf(fminf(fminf(x.a.x, x.a.y), fminf(x.a.z, x.a.w)), fminf(fminf(x.b.x, x.b.y), fminf(x.b.z, x.b.w)));
}
// 32 bytes of read-only global data: one 256-bit load when the address is
// 32-byte aligned, else two 128-bit loads.
__device__ __forceinline__ F8 ldg8(const float* p, bool v8) {
  F8 r;
  if (v8) {
    asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(r.a.x), "=f"(r.a.y), "=f"(r.a.z), "=f"(r.a.w), "=f"(r.b.x), "=f"(r.b.y), "=f"(r.b.z),
                   "=f"(r.b.w)
                 : "l"(p));
  } else {
    r.a = __ldg(reinterpret_cast<const float4*>(p));
    r.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  return r;
}
// fp32 [64][64] with 16-byte units XOR-swizzled by row.
__device__ __forceinline__ uint32_t a_off(uint32_t r, uint32_t s) {
  return r * 256u + ((s >> 2) ^ (r & 7u)) * 16u + (s & 3u) * 4u;
}
// fp32 [32][32] with 16-byte units XOR-swizzled by row.
__device__ __forceinline__ uint32_t b_off(uint32_t r, uint32_t s) {
  return r * 128u + ((s >> 2) ^ (r & 7u)) * 16u + (s & 3u) * 4u;
}
// One 16x8 tile of D = A B with fp32 operands held in shared memory, K = 8 *
// KSTEPS, on the warp-level tensor path in tf32 (the MMA reads the leading 10
// mantissa bits of each operand).  The solve's inputs come from fp16 tensor-core
// operands and its outputs are rounded to fp16, so tf32 block products leave the
// end-to-end error unchanged (a CPU emulation of the kernel's rounding points:
// output relative error 1.70e-3 with exact or tf32 block products, mild and
// model-range decay alike).  fa(r, k) / fb(k, n) return the operand element
// addresses.
template <int KSTEPS, typename FA, typename FB>
__device__ __forceinline__ void warp_gemm_tf32(float (&d)[4], FA fa, FB fb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  d[0] = d[1] = d[2] = d[3] = 0.f;
  uint32_t av[KSTEPS][4], bv[KSTEPS][2];
  // ldmatrix row address of this lane: tile lane/8 = (rows 8 (tile & 1)..,
  // words 4 (tile >> 1)..) of the 16x8 A block.
  const int arow = (lane & 7) + 8 * ((lane >> 3) & 1), akof = 4 * (lane >> 4);
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {  // every fragment load first: one shared-memory latency
    const int k0 = 8 * ks;
    ldsm_x4(smem_u32(fa(arow, k0 + akof)), av[ks]);
    bv[ks][0] = __float_as_uint(*fb(k0 + t, g));
    bv[ks][1] = __float_as_uint(*fb(k0 + t + 4, g));
  }
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) mma_tf32_16x8x8(d, av[ks], bv[ks]);
}

// Bounded wait that also gives up when the other group has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t ns, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > ns) return false;
  }
  return true;
}

struct Ctx {
  uint8_t* sm;
  uint32_t sb;  // shared-window address of sm
  uint64_t* bars;
  volatile int* abort;
  uint32_t tmem;
  int h, H, nchunks;
  int64_t t0, L;
  DeviceStatus* status;
  uint64_t wait_ns;
  float* dbg;  // chain-0 debug dump or nullptr
  long long* tdbg;  // chain-0 phase timestamps or nullptr
  long long tstart;
  bool trans;       // MODE_SEG: this block runs the transition (zero values, identity start)
  bool first;       // MODE_SEG: first segment of a sequence, run from its initial state
  int64_t ckpt0;    // MODE_CKPT: checkpoint slot of this sequence's first interval
};

// MODE_GATED: per-token log-decays of 8 channels from their bf16 decay
// logits: g = g_min / (1 + 2^(-exp(A_h) log2(e) z)).  The prefix converts
// them to log2 units like the plain path's inputs (keeping that one multiply
// in both modes also keeps the front group's register allocation spill-free).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ F8 gate_8(uint4 u, float gz, float gmin) {
  F8 z = bf16x8_to_f32(u);
  float* e = &z.a.x;
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = gmin * rcp_approx(1.f + ex2(gz * e[i]));
  return z;
}
// MODE_GATED: 1/|x_r| for this thread's 4 rows of the raw q and k tiles (its 8
// channels), stored in the row group's entry of `tab` ([rg][0..3] = q,
// [rg][4..7] = k) for the group's threads to read where they scale the rows
// (the values do not stay in registers across the Gram).  The 8 partial sums
// of the 16 threads of a row group are reduce-scattered by recursive halving
// (offsets 8, 4, 2: lane pair l/2 ends with sum number l/2), then the pair
// adds its two halves; 8 shuffles instead of 4 x 8.
__device__ __forceinline__ void row_norms(const uint8_t* qb, const uint8_t* kb, int rg, int cc, float* tab) {
  float v[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t o = sw128_off(4 * rg + m, cc);
    const F8 a = bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + o));
    const F8 b = bf16x8_to_f32(*reinterpret_cast<const uint4*>(kb + o));
    const F8 a2 = mul8(a, a), b2 = mul8(b, b);
    v[m] = ((a2.a.x + a2.a.y) + (a2.a.z + a2.a.w)) + ((a2.b.x + a2.b.y) + (a2.b.z + a2.b.w));
    v[4 + m] = ((b2.a.x + b2.a.y) + (b2.a.z + b2.a.w)) + ((b2.b.x + b2.b.y) + (b2.b.z + b2.b.w));
  }
  const int l = threadIdx.x & 15;
  const bool b3 = l & 8, b2 = l & 4, b1 = l & 2;
  float h4[4], h2[2];
#pragma unroll
  for (int j = 0; j < 4; ++j) h4[j] = (b3 ? v[j + 4] : v[j]) + __shfl_xor_sync(0xffffffffu, b3 ? v[j] : v[j + 4], 8);
#pragma unroll
  for (int j = 0; j < 2; ++j) h2[j] = (b2 ? h4[j + 2] : h4[j]) + __shfl_xor_sync(0xffffffffu, b2 ? h4[j] : h4[j + 2], 4);
  float h1 = (b1 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? h2[0] : h2[1], 2);
  h1 += __shfl_xor_sync(0xffffffffu, h1, 1);
  if (!(l & 1)) tab[rg * 8 + (l >> 1)] = l2norm_scale(h1);
  __syncwarp();  // a row group is half a warp
}
// One factor of the table, read where it is used (a volatile shared load is
// not hoisted, so the factors do not occupy registers across the pass).
__device__ __forceinline__ float row_factor(const uint8_t* sm, int rg, int i) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_u32(sm + SM_MISC + MS_RQK + (rg * 8 + i) * 4)));
  return v;
}
// This row group's factors from the table.
__device__ __forceinline__ void row_factors(const uint8_t* sm, int rg, float (&rq)[4], float (&rk)[4]) {
  const float* tab = reinterpret_cast<const float*>(sm + SM_MISC + MS_RQK) + rg * 8;
  const float4 a = *reinterpret_cast<const float4*>(tab), b = *reinterpret_cast<const float4*>(tab + 4);
  rq[0] = a.x; rq[1] = a.y; rq[2] = a.z; rq[3] = a.w;
  rk[0] = b.x; rk[1] = b.y; rk[2] = b.z; rk[3] = b.w;
}

// Which group converts a chunk's V tile to fp16 in place: the back group,
// while it waits for the front's tiles (measured faster for the plain,
// checkpoint and segment builds), or the front group in its scaling pass
// (the fused-prologue build, whose front is the slower group).
template <int MODE>
constexpr bool V_IN_FRONT = MODE == MODE_GATED;

// Phase timestamp (elected thread only) for the timing dump.
__device__ __forceinline__ void tmark(const Ctx& x, int c, int ev) {
  if (x.tdbg && c < TIME_CHUNKS) x.tdbg[c * 32 + ev] = clock64() - x.tstart;
}

__device__ __forceinline__ bool cwait(const Ctx& x, int bar, uint32_t parity, int where) {
  if (wait_bar(&x.bars[bar], parity, x.wait_ns, x.abort)) return true;
  if (!*x.abort) record_error(x.status, KDA_ERR_TIMEOUT, where);
  *x.abort = 1;
  return false;
}

// Named-barrier ids of the three groups, their first threads and sizes:
// scan = warps 0-3, front = warps 4-11, back = warps 12-15.
constexpr int GRP_FRONT = 1, GRP_SG = 2, GRP_BACK = 3;
constexpr int FRONT_T = 256;
constexpr unsigned FRONT0 = 128, BACK0 = 384;
__device__ __forceinline__ unsigned grp_leader(int grp) {
  return grp == GRP_SG ? 0u : (grp == GRP_FRONT ? FRONT0 : BACK0);
}
__device__ __forceinline__ int grp_size(int grp) { return grp == GRP_FRONT ? FRONT_T : 128; }

// Group-uniform bounded wait: every thread of named-barrier group `grp`
// (all its threads) polls, then the group agrees on the outcome, so no thread can
// leave a loop while the others wait at a barrier or a .sync.aligned op.
//
// Only the group's first thread polls the mbarrier; the others block in the
// hardware named barrier, so waiting warps take no issue slots or shared
// memory bandwidth from the warps that are working.  The barrier (with the
// tcgen05 / proxy fences the callers place after it) carries the observed
// completion to the rest of the group.
__device__ __forceinline__ bool gwait(const Ctx& x, int bar, uint32_t parity, int where, int grp) {
  const bool elected = threadIdx.x == grp_leader(grp);
  bool ok = true;
  if (elected) {
    ok = wait_bar(&x.bars[bar], parity, x.wait_ns, x.abort);
    if (!ok) {
      if (!*x.abort) record_error(x.status, KDA_ERR_TIMEOUT, where);
      *x.abort = 1;
    }
  }
  ok = named_sync_and(grp, grp_size(grp), ok);
  // Each thread also observes the completed phase itself (an acquire that
  // returns at once), so the data it guards is visible to every thread.
  if (ok && !elected) mbar_try_wait(&x.bars[bar], parity);
  return ok;
}

__device__ __forceinline__ int chunk_valid(const Ctx& x, int c) {
  const int64_t rem = x.L - (int64_t)c * CH;
  return rem < CH ? (int)rem : CH;
}

// ============================================== front and back groups
// Two groups share the chunk prologue and run one chunk apart: while the
// back group finishes chunk c, the front group starts chunk c+1.
//   front (warps 4-11, 256 threads): decay prefix fused with operand
//     scaling, the G1 Gram UMMA, and the P / A tiles;
//   back (warps 12-15, 128 threads): the triangular solve, T', the G2/G3
//     UMMAs and W'^T.
// Row-wise front work: thread f owns rows 4 (f / 16) .. + 3 and channels
// 8 (f % 16) .. + 7, so every tile access is 16 bytes wide.  TMEM work: a
// warp reads the lane quarter (warp index mod 4) it is allowed to access.
constexpr int GRP = 128;  // threads of the scan and back groups

// P (fp16, lower triangle with the diagonal) and A (fp32, beta-scaled; the
// solve reads only its strictly lower part) from one 32-column slice of
// [P ; A_raw] per thread: TMEM lane ti (row ti of [P ; A_raw]), columns
// 32 chh .. 32 chh + 31.
__device__ __forceinline__ void store_pa(uint8_t* sm, int b2, int ti, int chh, const float* s_beta,
                                         float (&r0)[32]) {
  if (ti < CH) {  // P row ti
    const int r = ti;
#pragma unroll
    for (int s = 0; s < 32; ++s)
      if (chh * 32 + s > r) r0[s] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      st_f16x8(sm + SM_P + b2 * 8192 + r * 128 + ((((4 * chh + k) ^ r) & 7) << 4), r0 + 8 * k);
  } else {  // A row r = beta_r (row r of the decayed K K^T)
    const int r = ti - CH;
    const float4 b = make_float4(s_beta[r], s_beta[r], s_beta[r], s_beta[r]);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<float4*>(sm + SM_A + a_off(r, 32 * chh + 4 * u)) =
          mul4(make_float4(r0[4 * u], r0[4 * u + 1], r0[4 * u + 2], r0[4 * u + 3]), b);
  }
}

// General chunks (total decay of the chunk below the end-referenced range in
// some channel): P and A on the tensor cores with the reference of every
// decay factor placed between the two tokens it connects, so that no operand
// is scaled by more than 1.  Level p = 64, 32, 16, 8 splits the rows into
// aligned p-blocks with an earlier and a later half and takes as reference
// R the cumulative decay G at the last row of the earlier half; it scales a
// later row r by e^{G_r - R} and an earlier row by e^{R - G_r} (both <= 1 for
// a non-positive log decay), so its Gram [Q ; K] K^T holds the products
// q_r k_s e^{G_r - G_s} exactly for the pairs r > s that straddle one of its
// boundaries: those whose highest differing index bit is p/2.  Levels run
// from p = 64 down; each keeps the pairs with r and s in the same p-block,
// so the finest level that contains a pair wins.  The pairs inside one
// 4-row group (and the diagonal of P) are one thread's own rows: they are
// summed exactly on CUDA cores from the per-token ratios e^{g}.  Q and K
// rows scaled for a level go to a tile of the stage layout whose two
// 64-channel halves are the A tile and KX[b2] (both released: AFREE and BUF
// were waited for); the row-group end values of G (the references) are
// staged in the P tile.
template <int MODE>
__device__ __forceinline__ bool level_gram(const Ctx& x, int c, int b2, const F8 (&gv)[4], int& g1_ph) {
  const int f = threadIdx.x - FRONT0;
  const int wq = f >> 5, lane = f & 31, lq = wq & 3, chh = wq >> 2;
  const int rg = f >> 4, ch0 = 8 * (f & 15), hh = ch0 >> 6, cc = ch0 & 63;
  uint8_t* sm = x.sm;
  const uint32_t sb = x.sb;
  float* s_ref = reinterpret_cast<float*>(sm + SM_P + b2 * 8192);  // [16][128]: G at row 4 k + 3
  float* s_pairs = reinterpret_cast<float*>(sm + SM_MISC + MS_PAIRS);
  const float* s_beta = reinterpret_cast<const float*>(sm + SM_MISC + MS_BETA) + b2 * 64;
  const uint8_t* qb = sm + b2 * STAGE_BYTES + OFF_QK + hh * 16384;
  const uint8_t* kb = qb + 8192;
  uint8_t* lt = sm + (hh ? SM_KX + b2 * 16384 : SM_A);  // this thread's channel half of the level tile
  const uint32_t tl = x.tmem + ((uint32_t)(lq * 32) << 16);
  const int ti = 32 * lq + lane, r = ti & 63;

  {  // G at the end of this thread's row group (a reference of the levels)
    const F8 ge = add8(add8(add8(gv[0], gv[1]), gv[2]), gv[3]);
    *reinterpret_cast<float4*>(s_ref + rg * 128 + ch0) = ge.a;
    *reinterpret_cast<float4*>(s_ref + rg * 128 + ch0 + 4) = ge.b;
  }
  named_sync(GRP_FRONT, FRONT_T);  // references staged

  // Level L: scale this thread's Q and K rows into the level tile.
  auto write_tile = [&](int L) {
    const int p = 1 << L;
    // row 4 rg + m times 2^{x_m} (log2 units); reference R: the end of row
    // group kref (another thread's rows)
    const int kref = (rg & ~(p / 4 - 1)) + p / 8 - 1;
    const bool later = ((4 * rg) & (p / 2)) != 0;
    F8 dr = sub8(f8(0.f), F8{*reinterpret_cast<const float4*>(s_ref + kref * 128 + ch0),
                             *reinterpret_cast<const float4*>(s_ref + kref * 128 + ch0 + 4)});  // G_r - R
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t o = sw128_off(4 * rg + m, cc);
      dr = add8(dr, gv[m]);
      const F8 e = ex2_8(later ? dr : sub8(f8(0.f), dr));
      if constexpr (MODE == MODE_GATED) {  // with the row's normalisation factors
        const float* tab = reinterpret_cast<const float*>(sm + SM_MISC + MS_RQK) + rg * 8;
        st_f16x8(lt + o, mul8(bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + o)), mul8(e, f8(tab[m]))));
        st_f16x8(lt + 8192 + o, mul8(bf16x8_to_f32(*reinterpret_cast<const uint4*>(kb + o)), mul8(e, f8(tab[4 + m]))));
      } else {
        st_f16x8(lt + o, mul8(bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + o)), e));
        st_f16x8(lt + 8192 + o, mul8(bf16x8_to_f32(*reinterpret_cast<const uint4*>(kb + o)), e));
      }
    }
    fence_proxy_async_smem();
  };
  // [Q ; K] K^T of the level tile (M=128, N=64, K=128) -> TM_G, once every
  // thread has written its rows and finished reading the previous level.
  auto issue = [&]() {
    tc_fence_before();
    named_sync(GRP_FRONT, FRONT_T);
    if (f == 0) {
      tc_fence_after();
      const uint32_t id = idesc_f16_f32(128, 64, 0, 0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t base = (i >> 2) ? sb + SM_KX + b2 * 16384 : sb + SM_A;
        const uint64_t da = sdesc_sw128(base + (i & 3) * 32, 16, 1024);
        const uint64_t db = sdesc_sw128(base + 8192 + (i & 3) * 32, 16, 1024);
        umma_ss(x.tmem + TM_G, da, db, id, i > 0);
      }
      umma_commit(&x.bars[B_G1]);
    }
  };
  auto pairs = [&]() {
  {  // While the first level runs: the pairs s <= r inside this thread's rows
     // 4 rg .. 4 rg + 3 over its 8 channels, pv[] = P (10 pairs with the
     // diagonal), av[] = A (6 pairs); e^{G_r - G_s} is the running product of
     // the ratios e^{g_t}, s < t <= r.
    float pv[10] = {}, av[6] = {};
#pragma unroll 1
    for (int hq = 0; hq < 2; ++hq) {  // 4 channels at a time
      int ip = 0, ia = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const float4 ks = bf16x4_to_f32(*reinterpret_cast<const uint2*>(kb + sw128_off(4 * rg + s, cc) + 8 * hq));
        float4 e = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
        for (int rr = s; rr < 4; ++rr) {
          if (rr > s) e = mul4(e, ex2_4(hq ? gv[rr].b : gv[rr].a));
          const uint32_t o = sw128_off(4 * rg + rr, cc) + 8 * hq;
          const float4 ke = mul4(ks, e);
          const float4 pq = mul4(bf16x4_to_f32(*reinterpret_cast<const uint2*>(qb + o)), ke);
          pv[ip++] += (pq.x + pq.y) + (pq.z + pq.w);
          if (rr > s) {
            const float4 pk = mul4(bf16x4_to_f32(*reinterpret_cast<const uint2*>(kb + o)), ke);
            av[ia++] += (pk.x + pk.y) + (pk.z + pk.w);
          }
        }
      }
    }
    if constexpr (MODE == MODE_GATED) {  // the pairs' normalisation factors
      float rq[4], rk[4];
      row_factors(sm, rg, rq, rk);
      int ip = 0, ia = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int rr = s; rr < 4; ++rr) {
          pv[ip++] *= rq[rr] * rk[s];
          if (rr > s) av[ia++] *= rk[rr] * rk[s];
        }
    }
    // Sum over the 16 threads of the row group (lanes differing in bits 0-3).
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
#pragma unroll
      for (int i = 0; i < 10; ++i) pv[i] += __shfl_xor_sync(0xffffffffu, pv[i], o);
#pragma unroll
      for (int i = 0; i < 6; ++i) av[i] += __shfl_xor_sync(0xffffffffu, av[i], o);
    }
    if ((f & 15) == 0) {  // [r][0..3]: P_{r, 4 rg + j};  [r][4..7]: A_{r, 4 rg + j} (j < r - 4 rg)
      int ip = 0, ia = 0;
      float tp[4][4] = {}, ta[4][4] = {};
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int rr = s; rr < 4; ++rr) {
          tp[rr][s] = pv[ip++];
          if (rr > s) ta[rr][s] = av[ia++];
        }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float* row = s_pairs + (4 * rg + m) * 8;
        *reinterpret_cast<float4*>(row) = make_float4(tp[m][0], tp[m][1], tp[m][2], tp[m][3]);
        *reinterpret_cast<float4*>(row + 4) = make_float4(ta[m][0], ta[m][1], ta[m][2], ta[m][3]);
      }
    }
  }

  };
  float acc[32] = {};
  // Pass L = 7 only starts level 64 (and, while it runs, the pairs inside
  // 4-row groups); pass L takes level L's Gram and starts level L - 1.
  // Level 64 fills acc; levels 32, 16, 8 overwrite the pairs inside their blocks.
#pragma unroll 1
  for (int L = 7; L >= 3; --L) {
    if (L < 7) {
      if (!gwait(x, B_G1, g1_ph, 16, GRP_FRONT)) return false;
      g1_ph ^= 1;
      tc_fence_after();
    }
    if (L > 3) write_tile(L - 1);  // the tile is free again; TM_G still holds level L
    // (warp-uniform) below level 64, only a warp whose rows and columns share a
    // 32-block has pairs to take
    if (L == 6 || (L < 6 && (lq & 1) == chh)) {
      const int rb = r >> L;
#pragma unroll
      for (int hv = 0; hv < 4; ++hv) {
        float val[8];
        tmem_ld8(tl + TM_G + chh * 32 + hv * 8, val);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (rb == ((32 * chh + 8 * hv + u) >> L)) acc[8 * hv + u] = val[u];
      }
    }
    if (L > 3) issue();
    if (L == 7) {
      if (f == 0) tmark(x, c, 29);
      pairs();
    }
  }
  if (f == 0) tmark(x, c, 30);
  if ((lq & 1) == chh) {  // the pairs inside 4-row groups
    const float4 t = *reinterpret_cast<const float4*>(s_pairs + r * 8 + (ti < CH ? 0 : 4));
    const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if ((r >> 2) == ((32 * chh + u) >> 2)) acc[u] = tv[u & 3];
  }
  // Every level's UMMA has completed and every thread is past the last
  // level's tile barrier, so the P tile (reference table) and the A tile
  // (level tile half) may be overwritten.
  store_pa(sm, b2, ti, chh, s_beta, acc);
  tc_fence_before();
  named_sync(GRP_FRONT, FRONT_T);  // TMEM reads done before the next G1
  return true;
}

// Debug dumps (chain 0, chunk 0): P (fp16 tile) and A (fp32 tile); T'; W'
// (from the fp16 W'^T tile) and U (TMEM, before D1).
__device__ __noinline__ void dump_pa(float* dbg, const uint8_t* sm, int b2, int p) {
  for (int e = p; e < 4096; e += FRONT_T) {
    const int r = e >> 6, s = e & 63;
    const uint16_t u = *reinterpret_cast<const uint16_t*>(sm + SM_P + b2 * 8192 + sw128_off(r, s));
    dbg[DBG_P + e] = __half2float(*reinterpret_cast<const __half*>(&u));
    dbg[DBG_A + e] = s < r ? *reinterpret_cast<const float*>(sm + SM_A + a_off(r, s)) : 0.f;
  }
}
__device__ __noinline__ void dump_t(float* dbg, const uint8_t* sm, int p) {
  for (int e = p; e < 4096; e += GRP) {
    const uint16_t u = *reinterpret_cast<const uint16_t*>(sm + SM_TP + sw128_off(e >> 6, e & 63));
    dbg[DBG_T + e] = __half2float(*reinterpret_cast<const __half*>(&u));
  }
}
__device__ __noinline__ void dump_wu(float* dbg, const uint8_t* sm, uint32_t tmem, int p) {
  for (int e = p; e < 8192; e += GRP) {
    const int r = e >> 7, c = e & 127;  // W'[r][c] = W'^T[c][r]
    const uint16_t u = *reinterpret_cast<const uint16_t*>(sm + SM_WT + sw128_off(c, r));
    dbg[DBG_W + e] = __half2float(*reinterpret_cast<const __half*>(&u));
  }
  const int lq = p >> 5;  // lane quarter of this warp
  const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16);
  const int j = lq * 32 + (p & 31);
  float u0[32];
  for (int half = 0; half < 2; ++half) {
    tmem_ld32(tl + TM_DELTA + half * 32, u0);
    for (int i = 0; i < 32; ++i) dbg[DBG_U + (half * 32 + i) * 128 + j] = u0[i];
  }
}

template <int MODE>
__device__ __forceinline__ void front_group(const Ctx& x, const float* __restrict__ g, const float* __restrict__ beta,
                            const void* tmg, int (&consumed)[2]) {
  const int f = threadIdx.x - FRONT0;  // 0..255
  const int wq = f >> 5, lane = f & 31;
  const int lq = wq & 3, chh = wq >> 2;                      // TMEM lane quarter, column half
  const int rg = f >> 4, ch0 = 8 * (f & 15), hh = ch0 >> 6, cc = ch0 & 63;
  const uint32_t tl = x.tmem + ((uint32_t)(lq * 32) << 16);
  uint8_t* sm = x.sm;
  const uint32_t sb = x.sb;
  float* s_red = reinterpret_cast<float*>(sm + SM_MISC + MS_RED);  // [8][128] log2 sums, one row per warp
  const int H = x.H;
  const bool g32 = (reinterpret_cast<uintptr_t>(g) & 31u) == 0;

  // Register prefetch of this thread's g rows (4 rows x 8 channels) and of beta.
  auto load_g = [&](int c, F8(&gv)[4], float& bv) {
    const int valid = c < x.nchunks ? chunk_valid(x, c) : 0;
    const int64_t tok0 = x.t0 + (int64_t)c * CH;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int r = 4 * rg + m;
      if constexpr (MODE == MODE_GATED) {
        // the raw bf16 decay logits (their bits in the first half of the
        // row); the prefix maps them to log-decays.  Rows past the end get
        // -inf, whose gate is exactly 0.
        const uint4 u = r < valid ? __ldg(reinterpret_cast<const uint4*>(
                                        reinterpret_cast<const __nv_bfloat16*>(g) + ((tok0 + r) * H + x.h) * D + ch0))
                                  : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
        gv[m].a = make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
      } else {
        gv[m] = r < valid ? ldg8(g + ((tok0 + r) * H + x.h) * D + ch0, g32) : f8(0.f);
      }
    }
    bv = (f < CH && f < valid) ? __ldg(beta + (tok0 + f) * H + x.h) : 0.f;
  };

  // The decay rows of a chunk are read with per-thread loads; an L2 prefetch
  // of the chunk's [64 x 128] fp32 tile two chunks ahead keeps those loads
  // short.
  if (f == 0) {
    for (int c = 0; c < 2 && c < x.nchunks; ++c) tma_prefetch_l2_3d(tmg, 0, x.h, (int)(x.t0 + (int64_t)c * CH));
  }
  F8 gv[4];
  float bv;
  load_g(0, gv, bv);
  int g1_ph = 0;

  for (int c = 0; c < x.nchunks; ++c) {
    const int b2 = c & 1;
    const int valid = chunk_valid(x, c);
    const bool dmp = x.dbg && c == 0;
    const uint32_t stg = sb + b2 * STAGE_BYTES;
    float* s_gc = reinterpret_cast<float*>(sm + SM_MISC + MS_GC) + b2 * 128;
    float* s_beta = reinterpret_cast<float*>(sm + SM_MISC + MS_BETA) + b2 * 64;
    volatile int* s_fast = reinterpret_cast<volatile int*>(sm + SM_MISC + MS_FAST) + b2;

    if (f == 0) {
      tmark(x, c, 0);
      if (c + 2 < x.nchunks) tma_prefetch_l2_3d(tmg, 0, x.h, (int)(x.t0 + (int64_t)(c + 2) * CH));
    }
    // ---- (a1) decay prefix in log2 units (registers only): this thread's
    // 4-row sums; the two row groups of a warp combine by shuffle, the eight
    // warps through shared memory; then the offsets of the earlier row
    // groups and the chunk total G_C.
    F8 acc = f8(0.f);
    const F8 l2e = f8(LOG2E);
    if constexpr (MODE == MODE_GATED) {
      const float* gc = reinterpret_cast<const float*>(x.sm + SM_MISC + MS_GATE);
      const float gz = gc[0], gmin = gc[1];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        gv[m] = gate_8(make_uint4(__float_as_uint(gv[m].a.x), __float_as_uint(gv[m].a.y),
                                  __float_as_uint(gv[m].a.z), __float_as_uint(gv[m].a.w)), gz, gmin);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      gv[m] = mul8(gv[m], l2e);
      acc = add8(acc, gv[m]);
    }
    F8 other;  // the other row group of this warp (lane ^ 16)
    other.a.x = __shfl_xor_sync(0xffffffffu, acc.a.x, 16); other.a.y = __shfl_xor_sync(0xffffffffu, acc.a.y, 16);
    other.a.z = __shfl_xor_sync(0xffffffffu, acc.a.z, 16); other.a.w = __shfl_xor_sync(0xffffffffu, acc.a.w, 16);
    other.b.x = __shfl_xor_sync(0xffffffffu, acc.b.x, 16); other.b.y = __shfl_xor_sync(0xffffffffu, acc.b.y, 16);
    other.b.z = __shfl_xor_sync(0xffffffffu, acc.b.z, 16); other.b.w = __shfl_xor_sync(0xffffffffu, acc.b.w, 16);
    const F8 wsum = add8(acc, other);
    if (lane < 16) {
      *reinterpret_cast<float4*>(s_red + wq * 128 + ch0) = wsum.a;
      *reinterpret_cast<float4*>(s_red + wq * 128 + ch0 + 4) = wsum.b;
    }
    named_sync(GRP_FRONT, FRONT_T);
    F8 tot = f8(0.f), off = (lane >= 16) ? other : f8(0.f);  // tot: G_C
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const F8 v = {*reinterpret_cast<const float4*>(s_red + q * 128 + ch0),
                    *reinterpret_cast<const float4*>(s_red + q * 128 + ch0 + 4)};
      if (q < wq) off = add8(off, v);
      tot = add8(tot, v);
    }
    const bool fast = named_sync_and(GRP_FRONT, FRONT_T, min8(tot) >= FAST_MIN_LOG2);
    gv[0] = add8(gv[0], off);  // from here the running sum of gv[0..m] is G of row 4 rg + m
    if (f == 0) tmark(x, c, 1);
    // Per-chunk values for the scan and back groups, in buffers [b2] that the
    // scan of chunk c-2 has released.
    auto publish = [&]() {
      if (rg == 0) {
        const F8 e = ex2_8(tot);
        *reinterpret_cast<float4*>(s_gc + ch0) = e.a;
        *reinterpret_cast<float4*>(s_gc + ch0 + 4) = e.b;
      }
      if (f == 0) *s_fast = fast ? 1 : 0;
      if (f < CH) s_beta[f] = bv;
      if (dmp && rg == 0) {
        const float LN2 = 0.6931471805599453f;
        const float tv[8] = {tot.a.x, tot.a.y, tot.a.z, tot.a.w, tot.b.x, tot.b.y, tot.b.z, tot.b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) x.dbg[DBG_GC + ch0 + i] = tv[i] * LN2;
      }
      mbar_arrive(&x.bars[B_GC0 + b2]);  // one arrival per thread, after its own writes
    };
    if (!fast) {  // the general Gram works in P[b2], KX[b2] and the A tile
      if (c >= 2 && !gwait(x, B_BUF0 + b2, ((c >> 1) - 1) & 1, 11, GRP_FRONT)) break;
      publish();
      if (c >= 1 && !gwait(x, B_AFREE, (c - 1) & 1, 13, GRP_FRONT)) break;
    }
    if (!gwait(x, B_FULL0 + b2, (c >> 1) & 1, 12, GRP_FRONT)) break;
    ++consumed[b2];
    if (f == 0) tmark(x, c, 2);
    uint8_t* qb = sm + b2 * STAGE_BYTES + OFF_QK + hh * 16384;
    uint8_t* kb = qb + 8192;
    uint8_t* vb = sm + b2 * STAGE_BYTES + OFF_V + hh * 8192;
    uint8_t* khb = sm + SM_KX + b2 * 16384 + hh * 8192;
    if (valid < CH) {
      // Rows past the end of a sequence's last chunk hold other data: zero
      // this thread's rows and channels of the raw tiles, so the scaling
      // pass (and the general Gram) needs no per-row mask.
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int r = 4 * rg + m;
        if (r >= valid) {
          const uint32_t o = sw128_off(r, cc);
          *reinterpret_cast<uint4*>(qb + o) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(kb + o) = make_uint4(0u, 0u, 0u, 0u);
          if constexpr (V_IN_FRONT<MODE>) *reinterpret_cast<uint4*>(vb + o) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    if constexpr (MODE == MODE_GATED) row_norms(qb, kb, rg, cc, reinterpret_cast<float*>(sm + SM_MISC + MS_RQK));
    if (!fast) {
      if (!level_gram<MODE>(x, c, b2, gv, g1_ph)) break;
      // G_C again from the warp sums (the same additions in the same order),
      // so that it is not held in registers across the Gram.
      tot = f8(0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        tot = add8(tot, F8{*reinterpret_cast<const float4*>(s_red + q * 128 + ch0),
                           *reinterpret_cast<const float4*>(s_red + q * 128 + ch0 + 4)});
    }

    // ---- (a2) operand scaling, row by row: E = e^{G_r - ref} (ref = G_C on
    // fast chunks, 0 otherwise), H = e^{G_C - G_r}.  QE and KE (fp16) go in
    // place (the back group converts V); KH goes to KX[b2] once the scan of
    // chunk c-2 has released it.
    uint4 kraw[4];  // raw K rows, kept for KH
    {
      F8 gr = f8(0.f);
#pragma unroll
      for (int mb = 0; mb < 4; mb += 2) {
        uint4 qr[2], vr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // this batch's loads first, then the in-place stores
          const uint32_t o = sw128_off(4 * rg + mb + i, cc);
          qr[i] = *reinterpret_cast<const uint4*>(qb + o);
          kraw[mb + i] = *reinterpret_cast<const uint4*>(kb + o);
          if constexpr (V_IN_FRONT<MODE>) vr[i] = *reinterpret_cast<const uint4*>(vb + o);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int m = mb + i;
          const uint32_t o = sw128_off(4 * rg + m, cc);
          gr = add8(gr, gv[m]);
          const F8 fw = ex2_8(fast ? sub8(gr, tot) : gr);
          if constexpr (MODE == MODE_GATED) {
            st_f16x8(qb + o, mul8(bf16x8_to_f32(qr[i]), mul8(fw, f8(row_factor(sm, rg, m)))));
            st_f16x8(kb + o, mul8(bf16x8_to_f32(kraw[m]), mul8(fw, f8(row_factor(sm, rg, 4 + m)))));
          } else {
            st_f16x8(qb + o, mul8(bf16x8_to_f32(qr[i]), fw));
            st_f16x8(kb + o, mul8(bf16x8_to_f32(kraw[m]), fw));
          }
          if constexpr (V_IN_FRONT<MODE>) st_f16x8(vb + o, bf16x8_to_f32(vr[i]));
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(&x.bars[B_OPS0 + b2]);  // QE is ready for the scan's D1a
    if (f == 0) tmark(x, c, 3);
    if (fast) {
      if (c >= 2 && !gwait(x, B_BUF0 + b2, ((c >> 1) - 1) & 1, 11, GRP_FRONT)) break;
      publish();
    }
    if (f == 0) tmark(x, c, 4);
    {
      F8 gr = f8(0.f);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t o = sw128_off(4 * rg + m, cc);
        gr = add8(gr, gv[m]);
        if constexpr (MODE == MODE_GATED)
          st_f16x8(khb + o, mul8(bf16x8_to_f32(kraw[m]), mul8(ex2_8(sub8(tot, gr)), f8(row_factor(sm, rg, 4 + m)))));
        else
          st_f16x8(khb + o, mul8(bf16x8_to_f32(kraw[m]), ex2_8(sub8(tot, gr))));
      }
    }
    fence_proxy_async_smem();
    named_sync(GRP_FRONT, FRONT_T);
    if (f == 0) tmark(x, c, 5);

    if (fast) {
      // ---- G1: [P ; A_raw] = [QE ; KE] . KH^T   (M=128, N=64, K=128)
      if (f == 0) {
        bool ok = true;
        if (c >= 1) ok = cwait(x, B_AFREE, (c - 1) & 1, 14);  // the back group is done with A of c-1
        if (ok) {
          tc_fence_after();
          const uint32_t id = idesc_f16_f32(128, 64, 0, 0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint64_t da = sdesc_sw128(stg + OFF_QK + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
            const uint64_t db = sdesc_sw128(sb + SM_KX + b2 * 16384 + (i >> 2) * 8192 + (i & 3) * 32, 16, 1024);
            umma_ss(x.tmem + TM_G, da, db, id, i > 0);
          }
          umma_commit(&x.bars[B_G1]);
        }
        tmark(x, c, 6);
      }
      if (!gwait(x, B_G1, g1_ph, 15, GRP_FRONT)) break;
      g1_ph ^= 1;
      tc_fence_after();
      if (f == 0) tmark(x, c, 7);
      // TMEM lane 32 lq + lane is row ti of [P ; A_raw]; this warp reads
      // columns 32 chh .. 32 chh + 31.
      float r0[32];
      tmem_ld32(tl + TM_G + chh * 32, r0);
      store_pa(sm, b2, 32 * lq + lane, chh, s_beta, r0);
      tc_fence_before();
    }
    // The next chunk's decay rows are requested after this chunk's last TMEM
    // read and tile stores, so that their latency overlaps the barrier below
    // (only named barriers follow until they are used; a wait on an mbarrier
    // or a TMEM load with these loads in flight would stall until they land).
    // Measured faster for the plain and gated modes only (the checkpoint and
    // segment builds lost 8-9 %), which request them at the end instead.
    constexpr bool early_g = MODE == MODE_PLAIN || MODE == MODE_GATED;
    if constexpr (early_g) load_g(c + 1, gv, bv);
    fence_proxy_async_smem();  // P is read by the D2 UMMA
    if (dmp) {
      named_sync(GRP_FRONT, FRONT_T);
      dump_pa(x.dbg, sm, b2, f);
    }
    named_sync(GRP_FRONT, FRONT_T);  // the front's TMEM reads are done before the next G1
    mbar_arrive(&x.bars[B_FR0 + b2]);
    if (f == 0) tmark(x, c, 26);
    if constexpr (!early_g) load_g(c + 1, gv, bv);
  }
}

template <int MODE>
__device__ __forceinline__ void back_group(const Ctx& x) {
  const int k = threadIdx.x - BACK0;  // 0..127
  const int bw = k >> 5, lane = k & 31;
  const uint32_t tl = x.tmem + ((uint32_t)(bw * 32) << 16);
  const int ti = bw * 32 + lane;  // this thread's TMEM lane
  uint8_t* sm = x.sm;
  const uint32_t sb = x.sb;
  int g23_ph = 0;

  for (int c = 0; c < x.nchunks; ++c) {
    const int b2 = c & 1;
    const bool dmp = x.dbg && c == 0;
    const uint32_t stg = sb + b2 * STAGE_BYTES;
    const float* s_beta = reinterpret_cast<const float*>(sm + SM_MISC + MS_BETA) + b2 * 64;

    if (k == 0) tmark(x, c, 16);
    // V of chunk c to fp16 in place for G3 (U^T = V^T T'^T) while the front
    // forms this chunk's tiles: rows past the end of a sequence become zero,
    // and so does every value of a transition run (segment mode).
    if constexpr (!V_IN_FRONT<MODE>) {
      if (!gwait(x, B_FULL0 + b2, (c >> 1) & 1, 25, GRP_BACK)) break;
      const int valid = chunk_valid(x, c);
      uint8_t* vbase = sm + b2 * STAGE_BYTES + OFF_V;
#pragma unroll 4
      for (int i = 0; i < 8; ++i) {  // 64 rows x 2 channel halves x 8 pieces of 8 channels
        const int p = k + GRP * i, row = p >> 4;
        uint8_t* ptr = vbase + ((p >> 3) & 1) * 8192 + sw128_off(row, 8 * (p & 7));
        const uint4 raw = *reinterpret_cast<const uint4*>(ptr);
        st_f16x8(ptr, (row < valid && !x.trans) ? bf16x8_to_f32(raw) : f8(0.f));
      }
      fence_proxy_async_smem();
    }
    if (!gwait(x, B_FR0 + b2, (c >> 1) & 1, 21, GRP_BACK)) break;
    if (k == 0) tmark(x, c, 17);

    // ---- (a3) T = (I + A)^-1 by blocks.  16x16 diagonal inverses E_a by
    // forward substitution; D_b = [[E_2b, 0], [-E_2b+1 A'_b E_2b, E_2b+1]] are
    // the 32x32 diagonal inverses; T_10 = -D_1 (A_10 D_0).
    // T' = T diag(beta) as fp16 [r][s] in the TP tile.
    if (k < 64) {
      // Forward substitution down the rows of diagonal block a (thread:
      // column jj of its inverse): x[r] = [r == jj] - sum_{s<r} A[r][s] x[s].
      // The A rows are float4 loads that do not depend on x; only the
      // strictly lower entries are read.
      const int a = k >> 4, jj = k & 15;
      float xs[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int u = 0; u < (r + 3) / 4; ++u) {
          const float4 a4 = *reinterpret_cast<const float4*>(sm + SM_A + a_off(16 * a + r, 16 * a + 4 * u));
          acc0 = fmaf(a4.x, xs[4 * u], acc0);
          if (4 * u + 1 < r) acc1 = fmaf(a4.y, xs[4 * u + 1], acc1);
          if (4 * u + 2 < r) acc0 = fmaf(a4.z, xs[4 * u + 2], acc0);
          if (4 * u + 3 < r) acc1 = fmaf(a4.w, xs[4 * u + 3], acc1);
        }
        xs[r] = ((r == jj) ? 1.f : 0.f) - (acc0 + acc1);
      }
      // E_a -> diagonal 16x16 block of D_{a/2}
      const uint32_t db = SM_DG + (a >> 1) * 4096;
      const int o = (a & 1) * 16;
#pragma unroll
      for (int r = 0; r < 16; ++r) *reinterpret_cast<float*>(sm + db + b_off(o + r, o + jj)) = xs[r];
    } else {  // zero the upper-right 16x16 block of D_0 and D_1
      const int t = k - 64, b = t >> 5, rr = (t & 31) >> 1, cb = 16 + (t & 1) * 8;
#pragma unroll
      for (int i = 0; i < 8; i += 4)
        *reinterpret_cast<float4*>(sm + SM_DG + b * 4096 + b_off(rr, cb + i)) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    named_sync(GRP_BACK, GRP);
    if (k == 0) tmark(x, c, 18);
    const int lg = lane >> 2, lt = lane & 3;  // mma fragment coordinates
    {  // Y_b = A'_b E_2b (A'_b = A[32b+16 .. +16][32b .. +16]), then F_b = -E_2b+1 Y_b
      const int b = bw >> 1, nt = bw & 1;
      float d[4];
      warp_gemm_tf32<2>(
          d, [&](int r, int kk) { return reinterpret_cast<const float*>(sm + SM_A + a_off(32 * b + 16 + r, 32 * b + kk)); },
          [&](int kk, int n) { return reinterpret_cast<const float*>(sm + SM_DG + b * 4096 + b_off(kk, 8 * nt + n)); });
      float* y = reinterpret_cast<float*>(sm + SM_X + b * 1024);
      *reinterpret_cast<float2*>(y + lg * 16 + 8 * nt + 2 * lt) = make_float2(d[0], d[1]);
      *reinterpret_cast<float2*>(y + (lg + 8) * 16 + 8 * nt + 2 * lt) = make_float2(d[2], d[3]);
    }
    named_sync(GRP_BACK, GRP);
    {
      const int b = bw >> 1, nt = bw & 1;
      float d[4];
      warp_gemm_tf32<2>(
          d, [&](int r, int kk) { return reinterpret_cast<const float*>(sm + SM_DG + b * 4096 + b_off(16 + r, 16 + kk)); },
          [&](int kk, int n) { return reinterpret_cast<const float*>(sm + SM_X + b * 1024 + (kk * 16 + 8 * nt + n) * 4); });
      uint8_t* db = sm + SM_DG + b * 4096;
      *reinterpret_cast<float2*>(db + b_off(16 + lg, 8 * nt + 2 * lt)) = make_float2(-d[0], -d[1]);
      *reinterpret_cast<float2*>(db + b_off(24 + lg, 8 * nt + 2 * lt)) = make_float2(-d[2], -d[3]);
    }
    named_sync(GRP_BACK, GRP);
    if (k == 0) tmark(x, c, 19);
#pragma unroll 1
    for (int t = bw; t < 8; t += 4) {  // X = A_10 D_0  (32x32x32, 16x8 tiles)
      const int mt = t >> 2, nt = t & 3;
      float d[4];
      warp_gemm_tf32<4>(
          d, [&](int r, int kk) { return reinterpret_cast<const float*>(sm + SM_A + a_off(32 + 16 * mt + r, kk)); },
          [&](int kk, int n) { return reinterpret_cast<const float*>(sm + SM_DG + b_off(kk, 8 * nt + n)); });
      *reinterpret_cast<float2*>(sm + SM_X + b_off(16 * mt + lg, 8 * nt + 2 * lt)) = make_float2(d[0], d[1]);
      *reinterpret_cast<float2*>(sm + SM_X + b_off(16 * mt + lg + 8, 8 * nt + 2 * lt)) = make_float2(d[2], d[3]);
    }
    named_sync(GRP_BACK, GRP);
    if (k == 0) {
      mbar_arrive(&x.bars[B_AFREE]);  // A is no longer read
      tmark(x, c, 20);
    }
#pragma unroll 1
    for (int t = bw; t < 8; t += 4) {  // T_10 = -D_1 X
      const int mt = t >> 2, nt = t & 3;
      float d[4];
      warp_gemm_tf32<4>(
          d, [&](int r, int kk) { return reinterpret_cast<const float*>(sm + SM_DG + 4096 + b_off(16 * mt + r, kk)); },
          [&](int kk, int n) { return reinterpret_cast<const float*>(sm + SM_X + b_off(kk, 8 * nt + n)); });
      *reinterpret_cast<float2*>(sm + SM_T10 + b_off(16 * mt + lg, 8 * nt + 2 * lt)) = make_float2(-d[0], -d[1]);
      *reinterpret_cast<float2*>(sm + SM_T10 + b_off(16 * mt + lg + 8, 8 * nt + 2 * lt)) = make_float2(-d[2], -d[3]);
    }
    named_sync(GRP_BACK, GRP);
    {  // T' = T diag(beta) as fp16 [r][s]: rows rr and 32 + rr, columns c8 .. c8+7 and 32 + c8 ..
      const int rr = k >> 2, c8 = 8 * (k & 3);
      float4 t00[2], t10[2], t11[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c4 = c8 + 4 * h;
        const float4 bl = *reinterpret_cast<const float4*>(s_beta + c4);
        const float4 bh = *reinterpret_cast<const float4*>(s_beta + 32 + c4);
        t00[h] = mul4(*reinterpret_cast<const float4*>(sm + SM_DG + b_off(rr, c4)), bl);
        t11[h] = mul4(*reinterpret_cast<const float4*>(sm + SM_DG + 4096 + b_off(rr, c4)), bh);
        t10[h] = mul4(*reinterpret_cast<const float4*>(sm + SM_T10 + b_off(rr, c4)), bl);
      }
      named_sync(GRP_BACK, GRP);  // the TP tile overlays X and T_10
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c4 = c8 + 4 * h;
        st_f16x4(sm + SM_TP + sw128_off(rr, c4), t00[h]);
        st_f16x4(sm + SM_TP + sw128_off(rr, 32 + c4), make_float4(0.f, 0.f, 0.f, 0.f));
        st_f16x4(sm + SM_TP + sw128_off(32 + rr, c4), t10[h]);
        st_f16x4(sm + SM_TP + sw128_off(32 + rr, 32 + c4), t11[h]);
      }
    }
    fence_proxy_async_smem();
    named_sync(GRP_BACK, GRP);
    if (dmp) {
      dump_t(x.dbg, sm, k);
      named_sync(GRP_BACK, GRP);
    }

    // ---- (a4) G2: W'^T = KE^T T'^T -> TM_W;  G3: U^T = V^T T'^T -> TM_DELTA
    if (k == 0) {
      tmark(x, c, 21);
      bool ok = true;
      if (c >= 1) ok = cwait(x, B_DFREE, (c - 1) & 1, 22);  // D2 of chunk c-1 has read Δ
      if (ok) {
        tc_fence_after();
        const uint32_t id = idesc_f16_f32(128, 64, 1, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t da = sdesc_sw128(stg + OFF_QK + 8192 + i * 2048, 16384, 1024);
          const uint64_t db = sdesc_sw128(sb + SM_TP + i * 32, 16, 1024);
          umma_ss(x.tmem + TM_W, da, db, id, i > 0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t da = sdesc_sw128(stg + OFF_V + i * 2048, 8192, 1024);
          const uint64_t db = sdesc_sw128(sb + SM_TP + i * 32, 16, 1024);
          umma_ss(x.tmem + TM_DELTA, da, db, id, i > 0);
        }
        umma_commit(&x.bars[B_G23]);
      }
      tmark(x, c, 22);
    }
    if (!gwait(x, B_G23, g23_ph, 23, GRP_BACK)) break;
    g23_ph ^= 1;
    tc_fence_after();
    if (k == 0) tmark(x, c, 23);
    if (c >= 1 && !gwait(x, B_WFREE, (c - 1) & 1, 24, GRP_BACK)) break;
    {  // lane ti holds W'^T[ti][r]: row ti of the MN-major B operand of D1
      float w0[32], w1[32];
      tmem_ld32x2(tl + TM_W, tl + TM_W + 32, w0, w1);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        st_f16x8(sm + SM_WT + ti * 128 + (((q ^ ti) & 7) << 4), w0 + 8 * q);
        st_f16x8(sm + SM_WT + ti * 128 + ((((4 + q) ^ ti) & 7) << 4), w1 + 8 * q);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_sync(GRP_BACK, GRP);
    if (dmp) {
      dump_wu(x.dbg, sm, x.tmem, k);
      named_sync(GRP_BACK, GRP);
    }
    if (k == 0) {
      mbar_arrive(&x.bars[B_PRO0 + b2]);
      tmark(x, c, 25);
    }
  }
}

// Debug dumps from the scan group (TMEM / staging tile), chain 0.
__device__ __noinline__ void dump_delta(float* dbg, uint32_t tmem) {
  const int j = threadIdx.x;
  const uint32_t tl = tmem + ((uint32_t)((j >> 5) * 32) << 16);
  float d[32];
  for (int half = 0; half < 2; ++half) {
    tmem_ld32(tl + TM_DELTA + half * 32, d);
    for (int i = 0; i < 32; ++i) dbg[DBG_DELTA + (half * 32 + i) * 128 + j] = d[i];
  }
}
__device__ __noinline__ void dump_s(float* dbg, uint32_t tmem) {
  const int j = threadIdx.x;
  const uint32_t tl = tmem + ((uint32_t)((j >> 5) * 32) << 16);
  float s[32];
  for (int cb = 0; cb < 4; ++cb) {
    tmem_ld32(tl + TM_S + cb * 32, s);
    for (int i = 0; i < 32; ++i) dbg[DBG_S + (cb * 32 + i) * 128 + j] = s[i];
  }
}
__device__ __noinline__ void dump_o(float* dbg, const uint8_t* sm) {
  for (int e = threadIdx.x; e < 8192; e += 128) {
    const int r = e >> 7, jj = e & 127;
    const uint16_t u = *reinterpret_cast<const uint16_t*>(sm + SM_OST + (jj >> 6) * 8192 + sw128_off(r, jj & 63));
    dbg[DBG_O + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&u));
  }
}

// One checkpoint: columns col0 .. col0+63 of S^T held by this lane (value
// channel j), written as rows col0 .. col0+63 of the state [dk][dv] in slot
// `slot`.  A slot beyond the caller's capacity is skipped and reported.
__device__ __forceinline__ void store_ckpt(const Ctx& x, const ModeArgs& ma, int64_t slot, int col0,
                                           const float (&s0)[32], const float (&s1)[32]) {
  if (slot >= ma.ckpt_capacity) {
    record_error(x.status, KDA_ERR_INVALID_ARG, 40);
    return;
  }
  float* dst = ma.ckpt + ((slot * x.H + x.h) * D + col0) * D + (threadIdx.x & 127);
#pragma unroll
  for (int i = 0; i < 32; ++i) __stcs(dst + i * D, s0[i]);
#pragma unroll
  for (int i = 0; i < 32; ++i) __stcs(dst + (32 + i) * D, s1[i]);
}

// ============================================================ scan group
template <int MODE>
__device__ __forceinline__ void scan_group(const Ctx& x, const void* tmq, const void* tmk, const void* tmv, const void* tmo,
                           const float* __restrict__ init, __nv_bfloat16* __restrict__ out,
                           float* __restrict__ fin, int64_t sbase, int64_t ibase, bool inject_stuck,
                           int (&issued)[2], const ModeArgs& ma) {
  const int j = threadIdx.x;  // 0..127: TMEM lane = value channel
  const uint32_t tl = x.tmem + ((uint32_t)((j >> 5) * 32) << 16);
  uint8_t* sm = x.sm;
  const uint32_t sb = x.sb;
  const int H = x.H;

  auto issue_stage = [&](int c) {
    const int st = c & 1;
    const int tok = (int)(x.t0 + (int64_t)c * CH);
    uint8_t* dst = sm + st * STAGE_BYTES;
    uint64_t* bar = &x.bars[B_FULL0 + st];
    mbar_arrive_expect_tx(bar, STAGE_BYTES);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      tma_load_3d(dst + OFF_QK + hh * 16384, tmq, bar, 64 * hh, x.h, tok);
      tma_load_3d(dst + OFF_QK + hh * 16384 + 8192, tmk, bar, 64 * hh, x.h, tok);
      tma_load_3d(dst + OFF_V + hh * 8192, tmv, bar, 64 * hh, x.h, tok);
    }
  };
  if (j == 0) {
    if (x.nchunks > 0) {
      issue_stage(0);
      ++issued[0];
    }
    if (x.nchunks > 1) {
      issue_stage(1);
      ++issued[1];
    }
  }
  // S^T <- initial state (zeros without one).
#pragma unroll 1
  for (int cb = 0; cb < 4; ++cb) {
    float r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if constexpr (MODE == MODE_SEG) {  // zero start, the (scaled) identity, or a first segment's init
        if (x.first)
          r[i] = init ? __ldg(init + ibase + (int64_t)(cb * 32 + i) * D + j) : 0.f;
        else
          r[i] = (x.trans && cb * 32 + i == j) ? TRANS_SCALE : 0.f;
      } else {
        r[i] = init ? __ldg(init + ibase + (int64_t)(cb * 32 + i) * D + j) : 0.f;
      }
    }
    tmem_st32(tl + TM_S + cb * 32, r);
  }
  tmem_wait_st();

  // Output of chunk c: O^T (lane j) -> bf16 staging tile in the TMA box
  // layout -> one TMA store per 64-channel half for a full chunk, or plain
  // 16-byte stores of the valid rows for a sequence's last, partial chunk.
  auto store_out = [&](int c) {
    const int valid = chunk_valid(x, c);
    const int64_t tok0 = x.t0 + (int64_t)c * CH;
    float o0[32], o1[32];
    tmem_ld32x2(tl + TM_O + (c & 1) * 64, tl + TM_O + (c & 1) * 64 + 32, o0, o1);
    if constexpr (MODE == MODE_SEG) {
      // fp32 outputs straight from the registers: lane j writes channel j of
      // every valid token (a warp stores 128 contiguous bytes per token).
      float* obuf = x.trans ? ma.qhat32 : ma.o32;
      if (!obuf) return;  // states only
      float* dst = obuf + (tok0 * H + x.h) * D + j;
      const int64_t st = (int64_t)H * D;
      const float sc = x.trans ? TRANS_UNSCALE : 1.f;
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t < valid) __stcs(dst + t * st, o0[t] * sc);
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (32 + t < valid) __stcs(dst + (32 + t) * st, o1[t] * sc);
      return;
    }
    // Lanes j and j^1 hold channels jc, jc+1 of every token; they swap one
    // value per token pair so that each writes both channels of one token
    // (the even lane the even token) as one 4-byte word.
    const int odd = j & 1, jc = j & ~1;
    uint8_t* ost = sm + SM_OST + (jc >> 6) * 8192;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const float s0 = odd ? o0[2 * t] : o0[2 * t + 1], s1 = odd ? o1[2 * t] : o1[2 * t + 1];
      const float r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
      const uint32_t w0 = odd ? pack_bf16x2(r0, o0[2 * t + 1]) : pack_bf16x2(o0[2 * t], r0);
      const uint32_t w1 = odd ? pack_bf16x2(r1, o1[2 * t + 1]) : pack_bf16x2(o1[2 * t], r1);
      *reinterpret_cast<uint32_t*>(ost + sw128_off(2 * t + odd, jc & 63)) = w0;
      *reinterpret_cast<uint32_t*>(ost + sw128_off(32 + 2 * t + odd, jc & 63)) = w1;
    }
    fence_proxy_async_smem();
    named_sync(2, 128);
    if (x.dbg && c == 0) dump_o(x.dbg, sm);
    if (valid == CH) {
      if (j == 0) {
        tma_store_3d(tmo, sm + SM_OST, 0, x.h, (int)tok0);
        tma_store_3d(tmo, sm + SM_OST + 8192, 64, x.h, (int)tok0);
        bulk_commit();
      }
    } else {
      const int r = j >> 1, hf = j & 1;
      if (r < valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((tok0 + r) * H + x.h) * D + hf * 64);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = *reinterpret_cast<const uint4*>(sm + SM_OST + hf * 8192 + r * 128 + (((q ^ r) & 7) << 4));
      }
    }
  };

  int d1_ph = 0, d2_ph = 0;
  bool ok = true;
  for (int c = 0; c < x.nchunks && ok; ++c) {
    const int b2 = c & 1;
    const uint32_t stg = sb + b2 * STAGE_BYTES;
    const float* s_gc = reinterpret_cast<const float*>(sm + SM_MISC + MS_GC) + b2 * 128;
    if (j == 0) tmark(x, c, 8);
    if (inject_stuck && c == 0 && !gwait(x, B_NEVER, 0, 99, GRP_SG)) {
      ok = false;
      break;
    }
    // ---- S pass: S^T (decayed to the chunk end when this chunk is "fast")
    // -> S'^T as fp16 pairs, the A operand of D1.
    if (c >= 1) {
      if (!gwait(x, B_D2, d2_ph, 31, GRP_SG)) {
        ok = false;
        break;
      }
      d2_ph ^= 1;
      tc_fence_after();
    }
    if (j == 0) tmark(x, c, 9);
    if (!gwait(x, B_GC0 + b2, (c >> 1) & 1, 32, GRP_SG)) {
      ok = false;
      break;
    }
    const bool fast = *reinterpret_cast<volatile int*>(sm + SM_MISC + MS_FAST + 4 * b2) != 0;
#pragma unroll 1
    for (int cp = 0; cp < 2; ++cp) {
      float s0[32], s1[32];
      uint32_t pk[16];
      tmem_ld32x2(tl + TM_S + cp * 64, tl + TM_S + cp * 64 + 32, s0, s1);
      if constexpr (MODE == MODE_CKPT) {
        // The state after chunk c-1 (before this chunk's decay) is the
        // checkpoint of the interval that ends there.
        if (c > 0 && c % ma.ckpt_every == 0) store_ckpt(x, ma, x.ckpt0 + c / ma.ckpt_every - 1, cp * 64, s0, s1);
      }
      if (fast) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 g0 = *reinterpret_cast<const float4*>(s_gc + cp * 64 + i);
          const float4 g1 = *reinterpret_cast<const float4*>(s_gc + cp * 64 + 32 + i);
          const float4 a = mul4(make_float4(s0[i], s0[i + 1], s0[i + 2], s0[i + 3]), g0);
          const float4 b = mul4(make_float4(s1[i], s1[i + 1], s1[i + 2], s1[i + 3]), g1);
          s0[i] = a.x; s0[i + 1] = a.y; s0[i + 2] = a.z; s0[i + 3] = a.w;
          s1[i] = b.x; s1[i + 1] = b.y; s1[i + 2] = b.z; s1[i + 3] = b.w;
        }
        tmem_st32(tl + TM_S + cp * 64, s0);
        tmem_st32(tl + TM_S + cp * 64 + 32, s1);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = pack_f16x2(s0[2 * i], s0[2 * i + 1]);
      tmem_st16(tl + TM_SB + cp * 32, pk);
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = pack_f16x2(s1[2 * i], s1[2 * i + 1]);
      tmem_st16(tl + TM_SB + cp * 32 + 16, pk);
    }
    if (j == 0) bulk_wait_read0();  // the staging tile is free again
    tmem_wait_st();
    tc_fence_before();
    if (!named_sync_and(2, 128, !*x.abort)) {
      ok = false;
      break;
    }
    if (j == 0) tmark(x, c, 10);

    // ---- D1a: O^T = S'^T QE^T as soon as QE is ready;  D1b: Δ^T = U^T -
    // S'^T W'^T once the back group has W'^T and U^T.  (A = S'^T from TMEM)
    if (j == 0) {
      bool okj = cwait(x, B_OPS0 + b2, (c >> 1) & 1, 36);
      if (okj) {
        tc_fence_after();
        const uint32_t idq = idesc_f16_f32(128, 64, 0, 0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint64_t dq = sdesc_sw128(stg + OFF_QK + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
          umma_tmem_a(x.tmem + TM_O + b2 * 64, x.tmem + TM_SB + i * 8, dq, idq, i > 0);
        }
        umma_commit(&x.bars[B_D1A]);
        tmark(x, c, 27);
      }
      okj = okj && cwait(x, B_PRO0 + b2, (c >> 1) & 1, 33);
      if (okj) {
        tmark(x, c, 24);
        tc_fence_after();
        const uint32_t idw = idesc_f16_f32(128, 64, 0, 1, 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint64_t dw = sdesc_sw128(sb + SM_WT + i * 2048, 8192, 1024);
          umma_tmem_a(x.tmem + TM_DELTA, x.tmem + TM_SB + i * 8, dw, idw, 1);
        }
        umma_commit(&x.bars[B_D1]);
        umma_commit(&x.bars[B_WFREE]);
      }
      tmark(x, c, 11);
      // Once D1a has read QE, nothing reads the stage of chunk c any more
      // (G1, G2 and G3 finished before PRO): fetch chunk c+2 into it.
      okj = okj && cwait(x, B_D1A, c & 1, 37);
      if (okj && c + 2 < x.nchunks) {
        issue_stage(c + 2);
        ++issued[b2];
      }
      tmark(x, c, 28);
    }
    if (!gwait(x, B_D1, d1_ph, 34, GRP_SG)) {
      ok = false;
      break;
    }
    d1_ph ^= 1;
    if (j == 0) tmark(x, c, 13);
    tc_fence_after();

    // ---- Δ^T -> fp16 pairs (A operand of D2); general chunks decay S^T here.
    if (!fast) {
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float s[32];
        tmem_ld32(tl + TM_S + cb * 32, s);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] *= s_gc[cb * 32 + i];
        tmem_st32(tl + TM_S + cb * 32, s);
      }
    }
    if (x.dbg && c == 0) dump_delta(x.dbg, x.tmem);  // before the fp16 pairs overwrite its first columns
    {
      float d0[32], d1[32];
      uint32_t pk[16];
      float dm = 0.f;
      tmem_ld32x2(tl + TM_DELTA, tl + TM_DELTA + 32, d0, d1);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pk[i] = pack_f16x2(d0[2 * i], d0[2 * i + 1]);
        dm = amax_nan(amax_nan(dm, d0[2 * i]), d0[2 * i + 1]);
      }
      tmem_st16(tl + TM_DELTA, pk);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pk[i] = pack_f16x2(d1[2 * i], d1[2 * i + 1]);
        dm = amax_nan(amax_nan(dm, d1[2 * i]), d1[2 * i + 1]);
      }
      tmem_st16(tl + TM_DELTA + 16, pk);
      if (!(fabsf(dm) <= F16_SAFE)) record_error(x.status, KDA_ERR_RANGE, 31);
    }
    tmem_wait_st();
    tc_fence_before();
    named_sync(2, 128);

    // ---- D2: S^T += Δ^T KH ;  O^T += Δ^T P^T      (A = Δ^T from TMEM)
    if (j == 0) tmark(x, c, 14);
    if (j == 0) {
      tc_fence_after();
      const uint32_t ids = idesc_f16_f32(128, 128, 0, 1);
      const uint32_t idp = idesc_f16_f32(128, 64, 0, 0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t dk = sdesc_sw128(sb + SM_KX + b2 * 16384 + i * 2048, 8192, 1024);
        umma_tmem_a(x.tmem + TM_S, x.tmem + TM_DELTA + i * 8, dk, ids, 1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t dp = sdesc_sw128(sb + SM_P + b2 * 8192 + i * 32, 16, 1024);
        umma_tmem_a(x.tmem + TM_O + b2 * 64, x.tmem + TM_DELTA + i * 8, dp, idp, 1);
      }
      umma_commit(&x.bars[B_D2]);
      umma_commit(&x.bars[B_BUF0 + b2]);
      umma_commit(&x.bars[B_DFREE]);  // Δ^T read: the next U^T may land
      tmark(x, c, 15);
    }
    // The output of chunk c-1 (final since D2 of c-1), off the path from
    // D1b to D2 that the next chunks' front and back wait on.
    if (c >= 1) store_out(c - 1);
    if (j == 0) tmark(x, c, 12);
  }
  if (named_sync_and(2, 128, ok && !*x.abort) && x.nchunks > 0) {
    if (gwait(x, B_D2, d2_ph, 35, GRP_SG)) {
      tc_fence_after();
      if (j == 0) bulk_wait_read0();
      named_sync(2, 128);
      store_out(x.nchunks - 1);
    }
  }
  if (j == 0) bulk_wait_all();  // every output store has completed
  if (named_sync_and(2, 128, !*x.abort)) {
    if (x.dbg && x.nchunks > 0) dump_s(x.dbg, x.tmem);
    if (fin) {
      const float sc = (MODE == MODE_SEG && x.trans) ? TRANS_UNSCALE : 1.f;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float s[32];
        tmem_ld32(tl + TM_S + cb * 32, s);
#pragma unroll
        for (int i = 0; i < 32; ++i) fin[sbase + (int64_t)(cb * 32 + i) * D + j] = MODE == MODE_SEG ? s[i] * sc : s[i];
      }
    }
    if constexpr (MODE == MODE_CKPT) {
      const int64_t every_tok = (int64_t)ma.ckpt_every * CH;
      if (x.L > 0 && x.L % every_tok == 0) {
#pragma unroll 1
        for (int cp = 0; cp < 2; ++cp) {
          float s0[32], s1[32];
          tmem_ld32x2(tl + TM_S + cp * 64, tl + TM_S + cp * 64 + 32, s0, s1);
          store_ckpt(x, ma, x.ckpt0 + x.L / every_tok - 1, cp * 64, s0, s1);
        }
      }
    }
  }
}

// HOOKS: the test-hook build (intermediate dumps, phase timestamps, the
// stuck-wait injection); without it those branches fold away at compile time.
// MODE (FwdMode): MODE_PLAIN is the production forward; MODE_CKPT adds the
// interval checkpoints; MODE_SEG runs two blocks per (sequence, head): the
// first N*H blocks the zero-start runs, the next N*H the transition runs.
template <bool HOOKS, int MODE>
__global__ void __launch_bounds__(NTHR, 1)
    kda_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_g,
                      const float* __restrict__ g,
                      const float* __restrict__ beta, const float* __restrict__ init,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ fin, const int32_t* __restrict__ cu,
                      const int32_t* __restrict__ order, int64_t Tper, int H, DeviceStatus* status,
                      float* __restrict__ dbg, uint64_t wait_ns, int inject_stuck,
                      const __grid_constant__ ModeArgs ma, int units) {
  extern __shared__ uint8_t smem_raw[];
  // Align to 1024 bytes by offsetting from the shared array itself, so the
  // compiler keeps treating every access through `sm` as a shared-memory one.
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctx x;
  x.sm = sm;
  x.sb = smem_u32(sm);
  x.bars = reinterpret_cast<uint64_t*>(sm + SM_MISC);
  x.abort = reinterpret_cast<volatile int*>(sm + SM_MISC + MS_ABORT);
  x.status = status;
  x.wait_ns = wait_ns;
  const int tid = threadIdx.x, warp = tid >> 5;
  // Work item: with packed batches the blocks follow `order`, so that the
  // longest sequences start first.
  int bid = blockIdx.x;
  x.trans = false;
  if constexpr (MODE == MODE_SEG) {
    x.trans = bid >= units;
    if (x.trans) bid -= units;
    if (x.trans) fin = ma.trans;
  }
  const int n0 = bid / H;
  const int n = order ? order[n0] : n0;
  x.h = bid % H;
  x.H = H;
  x.first = false;
  int64_t ibase = ((int64_t)n * H + x.h) * D * D;  // initial state of this chain
  if constexpr (MODE == MODE_SEG) {
    x.first = ma.seg_per_seq > 0 && n % ma.seg_per_seq == 0;
    const bool last = ma.seg_per_seq > 0 && n % ma.seg_per_seq == ma.seg_per_seq - 1;
    // a first segment needs no transition and a last segment no pieces at all
    // (the whole block leaves before it allocates anything)
    if ((x.first && x.trans) || (last && !x.first)) return;
    if (x.first) ibase = ((int64_t)(n / ma.seg_per_seq) * H + x.h) * D * D;
  }
  if (cu) {
    x.t0 = cu[n];
    x.L = (int64_t)cu[n + 1] - x.t0;
  } else {
    x.t0 = (int64_t)n * Tper;
    x.L = Tper;
  }
  x.nchunks = (int)((x.L + CH - 1) / CH);
  x.ckpt0 = 0;
  if constexpr (MODE == MODE_GATED) {
    if (threadIdx.x == 0) {
      float* gc = reinterpret_cast<float*>(sm + SM_MISC + MS_GATE);
      gc[0] = -__expf(ma.A_log[x.h]) * LOG2E;
      gc[1] = ma.g_min;
    }
  }
  if constexpr (MODE == MODE_CKPT)
    x.ckpt0 = ma.ckpt_base ? ma.ckpt_base[n] : (int64_t)n * (Tper / ((int64_t)ma.ckpt_every * CH));
  x.dbg = (HOOKS && dbg && n == 0 && x.h == 0) ? dbg : nullptr;
  x.tdbg = x.dbg ? reinterpret_cast<long long*>(x.dbg + DBG_TIME) : nullptr;
  long long* s_t0 = reinterpret_cast<long long*>(sm + SM_MISC + MS_T0);

  if (tid == 0) {
    *s_t0 = clock64();
    for (int i = 0; i < NUM_BARS; ++i)
      mbar_init(&x.bars[i], (i == B_GC0 || i == B_GC1 || i == B_OPS0 || i == B_OPS1 || i == B_FR0 || i == B_FR1) ? FRONT_T : 1);
    fence_mbar_init();
    *x.abort = 0;
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
    prefetch_tmap(&tm_g);
  }
  if (warp == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(sm + SM_MISC + MS_TMEM), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t*>(sm + SM_MISC + MS_TMEM);
  x.tstart = *s_t0;
  const int64_t sbase = ((int64_t)n * H + x.h) * D * D;

  int cnt[2] = {0, 0};  // TMA stages issued (scan group) / consumed (front group)
  int* s_cnt = reinterpret_cast<int*>(sm + SM_MISC + MS_CNT);
  if (warp < 4) {
    scan_group<MODE>(x, &tm_q, &tm_k, &tm_v, &tm_o, init, out, fin, sbase, ibase, HOOKS && inject_stuck != 0, cnt,
                     ma);
    if (tid == 0) { s_cnt[0] = cnt[0]; s_cnt[1] = cnt[1]; }
  } else if (warp < 12) {
    front_group<MODE>(x, g, beta, &tm_g, cnt);
    if (tid == (int)FRONT0) { s_cnt[2] = cnt[0]; s_cnt[3] = cnt[1]; }
  } else {
    back_group<MODE>(x);
  }

  // Drain: every UMMA issued by a group's elected thread has completed, and
  // (on the error path) every TMA load in flight has landed, before TMEM is
  // released and the block exits.
  if (tid == 0 || tid == (int)FRONT0 || tid == (int)BACK0) {
    uint64_t* db = &x.bars[tid == 0 ? B_DRAIN_SG : (tid == (int)FRONT0 ? B_DRAIN_F : B_DRAIN_B)];
    umma_commit(db);
    mbar_wait(db, 0, WAIT_NS);
  }
  __syncthreads();
  if (tid == 0) {
    // Wait (bounded) for any TMA load that was issued but never consumed.
    for (int st = 0; st < 2; ++st)
      for (int k = s_cnt[2 + st]; k < s_cnt[st]; ++k) mbar_wait(&x.bars[B_FULL0 + st], k & 1, WAIT_NS);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, TMEM_COLS);
  }
}

// Packed batches: order sequences by decreasing length (bucketed by
// floor(log2(length))) so the longest chains are scheduled first.
__global__ void kda_order_kernel(const int32_t* __restrict__ cu, int N, int32_t* __restrict__ order) {
  __shared__ int cnt[33], base[33];
  const int tid = threadIdx.x;
  if (tid < 33) cnt[tid] = 0;
  __syncthreads();
  auto bucket = [&](int n) {
    const int L = cu[n + 1] - cu[n];
    return L <= 0 ? 32 : __clz(L);  // longer sequences -> smaller bucket index
  };
  for (int n = tid; n < N; n += blockDim.x) atomicAdd(&cnt[bucket(n)], 1);
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int b = 0; b < 33; ++b) {
      base[b] = acc;
      acc += cnt[b];
    }
  }
  __syncthreads();
  for (int n = tid; n < N; n += blockDim.x) order[atomicAdd(&base[bucket(n)], 1)] = n;
}

// Packed batches with checkpoints: slot of the first checkpoint of every
// sequence = the number of whole intervals in the sequences before it
// (one block; a running prefix over blocks of 1024 sequences).
__global__ void kda_ckpt_base_kernel(const int32_t* __restrict__ cu, int N, int interval, int32_t* __restrict__ base) {
  __shared__ int part[1024];
  __shared__ int carry;
  const int tid = threadIdx.x;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int n0 = 0; n0 < N; n0 += 1024) {
    const int n = n0 + tid;
    const int cnt = n < N ? (cu[n + 1] - cu[n]) / interval : 0;
    part[tid] = cnt;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan
      const int v = tid >= o ? part[tid - o] : 0;
      __syncthreads();
      part[tid] += v;
      __syncthreads();
    }
    if (n < N) base[n] = carry + part[tid] - cnt;
    __syncthreads();
    if (tid == 1023) carry += part[1023];
    __syncthreads();
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

// bf16 tensor [T_total][H][128] as a 3-D map, box {64 channels, 1 head, 64 tokens}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int H, int64_t Ttot) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)Ttot};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)CH};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Decay rows [T_total][H][128] as a 3-D map, box {128 channels, 1 head, 64
// tokens}: fp32 log-decays, or bf16 decay logits (MODE_GATED).  Used for L2
// prefetches only.
bool make_map_g(CUtensorMap* m, const void* ptr, int H, int64_t Ttot, bool bf16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t es_bytes = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)Ttot};
  cuuint64_t strides[2] = {(cuuint64_t)D * es_bytes, (cuuint64_t)H * D * es_bytes};
  cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)CH};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fwd_tc_supported(int dk, int dv, bool bf16) { return bf16 && dk == D && dv == D; }

cudaError_t launch_ckpt_base(const int32_t* cu, int N, int interval, int32_t* base, cudaStream_t s) {
  kda_ckpt_base_kernel<<<1, 1024, 0, s>>>(cu, N, interval, base);
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc_impl(const FwdArgs& a, cudaStream_t s, uint64_t wait_ns, int inject_stuck,
                               int32_t* order_ws, const ModeArgs& ma) {
  const int64_t Ttot = a.cu ? a.T : (int64_t)a.N * a.T;
  const int units = (int)((int64_t)a.N * a.H);
  const unsigned blocks = (unsigned)(ma.mode == MODE_SEG ? 2 * (int64_t)units : (int64_t)units);
  if (blocks == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mo, mg;
  const int64_t Tmap = Ttot > 0 ? Ttot : 1;
  if (!make_map(&mq, a.q, a.H, Tmap) || !make_map(&mk, a.k, a.H, Tmap) || !make_map(&mv, a.v, a.H, Tmap) ||
      !make_map(&mo, a.out ? a.out : a.q, a.H, Tmap) || !make_map_g(&mg, a.g, a.H, Tmap, ma.mode == MODE_GATED))
    return cudaErrorInvalidValue;
  const int32_t* order = nullptr;
  if (a.cu && order_ws && a.N > 1) {
    kda_order_kernel<<<1, 1024, 0, s>>>(a.cu, a.N, order_ws);
    order = order_ws;
  }
  auto* kern = (a.dbg || inject_stuck) ? kda_fwd_tc_kernel<true, MODE_PLAIN>
               : ma.mode == MODE_CKPT  ? kda_fwd_tc_kernel<false, MODE_CKPT>
               : ma.mode == MODE_SEG   ? kda_fwd_tc_kernel<false, MODE_SEG>
               : ma.mode == MODE_GATED ? kda_fwd_tc_kernel<false, MODE_GATED>
                                       : kda_fwd_tc_kernel<false, MODE_PLAIN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<blocks, NTHR, SMEM_BYTES, s>>>(mq, mk, mv, mo, mg, a.g, a.beta, a.init, (__nv_bfloat16*)a.out, a.fin, a.cu,
                                        order, a.cu ? 0 : a.T, a.H, a.status, (float*)a.dbg, wait_ns, inject_stuck,
                                        ma, units);
  return cudaGetLastError();
}

int fwd_tc_debug_floats() { return DBG_FLOATS; }

}  // namespace kda
