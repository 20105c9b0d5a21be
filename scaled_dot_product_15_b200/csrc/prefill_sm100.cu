// Prefill attention on the 5th-generation tensor cores (sm_100a).
//
// What it computes is softmax(Q K^T * scale + mask) V with the per-row
// logsumexp (exactref.ai "scaled_dot_product_attention", "Full
// specification"), for fp16/bf16 with head size 64, 96 or 128 and the masks
// none / causal / block-diagonal (causal), without ever writing the L x S
// score matrix to HBM.  The keys are visited in tiles with the online-softmax
// recurrence described on the khchao.com NN-lab page ("FlashAttention Tiling &
// Online Softmax Algorithm"): a running row maximum m and running sum l are
// kept in fp32, and the output accumulator is rescaled by 2^(m_old - m_new)
// when the maximum grows.
//
// B200 mapping: a persistent kernel, one CTA per SM, 12 warps.  A work unit is
// 256 query rows (two 128-row sub-tiles) of one (batch, head) or segment.
// Units are listed longest first (last row blocks first under a causal mask)
// and handed out through a grid-wide atomic counter, so each CTA takes the
// next unit when it is ready for one: greedy longest-first scheduling.
//   warp 9      TMA producer: takes the next unit, publishes it to the other
//               roles through a small ring in shared memory, then loads K_0,
//               the unit's Q (each sub-tile's buffer as soon as the previous
//               unit's last scores of that sub-tile have read it), V_0, K_1,
//               V_1, ... as 128-key tiles through a ring of shared-memory
//               slots (128-byte swizzle, 64-column boxes).
//   warp 8      MMA issuer (one thread; at E = 128 the whole warp, one elected
//               lane issuing): S_i = Q_i K_j^T with both operands in
//               shared memory, O_i += P_i V_j with P_i read from tensor memory;
//               fp32 accumulators in tensor memory (S0 | S1 | O0 | O1 = 512
//               columns).  Sub-tiles interleave (PV0, S0 next, PV1, S1 next) so
//               the tensor core runs one while the other's softmax runs; a
//               sub-tile's first scores of the next unit are issued right
//               after its last PV of the current one.  Descriptors are built
//               once; each MMA advances them by compile-time offsets, so the
//               single issuing thread keeps pace with the tensor core.
//   warps 0-7   softmax, one thread per query row (warpgroup i owns sub-tile
//               i): tcgen05.ld of its 128 scores, masking on boundary tiles
//               only, row maximum, exp2 with scale*log2(e) folded into one
//               packed FMA (1 of every 8 pairs on the FMA pipe), P packed to
//               16 bits and stored over its own scores.  The output is
//               rescaled in tensor memory only when a row maximum grows by more
//               than 2^8 (exact: the final normalisation uses the same
//               maximum).  At the end of a unit it writes O / l in the output
//               dtype straight from tensor memory to global memory and
//               lse = (m + log2 l) * ln 2, while the next unit's first scores
//               are already being computed.
// Causal attention visits only key tiles at or left of the diagonal, per
// sub-tile: the last key tile of a 256-row unit lies wholly above sub-tile 0's
// rows, so sub-tile 0 skips its scores, softmax and PV.  A unit whose
// sub-tile 1 has no rows (the last block of a short segment or sequence)
// skips all of sub-tile 1's work.  Packed variable-length batches index tiles
// from each segment's first token.
//
// Every wait on an mbarrier is bounded (2 s); on a timeout the kernel records
// an error code, stops its other roles, drains what it issued and returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace sdpa15 {

__device__ int g_prefill_error = 0;

// Grid-wide work counters of the persistent prefill kernel, one pair per
// launch slot: units handed out, CTAs finished.  The last CTA of a launch
// resets its pair, so a slot is ready again for the next launch that uses
// it; launches take slots round robin, so up to kSchedSlots launches may run
// concurrently.
constexpr int kSchedSlots = 256;
__device__ unsigned int g_unit_next[kSchedSlots];
__device__ unsigned int g_cta_done[kSchedSlots];

namespace pf {

constexpr int BM = 128;  // query rows per sub-tile (tensor-memory lanes)
constexpr int BN = 128;  // keys per tile
constexpr int NSUB = 2;  // sub-tiles per work unit
constexpr int kThreads = 384;  // 3 warpgroups
constexpr int kWarpMma = 8;
constexpr int kWarpLoad = 9;
// Registers: the block is launched with 168 per thread (the largest multiple
// of 8 with 384 x 168 <= 65536), 64512 in all, and setmaxnreg.inc can only
// redistribute those: warpgroup 2 (MMA, load, two idle warps) drops to 72 so
// the two softmax warpgroups can rise to 216: 2 x 128 x 216 + 128 x 72 =
// 64512.  A split above the launch total would wait forever.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsCtl = 72;
constexpr int kRegsLaunch = (65536 / kThreads) / 8 * 8;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCtl <= kThreads * kRegsLaunch, "register split");
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;
// Exponential pairs of every 8 computed on the FMA pipe instead of the
// multi-function unit.
#ifndef PF_EMU
#define PF_EMU 1
#endif
constexpr int kEmuPer8 = PF_EMU;

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;        // 64-element column blocks per row
  static constexpr int BLOCK = 128 * 128;         // bytes of one [128 rows][64 elements] block
  static constexpr int TILE = NB * BLOCK;         // bytes of a 128-row tile
  static constexpr int NS = (D <= 64) ? 8 : 4;    // key/value ring slots
  static constexpr int KV_OFF = NSUB * TILE;
  static constexpr int BAR_OFF = KV_OFF + NS * TILE;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
};

constexpr int kUnitRing = 4;     // published unit indices in flight
constexpr int kUnitReaders = 9;  // MMA thread + 8 softmax warps

struct Bars {
  uint64_t q[2];         // Q of sub-tile i landed (one phase per unit)
  uint64_t q_free[2];    // the unit's last score MMAs of sub-tile i have read Q
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t s[2];         // S[sub] computed (one phase per key tile)
  uint64_t p[2];         // P[sub] written, O rescaled (one phase per key tile)
  uint64_t o[2];         // O[sub] final for a unit
  uint64_t unit_full[kUnitRing];   // a unit index published
  uint64_t unit_empty[kUnitRing];  // every role has read it
  uint64_t done;                   // every MMA of the CTA completed
  int unit[kUnitRing];
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// A work unit: 256 query rows of one (batch or segment, head).
struct Unit {
  int h, b, seq0, Lq, Sk, row0;
  int n_kv;  // key tiles of the unit
  int n0;    // key tiles of sub-tile 0: n_kv, or n_kv - 1 under a causal mask
             // when the last tile lies wholly above sub-tile 0's rows
  int n1;    // key tiles of sub-tile 1: n_kv, or 0 when it has no rows
};

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}


__device__ __forceinline__ void flag_error(Bars* bars, int code) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  atomicCAS(&g_prefill_error, 0, code);
}

__device__ __forceinline__ bool wait(Bars* bars, uint64_t* bar, uint32_t parity) {
  return ptx::mbar_wait(bar, parity, kTimeoutNs, &bars->abort);
}

// Wait of the producer, which runs ahead: polls with a short sleep in
// between, leaving issue slots to the softmax warps of its sub-partition.
__device__ __forceinline__ bool wait_idle(Bars* bars, uint64_t* bar, uint32_t parity) {
  const uint32_t a = ptx::smem_u32(bar);
  if (ptx::mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (;;) {
    __nanosleep(128);
    if (ptx::mbar_try_wait(a, parity)) return true;
    if (*reinterpret_cast<const volatile int*>(&bars->abort) != 0) return false;
    if (ptx::globaltimer_ns() - t0 > kTimeoutNs) return false;
  }
}

// Wait for this thread's own asynchronous copies or MMAs to finish before the
// CTA exits: bounded, but not cut short by another role's abort.
__device__ __forceinline__ bool drain(uint64_t* bar, uint32_t parity) {
  const int never = 0;
  return ptx::mbar_wait(bar, parity, kTimeoutNs, &never);
}

// kW: issued by the whole MMA warp (one elected lane issues each
// instruction), else by one thread.
// Lean issue: descriptors built once per CTA, operand addresses are the
// descriptor plus compile-time offsets (address >> 4 in the low 14 bits never
// carries inside shared memory).  S_i = Q_i K^T: A = Q_i (K-major), B = K
// tile (K-major), D = tensor-memory columns [i*128, i*128+128).
template <int D, bool kW, int KK = 0>
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint64_t dq_i, uint64_t dk, uint32_t idesc) {
  if constexpr (KK < D / 16) {
    constexpr uint32_t off = ((KK / 4) * Cfg<D>::BLOCK + (KK % 4) * 32) >> 4;
    if constexpr (kW)
      ptx::mma_ss_off_w<off, off>(tmem_s, dq_i, dk, idesc, KK > 0 ? 1u : 0u);
    else
      ptx::mma_ss_off<off, off>(tmem_s, dq_i, dk, idesc, KK > 0 ? 1u : 0u);
    issue_qk<D, kW, KK + 1>(tmem_s, dq_i, dk, idesc);
  }
}

// O_i += P_i V: A = P_i from tensor memory (16-bit, packed over S_i), B = V
// tile (MN-major).
template <bool kW, int KK = 0>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t dv, uint32_t acc0,
                                         uint32_t idesc) {
  if constexpr (KK < BN / 16) {
    if constexpr (kW)
      ptx::mma_ts_off_w<KK * 8, ((KK * 16 * 128) >> 4)>(tmem_o, tmem_p, dv, idesc, KK > 0 ? 1u : acc0);
    else
      ptx::mma_ts_off<KK * 8, ((KK * 16 * 128) >> 4)>(tmem_o, tmem_p, dv, idesc, KK > 0 ? 1u : acc0);
    issue_pv<kW, KK + 1>(tmem_o, tmem_p, dv, acc0, idesc);
  }
}

// Wait, outcome and commit of the MMA issuer in either form (kW: the whole
// warp, every outcome made warp-uniform; else one thread).
template <bool kW>
__device__ __forceinline__ bool mma_uniform(bool ok) {
  if constexpr (kW) return __all_sync(0xffffffffu, ok);
  return ok;
}
template <bool kW>
__device__ __forceinline__ bool mma_wait(Bars* bars, uint64_t* bar, uint32_t parity) {
  return mma_uniform<kW>(wait(bars, bar, parity));
}
template <bool kW>
__device__ __forceinline__ void mma_commit_as(uint64_t* bar) {
  if constexpr (kW)
    ptx::mma_commit_w(bar);
  else
    ptx::mma_commit(bar);
}

// All 128 columns of S (four 32-column blocks) with one instruction.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[4][32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,"
      "%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,"
      "%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,"
      "%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,"
      "%126,%127}, [%128];"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]), "=r"(r[0][7]),
        "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]), "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]),
        "=r"(r[0][16]), "=r"(r[0][17]), "=r"(r[0][18]), "=r"(r[0][19]), "=r"(r[0][20]), "=r"(r[0][21]), "=r"(r[0][22]), "=r"(r[0][23]),
        "=r"(r[0][24]), "=r"(r[0][25]), "=r"(r[0][26]), "=r"(r[0][27]), "=r"(r[0][28]), "=r"(r[0][29]), "=r"(r[0][30]), "=r"(r[0][31]),
        "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]), "=r"(r[1][7]),
        "=r"(r[1][8]), "=r"(r[1][9]), "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15]),
        "=r"(r[1][16]), "=r"(r[1][17]), "=r"(r[1][18]), "=r"(r[1][19]), "=r"(r[1][20]), "=r"(r[1][21]), "=r"(r[1][22]), "=r"(r[1][23]),
        "=r"(r[1][24]), "=r"(r[1][25]), "=r"(r[1][26]), "=r"(r[1][27]), "=r"(r[1][28]), "=r"(r[1][29]), "=r"(r[1][30]), "=r"(r[1][31]),
        "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[2][4]), "=r"(r[2][5]), "=r"(r[2][6]), "=r"(r[2][7]),
        "=r"(r[2][8]), "=r"(r[2][9]), "=r"(r[2][10]), "=r"(r[2][11]), "=r"(r[2][12]), "=r"(r[2][13]), "=r"(r[2][14]), "=r"(r[2][15]),
        "=r"(r[2][16]), "=r"(r[2][17]), "=r"(r[2][18]), "=r"(r[2][19]), "=r"(r[2][20]), "=r"(r[2][21]), "=r"(r[2][22]), "=r"(r[2][23]),
        "=r"(r[2][24]), "=r"(r[2][25]), "=r"(r[2][26]), "=r"(r[2][27]), "=r"(r[2][28]), "=r"(r[2][29]), "=r"(r[2][30]), "=r"(r[2][31]),
        "=r"(r[3][0]), "=r"(r[3][1]), "=r"(r[3][2]), "=r"(r[3][3]), "=r"(r[3][4]), "=r"(r[3][5]), "=r"(r[3][6]), "=r"(r[3][7]),
        "=r"(r[3][8]), "=r"(r[3][9]), "=r"(r[3][10]), "=r"(r[3][11]), "=r"(r[3][12]), "=r"(r[3][13]), "=r"(r[3][14]), "=r"(r[3][15]),
        "=r"(r[3][16]), "=r"(r[3][17]), "=r"(r[3][18]), "=r"(r[3][19]), "=r"(r[3][20]), "=r"(r[3][21]), "=r"(r[3][22]), "=r"(r[3][23]),
        "=r"(r[3][24]), "=r"(r[3][25]), "=r"(r[3][26]), "=r"(r[3][27]), "=r"(r[3][28]), "=r"(r[3][29]), "=r"(r[3][30]), "=r"(r[3][31])
      : "r"(taddr));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Row maximum of 128 scores held as 4 x 32 raw registers (4 independent
// chains of three-input max).
__device__ __forceinline__ float row_max128(const uint32_t (&s)[4][32]) {
  float a = -INFINITY, b = -INFINITY, c = -INFINITY, d = -INFINITY;
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      a = fmax3(a, __uint_as_float(s[k][i]), __uint_as_float(s[k][i + 1]));
      b = fmax3(b, __uint_as_float(s[k][i + 2]), __uint_as_float(s[k][i + 3]));
      c = fmax3(c, __uint_as_float(s[k][i + 4]), __uint_as_float(s[k][i + 5]));
      d = fmax3(d, __uint_as_float(s[k][i + 6]), __uint_as_float(s[k][i + 7]));
    }
  return fmax3(a, b, fmaxf(c, d));
}

// P = 2^(S * scale*log2(e) - m) for 128 scores, two at a time (packed fp32
// FMA), packed to 16-bit pairs in place over the scores (lower key in the low
// half) and stored over S in tensor memory; returns the row sum of the fp32
// weights.  With kEmu, kEmuPer8 of every 8 pairs take the FMA-pipe 2^x so the
// multi-function unit is not the bottleneck; masked tiles (-inf scores) use
// the multi-function unit only, whose 2^-inf is exactly 0.
template <typename T, bool kEmu>
__device__ __forceinline__ float exp_pack_store(uint32_t (&s)[4][32], float sl, float neg_m, uint32_t tS) {
  using namespace exp2poly;
  const uint64_t sl2 = pk(sl, sl), nm2 = pk(neg_m, neg_m);
  uint64_t acc0 = pk(0.f, 0.f), acc1 = pk(0.f, 0.f);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = 64 * hh + 2 * i;
      const uint64_t x = ffma2(pk(__uint_as_float(s[e >> 5][e & 31]), __uint_as_float(s[(e + 1) >> 5][(e + 1) & 31])),
                               sl2, nm2);
      float x0, x1, p0, p1;
      upk(x, x0, x1);
      if (kEmu && (i % 8) < kEmuPer8) {
        exp2_pair(x0, x1, p0, p1);
      } else {
        p0 = ptx::ex2(x0);
        p1 = ptx::ex2(x1);
      }
      if (i & 1) acc1 = fadd2(acc1, pk(p0, p1));
      else acc0 = fadd2(acc0, pk(p0, p1));
      s[2 * hh][i] = pack2<T>(p0, p1);  // s[2hh][>= i] and s[2hh+1] are read first
    }
    ptx::tmem_st32(tS + 32 * hh, s[2 * hh]);
  }
  float a, b, c, d;
  upk(acc0, a, b);
  upk(acc1, c, d);
  return (a + b) + (c + d);
}

// Unit `idx` in longest-first order (the row block outermost, last rows
// first), or false when it holds no rows (a short packed segment).
template <bool kVarlen>
__device__ __forceinline__ bool unit_at(const Params& p, int idx, int bx, int mblocks, bool causal, Unit& u) {
  const int per = bx * p.Hq;
  const int mb = mblocks - 1 - idx / per;
  const int rem = idx - (idx / per) * per;
  u.h = rem % p.Hq;
  const int g = rem / p.Hq;
  if (kVarlen) {
    const int c0 = min(max(__ldg(p.cu + g), 0), p.L);
    const int c1 = min(max(__ldg(p.cu + g + 1), c0), p.L);
    u.b = 0;
    u.seq0 = c0;
    u.Lq = u.Sk = c1 - c0;
  } else {
    u.b = g;
    u.seq0 = 0;
    u.Lq = p.L;
    u.Sk = p.S;
  }
  u.row0 = mb * (NSUB * BM);
  if (u.row0 >= u.Lq || u.Sk <= 0) return false;
  int n = (u.Sk + BN - 1) / BN, n0 = n;
  if (causal) {
    n = min(n, (min(u.row0 + NSUB * BM, u.Lq) - 1) / BN + 1);
    n0 = min(n, (min(u.row0 + BM, u.Lq) - 1) / BN + 1);  // n - 1 or n
  }
  u.n_kv = n;
  u.n0 = n0;
  u.n1 = u.row0 + BM < u.Lq ? n : 0;
  return true;
}

// The k-th unit of this CTA as published by the producer: its index in the
// longest-first list, or -1 when there is no more work.
__device__ __forceinline__ bool read_unit(Bars* bars, int k, int& idx) {
  const int e = k % kUnitRing;
  if (!wait(bars, &bars->unit_full[e], (k / kUnitRing) & 1)) return false;
  idx = *reinterpret_cast<volatile int*>(&bars->unit[e]);
  return true;
}

__device__ __forceinline__ bool publish_unit(Bars* bars, int k, int idx) {
  const int e = k % kUnitRing;
  if (!wait(bars, &bars->unit_empty[e], ((k / kUnitRing) & 1) ^ 1)) return false;
  *reinterpret_cast<volatile int*>(&bars->unit[e]) = idx;
  ptx::mbar_arrive(&bars->unit_full[e]);
  return true;
}

// End of a unit for one sub-tile, by its softmax warpgroup: once the last PV
// has landed, O / l to the output dtype from tensor memory straight to global
// memory and lse = (m + log2 l) * ln 2.  Returns false on a timeout.
template <typename T, int D>
__device__ __forceinline__ bool store_output(const Params& p, Bars* bars, const Unit& u, int sub, int k, int rin,
                                             uint32_t tO, float m_run, float l_run) {
  if (!__all_sync(0xffffffffu, wait(bars, &bars->o[sub], k & 1))) return false;
  ptx::tc_fence_after();
  const int r = u.row0 + sub * BM + rin;
  const bool row_ok = r < u.Lq;
  // No kept key: l = 0 (O = 0, lse = -inf).  A NaN score leaves l NaN, which
  // makes both O and lse NaN.
  const bool empty_row = (l_run == 0.f);
  const float inv = empty_row ? 0.f : 1.f / l_run;
  T* op = static_cast<T*>(p.o) + (int64_t)u.b * p.os[0] + (int64_t)u.h * p.os[1] + (int64_t)(u.seq0 + r) * p.os[2];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    ptx::tmem_ld32(tO + 32 * c, o);
    ptx::tmem_wait_ld();
    if (row_ok) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = pack2<T>(__uint_as_float(o[8 * v + 2 * i]) * inv, __uint_as_float(o[8 * v + 2 * i + 1]) * inv);
        *reinterpret_cast<uint4*>(op + 32 * c + 8 * v) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  if (row_ok) {
    const float lse = empty_row ? -INFINITY : (m_run + __log2f(l_run)) * kLn2;
    p.lse[((int64_t)u.b * p.Hq + u.h) * p.L + u.seq0 + r] = lse;
  }
  return true;
}

}  // namespace pf

template <typename T, int D, bool kVarlen>
__global__ void __launch_bounds__(pf::kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p, int n_units, int mblocks, int sched) {
  using C = pf::Cfg<D>;
  using namespace pf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::KV_OFF;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);

  const bool causal = (p.mask == SDPA_MASK_CAUSAL) || (p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL);
  constexpr bool kWI = D == 128;  // MMA issue by the whole warp
  const int bx = kVarlen ? p.n_seqs : p.B;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->q[s], 1);
      ptx::mbar_init(&bars->q_free[s], 1);
      ptx::mbar_init(&bars->s[s], 1);
      ptx::mbar_init(&bars->p[s], 128);
      ptx::mbar_init(&bars->o[s], 1);
    }
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    for (int e = 0; e < kUnitRing; ++e) {
      ptx::mbar_init(&bars->unit_full[e], 1);
      ptx::mbar_init(&bars->unit_empty[e], kUnitReaders);
    }
    ptx::mbar_init(&bars->done, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(&bars->tmem, 512);
    ptx::tmem_relinquish();
  }
  if (warp == kWarpLoad && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp >= 8) {
    // Every warp of a warpgroup changes its register count at the same
    // instruction, then the warpgroup splits by role.
    ptx::regs_dec<kRegsCtl>();
    if (warp == kWarpLoad && lane == 0) {
      // ---------------------------------------------------------- producer
      // Takes units from the grid-wide counter (longest first, whichever CTA
      // is ready next: greedy scheduling), publishes each to the other roles,
      // then loads K_0, the unit's Q (each sub-tile's buffer once the
      // previous unit's last scores have read it), V_0, K_1, V_1, ...
      int t = 0, ku = 0;
      int nq[NSUB] = {0, 0};  // Q loads issued per sub-tile
      bool ok = true;
      for (;;) {
        const int idx = (int)atomicAdd(&g_unit_next[sched], 1u);
        const bool more = idx < n_units;
        Unit u;
        if (more && !unit_at<kVarlen>(p, idx, bx, mblocks, causal, u)) continue;
        if (!publish_unit(bars, ku, more ? idx : -1)) {
          ok = false;
          break;
        }
        ++ku;
        if (!more) break;
        const int kvh = u.h / p.group;
        for (int j = 0; j < u.n_kv && ok; ++j) {
          for (int which = 0; which < 2; ++which, ++t) {
            if (j == 0 && which == 1) {
              for (int sub = 0; sub < NSUB; ++sub) {
                if (nq[sub] > 0 && !wait(bars, &bars->q_free[sub], (nq[sub] - 1) & 1)) {
                  ok = false;
                  break;
                }
                ptx::mbar_arrive_expect_tx(&bars->q[sub], C::TILE);
                for (int kb = 0; kb < C::NB; ++kb)
                  ptx::tma_load_4d(sQ + sub * C::TILE + kb * C::BLOCK, &tmQ, &bars->q[sub], 64 * kb,
                                   u.seq0 + u.row0 + sub * BM, u.h, u.b);
                ++nq[sub];
              }
              if (!ok) break;
            }
            const int slot = t % C::NS;
            if (!wait_idle(bars, &bars->empty[slot], ((t / C::NS) & 1) ^ 1)) {
              ok = false;
              break;
            }
            ptx::mbar_arrive_expect_tx(&bars->full[slot], C::TILE);
            const CUtensorMap* m = which ? &tmV : &tmK;
            for (int kb = 0; kb < C::NB; ++kb)
              ptx::tma_load_4d(sKV + slot * C::TILE + kb * C::BLOCK, m, &bars->full[slot], 64 * kb,
                               u.seq0 + j * BN, kvh, u.b);
          }
        }
        if (!ok) break;
      }
      if (!ok) flag_error(bars, 1);
      // Drain: the last load issued into each slot and each Q buffer has
      // landed before exit.
      for (int v = max(0, t - C::NS); v < t; ++v)
        if (!drain(&bars->full[v % C::NS], (v / C::NS) & 1)) flag_error(bars, 2);
      for (int sub = 0; sub < NSUB; ++sub)
        if (nq[sub] > 0 && !drain(&bars->q[sub], (nq[sub] - 1) & 1)) flag_error(bars, 2);
    } else if (warp == kWarpMma && (kWI || lane == 0)) {
      // ---------------------------------------------------------- MMA issuer
      // For E = 128 the whole warp runs this loop (every decision
      // warp-uniform) and one elected lane issues each tensor-core
      // instruction and commit, which keeps the issue up with the tensor
      // pipe while the softmax warps load the sub-partitions (measured: 1 %
      // faster at E = 128, 2-3 % slower at E = 64 and 96, where one thread
      // issues).
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_qk = ptx::idesc_f16(kBf16, BM, BN, false);
      constexpr uint32_t idesc_pv = ptx::idesc_f16(kBf16, BM, D, true);
      const uint64_t dq = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = ptx::sdesc_sw128(ptx::smem_u32(sKV), 16, 1024);
      const uint64_t dv0 = ptx::sdesc_sw128(ptx::smem_u32(sKV), C::BLOCK, 1024);
      constexpr uint64_t kSlotStep = C::TILE >> 4;
      constexpr uint64_t kSubStep = C::TILE >> 4;
      int t = 0, k = 0;  // ring position of the unit's K_0; units done
      int tile0 = 0, tile1 = 0;  // key tiles whose P each sub-tile has handed over
      int idx = -1;
      bool ok = mma_uniform<kWI>(read_unit(bars, 0, idx));
      if (ok && (!kWI || lane == 0)) ptx::mbar_arrive(&bars->unit_empty[0]);
      bool have = ok && idx >= 0;
      Unit u;
      if (have) {
        unit_at<kVarlen>(p, idx, bx, mblocks, causal, u);
        // Scores of the first unit's first key tile.
        ok = mma_wait<kWI>(bars, &bars->full[0], 0);
#pragma unroll 1
        for (int sub = 0; sub < NSUB && ok; ++sub) {
          // A sub-tile without tiles still takes its Q barrier's phase.
          if (!mma_wait<kWI>(bars, &bars->q[sub], 0)) {
            ok = false;
            break;
          }
          const int ns = sub ? u.n1 : u.n0;
          if (ns > 0) {
            ptx::tc_fence_after();
            issue_qk<D, kWI>(tmem + sub * 128, dq + sub * kSubStep, dk0, idesc_qk);
            mma_commit_as<kWI>(&bars->s[sub]);
          }
          if (ns <= 1) mma_commit_as<kWI>(&bars->q_free[sub]);
        }
        if (ok) mma_commit_as<kWI>(&bars->empty[0]);
      }
      while (have && ok) {
        const int n = u.n_kv;
        // Steady key tiles j < n-1: PV_i(j) then S_i(j+1), sub-tile by
        // sub-tile (S_i then holds only P that its PV has consumed).
        for (int j = 0; j + 1 < n && ok; ++j) {
          const int vt = t + 2 * j + 1, vslot = vt % C::NS;
          const int kt = t + 2 * (j + 1), kslot = kt % C::NS;
          const uint64_t dv = dv0 + vslot * kSlotStep, dk = dk0 + kslot * kSlotStep;
          const uint32_t acc = j > 0 ? 1u : 0u;
          // The first PV of a unit overwrites O: its P is written only after
          // the softmax warpgroup has read the previous unit's O out.
          ok = mma_wait<kWI>(bars, &bars->full[vslot], (vt / C::NS) & 1) && mma_wait<kWI>(bars, &bars->p[0], tile0 & 1);
          if (!ok) break;
          ++tile0;
          ptx::tc_fence_after();
          issue_pv<kWI>(tmem + 256, tmem, dv, acc, idesc_pv);
          if (!mma_wait<kWI>(bars, &bars->full[kslot], (kt / C::NS) & 1)) {
            ok = false;
            break;
          }
          if (j + 1 < u.n0) {  // sub-tile 0 may skip the unit's last key tile
            ptx::tc_fence_after();
            issue_qk<D, kWI>(tmem, dq, dk, idesc_qk);
            mma_commit_as<kWI>(&bars->s[0]);
            if (j + 2 == u.n0) mma_commit_as<kWI>(&bars->q_free[0]);  // its last scores of the unit
          }
          if (u.n1 > 0) {  // sub-tile 1 may have no rows (a short segment's last block)
            if (!mma_wait<kWI>(bars, &bars->p[1], tile1 & 1)) {
              ok = false;
              break;
            }
            ++tile1;
            ptx::tc_fence_after();
            issue_pv<kWI>(tmem + 384, tmem + 128, dv, acc, idesc_pv);
            issue_qk<D, kWI>(tmem + 128, dq + kSubStep, dk, idesc_qk);
            mma_commit_as<kWI>(&bars->s[1]);
            if (j + 2 == n) mma_commit_as<kWI>(&bars->q_free[1]);
          }
          mma_commit_as<kWI>(&bars->empty[vslot]);
          mma_commit_as<kWI>(&bars->empty[kslot]);
        }
        if (!ok) break;
        // Last key tile: PV_i(n-1) (sub-tile 0's last PV already ran above
        // when it skips this tile), then the next unit's first scores.
        const int vt = t + 2 * n - 1, vslot = vt % C::NS;
        const int kt = t + 2 * n, kslot = kt % C::NS;  // the next unit's K_0
        int nidx = -1;
        ok = mma_wait<kWI>(bars, &bars->full[vslot], (vt / C::NS) & 1) && mma_uniform<kWI>(read_unit(bars, k + 1, nidx));
        if (!ok) break;
        if (!kWI || lane == 0) ptx::mbar_arrive(&bars->unit_empty[(k + 1) % kUnitRing]);
        Unit nx;
        const bool nx_have = nidx >= 0;
        if (nx_have) unit_at<kVarlen>(p, nidx, bx, mblocks, causal, nx);
#pragma unroll 1
        for (int sub = 0; sub < NSUB; ++sub) {
          if ((sub ? u.n1 : u.n0) == n) {
            if (!mma_wait<kWI>(bars, &bars->p[sub], (sub ? tile1 : tile0) & 1)) {
              ok = false;
              break;
            }
            if (sub) ++tile1;
            else ++tile0;
            ptx::tc_fence_after();
            issue_pv<kWI>(tmem + 256 + sub * 128, tmem + sub * 128, dv0 + vslot * kSlotStep, n > 1 ? 1u : 0u,
                          idesc_pv);
          }
          mma_commit_as<kWI>(&bars->o[sub]);  // this sub-tile's output is final
          if (!nx_have) continue;
          if ((sub == 0 && !mma_wait<kWI>(bars, &bars->full[kslot], (kt / C::NS) & 1)) ||
              !mma_wait<kWI>(bars, &bars->q[sub], (k + 1) & 1)) {
            ok = false;
            break;
          }
          const int ns = sub ? nx.n1 : nx.n0;
          if (ns > 0) {
            ptx::tc_fence_after();
            issue_qk<D, kWI>(tmem + sub * 128, dq + sub * kSubStep, dk0 + kslot * kSlotStep, idesc_qk);
            mma_commit_as<kWI>(&bars->s[sub]);
          }
          if (ns <= 1) mma_commit_as<kWI>(&bars->q_free[sub]);  // the next unit's last scores
        }
        if (!ok) break;
        mma_commit_as<kWI>(&bars->empty[vslot]);
        if (!nx_have) break;
        mma_commit_as<kWI>(&bars->empty[kslot]);
        t += 2 * n;
        ++k;
        u = nx;
      }
      if (!ok) flag_error(bars, 3);
      // Every MMA issued above completes before tensor memory is freed.
      mma_commit_as<kWI>(&bars->done);
      if (!drain(&bars->done, 0)) flag_error(bars, 4);
    }
  } else {
    ptx::regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int sub = warp >> 2;
    const int rin = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + sub * 128 + lane_off;
    const uint32_t tO = tmem + 256 + sub * 128 + lane_off;
    const float sl = p.scale_log2;  // > 0 on this path
    int tile = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int idx = -1;
      ok = __all_sync(0xffffffffu, read_unit(bars, k, idx));
      if (!ok) break;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->unit_empty[k % kUnitRing]);
      if (idx < 0) break;
      Unit u;
      unit_at<kVarlen>(p, idx, bx, mblocks, causal, u);
      const int row_lo = u.row0 + sub * BM;
      const int r = row_lo + rin;  // query row within the sequence
      float m_run = -INFINITY, l_run = 0.f;
      const int n_sub = sub ? u.n1 : u.n0;
      for (int j = 0; j < n_sub; ++j, ++tile) {
        // Every wait's outcome is made warp-uniform, so a timeout can never
        // leave part of a warp inside a warp-collective tcgen05 instruction.
        if (!__all_sync(0xffffffffu, wait(bars, &bars->s[sub], tile & 1))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t s[4][32];
        tmem_ld128(tS, s);
        ptx::tmem_wait_ld();
        const int kv0 = j * BN;
        const bool masked = kv0 + BN > u.Sk || (causal && kv0 + BN - 1 > row_lo);  // warp-uniform
        if (masked) {
          const int lim = causal ? min(u.Sk, r + 1) : u.Sk;  // keys [0, lim) are kept
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (kv0 + 32 * c + i >= lim) s[c][i] = __float_as_uint(-INFINITY);
        }
        const float m_tile = row_max128(s) * sl;
        const float m_new = fmaxf(m_run, m_tile);
        const bool need = m_new > m_run + kRescaleLog2;  // false while both are -inf
        const bool any_need = __any_sync(0xffffffffu, need);
        const float factor = need ? ptx::ex2(m_run - m_new) : 1.f;
        if (need) {
          l_run *= factor;
          m_run = m_new;
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        const float rs =
            masked ? exp_pack_store<T, false>(s, sl, neg_m, tS) : exp_pack_store<T, true>(s, sl, neg_m, tS);
        // Output rescale (rare): only when some row's maximum grew by more
        // than 2^8.  The scores of this tile were issued after the previous
        // PV, so O holds the sum through the previous tile.
        if (any_need && j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + 32 * c, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            ptx::tmem_st32(tO + 32 * c, o);
          }
        }
        l_run += rs;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p[sub]);
      }
      if (!ok) break;
      ok = store_output<T, D>(p, bars, u, sub, k, rin, tO, m_run, l_run);
    }
    if (!ok) flag_error(bars, 6);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
  if (tid == 0) {
    // The last CTA to finish re-arms this launch's scheduler slot.
    __threadfence();
    if (atomicAdd(&g_cta_done[sched], 1u) == gridDim.x - 1) {
      atomicExch(&g_unit_next[sched], 0u);
      atomicExch(&g_cta_done[sched], 0u);
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------- host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// A 4-D map (feature, sequence, head, batch) with 64 x 128 boxes and 128-byte
// swizzle.  Strides are element strides (batch, head, sequence).
bool make_map(CUtensorMap* m, const void* base, bool bf16, int D, int seq, int H, int B, const int64_t* st) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)seq, (cuuint64_t)H, (cuuint64_t)B};
  int64_t s[3] = {st[2] * 2, st[1] * 2, st[0] * 2};
  // A stride of an axis of extent 1 is never used: give it a legal value.
  if (seq == 1) s[0] = 16;
  if (H == 1) s[1] = 16;
  if (B == 1) s[2] = 16;
  cuuint64_t strides[3] = {(cuuint64_t)s[0], (cuuint64_t)s[1], (cuuint64_t)s[2]};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scheduler slot of each launch, round robin over every prefill instantiation.
std::atomic<unsigned> g_launch_seq{0};

// SMs of the current device (one persistent CTA per SM).
int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 148;
  if (dev >= 0 && dev < 64) cached[dev] = v;
  return v;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

bool strides_ok(const int64_t* st) {
  for (int d = 0; d < 3; ++d)
    if ((st[d] * 2) % 16 != 0 || st[d] * 2 >= (int64_t(1) << 40)) return false;
  return true;
}

template <typename T, int D, bool V>
cudaError_t launch_t(const Params& p, cudaStream_t st) {
  using C = pf::Cfg<D>;
  const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap mq, mk, mv;
  const int Bm = V ? 1 : p.B;
  if (!make_map(&mq, p.q, bf16, D, p.L, p.Hq, Bm, p.qs) || !make_map(&mk, p.k, bf16, D, p.S, p.Hkv, Bm, p.ks) ||
      !make_map(&mv, p.v, bf16, D, p.S, p.Hkv, Bm, p.vs))
    return cudaErrorInvalidValue;
  auto kern = prefill_kernel<T, D, V>;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    // The warpgroups' setmaxnreg requests must fit in what the block is
    // launched with, or the increase would wait forever.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * pf::kThreads < 2 * 128 * pf::kRegsSoftmax + 128 * pf::kRegsCtl) return cudaErrorInvalidConfiguration;
    attr_set = true;
  }
  const int rows = V ? p.max_seqlen : p.L;
  const int mblocks = (rows + pf::NSUB * pf::BM - 1) / (pf::NSUB * pf::BM);
  const int64_t n_units = (int64_t)mblocks * (V ? p.n_seqs : p.B) * p.Hq;
  if (n_units <= 0 || n_units > (int64_t)(INT32_MAX / 2)) return cudaErrorInvalidValue;
  const int grid = (int)std::min<int64_t>(n_units, sm_count());
  const int sched = (int)(g_launch_seq.fetch_add(1) % kSchedSlots);
  kern<<<grid, pf::kThreads, C::SMEM, st>>>(mq, mk, mv, p, (int)n_units, mblocks, sched);
  return cudaGetLastError();
}

template <typename T, bool V>
cudaError_t launch_d(const Params& p, cudaStream_t st) {
  switch (p.E) {
    case 64: return launch_t<T, 64, V>(p, st);
    case 96: return launch_t<T, 96, V>(p, st);
    default: return launch_t<T, 128, V>(p, st);
  }
}

}  // namespace

// Reads and clears the error word the prefill kernels set when a bounded wait
// gives up (0 = none).  Synchronous.
cudaError_t prefill_take_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_prefill_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_prefill_error, &zero, sizeof(int));
}

bool prefill_supported(const Params& p, int dtype) {
  if (dtype != SDPA_F16 && dtype != SDPA_BF16) return false;
  if (p.E != p.Ev || (p.E != 64 && p.E != 96 && p.E != 128)) return false;
  if (p.mask == SDPA_MASK_FLOAT_BIAS) return false;
  if (!(p.scale > 0.f) || !isfinite(p.scale)) return false;
  if (p.L < 1 || p.S < 1) return false;
  if (!strides_ok(p.qs) || !strides_ok(p.ks) || !strides_ok(p.vs) || !strides_ok(p.os)) return false;
  if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(p.o)) return false;
  return true;
}

cudaError_t launch_prefill(const Params& p, int dtype, cudaStream_t st) {
  const bool varlen = p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL;
  if (dtype == SDPA_BF16)
    return varlen ? launch_d<__nv_bfloat16, true>(p, st) : launch_d<__nv_bfloat16, false>(p, st);
  return varlen ? launch_d<__half, true>(p, st) : launch_d<__half, false>(p, st);
}

}  // namespace sdpa15
