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
// B200 mapping (one CTA per 256 query rows of one head; 12 warps):
//   warp 9      TMA producer: Q (two 128-row sub-tiles) once, then K_j and V_j
//               128-key tiles through a ring of shared-memory slots (128-byte
//               swizzle, 64-column boxes).
//   warp 8      MMA issuer (one thread): S_i = Q_i K_j^T with both operands in
//               shared memory, and O_i += P_i V_j with P_i read from tensor
//               memory; fp32 accumulators live in tensor memory
//               (S0 | S1 | O0 | O1 = 4 x 128 columns).  The two sub-tiles are
//               interleaved (PV0, QK0 of the next tile, PV1, QK1) so the tensor
//               core works on one sub-tile while the other's softmax runs.
//   warps 0-7   softmax, one thread per query row (warpgroup i owns sub-tile
//               i): tcgen05.ld of its 128 scores, causal / segment / length
//               masking on boundary tiles only, row maximum, exp2 with
//               scale*log2(e) folded into one FMA, P packed to 16 bits and
//               stored back over its own scores in tensor memory.  The output
//               is rescaled in tensor memory only when the running maximum
//               grows by more than 2^8 (a stale maximum is exact because the
//               final normalisation uses the same one).  Epilogue: O / l to
//               the output dtype, lse = (m + log2 l) * ln 2.
// Causal attention visits only key tiles at or left of the diagonal; packed
// variable-length batches index tiles from each segment's first token.
//
// Every wait on an mbarrier is bounded (2 s); on a timeout the kernel records
// an error code, drains what it issued and returns.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace sdpa15 {

__device__ int g_prefill_error = 0;

namespace pf {

constexpr int BM = 128;  // query rows per sub-tile (tensor-memory lanes)
constexpr int BN = 128;  // keys per tile
constexpr int NSUB = 2;  // sub-tiles per CTA
constexpr int kThreads = 384;  // 3 warpgroups
constexpr int kWarpMma = 8;
constexpr int kWarpLoad = 9;
// Registers: launched with 168 per thread (384 x 168 = 64512); warpgroup 2
// (MMA, load and two idle warps) drops to 72 so the two softmax warpgroups
// can rise to 216: 2 x 128 x 216 + 128 x 72 = 64512.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = 72;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;        // 64-element column blocks per row
  static constexpr int BLOCK = 128 * 128;         // bytes of one [128 rows][64 elements] block
  static constexpr int TILE = NB * BLOCK;         // bytes of a 128-row tile
  static constexpr int NS = (D <= 64) ? 8 : 4;    // key/value ring slots
  static constexpr int KV_OFF = NSUB * TILE;
  static constexpr int BAR_OFF = KV_OFF + NS * TILE;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
};

struct Bars {
  uint64_t q;
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t s[2];
  uint64_t p[2];
  uint64_t o[2];
  uint32_t tmem;
  int abort;
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

// Lean issue: descriptors built once per CTA, operand addresses are the
// descriptor plus compile-time offsets (address >> 4 in the low 14 bits never
// carries inside shared memory).
template <int D, int SUB>
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint64_t dq, uint64_t dk, uint32_t idesc) {
  using C = Cfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * C::BLOCK + (kk % 4) * 32;
    const uint64_t a = dq + (uint64_t)((SUB * C::TILE + off) >> 4);
    const uint64_t bd = dk + (uint64_t)(off >> 4);
    ptx::mma_ss(tmem + SUB * 128, a, bd, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D, int SUB>
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint64_t dv, uint32_t acc0, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    const uint64_t bd = dv + (uint64_t)((kk * 16 * 128) >> 4);
    ptx::mma_ts(tmem + 256 + SUB * 128, tmem + SUB * 128 + kk * 8, bd, idesc, kk > 0 ? 1u : acc0);
  }
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
// weights.  With kEmu, 2 of every 8 pairs take the FMA-pipe 2^x so the
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
      if (kEmu && (i % 8) < 2) {
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

}  // namespace pf

template <typename T, int D, bool kVarlen>
__global__ void __launch_bounds__(pf::kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const Params p) {
  using C = pf::Cfg<D>;
  using namespace pf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::KV_OFF;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);

  // ---- work unit: 256 query rows of one (batch, head), or of one segment.
  // Blocks are dispatched in linear order (x fastest), so putting the row
  // block in z, last rows first, hands out the units with the most key tiles
  // (causal) first across all heads: greedy longest-first scheduling.
  const int mb = gridDim.z - 1 - blockIdx.z;
  const int h = blockIdx.x;
  int b, seq0, Lq, Sk;
  if (kVarlen) {
    const int sg = blockIdx.y;
    const int c0 = min(max(__ldg(p.cu + sg), 0), p.L);
    const int c1 = min(max(__ldg(p.cu + sg + 1), c0), p.L);
    b = 0;
    seq0 = c0;
    Lq = Sk = c1 - c0;
  } else {
    b = blockIdx.y;
    seq0 = 0;
    Lq = p.L;
    Sk = p.S;
  }
  const int row0 = mb * (NSUB * BM);
  if (row0 >= Lq || Sk <= 0) return;  // uniform over the CTA, before any barrier
  const bool causal = (p.mask == SDPA_MASK_CAUSAL) || (p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL);
  int n_kv = (Sk + BN - 1) / BN;
  if (causal) n_kv = min(n_kv, (min(row0 + NSUB * BM, Lq) - 1) / BN + 1);
  const int kvh = h / p.group;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    ptx::mbar_init(&bars->q, 1);
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->s[s], 1);
      ptx::mbar_init(&bars->p[s], 128);
      ptx::mbar_init(&bars->o[s], 1);
    }
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
    ptx::prefetch_tmap(&tmO);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem;
  if (warp >= 8) {
   // Warpgroup 2: every warp releases registers at the same instruction, then
   // splits by role.
   ptx::regs_dec<kRegsOther>();
   if (warp == kWarpLoad) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(&bars->q, NSUB * C::TILE);
      for (int sub = 0; sub < NSUB; ++sub)
        for (int kb = 0; kb < C::NB; ++kb)
          ptx::tma_load_4d(sQ + sub * C::TILE + kb * C::BLOCK, &tmQ, &bars->q, 64 * kb, seq0 + row0 + sub * BM, h,
                           b);
      int t = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int which = 0; which < 2; ++which, ++t) {
          const int slot = t % C::NS;
          if (!ptx::mbar_wait(&bars->empty[slot], ((t / C::NS) & 1) ^ 1, kTimeoutNs, &bars->abort)) {
            flag_error(bars, 1);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&bars->full[slot], C::TILE);
          const CUtensorMap* m = which ? &tmV : &tmK;
          for (int kb = 0; kb < C::NB; ++kb)
            ptx::tma_load_4d(sKV + slot * C::TILE + kb * C::BLOCK, m, &bars->full[slot], 64 * kb, seq0 + j * BN,
                             kvh, b);
        }
      }
      // Drain: the last load issued into each slot has landed before exit.
      for (int u = max(0, t - C::NS); u < t; ++u)
        if (!ptx::mbar_wait(&bars->full[u % C::NS], (u / C::NS) & 1, kTimeoutNs, &bars->abort)) flag_error(bars, 2);
      if (!ptx::mbar_wait(&bars->q, 0, kTimeoutNs, &bars->abort)) flag_error(bars, 2);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_qk = ptx::idesc_f16(kBf16, BM, BN, false);
      constexpr uint32_t idesc_pv = ptx::idesc_f16(kBf16, BM, D, true);
      const uint64_t dq = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = ptx::sdesc_sw128(ptx::smem_u32(sKV), 16, 1024);
      const uint64_t dv0 = ptx::sdesc_sw128(ptx::smem_u32(sKV), C::BLOCK, 1024);
      constexpr uint64_t kSlotStep = C::TILE >> 4;
      bool o_done[NSUB] = {false, false};
      bool ok = ptx::mbar_wait(&bars->q, 0, kTimeoutNs, &bars->abort) && ptx::mbar_wait(&bars->full[0], 0, kTimeoutNs, &bars->abort);
      if (ok) {
        ptx::tc_fence_after();
        issue_qk<D, 0>(tmem, dq, dk0, idesc_qk);
        ptx::mma_commit(&bars->s[0]);
        issue_qk<D, 1>(tmem, dq, dk0, idesc_qk);
        ptx::mma_commit(&bars->s[1]);
        ptx::mma_commit(&bars->empty[0]);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int vt = 2 * j + 1, vslot = vt % C::NS;
        if (!ptx::mbar_wait(&bars->full[vslot], (vt / C::NS) & 1, kTimeoutNs, &bars->abort)) { ok = false; break; }
        int kslot = -1;
        for (int sub = 0; sub < NSUB; ++sub) {
          if (!ptx::mbar_wait(&bars->p[sub], j & 1, kTimeoutNs, &bars->abort)) { ok = false; break; }
          ptx::tc_fence_after();
          if (sub == 0) issue_pv<D, 0>(tmem, dv0 + vslot * kSlotStep, j > 0 ? 1u : 0u, idesc_pv);
          else issue_pv<D, 1>(tmem, dv0 + vslot * kSlotStep, j > 0 ? 1u : 0u, idesc_pv);
          if (j + 1 == n_kv) {
            ptx::mma_commit(&bars->o[sub]);  // this sub-tile's output is final
            o_done[sub] = true;
          }
          if (j + 1 < n_kv) {
            if (sub == 0) {
              const int kt = 2 * (j + 1);
              kslot = kt % C::NS;
              if (!ptx::mbar_wait(&bars->full[kslot], (kt / C::NS) & 1, kTimeoutNs, &bars->abort)) { ok = false; break; }
              ptx::tc_fence_after();
            }
            if (sub == 0) issue_qk<D, 0>(tmem, dq, dk0 + kslot * kSlotStep, idesc_qk);
            else issue_qk<D, 1>(tmem, dq, dk0 + kslot * kSlotStep, idesc_qk);
            ptx::mma_commit(&bars->s[sub]);
          }
        }
        if (!ok) break;
        ptx::mma_commit(&bars->empty[vslot]);
        if (kslot >= 0) ptx::mma_commit(&bars->empty[kslot]);
      }
      if (!ok) flag_error(bars, 3);
      // On an abort, still complete the output barriers once every MMA issued
      // above has finished, so no waiter is left behind.
      for (int sub = 0; sub < NSUB; ++sub)
        if (!o_done[sub]) ptx::mma_commit(&bars->o[sub]);
      if (!ptx::mbar_wait(&bars->o[0], 0, kTimeoutNs, &bars->abort)) flag_error(bars, 4);
    }
   }
  } else {
    ptx::regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int sub = warp >> 2;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + sub * 128 + lane_off;
    const uint32_t tO = tmem + 256 + sub * 128 + lane_off;
    const int row_lo = row0 + sub * BM;
    const int r = row_lo + (warp & 3) * 32 + lane;  // query row within the sequence
    const float sl = p.scale_log2;                  // > 0 on this path
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      // Every wait's outcome is made warp-uniform, so a timeout can never
      // leave part of a warp inside a warp-collective tcgen05 instruction.
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bars->s[sub], j & 1, kTimeoutNs, &bars->abort))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + 32 * c, s[c]);
      ptx::tmem_wait_ld();
      const int kv0 = j * BN;
      const bool masked = kv0 + BN > Sk || (causal && kv0 + BN - 1 > row_lo);  // warp-uniform
      if (masked) {
        const int lim = causal ? min(Sk, r + 1) : Sk;  // keys [0, lim) are kept
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
      const float rs = masked ? exp_pack_store<T, false>(s, sl, neg_m, tS) : exp_pack_store<T, true>(s, sl, neg_m, tS);
      // Output rescale (rare): only when some row's maximum grew by > 2^8.
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
    // ------------------------------------------------------------ epilogue
    {
      // Warp-uniform: either the whole warp reads its rows of O or none does.
      const bool ep_ok = __all_sync(0xffffffffu, ok && ptx::mbar_wait(&bars->o[sub], 0, kTimeoutNs, &bars->abort));
      if (!ep_ok) flag_error(bars, 5);
      ptx::tc_fence_after();
      const bool row_ok = r < Lq;
      // No kept key: l = 0 (O = 0, lse = -inf).  A NaN score leaves l NaN,
      // which makes both O and lse NaN.
      const bool empty_row = (l_run == 0.f);
      const float inv = empty_row ? 0.f : 1.f / l_run;
      // Rows of this sub-tile that lie in its own sequence go out through
      // shared memory and one TMA tensor store (rows past the tensor's end
      // are clipped by the TMA); a packed sequence's last, partial tile is
      // written row by row so the next segment's rows are not touched.
      if (!kVarlen || row_lo + BM <= Lq) {
        uint8_t* so = sQ + sub * C::TILE;  // this sub-tile's Q tile: its last MMA has completed
        const uint32_t so_u = ptx::smem_u32(so);
        const int rin = (warp & 3) * 32 + lane;
        if (ep_ok) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + 32 * c, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                w[i] = pack2<T>(__uint_as_float(o[8 * v + 2 * i]) * inv, __uint_as_float(o[8 * v + 2 * i + 1]) * inv);
              const int ch = 4 * c + v;  // 16-byte chunk of the row
              const uint32_t addr = so_u + (ch >> 3) * C::BLOCK + rin * 128 + (((ch & 7) ^ (rin & 7)) << 4);
              ptx::st_shared_v4(addr, w[0], w[1], w[2], w[3]);
            }
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::named_barrier(1 + sub, 128);  // all 128 threads of the warpgroup, always
        if ((warp & 3) == 0 && lane == 0 && ep_ok && *reinterpret_cast<volatile int*>(&bars->abort) == 0) {
          for (int kb = 0; kb < C::NB; ++kb)
            ptx::tma_store_4d(&tmO, so + kb * C::BLOCK, 64 * kb, seq0 + row_lo, h, b);
          ptx::bulk_commit_group();
          ptx::bulk_wait_read_all();
        }
      } else if (ep_ok) {
        T* op = static_cast<T*>(p.o) + (int64_t)b * p.os[0] + (int64_t)h * p.os[1] + (int64_t)(seq0 + r) * p.os[2];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + 32 * c, o);
          ptx::tmem_wait_ld();
          if (row_ok) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack2<T>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(op + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
      }
      if (row_ok && ep_ok) {
        const float lse = empty_row ? -INFINITY : (m_run + __log2f(l_run)) * kLn2;
        p.lse[((int64_t)b * p.Hq + h) * p.L + seq0 + r] = lse;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
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
  const int seqq = p.L, seqk = p.S;
  const int Bm = V ? 1 : p.B;
  CUtensorMap mo;
  if (!make_map(&mq, p.q, bf16, D, seqq, p.Hq, Bm, p.qs) || !make_map(&mk, p.k, bf16, D, seqk, p.Hkv, Bm, p.ks) ||
      !make_map(&mv, p.v, bf16, D, seqk, p.Hkv, Bm, p.vs) || !make_map(&mo, p.o, bf16, D, seqq, p.Hq, Bm, p.os))
    return cudaErrorInvalidValue;
  auto kern = prefill_kernel<T, D, V>;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int rows = V ? p.max_seqlen : p.L;
  const int mblocks = (rows + pf::NSUB * pf::BM - 1) / (pf::NSUB * pf::BM);
  dim3 grid(p.Hq, V ? p.n_seqs : p.B, mblocks);
  kern<<<grid, pf::kThreads, C::SMEM, st>>>(mq, mk, mv, mo, p);
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
  if ((int64_t)(p.L + 255) / 256 > 65535) return false;  // row blocks go in grid.z
  if ((p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) && p.n_seqs > 65535) return false;
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
