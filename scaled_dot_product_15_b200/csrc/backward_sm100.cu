// Gradients of scaled dot-product attention on the 5th-generation tensor
// cores (sm_100a), for fp16/bf16 with E = Ev in {64, 96, 128} and the masks
// none / causal / block-diagonal (causal).  What is computed is the exactref.ai
// page "scaled_dot_product_attention", section "er.scaled_dot_product_
// attention.backward": with P the forward's weights (recomputed as
// exp(l - lse) from the forward's logsumexp), dP = grad V^T,
// D_i = grad_i . out_i, dS = P * (dP - D),
//     dq = scale dS K,   dk = scale dS^T Q,   dv = P^T grad.
// D comes from the row-dot kernel of backward_simt.cu, run first.
//
// Two kernels, each one CTA per 128-row tile, 12 warps:
//
// dQ kernel (a query tile, all its key tiles):
//   warp 5      TMA: Q and grad tiles once, K_j and V_j through two rings.
//   warp 4      MMA: S = Q K_j^T and dP = grad V_j^T (both operands in shared
//               memory) into tensor memory; dQ += dS K_j with dS read from
//               tensor memory and K_j as an MN-major operand.  S and dP of
//               the next key tile are computed while the current dS is
//               being formed (dS has columns of its own).
//   warps 0-7   elementwise, two threads per query row (warpgroup w takes
//               key columns 64w..64w+63): P = 2^(S scale log2e - lse log2e),
//               masked on boundary tiles, dS = P (dP - D), packed to 16 bits.
//   At the end the elementwise warps write dq = scale * dQ.
//
// dK/dV kernel (a key tile, all query tiles of every query head sharing it):
//   the same with the roles of rows and columns exchanged: S^T = K Q_i^T and
//   dP^T = V grad_i^T put the keys on the tensor-memory lanes, P^T and dS^T
//   are packed over them, and dV += P^T grad_i, dK += dS^T Q_i take Q_i and
//   grad_i as MN-major operands.  lse and D of the query tile are staged in
//   shared memory.  At the end dk = scale * dK and dv = dV are written.
//
// Every output element is written once (no atomics).  Every wait on an
// mbarrier is bounded (2 s); on a timeout the kernel records an error code in
// an error word (sdpa_take_device_error reports it), stops its other roles, drains what it
// issued and returns.
#include <algorithm>
#include <type_traits>

#include "backward.cuh"
#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace sdpa15 {

// Error word of the backward kernels (0 = none), read and cleared by
// backward_take_error().
__device__ int g_backward_error = 0;

namespace bw {

constexpr int BM = 128;  // rows of a tile (tensor-memory lanes)
constexpr int BN = 128;  // columns of a tile
constexpr int kThreads = 384;
constexpr int kWarpMma = 8;
constexpr int kWarpLoad = 9;
// The block is launched with 168 registers per thread (64512 in all);
// warpgroup 2 drops to 72 so the elementwise warpgroups can rise to 216.
constexpr int kRegsWork = 216;
constexpr int kRegsCtl = 72;
constexpr int kRegsLaunch = (65536 / kThreads) / 8 * 8;
static_assert(2 * 128 * kRegsWork + 128 * kRegsCtl <= kThreads * kRegsLaunch, "register split");
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int D>
struct Tile {
  static constexpr int NB = (D + 63) / 64;
  static constexpr int BLOCK = 128 * 128;  // bytes of a [128 rows][64 elements] block
  static constexpr int BYTES = NB * BLOCK;
};

struct BarsQ {
  uint64_t qg;                       // Q and grad tiles landed
  uint64_t kfull[3], kempty[3];      // key ring
  uint64_t vfull[2], vempty[2];      // value ring
  uint64_t sdp_ready;                // S and dP computed (one phase per key tile)
  uint64_t sdp_free;                 // S and dP read by every elementwise thread
  uint64_t ds_ready;                 // dS written
  uint64_t ds_free;                  // dQ MMA of the tile read dS
  uint64_t done;                     // every MMA completed
  uint32_t tmem;
  int abort;
};

struct BarsK {
  uint64_t kv;                       // K and V tiles landed
  uint64_t qfull[2], qempty[2];      // (Q_i, grad_i) ring
  uint64_t sdp_ready[2];             // S^T and dP^T of query columns 64h..64h+63 computed
  uint64_t pds_ready[2];             // warpgroup h's P^T and dS^T written
  uint64_t done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct CfgQ {
  static constexpr int T = Tile<D>::BYTES;
  static constexpr int Q_OFF = 0, G_OFF = T, K_OFF = 2 * T, V_OFF = 5 * T, BAR_OFF = 7 * T;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
};

template <int D>
struct CfgK {
  static constexpr int T = Tile<D>::BYTES;
  static constexpr int K_OFF = 0, V_OFF = T, R_OFF = 2 * T;  // ring: 2 x (Q_i, grad_i)
  static constexpr int VEC_OFF = 6 * T;                      // lse, D: [2 buffers][2 warpgroups][2][64] floats
  static constexpr int BAR_OFF = VEC_OFF + 2048;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
};

template <typename Bars>
__device__ __forceinline__ void flag_error(Bars* bars, int code) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  atomicCAS(&g_backward_error, 0, code);
}

template <typename Bars>
__device__ __forceinline__ bool wait(Bars* bars, uint64_t* bar, uint32_t parity) {
  return ptx::mbar_wait(bar, parity, kTimeoutNs, &bars->abort);
}

// wait() taken by a whole warp, which agrees on the outcome.
template <typename Bars>
__device__ __forceinline__ bool wait_w(Bars* bars, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, wait(bars, bar, parity));
}

__device__ __forceinline__ bool drain(uint64_t* bar, uint32_t parity) {
  const int never = 0;
  return ptx::mbar_wait(bar, parity, kTimeoutNs, &never);
}

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

// X = A B^T over a K dimension of D, both operands K-major in shared memory
// (descriptor plus compile-time offsets), into tensor-memory columns at d.
// kW: issued by a whole converged warp (ptx::mma_ss_off_w), else by one thread.
template <int D, bool kW = false, int KK = 0>
__device__ __forceinline__ void mma_kmajor(uint32_t d, uint64_t da, uint64_t db, uint32_t idesc) {
  if constexpr (KK < D / 16) {
    constexpr uint32_t off = ((KK / 4) * Tile<D>::BLOCK + (KK % 4) * 32) >> 4;
    if constexpr (kW)
      ptx::mma_ss_off_w<off, off>(d, da, db, idesc, KK > 0 ? 1u : 0u);
    else
      ptx::mma_ss_off<off, off>(d, da, db, idesc, KK > 0 ? 1u : 0u);
    mma_kmajor<D, kW, KK + 1>(d, da, db, idesc);
  }
}

// Acc += A B over K = 128 with A (16-bit, packed two per column) in tensor
// memory at a and B an MN-major shared-memory operand.  kSplit: A's K
// columns 0-63 are packed at a + [0, 32) and 64-127 at a + [64, 96) (each
// warpgroup's own half of the columns it read).
// KK in [KSTART, KEND) of the K = 128 products; the first one takes acc0.
// kW as for mma_kmajor.
template <bool kSplit = false, int KSTART = 0, int KEND = BN / 16, bool kW = false, int KK = KSTART>
__device__ __forceinline__ void mma_tmem_a(uint32_t acc, uint32_t a, uint64_t db, uint32_t idesc, uint32_t acc0) {
  if constexpr (KK < KEND) {
    constexpr uint32_t col = kSplit ? (KK / 4) * 64 + (KK % 4) * 8 : KK * 8;
    if constexpr (kW)
      ptx::mma_ts_off_w<col, ((KK * 16 * 128) >> 4)>(acc, a, db, idesc, KK > KSTART ? 1u : acc0);
    else
      ptx::mma_ts_off<col, ((KK * 16 * 128) >> 4)>(acc, a, db, idesc, KK > KSTART ? 1u : acc0);
    mma_tmem_a<kSplit, KSTART, KEND, kW, KK + 1>(acc, a, db, idesc, acc0);
  }
}

// One unit's rows [seq0, seq0 + n) of a (batch or segment).
struct Seg {
  int b, seq0, n;
};

template <bool kVarlen>
__device__ __forceinline__ Seg segment(const Params& p, int y) {
  Seg s;
  if (kVarlen) {
    const int c0 = min(max(__ldg(p.cu + y), 0), p.L);
    const int c1 = min(max(__ldg(p.cu + y + 1), c0), p.L);
    s.b = 0;
    s.seq0 = c0;
    s.n = c1 - c0;
  } else {
    s.b = y;
    s.seq0 = 0;
    s.n = p.L;
  }
  return s;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Barrier over the four warps of warpgroup w (named barrier 1 + w) that
// also ORs a flag over them, so every thread takes the same decision after it.
__device__ __forceinline__ bool wg_barrier_any(int w, bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "r"(1 + w)
      : "memory");
  return r != 0;
}

// 2^x on the multi-function unit.
__device__ __forceinline__ float exp2f_fast(float x) { return ptx::ex2(x); }

}  // namespace bw

// ---------------------------------------------------------------- dQ kernel

template <typename T, int D, bool kVarlen>
__global__ void __launch_bounds__(bw::kThreads, 1)
bwd_dq_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG, const Params p,
             const BwdParams g) {
  using namespace bw;
  using C = CfgQ<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BarsQ* bars = reinterpret_cast<BarsQ*>(smem + C::BAR_OFF);

  const int h = blockIdx.x;
  const Seg sg = segment<kVarlen>(p, blockIdx.y);
  const int Sk = kVarlen ? sg.n : p.S;
  const int row0 = (gridDim.z - 1 - blockIdx.z) * BM;  // longest tiles first under a causal mask
  if (row0 >= sg.n || Sk <= 0) return;  // uniform over the CTA, before any barrier
  const bool causal = p.mask == SDPA_MASK_CAUSAL || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL;
  int n = (Sk + BN - 1) / BN;
  if (causal) n = min(n, (min(row0 + BM, sg.n) - 1) / BN + 1);
  const int kvh = h / p.group;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    ptx::mbar_init(&bars->qg, 1);
    for (int s = 0; s < 3; ++s) {
      ptx::mbar_init(&bars->kfull[s], 1);
      ptx::mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->vfull[s], 1);
      ptx::mbar_init(&bars->vempty[s], 1);
    }
    ptx::mbar_init(&bars->sdp_ready, 1);
    ptx::mbar_init(&bars->sdp_free, 256);
    ptx::mbar_init(&bars->ds_ready, 256);
    ptx::mbar_init(&bars->ds_free, 1);
    ptx::mbar_init(&bars->done, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(&bars->tmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem;  // S @0, dP @128, dS @256 (64 packed columns), dQ @384

  if (warp >= 8) {
    ptx::regs_dec<kRegsCtl>();
    if (warp == kWarpLoad && lane == 0) {
      // ------------------------------------------------------------ TMA
      bool ok = true;
      ptx::mbar_arrive_expect_tx(&bars->qg, 2 * C::T);
      for (int kb = 0; kb < Tile<D>::NB; ++kb) {
        ptx::tma_load_4d(smem + C::Q_OFF + kb * Tile<D>::BLOCK, &tmQ, &bars->qg, 64 * kb, sg.seq0 + row0, h, sg.b);
        ptx::tma_load_4d(smem + C::G_OFF + kb * Tile<D>::BLOCK, &tmG, &bars->qg, 64 * kb, sg.seq0 + row0, h, sg.b);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int ks = j % 3, vs = j % 2;
        if (!wait(bars, &bars->kempty[ks], ((j / 3) & 1) ^ 1)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars->kfull[ks], C::T);
        for (int kb = 0; kb < Tile<D>::NB; ++kb)
          ptx::tma_load_4d(smem + C::K_OFF + ks * C::T + kb * Tile<D>::BLOCK, &tmK, &bars->kfull[ks], 64 * kb,
                           sg.seq0 + j * BN, kvh, sg.b);
        if (!wait(bars, &bars->vempty[vs], ((j / 2) & 1) ^ 1)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars->vfull[vs], C::T);
        for (int kb = 0; kb < Tile<D>::NB; ++kb)
          ptx::tma_load_4d(smem + C::V_OFF + vs * C::T + kb * Tile<D>::BLOCK, &tmV, &bars->vfull[vs], 64 * kb,
                           sg.seq0 + j * BN, kvh, sg.b);
      }
      if (!ok) flag_error(bars, 11);
      // Drain: the last load into every slot has landed before exit.
      if (!drain(&bars->qg, 0)) flag_error(bars, 12);
      for (int j = max(0, n - 3); j < n; ++j)
        if (!drain(&bars->kfull[j % 3], (j / 3) & 1)) flag_error(bars, 12);
      for (int j = max(0, n - 2); j < n; ++j)
        if (!drain(&bars->vfull[j % 2], (j / 2) & 1)) flag_error(bars, 12);
    } else if (warp == kWarpMma) {
      // ------------------------------------------------------------ MMA
      // The whole warp runs this loop and one elected lane issues each
      // tensor-core instruction.
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_s = ptx::idesc_f16(kBf16, BM, BN, false);
      constexpr uint32_t idesc_q = ptx::idesc_f16(kBf16, BM, D, true);
      const uint64_t dq_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::Q_OFF), 16, 1024);
      const uint64_t dg_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::G_OFF), 16, 1024);
      const uint64_t dk_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::K_OFF), 16, 1024);
      const uint64_t dkmn = ptx::sdesc_sw128(ptx::smem_u32(smem + C::K_OFF), Tile<D>::BLOCK, 1024);
      const uint64_t dv_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::V_OFF), 16, 1024);
      constexpr uint64_t kStep = C::T >> 4;
      bool ok = wait_w(bars, &bars->qg, 0) && wait_w(bars, &bars->kfull[0], 0);
      if (ok) {
        ptx::tc_fence_after();
        mma_kmajor<D, true>(tmem, dq_, dk_, idesc_s);
        ok = wait_w(bars, &bars->vfull[0], 0);
      }
      if (ok) {
        ptx::tc_fence_after();
        mma_kmajor<D, true>(tmem + 128, dg_, dv_, idesc_s);
        ptx::mma_commit_w(&bars->sdp_ready);
        ptx::mma_commit_w(&bars->vempty[0]);
      }
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) {
          // S and dP of the next key tile, once every thread has read this one's.
          const int ks = (j + 1) % 3, vs = (j + 1) % 2;
          ok = wait_w(bars, &bars->sdp_free, j & 1) && wait_w(bars, &bars->kfull[ks], ((j + 1) / 3) & 1);
          if (!ok) break;
          ptx::tc_fence_after();
          mma_kmajor<D, true>(tmem, dq_, dk_ + ks * kStep, idesc_s);
          if (!wait_w(bars, &bars->vfull[vs], ((j + 1) / 2) & 1)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          mma_kmajor<D, true>(tmem + 128, dg_, dv_ + vs * kStep, idesc_s);
          ptx::mma_commit_w(&bars->sdp_ready);
          ptx::mma_commit_w(&bars->vempty[vs]);
        }
        if (!wait_w(bars, &bars->ds_ready, j & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        mma_tmem_a<false, 0, BN / 16, true>(tmem + 384, tmem + 256, dkmn + (j % 3) * kStep, idesc_q, j > 0 ? 1u : 0u);
        ptx::mma_commit_w(&bars->ds_free);
        ptx::mma_commit_w(&bars->kempty[j % 3]);
      }
      if (!ok) flag_error(bars, 13);
      ptx::mma_commit_w(&bars->done);
      if (!drain(&bars->done, 0)) flag_error(bars, 14);
    }
  } else {
    ptx::regs_inc<kRegsWork>();
    // ------------------------------------------------------------ elementwise
    const int w = warp >> 2;                   // key columns 64w..64w+63
    const int r = (warp & 3) * 32 + lane;      // query row within the tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int rg = row0 + r;                   // row within the sequence
    const bool row_ok = rg < sg.n;
    const int64_t ridx = ((int64_t)sg.b * p.Hq + h) * p.L + sg.seq0 + rg;
    float lse2 = 0.f, Di = 0.f;
    if (row_ok) {
      const float l = p.lse[ridx];
      lse2 = (l == -INFINITY) ? INFINITY : l * kLog2e;  // no kept key: every weight 0
      Di = g.D[ridx];
    }
    const float sl = p.scale_log2;
    const uint64_t sl2 = exp2poly::pk(sl, sl), nl2 = exp2poly::pk(-lse2, -lse2), nD2 = exp2poly::pk(-Di, -Di);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!__all_sync(0xffffffffu, wait(bars, &bars->sdp_ready, j & 1))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      uint32_t s[2][32], dp[2][32];
      ptx::tmem_ld32(tmem + lane_off + 64 * w, s[0]);
      ptx::tmem_ld32(tmem + lane_off + 64 * w + 32, s[1]);
      ptx::tmem_ld32(tmem + lane_off + 128 + 64 * w, dp[0]);
      ptx::tmem_ld32(tmem + lane_off + 128 + 64 * w + 32, dp[1]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->sdp_free);
      const int kv0 = j * BN + 64 * w;
      const bool masked = !row_ok || kv0 + 64 > Sk || (causal && kv0 + 63 > row0);  // warp-uniform
      const int lim = !row_ok ? 0 : (causal ? min(Sk, rg + 1) : Sk);  // keys [0, lim) are kept
      const int cmax = lim - kv0;  // this tile's columns c < cmax are kept
      uint32_t ds[32];
      // Two straight-line copies of the loop (masked is warp-uniform): a mask
      // test between the pairs would split the unrolled loop into small blocks.
      auto form = [&](auto kMasked) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c0 = 2 * i, c1 = 2 * i + 1;
          // Pairs in packed fp32x2 arithmetic.
          const uint64_t x = exp2poly::ffma2(
              exp2poly::pk(__uint_as_float(s[c0 >> 5][c0 & 31]), __uint_as_float(s[c1 >> 5][c1 & 31])), sl2, nl2);
          float x0, x1;
          exp2poly::upk(x, x0, x1);
          float p0 = exp2f_fast(x0), p1 = exp2f_fast(x1);
          if constexpr (decltype(kMasked)::value) {
            p0 = c0 < cmax ? p0 : 0.f;
            p1 = c1 < cmax ? p1 : 0.f;
          }
          const uint64_t dd = exp2poly::fmul2(
              exp2poly::pk(p0, p1),
              exp2poly::fadd2(
                  exp2poly::pk(__uint_as_float(dp[c0 >> 5][c0 & 31]), __uint_as_float(dp[c1 >> 5][c1 & 31])), nD2));
          float d0, d1;
          exp2poly::upk(dd, d0, d1);
          ds[i] = pack2<T>(d0, d1);
        }
      };
      if (masked)
        form(std::true_type{});
      else
        form(std::false_type{});
      // dS has its own columns; the previous tile's dQ MMA must have read them.
      if (j > 0 && !__all_sync(0xffffffffu, wait(bars, &bars->ds_free, (j - 1) & 1))) {
        ok = false;
        break;
      }
      ptx::tmem_st32(tmem + lane_off + 256 + 32 * w, ds);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->ds_ready);
    }
    // dq = scale * dQ: warpgroup w writes the 32-column chunks c with c % 2 == w.
    if (ok) ok = __all_sync(0xffffffffu, wait(bars, &bars->done, 0));
    if (ok) {
      ptx::tc_fence_after();
      T* dqp = static_cast<T*>(g.dq) + (int64_t)sg.b * g.dqs[0] + (int64_t)h * g.dqs[1] +
               (int64_t)(sg.seq0 + (row_ok ? rg : 0)) * g.dqs[2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        if (c % 2 != w) continue;  // warp-uniform
        uint32_t o[32];
        ptx::tmem_ld32(tmem + lane_off + 384 + 32 * c, o);
        ptx::tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint32_t q4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              q4[i] = pack2<T>(__uint_as_float(o[8 * v4 + 2 * i]) * p.scale,
                               __uint_as_float(o[8 * v4 + 2 * i + 1]) * p.scale);
            *reinterpret_cast<uint4*>(dqp + 32 * c + 8 * v4) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
          }
        }
      }
    }
    if (!ok) flag_error(bars, 15);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK/dV kernel

template <typename T, int D, bool kVarlen>
__global__ void __launch_bounds__(bw::kThreads, 1)
bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG, const Params p,
               const BwdParams g) {
  using namespace bw;
  using C = CfgK<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BarsK* bars = reinterpret_cast<BarsK*>(smem + C::BAR_OFF);
  float* vec = reinterpret_cast<float*>(smem + C::VEC_OFF);  // [buffer][lse2 | D][128]

  const int kvh = blockIdx.x;
  const Seg sg = segment<kVarlen>(p, blockIdx.y);
  const int Sk = kVarlen ? sg.n : p.S;
  const int Lq = sg.n;
  const int key0 = blockIdx.z * BN;  // key tiles in order: the first see the most query tiles
  if (key0 >= Sk || Lq <= 0) return;  // uniform over the CTA, before any barrier
  const bool causal = p.mask == SDPA_MASK_CAUSAL || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL;
  const int qt_lo = causal ? key0 / BM : 0;  // query tiles that keep some key of this tile
  const int qt_hi = (Lq + BM - 1) / BM;
  const int per = max(0, qt_hi - qt_lo);
  const int iters = per * p.group;  // (query head of the group, query tile) pairs

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    ptx::mbar_init(&bars->kv, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars->qfull[s], 1);
      ptx::mbar_init(&bars->qempty[s], 1);
    }
    for (int hf = 0; hf < 2; ++hf) {
      ptx::mbar_init(&bars->sdp_ready[hf], 1);
      ptx::mbar_init(&bars->pds_ready[hf], 128);
    }
    ptx::mbar_init(&bars->done, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(&bars->tmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem;  // S^T @0, dP^T @128, dV @256, dK @384

  if (warp >= 8) {
    ptx::regs_dec<kRegsCtl>();
    if (warp == kWarpLoad && lane == 0) {
      // ------------------------------------------------------------ TMA
      bool ok = true;
      ptx::mbar_arrive_expect_tx(&bars->kv, 2 * C::T);
      for (int kb = 0; kb < Tile<D>::NB; ++kb) {
        ptx::tma_load_4d(smem + C::K_OFF + kb * Tile<D>::BLOCK, &tmK, &bars->kv, 64 * kb, sg.seq0 + key0, kvh, sg.b);
        ptx::tma_load_4d(smem + C::V_OFF + kb * Tile<D>::BLOCK, &tmV, &bars->kv, 64 * kb, sg.seq0 + key0, kvh, sg.b);
      }
      for (int it = 0; it < iters && ok; ++it) {
        const int h = kvh * p.group + it / per, q0 = (qt_lo + it % per) * BM;
        const int slot = it & 1;
        if (!wait(bars, &bars->qempty[slot], ((it >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars->qfull[slot], 2 * C::T);
        uint8_t* base = smem + C::R_OFF + slot * 2 * C::T;
        for (int kb = 0; kb < Tile<D>::NB; ++kb) {
          ptx::tma_load_4d(base + kb * Tile<D>::BLOCK, &tmQ, &bars->qfull[slot], 64 * kb, sg.seq0 + q0, h, sg.b);
          ptx::tma_load_4d(base + C::T + kb * Tile<D>::BLOCK, &tmG, &bars->qfull[slot], 64 * kb, sg.seq0 + q0, h,
                           sg.b);
        }
      }
      if (!ok) flag_error(bars, 21);
      if (!drain(&bars->kv, 0)) flag_error(bars, 22);
      for (int it = max(0, iters - 2); it < iters; ++it)
        if (!drain(&bars->qfull[it & 1], (it >> 1) & 1)) flag_error(bars, 22);
    } else if (warp == kWarpMma) {
      // ------------------------------------------------------------ MMA
      // The whole warp runs this loop and one elected lane issues each
      // tensor-core instruction.
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      // Query columns are handled in two halves (64 each), one per
      // elementwise warpgroup, so that one half's products overlap the other
      // half's elementwise work: S^T / dP^T of a half are N = 64 products
      // (the half's 64 query rows of Q_i / grad_i as B), dV / dK of a half
      // the K = 64 slice of the query dimension.
      constexpr uint32_t idesc_s = ptx::idesc_f16(kBf16, BM, BN / 2, false);
      constexpr uint32_t idesc_acc = ptx::idesc_f16(kBf16, BM, D, true);
      const uint64_t dk_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::K_OFF), 16, 1024);
      const uint64_t dv_ = ptx::sdesc_sw128(ptx::smem_u32(smem + C::V_OFF), 16, 1024);
      const uint32_t r0 = ptx::smem_u32(smem + C::R_OFF);
      const uint64_t dq_ = ptx::sdesc_sw128(r0, 16, 1024);                       // Q_i, K-major
      const uint64_t dg_ = ptx::sdesc_sw128(r0 + C::T, 16, 1024);                // grad_i, K-major
      const uint64_t dqmn = ptx::sdesc_sw128(r0, Tile<D>::BLOCK, 1024);          // Q_i, MN-major
      const uint64_t dgmn = ptx::sdesc_sw128(r0 + C::T, Tile<D>::BLOCK, 1024);   // grad_i, MN-major
      constexpr uint64_t kSlot = (2 * C::T) >> 4;
      constexpr uint64_t kHalfRows = (64 * 128) >> 4;  // 64 rows of a 128-byte-row block
      // S^T and dP^T of query half hf of the tile in ring slot ns.
      auto scores = [&](int ns, int hf) {
        const uint64_t off = ns * kSlot + hf * kHalfRows;
        mma_kmajor<D, true>(tmem + 64 * hf, dk_, dq_ + off, idesc_s);
        mma_kmajor<D, true>(tmem + 128 + 64 * hf, dv_, dg_ + off, idesc_s);
        ptx::mma_commit_w(&bars->sdp_ready[hf]);
      };
      bool ok = iters == 0 || (wait_w(bars, &bars->kv, 0) && wait_w(bars, &bars->qfull[0], 0));
      if (ok && iters > 0) {
        ptx::tc_fence_after();
        scores(0, 0);
        scores(0, 1);
      }
      for (int it = 0; it < iters && ok; ++it) {
        const int slot = it & 1, ns = (it + 1) & 1;
        const bool next = it + 1 < iters;
        // Half 0: dV += P^T grad_i and dK += dS^T Q_i over query rows 0-63,
        // then (the next tile's Q_i and grad_i loaded) its next S^T, dP^T.
        if (!wait_w(bars, &bars->pds_ready[0], it & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        mma_tmem_a<true, 0, 4, true>(tmem + 256, tmem, dgmn + slot * kSlot, idesc_acc, it > 0 ? 1u : 0u);
        mma_tmem_a<true, 0, 4, true>(tmem + 384, tmem + 128, dqmn + slot * kSlot, idesc_acc, it > 0 ? 1u : 0u);
        if (next) {
          if (!wait_w(bars, &bars->qfull[ns], ((it + 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          scores(ns, 0);  // overwrites only half 0's columns
        }
        // Half 1.
        if (!wait_w(bars, &bars->pds_ready[1], it & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        mma_tmem_a<true, 4, 8, true>(tmem + 256, tmem, dgmn + slot * kSlot, idesc_acc, 1u);
        mma_tmem_a<true, 4, 8, true>(tmem + 384, tmem + 128, dqmn + slot * kSlot, idesc_acc, 1u);
        ptx::mma_commit_w(&bars->qempty[slot]);
        if (next) scores(ns, 1);
      }
      if (!ok) flag_error(bars, 23);
      ptx::mma_commit_w(&bars->done);
      if (!drain(&bars->done, 0)) flag_error(bars, 24);
    }
  } else {
    ptx::regs_inc<kRegsWork>();
    // ------------------------------------------------------------ elementwise
    const int w = warp >> 2;                   // query columns 64w..64w+63
    const int r = (warp & 3) * 32 + lane;      // key row within the tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int kj = key0 + r;                   // key within the sequence
    const float sl = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < iters; ++it) {
      const int h = kvh * p.group + it / per, q0 = (qt_lo + it % per) * BM;
      // lse * log2(e) and D of this warpgroup's 64 query rows, staged by its
      // first 64 threads ([buffer][warpgroup][lse2 | D][64]).
      float* lv = vec + ((it & 1) * 2 + w) * 128;
      if (r < 64) {
        const int qi = q0 + 64 * w + r;
        float l2 = INFINITY, dd = 0.f;  // rows past the end: weight 0
        if (qi < Lq) {
          const int64_t ridx = ((int64_t)sg.b * p.Hq + h) * p.L + sg.seq0 + qi;
          const float l = p.lse[ridx];
          l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
          dd = g.D[ridx];
        }
        lv[r] = l2;
        lv[64 + r] = dd;
      }
      ok = __all_sync(0xffffffffu, wait(bars, &bars->sdp_ready[w], it & 1));
      ptx::tc_fence_after();
      uint32_t s[2][32], dp[2][32];
      if (ok) {
        ptx::tmem_ld32(tmem + lane_off + 64 * w, s[0]);
        ptx::tmem_ld32(tmem + lane_off + 64 * w + 32, s[1]);
        ptx::tmem_ld32(tmem + lane_off + 128 + 64 * w, dp[0]);
        ptx::tmem_ld32(tmem + lane_off + 128 + 64 * w + 32, dp[1]);
        ptx::tmem_wait_ld();
      }
      // The staged lse / D are visible to the warpgroup (every one of its
      // 128 threads reaches this barrier on every iteration, and all leave
      // together if any of them timed out).  Each thread packs its results
      // over columns it has read itself, so no other warpgroup is waited for.
      if (wg_barrier_any(w, !ok)) {
        ok = false;
        break;
      }
      // Query columns c < cmin of this thread's key row are masked out (all
      // of them for a key past the end; under a causal mask the columns of
      // queries before the key).  Columns of query rows past the end have
      // lse = +inf staged, so their weights are 2^-inf = 0 already.
      const int qc0 = q0 + 64 * w;
      const int cmin = kj >= Sk ? 64 : (causal ? kj - qc0 : 0);
      // Two straight-line copies of the loop, chosen per warp: a mask test
      // between the pairs would split the unrolled loop into small blocks.
      auto form = [&](auto kMasked) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pp[16], dsp[16];
#pragma unroll
          for (int qd = 0; qd < 8; ++qd) {  // 4 query columns at a time
            const int c = 32 * half + 4 * qd;
            const float4 l4 = *reinterpret_cast<const float4*>(lv + c);
            const float4 d4 = *reinterpret_cast<const float4*>(lv + 64 + c);
            const float ls[4] = {l4.x, l4.y, l4.z, l4.w}, ds[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
              const int c0 = c + 2 * pr, c1 = c0 + 1;
              float p0 = exp2f_fast(__uint_as_float(s[c0 >> 5][c0 & 31]) * sl - ls[2 * pr]);
              float p1 = exp2f_fast(__uint_as_float(s[c1 >> 5][c1 & 31]) * sl - ls[2 * pr + 1]);
              if constexpr (decltype(kMasked)::value) {
                p0 = c0 >= cmin ? p0 : 0.f;
                p1 = c1 >= cmin ? p1 : 0.f;
              }
              const float d0 = p0 * (__uint_as_float(dp[c0 >> 5][c0 & 31]) - ds[2 * pr]);
              const float d1 = p1 * (__uint_as_float(dp[c1 >> 5][c1 & 31]) - ds[2 * pr + 1]);
              pp[2 * qd + pr] = pack2<T>(p0, p1);
              dsp[2 * qd + pr] = pack2<T>(d0, d1);
            }
          }
          tmem_st16(tmem + lane_off + 64 * w + 16 * half, pp);
          tmem_st16(tmem + lane_off + 128 + 64 * w + 16 * half, dsp);
        }
      };
      if (__any_sync(0xffffffffu, cmin > 0))
        form(std::true_type{});
      else
        form(std::false_type{});
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->pds_ready[w]);
    }
    // dk = scale * dK, dv = dV: warpgroup w writes the 32-column chunks c
    // with c % 2 == w of both.
    if (ok && iters > 0) ok = __all_sync(0xffffffffu, wait(bars, &bars->done, 0));
    if (ok) {
      ptx::tc_fence_after();
      const bool key_ok = kj < Sk;
      const int64_t row = sg.seq0 + (key_ok ? kj : 0);
      T* dkp = static_cast<T*>(g.dk) + (int64_t)sg.b * g.dks[0] + (int64_t)kvh * g.dks[1] + row * g.dks[2];
      T* dvp = static_cast<T*>(g.dv) + (int64_t)sg.b * g.dvs[0] + (int64_t)kvh * g.dvs[1] + row * g.dvs[2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        if (c % 2 != w) continue;  // warp-uniform
        uint32_t ok_[32], ov[32];
        if (iters > 0) {
          ptx::tmem_ld32(tmem + lane_off + 384 + 32 * c, ok_);
          ptx::tmem_ld32(tmem + lane_off + 256 + 32 * c, ov);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ok_[i] = ov[i] = 0u;  // no query row keeps these keys
        }
        if (key_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint32_t a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              a[i] = pack2<T>(__uint_as_float(ok_[8 * v4 + 2 * i]) * p.scale,
                              __uint_as_float(ok_[8 * v4 + 2 * i + 1]) * p.scale);
              b[i] = pack2<T>(__uint_as_float(ov[8 * v4 + 2 * i]), __uint_as_float(ov[8 * v4 + 2 * i + 1]));
            }
            *reinterpret_cast<uint4*>(dkp + 32 * c + 8 * v4) = make_uint4(a[0], a[1], a[2], a[3]);
            *reinterpret_cast<uint4*>(dvp + 32 * c + 8 * v4) = make_uint4(b[0], b[1], b[2], b[3]);
          }
        }
      }
    }
    if (!ok) flag_error(bars, 25);
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

template <typename T, int D, bool V>
cudaError_t launch_bwd_t(const Params& p, const BwdParams& g, cudaStream_t st) {
  const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  const int Bm = V ? 1 : p.B;
  CUtensorMap mq, mk, mv, mg;
  if (!tmahost::make_map(&mq, p.q, bf16, D, p.L, p.Hq, Bm, p.qs) ||
      !tmahost::make_map(&mk, p.k, bf16, D, p.S, p.Hkv, Bm, p.ks) ||
      !tmahost::make_map(&mv, p.v, bf16, D, p.S, p.Hkv, Bm, p.vs) ||
      !tmahost::make_map(&mg, g.dO, bf16, D, p.L, p.Hq, Bm, g.dos))
    return cudaErrorInvalidValue;
  auto kq = bwd_dq_sm100<T, D, V>;
  auto kk = bwd_dkdv_sm100<T, D, V>;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, bw::CfgQ<D>::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, bw::CfgK<D>::SMEM);
    if (e != cudaSuccess) return e;
    // The warpgroups' setmaxnreg requests must fit in what the block is
    // launched with, or the increase would wait forever.
    cudaFuncAttributes fa, fb;
    if (cudaFuncGetAttributes(&fa, kq) != cudaSuccess || cudaFuncGetAttributes(&fb, kk) != cudaSuccess)
      return cudaErrorInvalidValue;
    const int need = 2 * 128 * bw::kRegsWork + 128 * bw::kRegsCtl;
    if (fa.numRegs * bw::kThreads < need || fb.numRegs * bw::kThreads < need) return cudaErrorInvalidConfiguration;
    attr_set = true;
  }
  const int rows = V ? p.max_seqlen : p.L;
  const int keys = V ? p.max_seqlen : p.S;
  const int y = V ? p.n_seqs : p.B;
  const int qtiles = (rows + bw::BM - 1) / bw::BM, ktiles = (keys + bw::BN - 1) / bw::BN;
  kk<<<dim3(p.Hkv, y, ktiles), bw::kThreads, bw::CfgK<D>::SMEM, st>>>(mq, mk, mv, mg, p, g);
  kq<<<dim3(p.Hq, y, qtiles), bw::kThreads, bw::CfgQ<D>::SMEM, st>>>(mq, mk, mv, mg, p, g);
  return cudaGetLastError();
}

template <typename T, bool V>
cudaError_t launch_bwd_d(const Params& p, const BwdParams& g, cudaStream_t st) {
  switch (p.E) {
    case 64: return launch_bwd_t<T, 64, V>(p, g, st);
    case 96: return launch_bwd_t<T, 96, V>(p, g, st);
    default: return launch_bwd_t<T, 128, V>(p, g, st);
  }
}

}  // namespace

// Problems the tensor-core backward takes; the rest go to the SIMT kernels.
bool backward_sm100_supported(const Params& p, const BwdParams& g, int dtype) {
  using tmahost::aligned16;
  using tmahost::strides_ok;
  if (dtype != SDPA_F16 && dtype != SDPA_BF16) return false;
  if (p.E != p.Ev || (p.E != 64 && p.E != 96 && p.E != 128)) return false;
  if (p.mask == SDPA_MASK_FLOAT_BIAS || p.mask == SDPA_MASK_BOOL) return false;
  if (!(p.scale > 0.f) || !isfinite(p.scale)) return false;
  if (p.L < 1 || p.S < 1) return false;
  const bool varlen = p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL;
  const int rows = varlen ? p.max_seqlen : p.L, keys = varlen ? p.max_seqlen : p.S;
  if ((rows + 127) / 128 > 65535 || (keys + 127) / 128 > 65535) return false;
  if (varlen && p.n_seqs > 65535) return false;
  if (!strides_ok(p.qs) || !strides_ok(p.ks) || !strides_ok(p.vs) || !strides_ok(g.dos)) return false;
  if (!strides_ok(g.dqs) || !strides_ok(g.dks) || !strides_ok(g.dvs)) return false;
  if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(g.dO)) return false;
  if (!aligned16(g.dq) || !aligned16(g.dk) || !aligned16(g.dv)) return false;
  return true;
}

// The dK/dV kernel, then the dQ kernel; the row-dot kernel (D) must have run.
cudaError_t launch_backward_sm100(const Params& p, const BwdParams& g, int dtype, cudaStream_t st) {
  const bool varlen = p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL;
  if (dtype == SDPA_BF16)
    return varlen ? launch_bwd_d<__nv_bfloat16, true>(p, g, st) : launch_bwd_d<__nv_bfloat16, false>(p, g, st);
  return varlen ? launch_bwd_d<__half, true>(p, g, st) : launch_bwd_d<__half, false>(p, g, st);
}

}  // namespace sdpa15

namespace sdpa15 {
// Reads and clears the backward kernels' error word.  Synchronous.
cudaError_t backward_take_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_backward_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_backward_error, &zero, sizeof(int));
}
}  // namespace sdpa15
