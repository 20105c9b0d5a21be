// Gradients of scaled dot-product attention (exactref.ai
// "scaled_dot_product_attention", section "er.scaled_dot_product_attention.
// backward"): with P the forward's weights, dP = grad V^T,
// D_i = sum_j P_ij dP_ij, dS = P * (dP - D),
//     grad_value = P^T grad, grad_query = scale dS K, grad_key = scale dS^T Q,
// summed over the query heads that share a key/value head.
//
// General SIMT kernels (every dtype, mask kind, head size up to 256 and any
// strides), fp32 arithmetic throughout:
//   1. bwd_rowdot: D_i = grad_i . O_i from the forward output (the same value
//      as sum_j P_ij dP_ij, since O_i = sum_j P_ij v_j), one warp per row.
//   2. bwd_dkdv: one warp per key j accumulates grad_value_j and grad_key_j
//      in registers over every query row (of every query head of its group)
//      that keeps the key, with P_ij = exp(l_ij - lse_i) recomputed from the
//      forward's logsumexp; query rows stream through shared memory.
//   3. bwd_dq: one warp per query row accumulates grad_query_i over its kept
//      keys; key/value rows stream through shared memory.
// No atomics: every output element is written once, so results are
// deterministic.  A row with no kept key (lse = -inf) contributes 0; a NaN
// forward row (lse NaN) makes what it touches NaN.  Removed keys are skipped,
// so a non-finite value under a removed key does not reach the gradients
// (the page's literal rule would make that row's D NaN).
#include "backward.cuh"

namespace sdpa15 {

constexpr int kBwdWarps = 8;     // warps per block
constexpr int kBwdTile = 16;     // rows per shared-memory tile
constexpr int kBwdMaxPL = 8;     // features per lane: head sizes up to 256

// Keys [lo, hi) that query row i keeps (forward semantics).
__device__ __forceinline__ void key_range(const Params& p, int i, int& lo, int& hi) {
  lo = 0;
  hi = p.S;
  if (p.mask == SDPA_MASK_CAUSAL) {
    hi = min(p.S, i + 1);
  } else if (p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
    const int sg = segment_of(p.cu, p.n_seqs, i);
    lo = max(0, min(p.S, __ldg(p.cu + sg)));
    hi = max(lo, min(p.S, __ldg(p.cu + sg + 1)));
    if (p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) hi = max(lo, min(hi, i + 1));
  }
}

// Query rows [lo, hi) that keep key j.
__device__ __forceinline__ void query_range(const Params& p, int j, int& lo, int& hi) {
  lo = 0;
  hi = p.L;
  if (p.mask == SDPA_MASK_CAUSAL) {
    lo = min(p.L, j);
  } else if (p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
    const int sg = segment_of(p.cu, p.n_seqs, j);
    lo = max(0, min(p.L, __ldg(p.cu + sg)));
    hi = max(lo, min(p.L, __ldg(p.cu + sg + 1)));
    if (p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) lo = min(hi, max(lo, j));
  }
}

// Weight P_ij from the logit and the row's logsumexp: 0 for a removed key or
// a row with no kept key, NaN for a NaN row.
__device__ __forceinline__ float weight(float logit, float lse) {
  if (logit == -INFINITY || lse == -INFINITY) return 0.f;
  return expf(logit - lse);
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_rowdot_kernel(Params p, BwdParams g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kBwdWarps + warp, h = blockIdx.y, b = blockIdx.z;
  if (i >= p.L) return;
  const T* op = static_cast<const T*>(p.o) + b * p.os[0] + h * p.os[1] + (int64_t)i * p.os[2];
  const T* gp = static_cast<const T*>(g.dO) + b * g.dos[0] + h * g.dos[1] + (int64_t)i * g.dos[2];
  float acc = 0.f;
  for (int e = lane; e < p.Ev; e += 32) acc = fmaf(to_f32<T>(gp[e]), to_f32<T>(op[e]), acc);
  acc = warp_sum(acc);
  if (lane == 0) g.D[((int64_t)b * p.Hq + h) * p.L + i] = acc;
}

// The same with 16-byte loads: LPR lanes (a power of two, LPR * 8 >= Ev)
// share a row, 32 / LPR rows per warp.  For 16-bit types with Ev % 8 == 0
// and 16-byte aligned rows.
template <typename T, int LPR>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_rowdot_vec_kernel(Params p, BwdParams g) {
  constexpr int kRows = 32 / LPR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = (blockIdx.x * kBwdWarps + warp) * kRows + lane / LPR, h = blockIdx.y, b = blockIdx.z;
  const int c = lane % LPR;  // 8-element chunk of the row
  float acc = 0.f;
  if (i < p.L && c * 8 < p.Ev) {
    const T* op = static_cast<const T*>(p.o) + b * p.os[0] + h * p.os[1] + (int64_t)i * p.os[2];
    const T* gp = static_cast<const T*>(g.dO) + b * g.dos[0] + h * g.dos[1] + (int64_t)i * g.dos[2];
    const uint4 ov = *reinterpret_cast<const uint4*>(op + 8 * c);
    const uint4 gv = *reinterpret_cast<const uint4*>(gp + 8 * c);
    const T* oe = reinterpret_cast<const T*>(&ov);
    const T* ge = reinterpret_cast<const T*>(&gv);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(to_f32<T>(ge[e]), to_f32<T>(oe[e]), acc);
  }
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (c == 0 && i < p.L) g.D[((int64_t)b * p.Hq + h) * p.L + i] = acc;
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkdv_kernel(Params p, BwdParams g) {
  extern __shared__ float smem[];
  float* sq = smem;                      // [kBwdTile][E]
  float* sg = smem + kBwdTile * p.E;     // [kBwdTile][Ev]
  __shared__ float s_lse[kBwdTile], s_D[kBwdTile];
  __shared__ int s_lo[kBwdWarps], s_hi[kBwdWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int j = blockIdx.x * kBwdWarps + warp;  // key of this warp
  const bool key_ok = j < p.S;
  int lo = p.L, hi = 0;
  if (key_ok) query_range(p, j, lo, hi);
  if (lane == 0) { s_lo[warp] = lo; s_hi[warp] = hi; }
  __syncthreads();
  int blo = p.L, bhi = 0;
#pragma unroll
  for (int w = 0; w < kBwdWarps; ++w) { blo = min(blo, s_lo[w]); bhi = max(bhi, s_hi[w]); }

  const T* kp = static_cast<const T*>(p.k) + b * p.ks[0] + kvh * p.ks[1] + (int64_t)(key_ok ? j : 0) * p.ks[2];
  const T* vp = static_cast<const T*>(p.v) + b * p.vs[0] + kvh * p.vs[1] + (int64_t)(key_ok ? j : 0) * p.vs[2];
  float kr[kBwdMaxPL], vr[kBwdMaxPL], dk[kBwdMaxPL], dv[kBwdMaxPL];
#pragma unroll
  for (int t = 0; t < kBwdMaxPL; ++t) {
    const int e = lane + 32 * t;
    kr[t] = (key_ok && e < p.E) ? to_f32<T>(kp[e]) : 0.f;
    vr[t] = (key_ok && e < p.Ev) ? to_f32<T>(vp[e]) : 0.f;
    dk[t] = 0.f;
    dv[t] = 0.f;
  }

  for (int hh = 0; hh < p.group; ++hh) {
    const int h = kvh * p.group + hh;
    const T* qb = static_cast<const T*>(p.q) + b * p.qs[0] + h * p.qs[1];
    const T* gb = static_cast<const T*>(g.dO) + b * g.dos[0] + h * g.dos[1];
    const float* lseb = p.lse + ((int64_t)b * p.Hq + h) * p.L;
    const float* Db = g.D + ((int64_t)b * p.Hq + h) * p.L;
    const float* biasb = (p.mask == SDPA_MASK_FLOAT_BIAS) ? p.bias + b * p.bs[0] + h * p.bs[1] : nullptr;
    // BOOL: bytes (nonzero = visible) in the bias pointer, a 0 / -inf bias
    const unsigned char* boolb = (p.mask == SDPA_MASK_BOOL)
                                     ? reinterpret_cast<const unsigned char*>(p.bias) + b * p.bs[0] + h * p.bs[1]
                                     : nullptr;
    for (int i0 = blo; i0 < bhi; i0 += kBwdTile) {
      const int ni = min(kBwdTile, bhi - i0);
      __syncthreads();  // previous tile consumed
      for (int idx = threadIdx.x; idx < ni * p.E; idx += blockDim.x) {
        const int ii = idx / p.E, e = idx - ii * p.E;
        sq[ii * p.E + e] = to_f32<T>(qb[(int64_t)(i0 + ii) * p.qs[2] + e]);
      }
      for (int idx = threadIdx.x; idx < ni * p.Ev; idx += blockDim.x) {
        const int ii = idx / p.Ev, e = idx - ii * p.Ev;
        sg[ii * p.Ev + e] = to_f32<T>(gb[(int64_t)(i0 + ii) * g.dos[2] + e]);
      }
      if (threadIdx.x < ni) {
        s_lse[threadIdx.x] = lseb[i0 + threadIdx.x];
        s_D[threadIdx.x] = Db[i0 + threadIdx.x];
      }
      __syncthreads();
      for (int ii = 0; ii < ni; ++ii) {
        const int i = i0 + ii;
        if (i < lo || i >= hi) continue;  // warp-uniform
        float dot = 0.f, dpd = 0.f;
#pragma unroll
        for (int t = 0; t < kBwdMaxPL; ++t) {
          const int e = lane + 32 * t;
          if (e < p.E) dot = fmaf(kr[t], sq[ii * p.E + e], dot);
          if (e < p.Ev) dpd = fmaf(vr[t], sg[ii * p.Ev + e], dpd);
        }
        dot = warp_sum(dot);
        dpd = warp_sum(dpd);
        float logit = p.E == 0 ? 0.f : dot * p.scale;  // E = 0: empty sums
        if (biasb) logit += __ldg(biasb + (int64_t)i * p.bs[2] + (int64_t)j * p.bs[3]);
        if (boolb) logit += __ldg(boolb + (int64_t)i * p.bs[2] + (int64_t)j * p.bs[3]) ? 0.f : -INFINITY;
        const float pij = weight(logit, s_lse[ii]);
        const float ds = pij * (dpd - s_D[ii]);
#pragma unroll
        for (int t = 0; t < kBwdMaxPL; ++t) {
          const int e = lane + 32 * t;
          if (e < p.Ev) dv[t] = fmaf(pij, sg[ii * p.Ev + e], dv[t]);
          if (e < p.E) dk[t] = fmaf(ds, sq[ii * p.E + e], dk[t]);
        }
      }
    }
  }
  if (!key_ok) return;
  T* dkp = static_cast<T*>(g.dk) + b * g.dks[0] + kvh * g.dks[1] + (int64_t)j * g.dks[2];
  T* dvp = static_cast<T*>(g.dv) + b * g.dvs[0] + kvh * g.dvs[1] + (int64_t)j * g.dvs[2];
#pragma unroll
  for (int t = 0; t < kBwdMaxPL; ++t) {
    const int e = lane + 32 * t;
    if (e < p.E) dkp[e] = from_f32<T>(dk[t] * p.scale);
    if (e < p.Ev) dvp[e] = from_f32<T>(dv[t]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(Params p, BwdParams g) {
  extern __shared__ float smem[];
  float* sk = smem;                      // [kBwdTile][E]
  float* sv = smem + kBwdTile * p.E;     // [kBwdTile][Ev]
  __shared__ int s_lo[kBwdWarps], s_hi[kBwdWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y, kvh = h / p.group;
  const int i = blockIdx.x * kBwdWarps + warp;
  const bool row_ok = i < p.L;
  int lo = p.S, hi = 0;
  if (row_ok) key_range(p, i, lo, hi);
  if (lane == 0) { s_lo[warp] = lo; s_hi[warp] = hi; }
  __syncthreads();
  int blo = p.S, bhi = 0;
#pragma unroll
  for (int w = 0; w < kBwdWarps; ++w) { blo = min(blo, s_lo[w]); bhi = max(bhi, s_hi[w]); }

  const int ri = row_ok ? i : 0;
  const T* qp = static_cast<const T*>(p.q) + b * p.qs[0] + h * p.qs[1] + (int64_t)ri * p.qs[2];
  const T* gp = static_cast<const T*>(g.dO) + b * g.dos[0] + h * g.dos[1] + (int64_t)ri * g.dos[2];
  const T* kb = static_cast<const T*>(p.k) + b * p.ks[0] + kvh * p.ks[1];
  const T* vb = static_cast<const T*>(p.v) + b * p.vs[0] + kvh * p.vs[1];
  const float lse = row_ok ? p.lse[((int64_t)b * p.Hq + h) * p.L + i] : 0.f;
  const float Di = row_ok ? g.D[((int64_t)b * p.Hq + h) * p.L + i] : 0.f;
  const float* biasp = (p.mask == SDPA_MASK_FLOAT_BIAS && row_ok)
                           ? p.bias + b * p.bs[0] + h * p.bs[1] + (int64_t)i * p.bs[2]
                           : nullptr;
  // BOOL: bytes (nonzero = visible) in the bias pointer, a 0 / -inf bias
  const unsigned char* boolp = (p.mask == SDPA_MASK_BOOL && row_ok)
                                   ? reinterpret_cast<const unsigned char*>(p.bias) + b * p.bs[0] + h * p.bs[1] +
                                         (int64_t)i * p.bs[2]
                                   : nullptr;
  float qr[kBwdMaxPL], gr[kBwdMaxPL], dq[kBwdMaxPL];
#pragma unroll
  for (int t = 0; t < kBwdMaxPL; ++t) {
    const int e = lane + 32 * t;
    qr[t] = (row_ok && e < p.E) ? to_f32<T>(qp[e]) : 0.f;
    gr[t] = (row_ok && e < p.Ev) ? to_f32<T>(gp[e]) : 0.f;
    dq[t] = 0.f;
  }
  for (int j0 = blo; j0 < bhi; j0 += kBwdTile) {
    const int nj = min(kBwdTile, bhi - j0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nj * p.E; idx += blockDim.x) {
      const int jj = idx / p.E, e = idx - jj * p.E;
      sk[jj * p.E + e] = to_f32<T>(kb[(int64_t)(j0 + jj) * p.ks[2] + e]);
    }
    for (int idx = threadIdx.x; idx < nj * p.Ev; idx += blockDim.x) {
      const int jj = idx / p.Ev, e = idx - jj * p.Ev;
      sv[jj * p.Ev + e] = to_f32<T>(vb[(int64_t)(j0 + jj) * p.vs[2] + e]);
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      const int j = j0 + jj;
      if (j < lo || j >= hi) continue;  // warp-uniform
      float dot = 0.f, dpd = 0.f;
#pragma unroll
      for (int t = 0; t < kBwdMaxPL; ++t) {
        const int e = lane + 32 * t;
        if (e < p.E) dot = fmaf(qr[t], sk[jj * p.E + e], dot);
        if (e < p.Ev) dpd = fmaf(gr[t], sv[jj * p.Ev + e], dpd);
      }
      dot = warp_sum(dot);
      dpd = warp_sum(dpd);
      float logit = p.E == 0 ? 0.f : dot * p.scale;  // E = 0: empty sums
      if (biasp) logit += __ldg(biasp + (int64_t)j * p.bs[3]);
      if (boolp) logit += __ldg(boolp + (int64_t)j * p.bs[3]) ? 0.f : -INFINITY;
      const float ds = weight(logit, lse) * (dpd - Di);
#pragma unroll
      for (int t = 0; t < kBwdMaxPL; ++t) {
        const int e = lane + 32 * t;
        if (e < p.E) dq[t] = fmaf(ds, sk[jj * p.E + e], dq[t]);
      }
    }
  }
  if (!row_ok) return;
  T* dqp = static_cast<T*>(g.dq) + b * g.dqs[0] + h * g.dqs[1] + (int64_t)i * g.dqs[2];
#pragma unroll
  for (int t = 0; t < kBwdMaxPL; ++t) {
    const int e = lane + 32 * t;
    if (e < p.E) dqp[e] = from_f32<T>(dq[t] * p.scale);
  }
}

template <typename T>
static cudaError_t launch_backward_t(const Params& p, const BwdParams& g, cudaStream_t st) {
  // With no query rows there is only dk = dv = 0 to write; with no keys only
  // dq = 0.
  const int threads = kBwdWarps * 32;
  const size_t smem = (size_t)kBwdTile * (p.E + p.Ev) * sizeof(float);
  if (p.L > 0) bwd_rowdot_kernel<T><<<dim3((p.L + kBwdWarps - 1) / kBwdWarps, p.Hq, p.B), threads, 0, st>>>(p, g);
  if (p.S > 0)
    bwd_dkdv_kernel<T><<<dim3((p.S + kBwdWarps - 1) / kBwdWarps, p.Hkv, p.B), threads, smem, st>>>(p, g);
  if (p.L > 0) bwd_dq_kernel<T><<<dim3((p.L + kBwdWarps - 1) / kBwdWarps, p.Hq, p.B), threads, smem, st>>>(p, g);
  return cudaGetLastError();
}

template <typename T, int LPR>
static void launch_rowdot_vec(const Params& p, const BwdParams& g, cudaStream_t st) {
  constexpr int rows_per_block = kBwdWarps * (32 / LPR);
  bwd_rowdot_vec_kernel<T, LPR>
      <<<dim3((p.L + rows_per_block - 1) / rows_per_block, p.Hq, p.B), kBwdWarps * 32, 0, st>>>(p, g);
}

template <typename T>
static cudaError_t launch_rowdot_t(const Params& p, const BwdParams& g, cudaStream_t st) {
  const bool vec = sizeof(T) == 2 && p.Ev % 8 == 0 && p.os[2] % 8 == 0 && g.dos[2] % 8 == 0 && p.os[1] % 8 == 0 &&
                   g.dos[1] % 8 == 0 && p.os[0] % 8 == 0 && g.dos[0] % 8 == 0 &&
                   (reinterpret_cast<uintptr_t>(p.o) & 15) == 0 && (reinterpret_cast<uintptr_t>(g.dO) & 15) == 0;
  if (vec && p.Ev <= 64) launch_rowdot_vec<T, 8>(p, g, st);
  else if (vec && p.Ev <= 128) launch_rowdot_vec<T, 16>(p, g, st);
  else if (vec) launch_rowdot_vec<T, 32>(p, g, st);
  else bwd_rowdot_kernel<T><<<dim3((p.L + kBwdWarps - 1) / kBwdWarps, p.Hq, p.B), kBwdWarps * 32, 0, st>>>(p, g);
  return cudaGetLastError();
}

cudaError_t launch_backward(const Params& p, const BwdParams& g, int dtype, cudaStream_t st, int* launches) {
  *launches = (p.L > 0 ? 2 : 0) + (p.S > 0 ? 1 : 0);
  switch (dtype) {
    case SDPA_F32: return launch_backward_t<float>(p, g, st);
    case SDPA_F16: return launch_backward_t<__half>(p, g, st);
    default: return launch_backward_t<__nv_bfloat16>(p, g, st);
  }
}

// Only the row dot products D (for the tensor-core backward kernels).
cudaError_t launch_rowdot(const Params& p, const BwdParams& g, int dtype, cudaStream_t st) {
  if (p.L == 0) return cudaSuccess;
  switch (dtype) {
    case SDPA_F32: return launch_rowdot_t<float>(p, g, st);
    case SDPA_F16: return launch_rowdot_t<__half>(p, g, st);
    default: return launch_rowdot_t<__nv_bfloat16>(p, g, st);
  }
}

size_t backward_workspace_bytes(int B, int Hq, int L) {
  return ((size_t)B * Hq * L * sizeof(float) + 255) / 256 * 256;
}

}  // namespace sdpa15
