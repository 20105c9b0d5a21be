// General SIMT attention kernel: every dtype (float32 included, which the
// tensor cores cannot take at float32 accuracy), every mask kind, any head
// size up to 256 and any strides.  One warp owns one query row and keeps its
// running maximum, running sum and output accumulator in fp32 registers while
// the block streams key/value tiles through shared memory (the online-softmax
// recurrence of the khchao.com NN-lab page, "FlashAttention Tiling & Online
// Softmax Algorithm", one key at a time).
//
// Special values follow the exactref "Full specification": a NaN logit makes
// the row NaN, a +inf logit makes it NaN with lse +inf, a row with no finite
// logit gets output 0 and lse -inf.  Removed keys (masked out or -inf bias)
// are skipped, so a non-finite value stored under a removed key does not reach
// the output.
#include "common.cuh"

namespace sdpa15 {

constexpr int kSimtRows = 8;    // warps (query rows) per block
constexpr int kSimtKeys = 16;   // keys per shared-memory tile
constexpr int kSimtMaxPL = 8;   // features per lane: head sizes up to 256

template <typename T>
__global__ void __launch_bounds__(kSimtRows * 32)
simt_attention_kernel(Params p) {
  extern __shared__ float smem[];
  float* sk = smem;                       // [kSimtKeys][E]
  float* sv = smem + kSimtKeys * p.E;     // [kSimtKeys][Ev]
  __shared__ int s_lo[kSimtRows], s_hi[kSimtRows];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int kvh = h / p.group;
  const int i = blockIdx.x * kSimtRows + warp;  // query row of this warp
  const bool row_ok = i < p.L;

  // Key range of this row.
  int lo = 0, hi = p.S;
  if (row_ok) {
    if (p.mask == SDPA_MASK_CAUSAL) {
      hi = min(p.S, i + 1);
    } else if (p.mask == SDPA_MASK_BLOCK_DIAG || p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
      int sgi = segment_of(p.cu, p.n_seqs, i);
      lo = max(0, min(p.S, __ldg(p.cu + sgi)));
      hi = max(lo, min(p.S, __ldg(p.cu + sgi + 1)));
      if (p.mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) hi = max(lo, min(hi, i + 1));
    }
  } else {
    lo = p.S;
    hi = 0;
  }
  if (lane == 0) { s_lo[warp] = lo; s_hi[warp] = hi; }
  __syncthreads();
  int blo = p.S, bhi = 0;
#pragma unroll
  for (int w = 0; w < kSimtRows; ++w) { blo = min(blo, s_lo[w]); bhi = max(bhi, s_hi[w]); }

  const T* qp = static_cast<const T*>(p.q) + b * p.qs[0] + h * p.qs[1] + (int64_t)(row_ok ? i : 0) * p.qs[2];
  const T* kp = static_cast<const T*>(p.k) + b * p.ks[0] + kvh * p.ks[1];
  const T* vp = static_cast<const T*>(p.v) + b * p.vs[0] + kvh * p.vs[1];

  float qr[kSimtMaxPL];
#pragma unroll
  for (int t = 0; t < kSimtMaxPL; ++t) {
    int e = lane + 32 * t;
    qr[t] = (row_ok && e < p.E) ? to_f32<T>(qp[e]) : 0.f;
  }
  float acc[kSimtMaxPL];
#pragma unroll
  for (int t = 0; t < kSimtMaxPL; ++t) acc[t] = 0.f;
  float m = -INFINITY, lsum = 0.f;
  bool bad_nan = false, bad_pinf = false;

  // FLOAT_BIAS: float32 bias; BOOL: bytes (nonzero = visible) in the same
  // pointer, applied as a 0 / -inf bias.
  const float* biasp = nullptr;
  const unsigned char* boolp = nullptr;
  if (p.mask == SDPA_MASK_FLOAT_BIAS && row_ok)
    biasp = p.bias + b * p.bs[0] + h * p.bs[1] + (int64_t)i * p.bs[2];
  if (p.mask == SDPA_MASK_BOOL && row_ok)
    boolp = reinterpret_cast<const unsigned char*>(p.bias) + b * p.bs[0] + h * p.bs[1] + (int64_t)i * p.bs[2];

  for (int j0 = blo; j0 < bhi; j0 += kSimtKeys) {
    const int nk = min(kSimtKeys, bhi - j0);
    __syncthreads();  // previous tile consumed
    for (int idx = threadIdx.x; idx < nk * p.E; idx += blockDim.x) {
      int jj = idx / p.E, e = idx - jj * p.E;
      sk[jj * p.E + e] = to_f32<T>(kp[(int64_t)(j0 + jj) * p.ks[2] + e]);
    }
    for (int idx = threadIdx.x; idx < nk * p.Ev; idx += blockDim.x) {
      int jj = idx / p.Ev, e = idx - jj * p.Ev;
      sv[jj * p.Ev + e] = to_f32<T>(vp[(int64_t)(j0 + jj) * p.vs[2] + e]);
    }
    __syncthreads();
    for (int jj = 0; jj < nk; ++jj) {
      const int j = j0 + jj;
      if (j < lo || j >= hi) continue;  // warp-uniform
      float dot = 0.f;
#pragma unroll
      for (int t = 0; t < kSimtMaxPL; ++t) {
        int e = lane + 32 * t;
        if (e < p.E) dot = fmaf(qr[t], sk[jj * p.E + e], dot);
      }
      dot = warp_sum(dot);
      float logit = (p.E == 0) ? 0.f : dot * p.scale;
      if (biasp) logit = logit + __ldg(biasp + (int64_t)j * p.bs[3]);
      if (boolp) logit = logit + (__ldg(boolp + (int64_t)j * p.bs[3]) ? 0.f : -INFINITY);
      if (isnan(logit)) { bad_nan = true; continue; }
      if (logit == INFINITY) { bad_pinf = true; continue; }
      if (logit == -INFINITY) continue;  // removed key: weight 0
      if (logit > m) {
        const float corr = (m == -INFINITY) ? 0.f : expf(m - logit);
        lsum *= corr;
#pragma unroll
        for (int t = 0; t < kSimtMaxPL; ++t) acc[t] *= corr;
        m = logit;
      }
      const float pj = expf(logit - m);
      lsum += pj;
#pragma unroll
      for (int t = 0; t < kSimtMaxPL; ++t) {
        int e = lane + 32 * t;
        if (e < p.Ev) acc[t] = fmaf(pj, sv[jj * p.Ev + e], acc[t]);
      }
    }
  }

  if (!row_ok) return;
  T* op = static_cast<T*>(p.o) + b * p.os[0] + h * p.os[1] + (int64_t)i * p.os[2];
  float lse;
  if (bad_nan || bad_pinf) {
    lse = bad_nan ? NAN : INFINITY;
#pragma unroll
    for (int t = 0; t < kSimtMaxPL; ++t) acc[t] = NAN;
  } else if (m == -INFINITY) {
    lse = -INFINITY;
#pragma unroll
    for (int t = 0; t < kSimtMaxPL; ++t) acc[t] = 0.f;
  } else {
    lse = m + logf(lsum);
    const float inv = 1.f / lsum;
#pragma unroll
    for (int t = 0; t < kSimtMaxPL; ++t) acc[t] *= inv;
  }
#pragma unroll
  for (int t = 0; t < kSimtMaxPL; ++t) {
    int e = lane + 32 * t;
    if (e < p.Ev) op[e] = from_f32<T>(acc[t]);
  }
  if (lane == 0) p.lse[((int64_t)b * p.Hq + h) * p.L + i] = lse;
}

template <typename T>
static cudaError_t launch_simt_t(const Params& p, cudaStream_t st) {
  dim3 grid((p.L + kSimtRows - 1) / kSimtRows, p.Hq, p.B);
  size_t smem = (size_t)kSimtKeys * (p.E + p.Ev) * sizeof(float);
  simt_attention_kernel<T><<<grid, kSimtRows * 32, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_simt(const Params& p, int dtype, cudaStream_t st) {
  switch (dtype) {
    case SDPA_F32: return launch_simt_t<float>(p, st);
    case SDPA_F16: return launch_simt_t<__half>(p, st);
    default: return launch_simt_t<__nv_bfloat16>(p, st);
  }
}

}  // namespace sdpa15
