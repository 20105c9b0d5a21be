// Shared definitions of the CUDA side: launch parameters, element access and
// small device helpers.  Included by every kernel translation unit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sdpa15.h"

namespace sdpa15 {

// Everything a kernel needs about one sdpa_fwd() call, by value.
struct Params {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, Hq, Hkv, L, S, E, Ev;
  int group;  // Hq / Hkv: query heads per key/value head (contiguous grouping)
  int64_t qs[4], ks[4], vs[4], os[4];  // element strides (batch, head, seq, feature)
  float scale;       // factor on the raw dot products
  float scale_log2;  // scale * log2(e): logits in base-2 units
  int mask;          // sdpa_mask_kind
  const int32_t* cu;  // block-diagonal segment starts (device), n_seqs + 1 entries
  int n_seqs;
  int max_seqlen;
  const float* bias;  // FLOAT_BIAS: float32 bias with element strides bs
  int64_t bs[4];
  void* ws;  // workspace
  size_t ws_bytes;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Segment of packed token i: the last s with cu[s] <= i, found by bisection,
// clamped so a malformed cu_seqlens array can never index out of range.
__device__ __forceinline__ int segment_of(const int32_t* cu, int n_seqs, int i) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

}  // namespace sdpa15
