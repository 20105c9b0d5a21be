// Host-side helpers for the tensor-memory-accelerator kernels: the driver's
// tensor-map encoder, 4-D maps over (feature, sequence, head, batch) with
// 64 x 128 boxes and 128-byte swizzle, and the alignment rules those maps
// need.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdpa15 {
namespace tmahost {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// A 4-D map of a 16-bit tensor with element strides st = (batch, head, seq).
inline bool make_map(CUtensorMap* m, const void* base, bool bf16, int D, int seq, int H, int B, const int64_t* st) {
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

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

// Byte strides of a 16-bit tensor that a map (and 16-byte row stores) accept.
inline bool strides_ok(const int64_t* st) {
  for (int d = 0; d < 3; ++d)
    if ((st[d] * 2) % 16 != 0 || st[d] * 2 >= (int64_t(1) << 40)) return false;
  return true;
}

}  // namespace tmahost
}  // namespace sdpa15
