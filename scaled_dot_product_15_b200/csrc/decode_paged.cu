// C ABI of decode attention over a paged key/value cache (declared in
// include/sdpa15.h): argument checks, then the split-S decode and combine
// kernels of decode.cu reading keys and values through the block table.
#include <math.h>
#include <string.h>

#include "common.cuh"

namespace sdpa15 {
bool decode_supported(const Params& p, int dtype);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Ev);
cudaError_t launch_decode_paged(const Params& p, const int32_t* table, const int32_t* lens, int max_pages,
                                int num_pages, int page_shift, int dtype, cudaStream_t st, int* launches);
void set_last_launches(int n);
}  // namespace sdpa15

using namespace sdpa15;

namespace {

constexpr int kMaxPageShift = 16;  // page sizes 1 .. 65536 tokens

// log2(page_size) for a power of two in range, else -1.
int page_shift(int page_size) {
  for (int s = 0; s <= kMaxPageShift; ++s)
    if (page_size == (1 << s)) return s;
  return -1;
}

// Checks that need no device data; fills p on success.
int check_paged(const void* q, const void* kp, const void* vp, void* out, float* lse, int B, int Hq, int Hkv, int L,
                int E, int Ev, int num_pages, int page_size, int max_pages, const int64_t* qs, const int64_t* ks,
                const int64_t* vs, const int64_t* os, int has_scale, float scale, int dtype, Params& p) {
  if (dtype != SDPA_F32 && dtype != SDPA_F16 && dtype != SDPA_BF16) return SDPA_ERR_INVALID;
  if (B < 0 || Hq < 1 || Hkv < 1 || L < 0 || E < 1 || Ev < 1 || num_pages < 1 || page_size < 1 || max_pages < 1)
    return SDPA_ERR_INVALID;
  if (Hq % Hkv != 0) return SDPA_ERR_INVALID;
  if (!qs || !ks || !vs || !os) return SDPA_ERR_INVALID;
  const int64_t* st[4] = {qs, ks, vs, os};
  for (int t = 0; t < 4; ++t) {
    if (st[t][3] != 1) return SDPA_ERR_INVALID;
    for (int d = 0; d < 3; ++d)
      if (st[t][d] < 0) return SDPA_ERR_INVALID;
  }
  if (has_scale && !isfinite(scale)) return SDPA_ERR_INVALID;
  const int shift = page_shift(page_size);
  if (shift < 0) return SDPA_ERR_UNSUPPORTED;
  // At most 2^20 tokens per row keeps every key chunk within 1024 keys (the
  // split kernel's page list holds a chunk's pages).
  if ((int64_t)max_pages * page_size > (1 << 20)) return SDPA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = kp; p.v = vp; p.o = out; p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.E = E; p.Ev = Ev;
  p.S = max_pages * page_size;
  p.group = Hq / Hkv;
  for (int d = 0; d < 4; ++d) { p.qs[d] = qs[d]; p.ks[d] = ks[d]; p.vs[d] = vs[d]; p.os[d] = os[d]; }
  p.mask = SDPA_MASK_NONE;
  p.scale = has_scale ? scale : (float)(1.0 / sqrt((double)E));
  p.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  // The decode kernel's own conditions (16-bit, E = Ev in {64, 128, 256},
  // (Hq/Hkv) * L <= 8, 16-byte aligned rows); the pools' page stride counts
  // as their batch stride.
  if (!decode_supported(p, dtype)) return SDPA_ERR_UNSUPPORTED;
  return SDPA_OK;
}

}  // namespace

extern "C" {

size_t sdpa_decode_paged_workspace_size(int B, int Hq, int Hkv, int L, int E, int Ev, int page_size, int max_pages,
                                        int dtype) {
  if (dtype != SDPA_F16 && dtype != SDPA_BF16) return 0;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || L < 1 || E != Ev) return 0;
  if (E != 64 && E != 128 && E != 256) return 0;
  if ((Hq / Hkv) * L > 8 || page_shift(page_size) < 0 || max_pages < 1) return 0;
  if ((int64_t)max_pages * page_size > (1 << 20)) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, L, max_pages * page_size, Ev);
}

int sdpa_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int L, int E, int Ev,
                      int num_pages, int page_size, int max_pages, const int64_t q_stride[4],
                      const int64_t kp_stride[4], const int64_t vp_stride[4], const int64_t o_stride[4],
                      int has_scale, float scale, int dtype, void* workspace, size_t workspace_bytes,
                      void* stream) {
  set_last_launches(0);
  Params p;
  int st = check_paged(q, k_pages, v_pages, out, lse, B, Hq, Hkv, L, E, Ev, num_pages, page_size, max_pages,
                       q_stride, kp_stride, vp_stride, o_stride, has_scale, scale, dtype, p);
  if (st != SDPA_OK) return st;
  if (B == 0 || L == 0) return SDPA_OK;
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out || !lse) return SDPA_ERR_INVALID;
  const size_t need = decode_workspace_bytes(B, Hq, Hkv, L, p.S, Ev);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256 != 0))
    return SDPA_ERR_WORKSPACE;
  // No usable device, or not an sm_100 one: unsupported (as for sdpa_fwd()).
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SDPA_ERR_UNSUPPORTED;
  if (major != 10 || minor != 0) return SDPA_ERR_UNSUPPORTED;
  p.ws = workspace;
  p.ws_bytes = workspace_bytes;
  int launches = 0;
  if (launch_decode_paged(p, block_table, seq_lens, max_pages, num_pages, page_shift(page_size), dtype,
                          static_cast<cudaStream_t>(stream), &launches) != cudaSuccess)
    return SDPA_ERR_CUDA;
  set_last_launches(launches);
  return SDPA_OK;
}

}  // extern "C"
