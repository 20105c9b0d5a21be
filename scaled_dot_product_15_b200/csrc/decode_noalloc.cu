// Allocation-free entry point for decode attention.
//
// sdpa_fwd() asks its caller for a workspace: the split-S decode kernel keeps
// each key chunk's partial output and logsumexp there before the combine
// kernel merges them.  Some callers cannot provide one, because they cannot
// allocate device memory when the call is made: a runtime that reserves all
// of its device memory up front and forbids later allocations, or a plugin
// interface that hands over only the input and output buffers.  For them,
// sdpa_decode_fwd_noalloc() runs the same two decode kernels with their
// scratch in a fixed array compiled into this library.
//
// That array (SDPA_NOALLOC_SCRATCH_BYTES, 32 MiB) is a file-scope __device__
// variable: every GPU on which this library's code is loaded holds it until
// the process exits, whether or not the entry point is ever called.  Host
// code cannot use the array's name as a device address, so the first call on
// each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; make that first call before any stream
// capture.  All calls share the one array, and the split kernel writes every
// element the combine kernel reads, so nothing needs clearing between calls;
// calls whose kernels overlap on the GPU (different streams, or different
// host threads) race on the array and must be serialised by the caller.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"

namespace sdpa15 {
bool decode_supported(const Params& p, int dtype);
cudaError_t launch_decode(const Params& p, int dtype, cudaStream_t st, int* launches);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Ev);
}  // namespace sdpa15

static __device__ __align__(256) unsigned char g_decode_scratch[SDPA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device).
cudaError_t scratch_address(int dev, void** addr) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* a = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&a, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = a;
  }
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int sdpa_decode_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                                       int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                                       const int64_t q_stride[4], const int64_t k_stride[4],
                                       const int64_t v_stride[4], const int64_t o_stride[4], int has_scale,
                                       float scale, int dtype, void* stream) {
  using namespace sdpa15;
  if (dtype != SDPA_F32 && dtype != SDPA_F16 && dtype != SDPA_BF16) return SDPA_ERR_INVALID;
  if (B < 0 || Hq < 1 || Hkv < 1 || L < 0 || S < 0 || E < 1 || Ev < 1) return SDPA_ERR_INVALID;
  if (Hq % Hkv != 0) return SDPA_ERR_INVALID;
  if (!q_stride || !k_stride || !v_stride || !o_stride) return SDPA_ERR_INVALID;
  const int64_t* st[4] = {q_stride, k_stride, v_stride, o_stride};
  for (int t = 0; t < 4; ++t) {
    if (st[t][3] != 1) return SDPA_ERR_INVALID;
    for (int d = 0; d < 3; ++d)
      if (st[t][d] < 0) return SDPA_ERR_INVALID;
  }
  if (has_scale && !isfinite(scale)) return SDPA_ERR_INVALID;
  if (B > 65535 || Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  if (B == 0 || L == 0) return SDPA_OK;
  if (!q || !k || !v || !out || !lse) return SDPA_ERR_INVALID;

  Params p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.S = S; p.E = E; p.Ev = Ev;
  p.group = Hq / Hkv;
  for (int d = 0; d < 4; ++d) {
    p.qs[d] = q_stride[d]; p.ks[d] = k_stride[d]; p.vs[d] = v_stride[d]; p.os[d] = o_stride[d];
  }
  p.mask = SDPA_MASK_NONE;
  p.scale = has_scale ? scale : (float)(1.0 / sqrt((double)E));
  p.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  // Only problems the split-S decode kernel takes (16-bit, no mask,
  // E = Ev in {64, 128, 256}, at most 8 query rows per key/value head).
  if (!decode_supported(p, dtype)) return SDPA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, Hq, Hkv, L, S, Ev);
  if (need > (size_t)SDPA_NOALLOC_SCRATCH_BYTES) return SDPA_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SDPA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SDPA_ERR_CUDA;
  if (major != 10 || minor != 0) return SDPA_ERR_UNSUPPORTED;
  if (dev < 0 || dev >= kMaxDevices) return SDPA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return SDPA_ERR_CUDA;
  p.ws = scratch;
  p.ws_bytes = SDPA_NOALLOC_SCRATCH_BYTES;
  int launches = 0;
  if (launch_decode(p, dtype, static_cast<cudaStream_t>(stream), &launches) != cudaSuccess) return SDPA_ERR_CUDA;
  return SDPA_OK;
}
