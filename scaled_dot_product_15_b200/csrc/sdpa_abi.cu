// The extern "C" boundary declared in include/sdpa15.h: argument checks,
// choice of kernel by shape and dtype, and launch on the caller's stream.
// No device memory is allocated here and nothing synchronises.
#include <math.h>
#include <string.h>

#include "backward.cuh"

namespace sdpa15 {
cudaError_t launch_simt(const Params& p, int dtype, cudaStream_t st);
bool decode_supported(const Params& p, int dtype);
cudaError_t launch_decode(const Params& p, int dtype, cudaStream_t st, int* launches);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Ev);
bool prefill_supported(const Params& p, int dtype);
cudaError_t launch_prefill(const Params& p, int dtype, cudaStream_t st);
cudaError_t prefill_take_error(int* code);
cudaError_t launch_backward(const Params& p, const BwdParams& g, int dtype, cudaStream_t st, int* launches);
size_t backward_workspace_bytes(int B, int Hq, int L);
cudaError_t launch_rowdot(const Params& p, const BwdParams& g, int dtype, cudaStream_t st);
bool backward_sm100_supported(const Params& p, const BwdParams& g, int dtype);
cudaError_t launch_backward_sm100(const Params& p, const BwdParams& g, int dtype, cudaStream_t st);
cudaError_t backward_take_error(int* code);
cudaError_t decode_take_error(int* code);
}  // namespace sdpa15

using namespace sdpa15;

namespace {

constexpr int kAbiVersion = 2;
thread_local int t_last_launches = 0;

enum Plan { kPlanPrefill = 1, kPlanDecode = 2, kPlanSimt = 3 };

bool valid_dtype(int d) { return d == SDPA_F32 || d == SDPA_F16 || d == SDPA_BF16; }
bool valid_mask(int m) { return m >= SDPA_MASK_NONE && m <= SDPA_MASK_BOOL; }
bool has_bias(int m) { return m == SDPA_MASK_FLOAT_BIAS || m == SDPA_MASK_BOOL; }

// Checks shapes and strides that do not need device data.  Returns SDPA_OK or
// an error status.
int check_shapes(int B, int Hq, int Hkv, int L, int S, int E, int Ev, const int64_t* qs,
                 const int64_t* ks, const int64_t* vs, const int64_t* os, int mask, int dtype) {
  if (!valid_dtype(dtype) || !valid_mask(mask)) return SDPA_ERR_INVALID;
  if (B < 0 || Hq < 0 || Hkv < 0 || L < 0 || S < 0 || E < 0 || Ev < 0) return SDPA_ERR_INVALID;
  if (Hkv == 0 || Hq == 0 || Hq % Hkv != 0) return SDPA_ERR_INVALID;
  if (B > 65535 || Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  if (E > 256 || Ev == 0 || Ev > 256) return SDPA_ERR_UNSUPPORTED;
  if (!qs || !ks || !vs || !os) return SDPA_ERR_INVALID;
  if (qs[3] != 1 || ks[3] != 1 || vs[3] != 1 || os[3] != 1) return SDPA_ERR_INVALID;
  for (int d = 0; d < 3; ++d)
    if (qs[d] < 0 || ks[d] < 0 || vs[d] < 0 || os[d] < 0) return SDPA_ERR_INVALID;
  if (mask == SDPA_MASK_BLOCK_DIAG || mask == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
    if (B != 1 || L != S) return SDPA_ERR_INVALID;
  }
  return SDPA_OK;
}

void fill_params(Params& p, const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int Hq, int Hkv, int L, int S, int E, int Ev, const int64_t* qs,
                 const int64_t* ks, const int64_t* vs, const int64_t* os, int mask) {
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.S = S; p.E = E; p.Ev = Ev;
  p.group = Hq / Hkv;
  for (int d = 0; d < 4; ++d) { p.qs[d] = qs[d]; p.ks[d] = ks[d]; p.vs[d] = vs[d]; p.os[d] = os[d]; }
  p.mask = mask;
  p.scale = E > 0 ? (float)(1.0 / sqrt((double)E)) : 1.f;  // the default; sdpa_fwd() sets the real one
  p.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
}

int choose_plan(const Params& p, int dtype) {
  if (p.mask == SDPA_MASK_BOOL) return kPlanSimt;  // bool masks run on the general kernels only
  if (dtype != SDPA_F32) {
    if (decode_supported(p, dtype)) return kPlanDecode;
    if (prefill_supported(p, dtype)) return kPlanPrefill;
  }
  return kPlanSimt;
}

bool is_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0;
}

}  // namespace

namespace sdpa15 {
// Kernel launches of this thread's last call (for sdpa_last_launch_count).
void set_last_launches(int n) { t_last_launches = n; }
}  // namespace sdpa15

extern "C" {

int sdpa_abi_version(void) { return kAbiVersion; }

const char* sdpa_status_string(int status) {
  switch (status) {
    case SDPA_OK: return "ok";
    case SDPA_ERR_INVALID: return "invalid argument";
    case SDPA_ERR_UNSUPPORTED: return "unsupported problem or device";
    case SDPA_ERR_CUDA: return "CUDA error";
    case SDPA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int sdpa_last_launch_count(void) { return t_last_launches; }

int sdpa_take_device_error(int* code) {
  if (!code) return SDPA_ERR_INVALID;
  *code = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return SDPA_ERR_CUDA;
  int c1 = 0, c2 = 0, c3 = 0;
  if (prefill_take_error(&c1) != cudaSuccess || backward_take_error(&c2) != cudaSuccess ||
      decode_take_error(&c3) != cudaSuccess)
    return SDPA_ERR_CUDA;
  *code = c1 ? c1 : (c2 ? c2 : c3);
  return SDPA_OK;
}

size_t sdpa_fwd_workspace_size(int B, int Hq, int Hkv, int L, int S, int E, int Ev, int mask_kind,
                               int dtype) {
  const int64_t z[4] = {0, 0, 0, 1};
  if (check_shapes(B, Hq, Hkv, L, S, E, Ev, z, z, z, z, mask_kind, dtype) != SDPA_OK) return 0;
  // Only the decode path uses scratch.  Its eligibility also depends on
  // strides and alignment; the size assumes it may be taken.
  if (dtype == SDPA_F32 || mask_kind != SDPA_MASK_NONE || E != Ev) return 0;
  if (E != 64 && E != 128 && E != 256) return 0;
  if ((Hq / Hkv) * L > 8 || S < 1) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, L, S, Ev);
}

int sdpa_fwd_plan(int B, int Hq, int Hkv, int L, int S, int E, int Ev, const int64_t q_stride[4],
                  const int64_t k_stride[4], const int64_t v_stride[4], const int64_t o_stride[4],
                  int mask_kind, int dtype, const void* q, const void* k, const void* v,
                  const void* out) {
  int st = check_shapes(B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, o_stride, mask_kind, dtype);
  if (st != SDPA_OK) return -st;
  Params p;
  fill_params(p, q, k, v, const_cast<void*>(out), nullptr, B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride,
              v_stride, o_stride, mask_kind);
  return choose_plan(p, dtype);
}

int sdpa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
             int Hkv, int L, int S, int E, int Ev, const int64_t q_stride[4],
             const int64_t k_stride[4], const int64_t v_stride[4], const int64_t o_stride[4],
             int has_scale, float scale, int mask_kind, const int32_t* cu_seqlens, int n_seqs,
             int max_seqlen, const void* bias, const int64_t bias_stride[4], int dtype,
             void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  int st = check_shapes(B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, o_stride, mask_kind, dtype);
  if (st != SDPA_OK) return st;
  if (has_scale && !isfinite(scale)) return SDPA_ERR_INVALID;
  if (B == 0 || L == 0) return SDPA_OK;  // nothing to compute
  // Tensors without elements may have NULL data: q and k when E = 0 (the
  // scores are empty sums), k and v when S = 0 (every row keeps no key).
  if ((E > 0 && !q) || (E > 0 && S > 0 && !k) || (S > 0 && !v) || !out || !lse) return SDPA_ERR_INVALID;
  if (mask_kind == SDPA_MASK_BLOCK_DIAG || mask_kind == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
    if (!cu_seqlens || n_seqs < 1 || max_seqlen < 1) return SDPA_ERR_INVALID;
  }
  if (has_bias(mask_kind)) {
    if (!bias || !bias_stride) return SDPA_ERR_INVALID;
    for (int d = 0; d < 4; ++d)
      if (bias_stride[d] < 0) return SDPA_ERR_INVALID;
  }
  if (!is_sm100()) return SDPA_ERR_UNSUPPORTED;

  Params p;
  fill_params(p, q, k, v, out, lse, B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, o_stride,
              mask_kind);
  p.scale = has_scale ? scale : (E > 0 ? (float)(1.0 / sqrt((double)E)) : 1.f);
  p.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  p.cu = cu_seqlens;
  p.n_seqs = n_seqs;
  p.max_seqlen = max_seqlen;
  if (has_bias(mask_kind)) {
    // BOOL: the byte mask travels in the bias pointer; the kernels read it
    // as bytes when p.mask says so.
    p.bias = static_cast<const float*>(bias);
    for (int d = 0; d < 4; ++d) p.bs[d] = bias_stride[d];
  }
  p.ws = workspace;
  p.ws_bytes = workspace_bytes;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  const int plan = S == 0 ? kPlanSimt : choose_plan(p, dtype);
  cudaError_t err = cudaSuccess;
  int launches = 1;
  if (plan == kPlanDecode) {
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, L, S, Ev);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                     reinterpret_cast<uintptr_t>(workspace) % 256 != 0))
      return SDPA_ERR_WORKSPACE;
    err = launch_decode(p, dtype, cs, &launches);
  } else if (plan == kPlanPrefill) {
    err = launch_prefill(p, dtype, cs);
  } else {
    err = launch_simt(p, dtype, cs);
  }
  if (err != cudaSuccess) return SDPA_ERR_CUDA;
  t_last_launches = launches;
  return SDPA_OK;
}

size_t sdpa_bwd_workspace_size(int B, int Hq, int Hkv, int L, int S, int E, int Ev, int mask_kind,
                               int dtype) {
  const int64_t z[4] = {0, 0, 0, 1};
  if (check_shapes(B, Hq, Hkv, L, S, E, Ev, z, z, z, z, mask_kind, dtype) != SDPA_OK) return 0;
  return backward_workspace_bytes(B, Hq, L);
}

int sdpa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int L, int S,
             int E, int Ev, const int64_t q_stride[4], const int64_t k_stride[4],
             const int64_t v_stride[4], const int64_t o_stride[4], const int64_t do_stride[4],
             const int64_t dq_stride[4], const int64_t dk_stride[4], const int64_t dv_stride[4],
             int has_scale, float scale, int mask_kind, const int32_t* cu_seqlens, int n_seqs,
             int max_seqlen, const void* bias, const int64_t bias_stride[4], int dtype,
             void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  int st = check_shapes(B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, o_stride, mask_kind, dtype);
  if (st != SDPA_OK) return st;
  // The gradients' strides follow the same rules as the forward's tensors.
  st = check_shapes(B, Hq, Hkv, L, S, E, Ev, dq_stride, dk_stride, dv_stride, do_stride, mask_kind, dtype);
  if (st != SDPA_OK) return st;
  if (has_scale && !isfinite(scale)) return SDPA_ERR_INVALID;
  if (B == 0) return SDPA_OK;
  // Tensors without elements may have NULL data (E = 0: q, k, dq, dk;
  // S = 0: k, v, dk, dv; L = 0: q, out, lse, dout, dq).
  const bool rows = L > 0, keys = S > 0, feat = E > 0;
  if ((rows && feat && (!q || !dq)) || (keys && feat && (!k || !dk)) || (keys && (!v || !dv)) ||
      (rows && (!out || !lse || !dout)))
    return SDPA_ERR_INVALID;
  if (mask_kind == SDPA_MASK_BLOCK_DIAG || mask_kind == SDPA_MASK_BLOCK_DIAG_CAUSAL) {
    if (!cu_seqlens || n_seqs < 1 || max_seqlen < 1) return SDPA_ERR_INVALID;
  }
  if (has_bias(mask_kind)) {
    if (!bias || !bias_stride) return SDPA_ERR_INVALID;
    for (int d = 0; d < 4; ++d)
      if (bias_stride[d] < 0) return SDPA_ERR_INVALID;
  }
  const size_t need = backward_workspace_bytes(B, Hq, L);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                   reinterpret_cast<uintptr_t>(workspace) % 256 != 0))
    return SDPA_ERR_WORKSPACE;
  if (!is_sm100()) return SDPA_ERR_UNSUPPORTED;

  Params p;
  fill_params(p, q, k, v, const_cast<void*>(out), const_cast<float*>(lse), B, Hq, Hkv, L, S, E, Ev, q_stride,
              k_stride, v_stride, o_stride, mask_kind);
  p.scale = has_scale ? scale : (E > 0 ? (float)(1.0 / sqrt((double)E)) : 1.f);
  p.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  p.cu = cu_seqlens;
  p.n_seqs = n_seqs;
  p.max_seqlen = max_seqlen;
  if (has_bias(mask_kind)) {
    // BOOL: the byte mask travels in the bias pointer; the kernels read it
    // as bytes when p.mask says so.
    p.bias = static_cast<const float*>(bias);
    for (int d = 0; d < 4; ++d) p.bs[d] = bias_stride[d];
  }
  BwdParams g;
  memset(&g, 0, sizeof(g));
  g.dO = dout;
  g.dq = dq;
  g.dk = dk;
  g.dv = dv;
  for (int d = 0; d < 4; ++d) {
    g.dos[d] = do_stride[d];
    g.dqs[d] = dq_stride[d];
    g.dks[d] = dk_stride[d];
    g.dvs[d] = dv_stride[d];
  }
  g.D = static_cast<float*>(workspace);
  int launches = 0;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (backward_sm100_supported(p, g, dtype)) {
    if (launch_rowdot(p, g, dtype, cs) != cudaSuccess || launch_backward_sm100(p, g, dtype, cs) != cudaSuccess)
      return SDPA_ERR_CUDA;
    launches = 3;
  } else if (launch_backward(p, g, dtype, cs, &launches) != cudaSuccess) {
    return SDPA_ERR_CUDA;
  }
  t_last_launches = launches;
  return SDPA_OK;
}

int sdpa_bwd_plan(int B, int Hq, int Hkv, int L, int S, int E, int Ev, const int64_t q_stride[4],
                  const int64_t k_stride[4], const int64_t v_stride[4], const int64_t do_stride[4],
                  const int64_t dq_stride[4], const int64_t dk_stride[4], const int64_t dv_stride[4],
                  int mask_kind, int dtype, const void* q, const void* k, const void* v, const void* dout,
                  const void* dq, const void* dk, const void* dv) {
  int st = check_shapes(B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, do_stride, mask_kind, dtype);
  if (st == SDPA_OK)
    st = check_shapes(B, Hq, Hkv, L, S, E, Ev, dq_stride, dk_stride, dv_stride, do_stride, mask_kind, dtype);
  if (st != SDPA_OK) return -st;
  Params p;
  fill_params(p, q, k, v, nullptr, nullptr, B, Hq, Hkv, L, S, E, Ev, q_stride, k_stride, v_stride, do_stride,
              mask_kind);
  BwdParams g;
  memset(&g, 0, sizeof(g));
  g.dO = dout;
  g.dq = const_cast<void*>(dq);
  g.dk = const_cast<void*>(dk);
  g.dv = const_cast<void*>(dv);
  for (int d = 0; d < 4; ++d) {
    g.dos[d] = do_stride[d];
    g.dqs[d] = dq_stride[d];
    g.dks[d] = dk_stride[d];
    g.dvs[d] = dv_stride[d];
  }
  return backward_sm100_supported(p, g, dtype) ? kPlanPrefill : kPlanSimt;
}

}  // extern "C"
