// Arguments of the backward kernels beyond the forward's Params.
#pragma once

#include "common.cuh"

namespace sdpa15 {

// The extra arguments of one sdpa_bwd() call: the output gradient, the three
// input gradients (element strides batch, head, seq, feature) and the row
// dot products D_i = grad_i . O_i in the workspace (float32, B x Hq x L).
struct BwdParams {
  const void* dO;
  int64_t dos[4];
  void* dq;
  int64_t dqs[4];
  void* dk;
  int64_t dks[4];
  void* dv;
  int64_t dvs[4];
  float* D;
};

}  // namespace sdpa15
