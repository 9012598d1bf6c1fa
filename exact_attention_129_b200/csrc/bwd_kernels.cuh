// bwd_kernels.cuh -- backward pass (placeholder until the kernels land).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "attn.h"

namespace attn {

struct BwdArgs {
  const void *q, *k, *v, *out, *dout;
  const float* lse;
  const int32_t *cu_q, *cu_k;
  int batch, total_q, total_k, max_q, max_k, hq, hkv, d;
  float scale;
  bool causal;
  void *dq, *dk, *dv, *workspace;
  uint32_t* err;
  uint64_t timeout_ns;
};

inline size_t bwd_workspace_bytes(int batch, int total_q, int hq, int d) {
  (void)batch; (void)total_q; (void)hq; (void)d;
  return 256;
}

inline attn_status_t bwd_launch(const BwdArgs&, cudaStream_t) { return ATTN_ERR_UNSUPPORTED; }

}  // namespace attn
