// Tensor-core (tcgen05 / TMEM / TMA) path of the Infini-attention forward.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/infini_attn.h"
#include "common.cuh"

namespace infini {

// Set once the tensor-core kernels are in place.
constexpr bool kTcPathBuilt = false;

struct TcArgs {
  int64_t B, H, L, N, S;
  const void *q, *k, *v;
  const float* beta;
  const float *M_in, *z_in;
  void* out;
  float *M_out, *z_out;
  float *dM, *dz;
  __nv_bfloat16* Mp;
  float* zp;
};

inline int tc_launch_count() { return 3; }

inline int tc_forward(const TcArgs&, cudaStream_t, const Trace&) { return INFINI_ERR_UNSUPPORTED; }

}  // namespace infini
