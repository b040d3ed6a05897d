// Host side of the tensor-core backward for d = 64 with 64-token segments
// (tc_bwd64_kernels.cuh); included after tc_kernels.cuh, whose tensor maps,
// epochs and d = 64 constants it uses.
#pragma once

#include "tc_kernels.cuh"
#include "tc_bwd64_kernels.cuh"

namespace infini {

// The tensor-core backward for d = 64 with 64-token segments, an even number
// per sequence (tc_bwd64_kernels.cuh): the state recompute (tc_forward64's
// state-only path writes M_{s-1} in bf16 and z_{s-1}), then the pair kernel
// (dq, the local dk and dv, each segment's G and Gz, dbeta), the reverse scan
// over segments (bwd_rscan_kernel, by the caller between rscan = false and
// rscan = true), and the state kernel (dk, dv += the state terms).
struct TcBwd64Args {
  int64_t B, H, L, S;
  const void *q, *k, *v, *dout;
  const __nv_bfloat16* Mp;
  const float *beta, *zp;
  float *G, *Gz, *dq, *dk, *dv, *dbeta;
};

inline int tc_backward64(const TcBwd64Args& a, cudaStream_t st, bool state_terms) {
  using namespace tc;
  const int64_t BH = a.B * a.H, rows = BH * a.L;
  const int64_t pairs = BH * (a.S / 2);
  if (pairs >= (int64_t(1) << 31) || rows >= (int64_t(1) << 31)) return INFINI_ERR_SIZE;
  const uint32_t epoch = next_epoch();
  const int L = (int)a.L, S = (int)a.S, H = (int)a.H;
  CUtensorMap mk, mv;
  if (!make_map(&mk, a.k, rows, 128, kD64) || !make_map(&mv, a.v, rows, 128, kD64)) return INFINI_ERR_CUDA;
  if (state_terms) {
    if (cudaFuncSetAttribute(tc_bwd64_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kB64StateSmem) != cudaSuccess)
      return INFINI_ERR_CUDA;
    tc_bwd64_state_kernel<<<(unsigned)pairs, kB64Threads, kB64StateSmem, st>>>(mk, mv, a.G, a.Gz, a.dk, a.dv, L, S,
                                                                                epoch);
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
  }
  CUtensorMap mq, mo, mm128, mm64;
  if (!make_map(&mq, a.q, rows, 128, kD64) || !make_map(&mo, a.dout, rows, 128, kD64) ||
      !make_map(&mm128, a.Mp, BH * a.S * kD64, 128, kD64) || !make_map(&mm64, a.Mp, BH * a.S * kD64, 64, kD64))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_bwd64_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kB64Smem) !=
      cudaSuccess)
    return INFINI_ERR_CUDA;
  tc_bwd64_pair_kernel<<<(unsigned)pairs, kB64Threads, kB64Smem, st>>>(mq, mk, mv, mo, mm128, mm64, a.beta, a.zp,
                                                                        a.dq, a.dk, a.dv, a.G, a.Gz, a.dbeta, L, S, H,
                                                                        epoch);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

}  // namespace infini
