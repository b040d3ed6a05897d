// Host side of the tensor-core backward: d = 128 (tc_bwd_kernels.cuh) and
// d = 64 with 64-token segments (tc_bwd64_kernels.cuh); included after
// tc_kernels.cuh, whose tensor maps, epochs and constants it uses.
#pragma once

#include "tc_kernels.cuh"
#include "tc_bwd64_kernels.cuh"

namespace infini {

// The tensor-core backward's launches after the statistics pass (tc_forward
// with bwd set), tc_bwd_kernels.cuh: kv = false launches the dQ kernel (dq,
// and each segment's sigma(Q)^T dnum, sigma(Q)^T dden added into the zeroed
// G, Gz); kv = true, after the reverse scan has made G_s, Gz_s of those, the
// dK/dV kernel. bf16 I/O, d = 128, seg_len % 128 == 0.
struct TcBwdArgs {
  int64_t B, H, L, N, S;
  const void *q, *k, *v, *dout;
  const __nv_bfloat16 *dnum16, *Mp;
  const float *beta, *zp, *lse, *delta, *dden;
  float *G, *Gz;
  float *dq, *dk, *dv;
};

// A [rows, cols] fp32 row-major matrix (cols 128 or 64) stored through
// 32-column x 128-row boxes in the 128-byte swizzle (the backward kernels'
// output tiles).
inline bool make_map_f32_out(CUtensorMap* m, void* base, int64_t rows, int cols = tc::kD) {
  auto enc = tc::tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)tc::kTile};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

inline int tc_backward_local(const TcBwdArgs& a, cudaStream_t st, bool kv) {
  using namespace tc;
  const int64_t BH = a.B * a.H, rows = BH * a.L, n_segs = BH * a.S;
  const int n_qt = (int)(a.N / kTile);
  const int64_t units = n_segs * n_qt;
  if (units >= (int64_t(1) << 31)) return INFINI_ERR_SIZE;
  CUtensorMap mq, mo, mk, mv, mn, mm;
  if (!make_map(&mq, a.q, rows) || !make_map(&mo, a.dout, rows) || !make_map(&mk, a.k, rows) ||
      !make_map(&mv, a.v, rows) || !make_map(&mn, a.dnum16, rows) || !make_map(&mm, a.Mp, n_segs * kD))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDqSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kKvSmem) !=
          cudaSuccess)
    return INFINI_ERR_CUDA;
  const uint32_t epoch = next_epoch();
  const int L = (int)a.L, N = (int)a.N, S = (int)a.S, H = (int)a.H;
  if (!kv) {
    // G as [n_segs * d rows (segment, d_k), d columns d_v]: each CTA adds its
    // 128 x 128 share by a TMA reduce-add at row seg * d (an int32 coordinate).
    if (rows >= (int64_t(1) << 31) || n_segs * kD >= (int64_t(1) << 31)) return INFINI_ERR_SIZE;
    CUtensorMap mdq, mg;
    if (!make_map_f32_out(&mdq, a.dq, rows) || !make_map_f32_out(&mg, a.G, n_segs * kD)) return INFINI_ERR_CUDA;
    tc_bwd_dq_kernel<<<(unsigned)units, kBwdTcThreads, kDqSmem, st>>>(mq, mo, mk, mv, mn, mm, mdq, mg, a.beta, a.zp,
                                                                       a.lse, a.delta, a.dden, a.Gz, L, N, S, H,
                                                                       (int)n_segs, epoch);
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
  }
  CUtensorMap mdk, mdv;
  if (!make_map_f32_out(&mdk, a.dk, rows) || !make_map_f32_out(&mdv, a.dv, rows)) return INFINI_ERR_CUDA;
  tc_bwd_kv_kernel<<<(unsigned)units, kBwdTcThreads, kKvSmem, st>>>(mq, mo, mk, mv, mdk, mdv, a.beta, a.lse, a.delta,
                                                                     a.G, a.Gz, L, N, S, H, (int)n_segs, epoch);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

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
  if (state_terms) {  // 64-row boxes: each segment's rows land in their diagonal block
    CUtensorMap mdk, mdv;
    if (!make_map(&mk, a.k, rows, 64, kD64) || !make_map(&mv, a.v, rows, 64, kD64) ||
        !make_map_f32_out(&mdk, a.dk, rows, kD64) || !make_map_f32_out(&mdv, a.dv, rows, kD64))
      return INFINI_ERR_CUDA;
    if (cudaFuncSetAttribute(tc_bwd64_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kB64StateSmem) != cudaSuccess)
      return INFINI_ERR_CUDA;
    tc_bwd64_state_kernel<<<(unsigned)pairs, kB64Threads, kB64StateSmem, st>>>(mk, mv, mdk, mdv, a.G, a.Gz, L, S,
                                                                                epoch);
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
  }
  if (!make_map(&mk, a.k, rows, 128, kD64) || !make_map(&mv, a.v, rows, 128, kD64)) return INFINI_ERR_CUDA;
  CUtensorMap mq, mo, mm128, mm64, mdq, mdk, mdv, mg;
  if (!make_map(&mq, a.q, rows, 128, kD64) || !make_map(&mo, a.dout, rows, 128, kD64) ||
      !make_map(&mm128, a.Mp, BH * a.S * kD64, 128, kD64) || !make_map(&mm64, a.Mp, BH * a.S * kD64, 64, kD64))
    return INFINI_ERR_CUDA;
  // fp32 outputs: dq, dk, dv [B*H*L, 64] and G as [B*H*S*64 rows (segment, d_k), 64 columns d_v].
  if (!make_map_f32_out(&mdq, a.dq, rows, kD64) || !make_map_f32_out(&mdk, a.dk, rows, kD64) ||
      !make_map_f32_out(&mdv, a.dv, rows, kD64) || !make_map_f32_out(&mg, a.G, BH * a.S * kD64, kD64))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_bwd64_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kB64Smem) !=
      cudaSuccess)
    return INFINI_ERR_CUDA;
  tc_bwd64_pair_kernel<<<(unsigned)pairs, kB64Threads, kB64Smem, st>>>(mq, mk, mv, mo, mm128, mm64, mdq, mdk, mdv,
                                                                        mg, a.beta, a.zp, a.Gz, a.dbeta, L, S, H,
                                                                        sm_count(), epoch);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

}  // namespace infini
