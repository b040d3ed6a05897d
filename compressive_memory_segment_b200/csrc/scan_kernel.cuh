// Cross-segment exclusive prefix of the memory state (fp32, HBM-bound).
//
// For every (b, h) and every element e of the D x D matrix M and the D-vector z:
//   Mp[s][e] = M_in[e] + sum_{j < s} dM[j][e]      (the M_{s-1} each segment reads)
//   M_out[e] = M_in[e] + sum_{j < S} dM[j][e]
// and likewise for z. The sum runs over s in order, in fp32, one element per
// lane, so the result does not depend on the launch shape. This is the
// "Memory Update" / "State Transfer" chain of "Hugging Face Infini-Attention
// reproduction analysis" (Infini-Attention mechanism) computed for all segments
// at once from the per-segment increments instead of walking the segments.
//
// Each thread owns 4 consecutive elements (16-byte loads) and keeps kUnroll
// segments' loads in flight. M_out may be M_in (in place): each element is read
// before it is written, by the same thread.
#pragma once

#include "common.cuh"

namespace infini {

constexpr int kScanThreads = 256;
constexpr int kScanUnroll = 8;

template <typename TM>
__device__ __forceinline__ void store4(TM* p, float4 x);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 x) {
  *reinterpret_cast<float4*>(p) = x;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 x) {
  __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// One flat index space over (bh, part, element/4): part 0 = M (D*D), part 1 = z (D).
// TM: element type of Mp (fp32 for the CUDA-core path, bf16 for the tensor-core
// path, whose retrieval MMA takes bf16 operands). zp is always fp32.
template <typename TM>
__global__ void __launch_bounds__(kScanThreads)
scan_state_kernel(const float* __restrict__ dM, const float* __restrict__ dz,
                  const float* M_in, const float* z_in, TM* __restrict__ Mp,
                  float* __restrict__ zp, float* M_out, float* z_out, int64_t BH, int S, int D) {
  const int64_t per_bh = ((int64_t)D * D + D) / 4;
  const int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= BH * per_bh) return;
  const int64_t bh = f / per_bh;
  const int64_t r = f % per_bh;
  const bool is_m = r < (int64_t)D * D / 4;
  const int64_t e = is_m ? r * 4 : (r - (int64_t)D * D / 4) * 4;  // element within M or z
  const int64_t width = is_m ? (int64_t)D * D : D;                 // stride between segments
  const float* src = (is_m ? dM : dz) + bh * S * width + e;
  const float* init = is_m ? M_in : z_in;
  float* fin = (is_m ? M_out : z_out) + bh * width + e;

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (init != nullptr) acc = *reinterpret_cast<const float4*>(init + bh * width + e);

  int s = 0;
  for (; s + kScanUnroll <= S; s += kScanUnroll) {
    float4 x[kScanUnroll];
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u)
      x[u] = __ldcs(reinterpret_cast<const float4*>(src + (int64_t)(s + u) * width));
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u) {
      const int64_t o = (bh * S + s + u) * width + e;
      if (!INFINI_CHECK(o + 4 <= BH * S * width)) continue;
      if (is_m) store4<TM>(Mp + o, acc); else store4<float>(zp + o, acc);
      acc.x += x[u].x; acc.y += x[u].y; acc.z += x[u].z; acc.w += x[u].w;
    }
  }
  for (; s < S; ++s) {
    const float4 x = __ldcs(reinterpret_cast<const float4*>(src + (int64_t)s * width));
    const int64_t o = (bh * S + s) * width + e;
    if (is_m) store4<TM>(Mp + o, acc); else store4<float>(zp + o, acc);
    acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
  }
  *reinterpret_cast<float4*>(fin) = acc;
}

// Sequence split over P parts (e.g. one block of consecutive segments per
// GPU): part p's incoming state is the caller's state plus the totals of the
// parts before it, off[e] = base[e] + sum_{r < part} totals[r][e], added in
// part order. The same exclusive prefix the scan above takes over segments,
// taken over parts.
__global__ void __launch_bounds__(kScanThreads)
exscan_parts_kernel(const float* __restrict__ totals, int64_t n, int part, const float* __restrict__ base,
                    float* __restrict__ off) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float acc = base ? base[e] : 0.f;
    for (int r = 0; r < part; ++r) acc += totals[(int64_t)r * n + e];
    off[e] = acc;
  }
}

}  // namespace infini
