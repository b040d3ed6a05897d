// Shared device helpers for the Infini-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infini {

// Device status word: bit 0 = a bounded wait gave up. Read and cleared by
// infini_attn_device_status(). The library is one translation unit, so the
// word is defined here.
__device__ unsigned int g_status = 0u;
constexpr unsigned int kStatusTimeout = 1u;

// Abort word for bounded waits: the host gives every call a fresh nonzero
// epoch; a wait that gives up stores the call's epoch here, and every other
// wait of the same call sees it and returns at once, so one stuck CTA does not
// make each later CTA wait out its own deadline. Stale values from earlier
// calls never match the current epoch.
__device__ unsigned int g_abort_epoch = 0u;

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_status, kStatusTimeout); }

// Optional event trace of a forward call: events[i] is recorded on the stream
// after launch i (events[0] before the first launch). Host side only.
struct Trace {
  void* const* events;
  int n;
  bool mark(int i, cudaStream_t st) const {
    if (events == nullptr || i >= n) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
  }
};

// Load one I/O element as fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// sigma(x) = ELU(x) + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise.
__device__ __forceinline__ float elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float elu1_accurate(float x) { return x > 0.f ? x + 1.f : expf(x); }

// g = sigmoid(beta); beta = +inf -> 1, -inf -> 0 under IEEE arithmetic.
__device__ __forceinline__ float gate_of(float beta) { return 1.f / (1.f + expf(-beta)); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace infini
