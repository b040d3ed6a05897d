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

// ROWS rows of a [*, D] tensor (rows tok_row0 .. ; rows >= valid read as
// zero) moved into shared memory as fp32 at row stride ST in two steps:
// issue() starts every 16-byte load of the calling thread (into registers),
// store() converts and writes them. A loop can put the work on the previous
// tile between the two, so the loads overlap it. NT threads take part.
template <typename T, int D, int ST, int ROWS, int NT>
struct RowTile {
  static constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte vector
  static constexpr int VPR = D / VE;              // vectors per row
  static_assert((ROWS * VPR) % NT == 0, "tile vectors per thread");
  static_assert(ST % 4 == 0, "16-byte aligned shared-memory rows");
  static constexpr int PER = ROWS * VPR / NT;
  uint4 r[PER];

  __device__ __forceinline__ void issue(const T* __restrict__ a, int64_t tok_row0, int valid, int tid) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int vec = tid + u * NT, row = vec / VPR, cv = vec % VPR;
      r[u] = row < valid ? *reinterpret_cast<const uint4*>(a + (tok_row0 + row) * D + cv * VE)
                         : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ __forceinline__ static void put(const uint4& x, float* d) {
    if constexpr (VE == 8) {  // bf16: the high half of an fp32 is the bf16 value
      *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u),
                                                  __uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u));
      *reinterpret_cast<float4*>(d + 4) = make_float4(__uint_as_float(x.z << 16), __uint_as_float(x.z & 0xffff0000u),
                                                      __uint_as_float(x.w << 16), __uint_as_float(x.w & 0xffff0000u));
    } else {
      *reinterpret_cast<uint4*>(d) = x;
    }
  }
  __device__ __forceinline__ void store(float* __restrict__ sa, int tid) const {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int vec = tid + u * NT, row = vec / VPR, cv = vec % VPR;
      put(r[u], sa + row * ST + cv * VE);
    }
  }
};

// The same for two tensors with the same rows (K and V, or Q and dout).
template <typename T, int D, int ST, int ROWS, int NT>
struct RowTilePair {
  RowTile<T, D, ST, ROWS, NT> ta, tb;
  __device__ __forceinline__ void issue(const T* __restrict__ a, const T* __restrict__ b, int64_t tok_row0,
                                        int valid, int tid) {
    ta.issue(a, tok_row0, valid, tid);
    tb.issue(b, tok_row0, valid, tid);
  }
  __device__ __forceinline__ void store(float* __restrict__ sa, float* __restrict__ sb, int tid) const {
    ta.store(sa, tid);
    tb.store(sb, tid);
  }
};

}  // namespace infini
