// Streaming decode step of the Infini-attention layer: one new token per
// (b, h) at position `pos` of its segment. The token attends causally to the
// segment's cached keys 0..pos-1 and to itself, reads the memory of earlier
// segments (M_{s-1}, z_{s-1}), and is gated; its key and value are appended to
// the cache. ("Hugging Face Infini-Attention reproduction analysis", section
// "Infini-Attention mechanism": Local Attention, Memory Retrieval, Integration,
// State Transfer; "KV linear-addition Infini-attention": streaming with a
// bounded local context.) After a segment's last token the library folds the
// cached segment into (M, z) with the forward's state and scan kernels.
//
// The step is memory-bound: per (b, h) it reads the cache rows 0..pos-1 of K
// and V (2 * pos * d elements), M (d * d fp32) and z, and writes one output row
// and one cache row. One CTA per (b, h), 256 threads:
//   - scores: one key per thread (the whole d-long dot product in registers,
//     16-byte loads), so 256 cache rows are in flight per CTA;
//   - the softmax over the pos + 1 scores in shared memory (block max, sum);
//   - P V and sigma(q) M: each warp takes every 8th row (of V or of M), each
//     lane d/32 consecutive columns, so every row is one coalesced load; the
//     eight warps' partial sums meet in shared memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"

namespace infini {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;

// Shared memory of one step CTA: q and sigma(q) [D], the warps' partial rows
// [8][D], the scores [N], the reduction slots.
template <int D>
constexpr size_t decode_smem_bytes(int N) {
  return (size_t)(2 * D + kDecodeWarps * D + N + 2 * kDecodeWarps) * sizeof(float);
}

// 16 bytes of a row as floats: 4 fp32 or 8 bf16 values.
template <typename T>
struct Row16;
template <>
struct Row16<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float* o) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  }
};
template <>
struct Row16<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float* o) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

__device__ __forceinline__ float block_reduce(float x, float* slots, bool is_max) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  x = is_max ? warp_max(x) : warp_sum(x);
  if (lane == 0) slots[warp] = x;
  __syncthreads();
  float r = slots[0];
#pragma unroll
  for (int w = 1; w < kDecodeWarps; ++w) r = is_max ? fmaxf(r, slots[w]) : r + slots[w];
  __syncthreads();
  return r;
}

// grid: B * H CTAs (blockIdx.x = b * H + h), kDecodeThreads threads,
// decode_smem_bytes<D>(N) dynamic shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ beta, T* __restrict__ k_cache, T* __restrict__ v_cache, int H, int N,
                   int pos, const float* __restrict__ M, const float* __restrict__ z, T* __restrict__ out) {
  static_assert(D % 32 == 0, "head dim");
  extern __shared__ float dsm[];
  float* qf = dsm;                         // [D] q
  float* sqf = qf + D;                     // [D] sigma(q)
  float* part = sqf + D;                   // [8][D] per-warp partial rows
  float* sc = part + kDecodeWarps * D;     // [N] scores, then p
  float* slots = sc + N;                   // [2][8] reductions
  const int bh = blockIdx.x, h = bh % H;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const T* qb = q + (int64_t)bh * D;
  const T* kb = k + (int64_t)bh * D;
  const T* vb = v + (int64_t)bh * D;
  T* kcb = k_cache + (int64_t)bh * N * D;
  T* vcb = v_cache + (int64_t)bh * N * D;

  // q, sigma(q) to shared memory; this token's key and value to cache row pos.
  for (int c = t; c < D; c += kDecodeThreads) {
    const float x = to_f32(qb[c]);
    qf[c] = x;
    sqf[c] = elu1(x);
    kcb[(int64_t)pos * D + c] = kb[c];
    vcb[(int64_t)pos * D + c] = vb[c];
  }
  __syncthreads();

  // Scores s_j = q . k_j * log2(e) / sqrt(d) for j <= pos (row pos is this
  // token's key, read from the input rather than the row just written).
  const float scale2 = 1.4426950408889634f * rsqrtf((float)D);
  constexpr int V16 = Row16<T>::n;
  float mloc = -INFINITY;
  for (int j = t; j <= pos; j += kDecodeThreads) {
    const T* kr = j < pos ? kcb + (int64_t)j * D : kb;
    float acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < D; c += V16) {
      float x[V16];
      Row16<T>::load(kr + c, x);
#pragma unroll
      for (int e = 0; e < V16; ++e) acc = fmaf(qf[c + e], x[e], acc);
    }
    acc *= scale2;
    sc[j] = acc;
    mloc = fmaxf(mloc, acc);
  }
  const float m = block_reduce(mloc, slots, true);
  float lloc = 0.f;
  for (int j = t; j <= pos; j += kDecodeThreads) {
    const float p = exp2f(sc[j] - m);
    sc[j] = p;
    lloc += p;
  }
  const float l = block_reduce(lloc, slots + kDecodeWarps, false);  // also orders the p writes

  // A_dot = sum_j p_j v_j / l: warp w takes rows j = w, w + 8, ...; lane
  // handles columns [lane * CPL, lane * CPL + CPL).
  constexpr int CPL = D / 32;
  float acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
  for (int j = warp; j <= pos; j += kDecodeWarps) {
    const T* vr = (j < pos ? vcb + (int64_t)j * D : vb) + lane * CPL;
    const float p = sc[j];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = fmaf(p, to_f32(vr[e]), acc[e]);
  }
#pragma unroll
  for (int e = 0; e < CPL; ++e) part[warp * D + lane * CPL + e] = acc[e];
  __syncthreads();
  float adot = 0.f;
  if (t < D) {
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) adot += part[w * D + t];
    adot /= l;
  }
  __syncthreads();

  // Retrieval: num = sigma(q) M (M is [d_k][d_v], row i scaled by sigma(q)_i),
  // den = sigma(q) . z.
  const float* Mb = M + (int64_t)bh * D * D;
#pragma unroll
  for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
  for (int i = warp; i < D; i += kDecodeWarps) {
    const float s = sqf[i];
    const float* mr = Mb + (int64_t)i * D + lane * CPL;
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = fmaf(s, mr[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < CPL; ++e) part[warp * D + lane * CPL + e] = acc[e];
  float dloc = 0.f;
  for (int i = t; i < D; i += kDecodeThreads) dloc = fmaf(sqf[i], z[(int64_t)bh * D + i], dloc);
  const float den = block_reduce(dloc, slots, false);  // its barrier also publishes part
  if (t < D) {
    float num = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) num += part[w * D + t];
    const float g = gate_of(beta[h]);
    const float amem = den != 0.f ? num / den : 0.f;
    out[(int64_t)bh * D + t] = from_f32<T>(g * amem + (1.f - g) * adot);
  }
}

}  // namespace infini
