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
// and one cache row. To keep enough loads in flight it is split over CTAs
// (grid: chunks + 1 per (b, h)):
//   - chunk CTAs: 128 keys each, in one pass: every K and V row is one
//     coalesced warp load, each warp keeps an online softmax over its keys,
//     and the chunk's (m_c, l_c, acc_c[d]) is written out;
//   - one retrieval CTA: sigma(q) M and sigma(q) . z (each warp every 8th row
//     of M);
//   - a combine kernel (one CTA per (b, h)) merges the chunks with the
//     online-softmax rule, adds the gated retrieval and writes the output.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"

namespace infini {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;

constexpr int kDecodeChunk = 128;  // keys per chunk CTA (eight warps, 16 keys each)

// Per (b, h): for each chunk (m, l, acc[D]) then the retrieval (den, num[D]).
template <int D>
constexpr size_t decode_partial_floats(int max_chunks) {
  return (size_t)max_chunks * (D + 2) + (D + 1);
}

// CPL consecutive elements of a row as floats, in one vector load of
// CPL * sizeof(T) bytes (4, 8 or 16; the callers' offsets are multiples of it).
template <typename T, int CPL>
__device__ __forceinline__ void load_cols(const T* p, float* o);
template <>
__device__ __forceinline__ void load_cols<__nv_bfloat16, 4>(const __nv_bfloat16* p, float* o) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  o[0] = __uint_as_float(x.x << 16); o[1] = __uint_as_float(x.x & 0xffff0000u);
  o[2] = __uint_as_float(x.y << 16); o[3] = __uint_as_float(x.y & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_cols<__nv_bfloat16, 2>(const __nv_bfloat16* p, float* o) {
  const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
  o[0] = __uint_as_float(x << 16); o[1] = __uint_as_float(x & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_cols<float, 4>(const float* p, float* o) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
}
template <>
__device__ __forceinline__ void load_cols<float, 2>(const float* p, float* o) {
  const float2 x = *reinterpret_cast<const float2*>(p);
  o[0] = x.x; o[1] = x.y;
}

// The same columns kept as loaded (packed bf16 or fp32) until they are used,
// so a warp can have many rows in flight for few registers.
template <typename T, int CPL>
struct RawCols;
template <>
struct RawCols<__nv_bfloat16, 4> {
  uint2 x;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { x = *reinterpret_cast<const uint2*>(p); }
  __device__ __forceinline__ void zero() { x = make_uint2(0u, 0u); }
  __device__ __forceinline__ float get(int e) const {
    const uint32_t w = e < 2 ? x.x : x.y;
    return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <>
struct RawCols<__nv_bfloat16, 2> {
  uint32_t x;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { x = *reinterpret_cast<const uint32_t*>(p); }
  __device__ __forceinline__ void zero() { x = 0u; }
  __device__ __forceinline__ float get(int e) const { return __uint_as_float(e ? (x & 0xffff0000u) : (x << 16)); }
};
template <>
struct RawCols<float, 4> {
  float4 x;
  __device__ __forceinline__ void load(const float* p) { x = *reinterpret_cast<const float4*>(p); }
  __device__ __forceinline__ void zero() { x = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float get(int e) const { return e == 0 ? x.x : e == 1 ? x.y : e == 2 ? x.z : x.w; }
};
template <>
struct RawCols<float, 2> {
  float2 x;
  __device__ __forceinline__ void load(const float* p) { x = *reinterpret_cast<const float2*>(p); }
  __device__ __forceinline__ void zero() { x = make_float2(0.f, 0.f); }
  __device__ __forceinline__ float get(int e) const { return e == 0 ? x.x : x.y; }
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

// grid: (n_chunks + 1, B * H) with n_chunks = ceil((pos + 1) / kDecodeChunk);
// kDecodeThreads threads. part: [B*H][decode_partial_floats<D>(max_chunks)].
template <typename T, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_partial_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      T* __restrict__ k_cache, T* __restrict__ v_cache, int N, int pos, int max_chunks,
                      const float* __restrict__ M, const float* __restrict__ z, float* __restrict__ part) {
  static_assert(D % 32 == 0, "head dim");
  __shared__ float qf[D];
  __shared__ float red[kDecodeWarps * D];
  __shared__ float slots[2 * kDecodeWarps];
  const int bh = blockIdx.y, c = blockIdx.x;
  const int n_chunks = (pos + kDecodeChunk) / kDecodeChunk;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const T* qb = q + (int64_t)bh * D;
  const T* kb = k + (int64_t)bh * D;
  const T* vb = v + (int64_t)bh * D;
  const T* kcb = k_cache + (int64_t)bh * N * D;
  const T* vcb = v_cache + (int64_t)bh * N * D;
  float* pb = part + (int64_t)bh * decode_partial_floats<D>(max_chunks);
  constexpr int CPL = D / 32;

  if (c == n_chunks) {
    // Retrieval CTA: num = sigma(q) M ([d_k][d_v], row i scaled by
    // sigma(q)_i), den = sigma(q) . z; this CTA also appends the token's key
    // and value to cache row pos (no chunk CTA reads that row: it takes this
    // token's key and value from the inputs).
    for (int i = t; i < D; i += kDecodeThreads) {
      qf[i] = elu1(to_f32(qb[i]));
      k_cache[((int64_t)bh * N + pos) * D + i] = kb[i];
      v_cache[((int64_t)bh * N + pos) * D + i] = vb[i];
    }
    __syncthreads();
    const float* Mb = M + (int64_t)bh * D * D;
    float acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = warp; i < D; i += kDecodeWarps) {  // all d / 8 rows of a warp in flight at once
      const float s = qf[i];
      float mr[CPL];
      load_cols<float, CPL>(Mb + (int64_t)i * D + lane * CPL, mr);
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[e] = fmaf(s, mr[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) red[warp * D + lane * CPL + e] = acc[e];
    float dloc = 0.f;
    for (int i = t; i < D; i += kDecodeThreads) dloc = fmaf(qf[i], z[(int64_t)bh * D + i], dloc);
    const float den = block_reduce(dloc, slots, false);  // its barrier also publishes red
    float* rb = pb + (int64_t)max_chunks * (D + 2);
    if (t < D) {
      float num = 0.f;
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) num += red[w * D + t];
      rb[1 + t] = num;
    }
    if (t == 0) rb[0] = den;
    return;
  }

  // Chunk CTA: keys j0 .. j1-1 of the segment (key pos is this token's).
  // Warp w takes keys j0 + 8w + 64i .. +7 (i = 0, 1, ...): each lane holds
  // d/32 consecutive columns of q, so one load instruction fetches a whole K
  // or V row; the eight keys' K and V rows (4 KB at d = 128 in bf16) are
  // requested together and kept as loaded until used. A dot product is a
  // butterfly sum over the lanes; each warp keeps its own online softmax
  // (running max m, sum l and P V row), and the eight warps merge in shared
  // memory at the end.
  const int j0 = c * kDecodeChunk, j1 = min(j0 + kDecodeChunk, pos + 1);
  const float scale2 = 1.4426950408889634f * rsqrtf((float)D);
  float qv[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) qv[e] = to_f32(qb[lane * CPL + e]) * scale2;
  float m_w = -INFINITY, l_w = 0.f, acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
  constexpr int KB = 8;  // keys per warp per batch
  for (int jb = j0 + KB * warp; jb < j1; jb += KB * kDecodeWarps) {
    RawCols<T, CPL> kx[KB], vx[KB];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const int j = jb + u;
      if (j < j1) {
        kx[u].load((j < pos ? kcb + (int64_t)j * D : kb) + lane * CPL);
        vx[u].load((j < pos ? vcb + (int64_t)j * D : vb) + lane * CPL);
      } else {
        kx[u].zero();
        vx[u].zero();
      }
    }
    float sc[KB];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) dot = fmaf(qv[e], kx[u].get(e), dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      sc[u] = jb + u < j1 ? dot : -INFINITY;
    }
    float m_new = m_w;
#pragma unroll
    for (int u = 0; u < KB; ++u) m_new = fmaxf(m_new, sc[u]);
    const float alpha = exp2f(m_w - m_new);
    l_w *= alpha;
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] *= alpha;
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const float p = exp2f(sc[u] - m_new);
      l_w += p;
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[e] = fmaf(p, vx[u].get(e), acc[e]);
    }
    m_w = m_new;
  }
#pragma unroll
  for (int e = 0; e < CPL; ++e) red[warp * D + lane * CPL + e] = acc[e];
  if (lane == 0) {
    slots[warp] = m_w;
    slots[kDecodeWarps + warp] = l_w;
  }
  __syncthreads();
  float m = -INFINITY;
#pragma unroll
  for (int w = 0; w < kDecodeWarps; ++w) m = fmaxf(m, slots[w]);
  float* cb = pb + (int64_t)c * (D + 2);
  if (t < D) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) a = fmaf(exp2f(slots[w] - m), red[w * D + t], a);
    cb[2 + t] = a;
  }
  if (t == 0) {
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) l = fmaf(exp2f(slots[w] - m), slots[kDecodeWarps + w], l);
    cb[0] = m;
    cb[1] = l;
  }
}

// grid: B * H CTAs of D threads. Merges the chunks (softmax over all keys =
// sum_c 2^(m_c - m) acc_c / sum_c 2^(m_c - m) l_c with m = max_c m_c), then
// out = g A_mem + (1 - g) A_dot with A_mem = num / den (0 when den = 0).
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part, int pos, int max_chunks, int H, const float* __restrict__ beta,
                      T* __restrict__ out) {
  const int bh = blockIdx.x, t = threadIdx.x;
  const int n_chunks = (pos + kDecodeChunk) / kDecodeChunk;
  const float* pb = part + (int64_t)bh * decode_partial_floats<D>(max_chunks);
  float m = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) m = fmaxf(m, pb[(int64_t)c * (D + 2)]);
  float l = 0.f, a = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const float* cb = pb + (int64_t)c * (D + 2);
    const float w = exp2f(cb[0] - m);
    l = fmaf(w, cb[1], l);
    a = fmaf(w, cb[2 + t], a);
  }
  const float* rb = pb + (int64_t)max_chunks * (D + 2);
  const float den = rb[0], num = rb[1 + t];
  const float g = gate_of(beta[bh % H]);
  const float amem = den != 0.f ? num / den : 0.f;
  out[(int64_t)bh * D + t] = from_f32<T>(g * amem + (1.f - g) * (a / l));
}

}  // namespace infini
