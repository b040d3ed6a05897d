// CUDA-core (fp32 FFMA) kernels of the Infini-attention forward.
//
// These cover every supported shape and both I/O dtypes, and are the path for
// fp32 I/O, whose 1e-4 tolerance the bf16 tensor-core operands cannot meet.
// All arithmetic is fp32; the I/O dtype only changes loads and stores.
//
//   simt_state_kernel : per (b, h, segment s): dM_s = sigma(K_s)^T V_s and
//                       dz_s = sum_t sigma(K_s,t) ("Hugging Face
//                       Infini-Attention reproduction analysis", Infini-Attention
//                       mechanism: Memory Update).
//   simt_attn_kernel  : per (b, h, s, 32-row block): causal softmax attention
//                       inside the segment with an online softmax over 32-key
//                       tiles (the running-max/normaliser merge of the
//                       "Attention-State Memory" page, Methodology), retrieval
//                       sigma(q) M_{s-1} / (sigma(q) . z_{s-1}) with 0 for a zero
//                       denominator, and the sigmoid(beta) gate (Local Attention,
//                       Memory Retrieval, Integration).
#pragma once

#include "common.cuh"

namespace infini {

constexpr int kSimtStateThreads = 256;
constexpr int kSimtStateChunk = 32;  // tokens staged per iteration

// grid (S, H, B), block 256 = 16 x 16 threads; thread (ty, tx) owns rows
// c = ty + 16 r1 and columns j = tx + 16 r2 of the D x D increment.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtStateThreads)
simt_state_kernel(const T* __restrict__ k, const T* __restrict__ v, int64_t L, int N,
                  float* __restrict__ dM, float* __restrict__ dz) {
  constexpr int R = D / 16;
  __shared__ float sk[kSimtStateChunk][D];
  __shared__ float sv[kSimtStateChunk][D];
  const int s = blockIdx.x, S = gridDim.x;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t tok0 = bh * L + (int64_t)s * N;  // first token row of the segment

  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  float zacc = 0.f;

  for (int t0 = 0; t0 < N; t0 += kSimtStateChunk) {
    for (int e = tid; e < kSimtStateChunk * D; e += kSimtStateThreads) {
      const int t = e / D, c = e % D;
      float kv = 0.f, vv = 0.f;  // tokens past the segment contribute nothing
      if (t0 + t < N) {
        const int64_t off = (tok0 + t0 + t) * D + c;
        kv = elu1_accurate(to_f32(k[off]));
        vv = to_f32(v[off]);
      }
      sk[t][c] = kv;
      sv[t][c] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kSimtStateChunk; ++t) {
      float a[R], b[R];
#pragma unroll
      for (int r = 0; r < R; ++r) { a[r] = sk[t][ty + 16 * r]; b[r] = sv[t][tx + 16 * r]; }
#pragma unroll
      for (int r1 = 0; r1 < R; ++r1)
#pragma unroll
        for (int r2 = 0; r2 < R; ++r2) acc[r1][r2] = fmaf(a[r1], b[r2], acc[r1][r2]);
    }
    if (tid < D) {
      for (int t = 0; t < kSimtStateChunk; ++t) zacc += sk[t][tid];
    }
    __syncthreads();
  }
  float* dMs = dM + (bh * S + s) * (int64_t)D * D;
#pragma unroll
  for (int r1 = 0; r1 < R; ++r1)
#pragma unroll
    for (int r2 = 0; r2 < R; ++r2) dMs[(ty + 16 * r1) * D + tx + 16 * r2] = acc[r1][r2];
  if (tid < D) dz[(bh * S + s) * D + tid] = zacc;
}

constexpr int kSimtAttnWarps = 8;
constexpr int kSimtAttnRowsPerWarp = 4;
constexpr int kSimtAttnRows = kSimtAttnWarps * kSimtAttnRowsPerWarp;  // 32 query rows per CTA
constexpr int kSimtAttnKeys = 32;                                     // keys per tile

template <int D>
constexpr size_t simt_attn_smem_bytes() {
  // q rows, K tile (padded), V tile, M_{s-1}, z_{s-1}; all fp32.
  return sizeof(float) * ((size_t)kSimtAttnRows * D + (size_t)kSimtAttnKeys * (D + 1) +
                          (size_t)kSimtAttnKeys * D + (size_t)D * D + D);
}

// grid (S * ceil(N/32), H, B), block 256. Mp/zp: M_{s-1} (fp32 [BH,S,D,D]) and
// z_{s-1} ([BH,S,D]) from the cross-segment scan.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtAttnWarps * 32)
simt_attn_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ Mp,
                 const float* __restrict__ zp, int64_t L, int N, int S, T* __restrict__ out) {
  constexpr int C = D / 32;  // output columns per lane: j = lane + 32 cc
  extern __shared__ float smem[];
  float* sq = smem;                                   // [32][D]
  float* sk = sq + kSimtAttnRows * D;                 // [32][D+1]
  float* sv = sk + kSimtAttnKeys * (D + 1);           // [32][D]
  float* sM = sv + kSimtAttnKeys * D;                 // [D][D]
  float* sz = sM + D * D;                             // [D]

  const int blocks_per_seg = (N + kSimtAttnRows - 1) / kSimtAttnRows;
  const int s = blockIdx.x / blocks_per_seg;
  const int rb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int row_lo = rb * kSimtAttnRows;
  const int row_hi = min(row_lo + kSimtAttnRows, N);  // exclusive

  for (int e = tid; e < kSimtAttnRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    sq[e] = (row_lo + r < N) ? to_f32(q[(tok0 + row_lo + r) * D + c]) : 0.f;
  }

  const float scale = rsqrtf((float)D);
  float m[kSimtAttnRowsPerWarp], l[kSimtAttnRowsPerWarp], o[kSimtAttnRowsPerWarp][C];
#pragma unroll
  for (int i = 0; i < kSimtAttnRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) o[i][cc] = 0.f;
  }

  const int n_tiles = (row_hi + kSimtAttnKeys - 1) / kSimtAttnKeys;  // keys 0 .. row_hi-1
  for (int kt = 0; kt < n_tiles; ++kt) {
    __syncthreads();  // previous tile fully consumed (and sq written on the first pass)
    for (int e = tid; e < kSimtAttnKeys * D; e += blockDim.x) {
      const int j = e / D, c = e % D;
      const int key = kt * kSimtAttnKeys + j;
      float kv = 0.f, vv = 0.f;
      if (key < N) {
        const int64_t off = (tok0 + key) * D + c;
        kv = to_f32(k[off]);
        vv = to_f32(v[off]);
      }
      sk[j * (D + 1) + c] = kv;
      sv[j * D + c] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kSimtAttnRowsPerWarp; ++i) {
      const int r = warp * kSimtAttnRowsPerWarp + i;
      const int row = row_lo + r;
      if (row >= N) continue;  // warp-uniform
      const int key = kt * kSimtAttnKeys + lane;
      float sc = 0.f;
      const float* qr = sq + r * D;
      const float* kr = sk + lane * (D + 1);
#pragma unroll 8
      for (int c = 0; c < D; ++c) sc = fmaf(qr[c], kr[c], sc);
      sc = (key <= row) ? sc * scale : -INFINITY;
      const float mt = warp_max(sc);
      const float mn = fmaxf(m[i], mt);
      if (mn == -INFINITY) continue;  // no visible key yet (cannot happen at kt = 0)
      const float p = (key <= row) ? expf(sc - mn) : 0.f;
      const float corr = expf(m[i] - mn);  // exp(-inf) = 0 on the first tile
      l[i] = l[i] * corr + warp_sum(p);
      m[i] = mn;
#pragma unroll
      for (int cc = 0; cc < C; ++cc) o[i][cc] *= corr;
#pragma unroll 8
      for (int j = 0; j < kSimtAttnKeys; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) o[i][cc] = fmaf(pj, sv[j * D + lane + 32 * cc], o[i][cc]);
      }
    }
  }

  // Memory retrieval with M_{s-1}, z_{s-1}.
  __syncthreads();
  const float* Ms = Mp + (bh * S + s) * (int64_t)D * D;
  const float* zs = zp + (bh * S + s) * D;
  for (int e = tid; e < D * D; e += blockDim.x) sM[e] = Ms[e];
  for (int e = tid; e < D; e += blockDim.x) sz[e] = zs[e];
  __syncthreads();
  const float g = gate_of(beta[h]);
#pragma unroll
  for (int i = 0; i < kSimtAttnRowsPerWarp; ++i) {
    const int r = warp * kSimtAttnRowsPerWarp + i;
    const int row = row_lo + r;
    if (row >= N) continue;
    const float* qr = sq + r * D;
    float num[C], den = 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) num[cc] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float sqc = elu1_accurate(qr[c]);
      den = fmaf(sqc, sz[c], den);
#pragma unroll
      for (int cc = 0; cc < C; ++cc) num[cc] = fmaf(sqc, sM[c * D + lane + 32 * cc], num[cc]);
    }
    const float inv_l = 1.f / l[i];
    T* orow = out + (tok0 + row) * D;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      const float amem = (den == 0.f) ? 0.f : num[cc] / den;
      const float adot = o[i][cc] * inv_l;
      orow[lane + 32 * cc] = from_f32<T>(g * amem + (1.f - g) * adot);
    }
  }
}

}  // namespace infini
