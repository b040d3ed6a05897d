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

#include <type_traits>

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
  __shared__ __align__(16) float sk[kSimtStateChunk][D];
  __shared__ __align__(16) float sv[kSimtStateChunk][D];
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
    // 16-byte loads of the chunk's K and V rows (rows past the segment read as
    // zero and contribute nothing), then sigma on the rows inside it.
    RowTilePair<T, D, D, kSimtStateChunk, kSimtStateThreads> kv;
    kv.issue(k, v, tok0 + t0, N - t0, tid);
    kv.store(&sk[0][0], &sv[0][0], tid);
    __syncthreads();
    for (int e = tid; e < kSimtStateChunk * D; e += kSimtStateThreads) {
      const int t = e / D, c = e % D;
      if (t0 + t < N) sk[t][c] = elu1_accurate(sk[t][c]);
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

// Shared-memory rows are padded to D + 4 floats (16-byte aligned; 32 lanes
// reading 32 rows at one offset hit different banks per quarter-warp), and a
// lane owns D / 32 consecutive output columns, so dot products and
// accumulations use 128-bit (D = 128) or 64-bit (D = 64) loads.
template <int D>
constexpr int simt_stride() { return D + 4; }

template <int D>
constexpr size_t simt_attn_smem_bytes() {
  // q rows, sigma(q) rows, K tile, V tile, M_{s-1}, z_{s-1}; then the
  // tensor-core scratch: a [32][33] score block, a [32][36] P block and the
  // rows' rescale factors. All fp32.
  return sizeof(float) * ((size_t)(2 * kSimtAttnRows + 2 * kSimtAttnKeys + D) * simt_stride<D>() + D +
                          (size_t)kSimtAttnRows * (kScoreStride + kAccStride) + kSimtAttnRows);
}

template <int CPL>
__device__ __forceinline__ void simt_ldv(const float* p, float (&o)[CPL]) {
  if constexpr (CPL == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  } else {
    static_assert(CPL == 2, "columns per lane");
    const float2 x = *reinterpret_cast<const float2*>(p);
    o[0] = x.x; o[1] = x.y;
  }
}
__device__ __forceinline__ float simt_dot4(const float* a, const float* b, float acc) {
  const float4 x = *reinterpret_cast<const float4*>(a), y = *reinterpret_cast<const float4*>(b);
  return fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, acc))));
}

// grid (S * ceil(N/32), H, B), block 256: 32 query rows, 4 per warp. Mp/zp:
// M_{s-1} (fp32 [BH,S,D,D]) and z_{s-1} ([BH,S,D]) from the cross-segment scan.
// d = 64 keeps three CTAs per SM (52 KB of shared memory each, 80 registers);
// d = 128 needs 135 KB per CTA, so it runs one CTA per SM with the registers
// that allows.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtAttnWarps * 32, D == 64 ? 3 : 1)
simt_attn_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ Mp,
                 const float* __restrict__ zp, int64_t L, int N, int S, T* __restrict__ out) {
  constexpr int CPL = D / 32;  // output columns per lane: lane * CPL .. + CPL
  constexpr int ST = simt_stride<D>();
  constexpr int RW = kSimtAttnRowsPerWarp;
  extern __shared__ __align__(16) float smem[];
  float* sq = smem;                          // [32][ST] q rows
  float* ssq = sq + kSimtAttnRows * ST;      // [32][ST] sigma(q) rows
  float* sk = ssq + kSimtAttnRows * ST;      // [32][ST] K tile
  float* sv = sk + kSimtAttnKeys * ST;       // [32][ST] V tile
  float* sM = sv + kSimtAttnKeys * ST;       // [D][ST] M_{s-1}
  float* sz = sM + D * ST;                   // [D] z_{s-1}
  const int blocks_per_seg = (N + kSimtAttnRows - 1) / kSimtAttnRows;
  const int s = blockIdx.x / blocks_per_seg;
  const int rb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int row_lo = rb * kSimtAttnRows;
  const int row_hi = min(row_lo + kSimtAttnRows, N);  // exclusive
  const int c0 = lane * CPL, r0 = warp * RW;

  // 16-byte loads throughout: the q rows, M_{s-1} and the first K/V tile are
  // all requested before any is stored, and each later tile is requested
  // before the work on the one before.
  constexpr int NT = kSimtAttnWarps * 32;
  RowTile<T, D, ST, kSimtAttnRows, NT> qtile;
  qtile.issue(q, tok0 + row_lo, N - row_lo, tid);
  RowTilePair<T, D, ST, kSimtAttnKeys, NT> kv_next;
  kv_next.issue(k, v, tok0, N, tid);
  const float* Ms = Mp + (bh * S + s) * (int64_t)D * D;
  for (int e = tid * 4; e < D * D; e += NT * 4)
    *reinterpret_cast<float4*>(sM + (e / D) * ST + e % D) = *reinterpret_cast<const float4*>(Ms + e);
  for (int e = tid; e < D; e += blockDim.x) sz[e] = zp[(bh * S + s) * D + e];
  qtile.store(sq, tid);
  __syncthreads();
  for (int e = tid; e < kSimtAttnRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    ssq[r * ST + c] = elu1_accurate(sq[r * ST + c]);
  }
  const float scale = rsqrtf((float)D);
  float m[RW], l[RW], o[RW][CPL];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) o[i][e] = 0.f;
  }
  const int n_tiles = (row_hi + kSimtAttnKeys - 1) / kSimtAttnKeys;  // keys 0 .. row_hi-1
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // bf16 inputs: the tile's scores and the P V accumulation on tensor cores
    // (TF32 mma.sync; q, k, v are exact in TF32, P is split into two TF32
    // parts). Each warp's 4 rows keep their online softmax in the lane layout;
    // P and the rows' rescale factors go through shared memory, and warp w
    // rescales and accumulates rows 16 (w % 2).. and columns (w / 2) D / 4 ..
    // of O. O returns to the lane layout through the K tile at the end. Every
    // warp takes part in every barrier.
    constexpr int NTW = D / 32;
    const int mi = warp & 1, cb = (warp >> 1) * (D / 4);
    float* ssc = sz + D;                                 // [32][33] scores
    float* spb = ssc + kSimtAttnRows * kScoreStride;     // [32][36] P
    float* salpha = spb + kSimtAttnRows * kAccStride;    // [32] rescale factors
    float co[NTW][4];
#pragma unroll
    for (int n = 0; n < NTW; ++n) co[n][0] = co[n][1] = co[n][2] = co[n][3] = 0.f;
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();  // previous tile fully consumed (and sigma(q) written on the first pass)
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kSimtAttnKeys, N - (kt + 1) * kSimtAttnKeys, tid);
      score_block_tf32<D, ST>(sq, sk, ssc, warp, lane);
      __syncthreads();
      const int key = kt * kSimtAttnKeys + lane;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const bool vis = key <= row && row < N;
        const float x = vis ? ssc[(r0 + i) * kScoreStride + lane] * scale : -INFINITY;
        const float mn = fmaxf(m[i], warp_max(x));
        const float corr = mn == -INFINITY ? 1.f : expf(m[i] - mn);  // exp(-inf) = 0 on the first tile
        const float pv = vis ? expf(x - mn) : 0.f;
        l[i] = l[i] * corr + warp_sum(pv);
        m[i] = mn;
        spb[(r0 + i) * kAccStride + lane] = pv;
        if (lane == 0) salpha[r0 + i] = corr;
      }
      __syncthreads();
      const float a0 = salpha[16 * mi + (lane >> 2)], a1 = salpha[16 * mi + (lane >> 2) + 8];
#pragma unroll
      for (int n = 0; n < NTW; ++n) {
        co[n][0] *= a0;
        co[n][1] *= a0;
        co[n][2] *= a1;
        co[n][3] *= a1;
      }
      mma_acc_split<NTW, ST>(co, spb + 16 * mi * kAccStride, sv + cb, lane);
    }
    __syncthreads();
    store_acc<NTW, ST>(co, sk + 16 * mi * ST + cb, lane);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RW; ++i) simt_ldv<CPL>(sk + (r0 + i) * ST + c0, o[i]);
  } else {
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();  // previous tile fully consumed (and sigma(q) written on the first pass)
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kSimtAttnKeys, N - (kt + 1) * kSimtAttnKeys, tid);
      if (row_lo + r0 >= N) continue;  // warp-uniform: none of the warp's rows exist
      // Scores of the warp's 4 rows against key `lane` of the tile.
      float sc[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) sc[i] = 0.f;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
#pragma unroll
        for (int i = 0; i < RW; ++i) sc[i] = simt_dot4(sq + (r0 + i) * ST + c, sk + lane * ST + c, sc[i]);
      }
      const int key = kt * kSimtAttnKeys + lane;
      float p[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const bool vis = key <= row && row < N;
        const float x = vis ? sc[i] * scale : -INFINITY;
        const float mn = fmaxf(m[i], warp_max(x));
        const float corr = mn == -INFINITY ? 1.f : expf(m[i] - mn);  // exp(-inf) = 0 on the first tile
        p[i] = vis ? expf(x - mn) : 0.f;
        l[i] = l[i] * corr + warp_sum(p[i]);
#pragma unroll
        for (int e = 0; e < CPL; ++e) o[i][e] *= corr;
        m[i] = mn;
      }
#pragma unroll 4
      for (int j = 0; j < kSimtAttnKeys; ++j) {
        float vj[CPL];
        simt_ldv<CPL>(sv + j * ST + c0, vj);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          const float pj = __shfl_sync(0xffffffffu, p[i], j);
#pragma unroll
          for (int e = 0; e < CPL; ++e) o[i][e] = fmaf(pj, vj[e], o[i][e]);
        }
      }
    }
  }

  // Memory retrieval with M_{s-1}, z_{s-1}: num = sigma(q) M over the lane's
  // columns, den = sigma(q) . z, then the gate.
  const float g = gate_of(beta[h]);
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int r = r0 + i;
    const int row = row_lo + r;
    if (row >= N) continue;  // warp-uniform
    float num[CPL], sqv[CPL], den = 0.f;
    simt_ldv<CPL>(ssq + r * ST + c0, sqv);
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      den = fmaf(sqv[e], sz[c0 + e], den);
      num[e] = 0.f;
    }
    den = warp_sum(den);
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      const float4 s4 = *reinterpret_cast<const float4*>(ssq + r * ST + c);
      const float sc4[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float mr[CPL];
        simt_ldv<CPL>(sM + (c + u) * ST + c0, mr);
#pragma unroll
        for (int e = 0; e < CPL; ++e) num[e] = fmaf(sc4[u], mr[e], num[e]);
      }
    }
    const float inv_l = 1.f / l[i];
    T* orow = out + (tok0 + row) * D + c0;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      const float amem = (den == 0.f) ? 0.f : num[e] / den;
      orow[e] = from_f32<T>(g * amem + (1.f - g) * (o[i][e] * inv_l));
    }
  }
}

}  // namespace infini
