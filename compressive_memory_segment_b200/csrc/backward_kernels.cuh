// Backward of the Infini-attention layer (fp32 gradients). With fp32 inputs
// all arithmetic is fp32 FFMA; with bf16 inputs the 32 x 32 tile products of
// the local attention (scores, dout V^T, P V, dS K, dS^T Q, P^T dout) run on
// TF32 mma.sync tensor-core instructions (exact products of bf16 values; the
// fp32 factors P and dS split into two TF32 parts). The pages give no
// gradient; the formulas follow from the
// forward's steps by the chain rule ("Hugging Face Infini-Attention
// reproduction analysis", section "Infini-Attention mechanism": Local
// Attention, Memory Retrieval, Integration, Memory Update, State Transfer):
//
//   out_t = g A_mem,t + (1 - g) A_dot,t, g = sigmoid(beta_h)
//     dbeta += g (1 - g) dout_t . (A_mem,t - A_dot,t)
//   local part, with dA_t = (1 - g) dout_t, P the causal softmax, lse_t its
//   log-normaliser and Delta_t = dA_t . A_dot,t:
//     dS_tj = P_tj (dA_t . v_j - Delta_t),
//     dq_t += sum_j dS_tj k_j / sqrt(d), dk_j += sum_t dS_tj q_t / sqrt(d),
//     dv_j += sum_t P_tj dA_t
//   retrieval, with dA'_t = g dout_t (nothing where den = 0):
//     dnum = dA' / den, dden = -(dA' . A_mem) / den,
//     dq_t += (M_{s-1} dnum + z_{s-1} dden) * sigma'(q_t),
//     the gradient reaching M_{s-1}: sum_t sigma(q_t) dnum_t^T (z: sigma(q_t) dden_t)
//   state chain: G_s, the gradient reaching M_s, is dM_out plus those of all
//     later segments; dv_t += G_s^T sigma(k_t),
//     dk_t += (G_s v_t + Gz_s) * sigma'(k_t); dM_in is G reaching M_in.
//
// Launch sequence (one call): the forward's state and scan kernels recompute
// M_{s-1}, z_{s-1}; bwd_rows_kernel (per 32 query rows) recomputes each row's
// softmax statistics and output, writes dq, lse, Delta, dnum, dden and adds
// its rows' dbeta; bwd_state_grad_kernel forms each segment's
// sigma(Q)^T dnum; bwd_rscan_kernel turns those into G in place (and dM_in);
// bwd_keys_kernel (per 32 keys) writes dk and dv.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace infini {

constexpr int kBwdWarps = 8;
constexpr int kBwdRowsPerWarp = 4;
constexpr int kBwdRows = kBwdWarps * kBwdRowsPerWarp;  // query rows (or keys) per CTA
constexpr int kBwdTile = 32;                            // keys (or query rows) per inner tile

__device__ __forceinline__ float dsigma(float x) { return x > 0.f ? 1.f : __expf(x); }

// Shared-memory rows are padded to D + 4 floats: 16-byte aligned for 128-bit
// loads, and 32 lanes reading 32 different rows at the same offset touch
// different banks within each quarter-warp. A lane owns CPL = D / 32
// consecutive columns, so a row slice is one 128-bit (CPL = 4) or 64-bit
// (CPL = 2) load.
template <int D>
constexpr int bwd_stride() { return D + 4; }

// With bf16 inputs every operand of the score-shaped products (q, k, v, dout,
// widened to fp32 in shared memory) has at most 8 significant bits, so TF32
// tensor-core products of them are exact and only the fp32 summation order
// differs from the FFMA loops; the accumulating products split their fp32
// factor in two (mma_acc_split). fp32 inputs keep the FFMA loops.
template <typename T>
constexpr bool kBwdTf32 = std::is_same<T, __nv_bfloat16>::value;

// The K/V (or Q/dout) tiles: 32 rows of two [*, D] tensors, issued ahead of
// the work on the tile before (RowTilePair in common.cuh).
static_assert(kBwdRows == kBwdTile, "a CTA's own rows and an inner tile are both 32 rows");
template <typename T, int D>
using TilePair = RowTilePair<T, D, bwd_stride<D>(), kBwdTile, kBwdWarps * 32>;

template <typename T, int D>
__device__ __forceinline__ void load_tile_pair(const T* __restrict__ a, const T* __restrict__ b, int64_t tok_row0,
                                               int valid, float* __restrict__ sa, float* __restrict__ sb,
                                               int tid) {
  TilePair<T, D> tp;
  tp.issue(a, b, tok_row0, valid, tid);
  tp.store(sa, sb, tid);
}


template <int CPL>
__device__ __forceinline__ void ldv(const float* p, float (&o)[CPL]) {
  if constexpr (CPL == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  } else {
    static_assert(CPL == 2, "columns per lane");
    const float2 x = *reinterpret_cast<const float2*>(p);
    o[0] = x.x; o[1] = x.y;
  }
}
template <int CPL>
__device__ __forceinline__ void stv(float* p, const float (&o)[CPL]) {
  if constexpr (CPL == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
  } else {
    *reinterpret_cast<float2*>(p) = make_float2(o[0], o[1]);
  }
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Shared memory of bwd_rows_kernel: q, dout, dA and scratch rows, a K and a V
// tile, M_{s-1} and z_{s-1}.
template <int D>
constexpr size_t bwd_rows_smem_bytes() {
  return sizeof(float) * ((size_t)6 * kBwdRows * bwd_stride<D>() + (size_t)D * bwd_stride<D>() + D);
}

// grid (S * ceil(N / 32), H, B), 256 threads: 32 query rows per CTA, 4 per
// warp. Writes dq (fp32, [B,H,L,D]), lse and Delta ([BH, L]), dnum
// ([BH, L, D]) and dden ([BH, L]); adds this CTA's share of dbeta[h] with one
// atomic.
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32, D == 64 ? 2 : 1)
bwd_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ beta, const float* __restrict__ Mp, const float* __restrict__ zp,
                const T* __restrict__ dout, int64_t L, int N, int S, float* __restrict__ dq,
                float* __restrict__ lse_out, float* __restrict__ delta_out, float* __restrict__ dnum_out,
                float* __restrict__ dden_out, float* __restrict__ dbeta) {
  constexpr int CPL = D / 32;  // columns per lane: lane * CPL .. + CPL
  constexpr int ST = bwd_stride<D>();
  constexpr int RW = kBwdRowsPerWarp;
  extern __shared__ __align__(16) float smem[];
  float* sq = smem;                      // [32][ST] q rows
  float* sdo = sq + kBwdRows * ST;       // [32][ST] dout rows
  float* sx = sdo + kBwdRows * ST;       // [32][ST] dA = (1 - g) dout (FFMA loops), or the score,
                                         // P and rescale scratch and at the end the dq block
                                         // (tensor-core form; O returns through the K tile)
  float* sy = sx + kBwdRows * ST;        // [32][ST] sigma(q), then dnum
  float* sk = sy + kBwdRows * ST;        // [32][ST] K tile
  float* sv = sk + kBwdTile * ST;        // [32][ST] V tile
  float* sM = sv + kBwdTile * ST;        // [D][ST] M_{s-1}; in pass 2 the dS block (tensor-core form)
  float* sz = sM + D * ST;               // [D] z_{s-1}
  const int blocks_per_seg = (N + kBwdRows - 1) / kBwdRows;
  const int s = blockIdx.x / blocks_per_seg, rb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int row_lo = rb * kBwdRows, row_hi = min(row_lo + kBwdRows, N);
  const float g = gate_of(beta[h]);
  const float scale = rsqrtf((float)D);
  const int c0 = lane * CPL;

  load_tile_pair<T, D>(q, dout, tok0 + row_lo, N - row_lo, sq, sdo, tid);
  __syncthreads();
  for (int e = tid; e < kBwdRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    if constexpr (!kBwdTf32<T>) sx[r * ST + c] = (1.f - g) * sdo[r * ST + c];
    sy[r * ST + c] = elu1(sq[r * ST + c]);
  }
  const float* Ms = Mp + (bh * S + s) * (int64_t)D * D;
  for (int e = tid; e < D * D; e += blockDim.x) sM[(e / D) * ST + e % D] = Ms[e];
  for (int e = tid; e < D; e += blockDim.x) sz[e] = zp[(bh * S + s) * D + e];

  // Pass 1: the forward's online softmax for the warp's 4 rows (lane = key of
  // the tile for the scores, lane's CPL columns for the output).
  float m[RW], l[RW], o[RW][CPL];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) o[i][e] = 0.f;
  }
  const int r0 = warp * RW;
  const int n_tiles = (row_hi + kBwdTile - 1) / kBwdTile;
  TilePair<T, D> kv_next;
  kv_next.issue(k, v, tok0, N, tid);
  if constexpr (kBwdTf32<T>) {
    // Tensor-core form. Per tile: the score block, then each warp's rows'
    // online softmax in the lane layout; P (over the score block once every
    // warp has read it) and the rows' rescale factors go through shared
    // memory; warp w rescales and accumulates rows 16 (w % 2).. and columns
    // (w / 2) D / 4 .. of O with accumulating MMAs. O returns to the lane
    // layout through the K tile at the end. Every warp takes part in every
    // barrier.
    constexpr int NTW = D / 32;
    const int mi = warp & 1, cb = (warp >> 1) * (D / 4);
    float* spb = sx;                               // [32][kAccStride] P
    float* salpha = sx + kBwdRows * kAccStride;    // [32] rescale factors
    float co[NTW][4];
#pragma unroll
    for (int n = 0; n < NTW; ++n) co[n][0] = co[n][1] = co[n][2] = co[n][3] = 0.f;
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kBwdTile, N - (kt + 1) * kBwdTile, tid);
      score_block_tf32<D, ST>(sq, sk, sx, warp, lane);
      __syncthreads();
      float sc[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) sc[i] = sx[(r0 + i) * kScoreStride + lane];
      __syncthreads();  // every score read before P overwrites the block
      const int key = kt * kBwdTile + lane;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const bool vis = key <= row && row < N;
        const float x = vis ? sc[i] * scale : -INFINITY;
        const float mn = fmaxf(m[i], warp_max(x));
        const float alpha = mn == -INFINITY ? 1.f : __expf(m[i] - mn);
        const float pv = vis ? __expf(x - mn) : 0.f;
        l[i] = l[i] * alpha + warp_sum(pv);
        m[i] = mn;
        spb[(r0 + i) * kAccStride + lane] = pv;
        if (lane == 0) salpha[r0 + i] = alpha;
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
    for (int i = 0; i < RW; ++i) ldv<CPL>(sk + (r0 + i) * ST + c0, o[i]);
  } else {
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kBwdTile, N - (kt + 1) * kBwdTile, tid);
      if (row_lo + r0 >= N) continue;  // warp-uniform: none of the warp's rows exist
      float sc[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) sc[i] = 0.f;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 kv = ld4(sk + lane * ST + c);
#pragma unroll
        for (int i = 0; i < RW; ++i) sc[i] = dot4(ld4(sq + (r0 + i) * ST + c), kv, sc[i]);
      }
      const int key = kt * kBwdTile + lane;
      float p[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const bool vis = key <= row && row < N;
        const float x = vis ? sc[i] * scale : -INFINITY;
        const float mn = fmaxf(m[i], warp_max(x));
        const float alpha = mn == -INFINITY ? 1.f : __expf(m[i] - mn);
        p[i] = vis ? __expf(x - mn) : 0.f;
        l[i] = l[i] * alpha + warp_sum(p[i]);
#pragma unroll
        for (int e = 0; e < CPL; ++e) o[i][e] *= alpha;
        m[i] = mn;
      }
      for (int j = 0; j < kBwdTile; ++j) {
        float vj[CPL];
        ldv<CPL>(sv + j * ST + c0, vj);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          const float pj = __shfl_sync(0xffffffffu, p[i], j);
#pragma unroll
          for (int e = 0; e < CPL; ++e) o[i][e] = fmaf(pj, vj[e], o[i][e]);
        }
      }
    }
  }

  // Per row: A_dot, retrieval, gate gradient, Delta, dnum/dden and the
  // retrieval part of dq.
  float dbeta_acc = 0.f;
  float lse[RW], delta[RW], dqa[RW][CPL];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int r = r0 + i, row = row_lo + r;
#pragma unroll
    for (int e = 0; e < CPL; ++e) dqa[i][e] = 0.f;
    lse[i] = 0.f;
    delta[i] = 0.f;
    if (row >= N) continue;  // warp-uniform
    const int64_t tok = tok0 + row;
    const float inv_l = 1.f / l[i];
    lse[i] = m[i] + __logf(l[i]);
    float adot[CPL], sqv[CPL], zv[CPL], num[CPL], go[CPL], dnum[CPL];
    ldv<CPL>(sy + r * ST + c0, sqv);
    ldv<CPL>(sdo + r * ST + c0, go);
    float den = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      adot[e] = o[i][e] * inv_l;
      zv[e] = sz[c0 + e];
      den = fmaf(sqv[e], zv[e], den);
      num[e] = 0.f;
    }
    den = warp_sum(den);
    // num_j = sum_c sigma(q)_c M[c][j] over the lane's columns j.
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      const float4 sq4 = ld4(sy + r * ST + c);
      const float sqc[4] = {sq4.x, sq4.y, sq4.z, sq4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float mr[CPL];
        ldv<CPL>(sM + (c + u) * ST + c0, mr);
#pragma unroll
        for (int e = 0; e < CPL; ++e) num[e] = fmaf(sqc[u], mr[e], num[e]);
      }
    }
    float bsum = 0.f, dl = 0.f, dden = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      const float amem = den != 0.f ? num[e] / den : 0.f;
      bsum = fmaf(go[e], amem - adot[e], bsum);
      dl = fmaf((1.f - g) * go[e], adot[e], dl);
      const float dAm = g * go[e];
      dnum[e] = den != 0.f ? dAm / den : 0.f;
      dden = fmaf(dAm, amem, dden);
    }
    dbeta_acc += g * (1.f - g) * warp_sum(bsum);
    delta[i] = warp_sum(dl);
    dden = den != 0.f ? -warp_sum(dden) / den : 0.f;
    stv<CPL>(dnum_out + tok * D + c0, dnum);
    if (lane == 0) {
      dden_out[tok] = dden;
      lse_out[tok] = lse[i];
      delta_out[tok] = delta[i];
    }
    // dsigma(q)_c = sum_j M[c][j] dnum_j + z_c dden over the lane's columns c
    // (dnum goes through the row's scratch for broadcast reads).
    __syncwarp();
    stv<CPL>(sy + r * ST + c0, dnum);
    __syncwarp();
#pragma unroll
    for (int e = 0; e < CPL; ++e) dqa[i][e] = zv[e] * dden;
#pragma unroll 2
    for (int j = 0; j < D; j += 4) {
      const float4 dn = ld4(sy + r * ST + j);
#pragma unroll
      for (int e = 0; e < CPL; ++e) dqa[i][e] = dot4(ld4(sM + (c0 + e) * ST + j), dn, dqa[i][e]);
    }
    float qv[CPL];
    ldv<CPL>(sq + r * ST + c0, qv);
#pragma unroll
    for (int e = 0; e < CPL; ++e) dqa[i][e] *= dsigma(qv[e]);
  }

  // Pass 2: dq_t += sum_j dS_tj k_j / sqrt(d) over the causal keys.
  if constexpr (kBwdTf32<T>) {
    // dS goes through shared memory (M_{s-1} is no longer needed) into
    // accumulating MMAs: warp w owns rows 16 (w % 2).. and columns
    // (w / 2) D / 4 .. of the block. Every warp takes part in every barrier.
    constexpr int NTW = D / 32;
    const int mi = warp & 1, cb = (warp >> 1) * (D / 4);
    float* sds = sM;
    float cq[NTW][4];
#pragma unroll
    for (int n = 0; n < NTW; ++n) cq[n][0] = cq[n][1] = cq[n][2] = cq[n][3] = 0.f;
    kv_next.issue(k, v, tok0, N, tid);
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kBwdTile, N - (kt + 1) * kBwdTile, tid);
      score_block_tf32<D, ST>(sq, sk, sx, warp, lane);
      score_block_tf32<D, ST>(sdo, sv, sx + kBwdRows * kScoreStride, warp, lane);
      __syncthreads();
      const int key = kt * kBwdTile + lane;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const float sc = sx[(r0 + i) * kScoreStride + lane];
        const float dp = (1.f - g) * sx[kBwdRows * kScoreStride + (r0 + i) * kScoreStride + lane];
        const float p = (key <= row && row < N) ? __expf(sc * scale - lse[i]) : 0.f;
        sds[(r0 + i) * kAccStride + lane] = p * (dp - delta[i]) * scale;
      }
      __syncthreads();
      mma_acc_split<NTW, ST>(cq, sds + 16 * mi * kAccStride, sk + cb, lane);
    }
    __syncthreads();
    store_acc<NTW, ST>(cq, sx + 16 * mi * ST + cb, lane);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      float add[CPL];
      ldv<CPL>(sx + (r0 + i) * ST + c0, add);
#pragma unroll
      for (int e = 0; e < CPL; ++e) dqa[i][e] += add[e];
    }
  } else {
    kv_next.issue(k, v, tok0, N, tid);
    for (int kt = 0; kt < n_tiles; ++kt) {
      __syncthreads();
      kv_next.store(sk, sv, tid);
      __syncthreads();
      if (kt + 1 < n_tiles) kv_next.issue(k, v, tok0 + (kt + 1) * kBwdTile, N - (kt + 1) * kBwdTile, tid);
      if (row_lo + r0 >= N) continue;
      float sc[RW], dp[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) sc[i] = dp[i] = 0.f;
#pragma unroll 2
      for (int c = 0; c < D; c += 4) {
        const float4 kv = ld4(sk + lane * ST + c), vv = ld4(sv + lane * ST + c);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          sc[i] = dot4(ld4(sq + (r0 + i) * ST + c), kv, sc[i]);
          dp[i] = dot4(ld4(sx + (r0 + i) * ST + c), vv, dp[i]);
        }
      }
      const int key = kt * kBwdTile + lane;
      float ds[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = row_lo + r0 + i;
        const float p = (key <= row && row < N) ? __expf(sc[i] * scale - lse[i]) : 0.f;
        ds[i] = p * (dp[i] - delta[i]) * scale;
      }
      for (int j = 0; j < kBwdTile; ++j) {
        float kj[CPL];
        ldv<CPL>(sk + j * ST + c0, kj);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          const float dsj = __shfl_sync(0xffffffffu, ds[i], j);
#pragma unroll
          for (int e = 0; e < CPL; ++e) dqa[i][e] = fmaf(dsj, kj[e], dqa[i][e]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int row = row_lo + r0 + i;
    if (row >= N) continue;
    stv<CPL>(dq + (tok0 + row) * D + c0, dqa[i]);
  }
  // One dbeta atomic per CTA.
  __syncthreads();
  if (lane == 0) sz[warp] = dbeta_acc;  // sz is no longer needed
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kBwdWarps; ++w) t += sz[w];
    atomicAdd(&dbeta[h], t);
  }
}

// Per (b, h, segment s): dMq_s = sum_t sigma(q_t) dnum_t^T and
// dzq_s = sum_t sigma(q_t) dden_t (the gradient reaching M_{s-1}, z_{s-1}
// from segment s's queries). grid (S, H, B), 256 threads as 16 x 16.
template <typename T, int D>
__global__ void __launch_bounds__(256)
bwd_state_grad_kernel(const T* __restrict__ q, const float* __restrict__ dnum, const float* __restrict__ dden,
                      int64_t L, int N, float* __restrict__ dMq, float* __restrict__ dzq) {
  constexpr int R = D / 16;
  constexpr int CH = 32;
  __shared__ float sa[CH][D];
  __shared__ float sb[CH][D];
  __shared__ float sd[CH];
  const int s = blockIdx.x, S = gridDim.x;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  float zacc = 0.f;
  for (int t0 = 0; t0 < N; t0 += CH) {
    for (int e = tid; e < CH * D; e += 256) {
      const int t = e / D, c = e % D;
      const bool in = t0 + t < N;
      sa[t][c] = in ? elu1_accurate(to_f32(q[(tok0 + t0 + t) * D + c])) : 0.f;
      sb[t][c] = in ? dnum[(tok0 + t0 + t) * D + c] : 0.f;
    }
    for (int t = tid; t < CH; t += 256) sd[t] = t0 + t < N ? dden[tok0 + t0 + t] : 0.f;
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < CH; ++t) {
      float a[R], b[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        a[r] = sa[t][ty + 16 * r];
        b[r] = sb[t][tx + 16 * r];
      }
#pragma unroll
      for (int r1 = 0; r1 < R; ++r1)
#pragma unroll
        for (int r2 = 0; r2 < R; ++r2) acc[r1][r2] = fmaf(a[r1], b[r2], acc[r1][r2]);
    }
    if (tid < D)
      for (int t = 0; t < CH; ++t) zacc = fmaf(sa[t][tid], sd[t], zacc);
    __syncthreads();
  }
  float* out = dMq + (bh * S + s) * (int64_t)D * D;
#pragma unroll
  for (int r1 = 0; r1 < R; ++r1)
#pragma unroll
    for (int r2 = 0; r2 < R; ++r2) out[(ty + 16 * r1) * D + tx + 16 * r2] = acc[r1][r2];
  if (tid < D) dzq[(bh * S + s) * D + tid] = zacc;
}

// In place over segments, from the last: X[s] <- G_s = g_out + sum_{s' > s} X[s']
// (the gradient reaching M_s), and g_in = g_out + sum_s X[s] (reaching M_in).
// One thread per four consecutive elements idx4 .. idx4 + 3 of the (b, h)
// matrices or vectors (n, the elements per (b, h) and segment, is a multiple
// of 4, and X, g_out and g_in are 16-byte aligned); each element's sum runs
// over the segments in the same order as a scalar walk.
__device__ __forceinline__ void bwd_rscan_one(float* __restrict__ X, int64_t BH, int S, int64_t n,
                                              const float* __restrict__ g_out, float* __restrict__ g_in,
                                              int64_t idx4) {
  const int64_t idx = idx4 * 4;
  if (idx >= BH * n) return;
  const int64_t bh = idx / n, e = idx % n;
  float4 acc = g_out ? *reinterpret_cast<const float4*>(g_out + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
  float* xb = X + bh * S * n + e;
  // Eight segments' values are loaded before any is used, so a thread has
  // eight 16-byte loads in flight instead of one per round trip.
  constexpr int U = 8;
  int s = S - 1;
  for (; s >= U - 1; s -= U) {
    float4 t[U];
#pragma unroll
    for (int u = 0; u < U; ++u) t[u] = *reinterpret_cast<const float4*>(xb + (int64_t)(s - u) * n);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      *reinterpret_cast<float4*>(xb + (int64_t)(s - u) * n) = acc;
      acc.x += t[u].x; acc.y += t[u].y; acc.z += t[u].z; acc.w += t[u].w;
    }
  }
  for (; s >= 0; --s) {
    const float4 t = *reinterpret_cast<const float4*>(xb + (int64_t)s * n);
    *reinterpret_cast<float4*>(xb + (int64_t)s * n) = acc;
    acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
  }
  *reinterpret_cast<float4*>(g_in + idx) = acc;
}

// Both reverse scans in one launch of 256-thread blocks: the first nb_z
// blocks take the vectors Gz (d per (b, h) and segment; few blocks, each a
// chain of dependent round trips, so they start first), the rest the matrices
// G (d * d).
__global__ void __launch_bounds__(256)
bwd_rscan_kernel(float* __restrict__ G, float* __restrict__ Gz, int64_t BH, int S, int D,
                 const float* __restrict__ dM_out, float* __restrict__ dM_in, const float* __restrict__ dz_out,
                 float* __restrict__ dz_in, unsigned nb_z) {
  if (blockIdx.x < nb_z)
    bwd_rscan_one(Gz, BH, S, D, dz_out, dz_in, (int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  else
    bwd_rscan_one(G, BH, S, (int64_t)D * D, dM_out, dM_in, (int64_t)(blockIdx.x - nb_z) * blockDim.x + threadIdx.x);
}

inline cudaError_t launch_bwd_rscan(float* G, float* Gz, int64_t BH, int S, int D, const float* dM_out,
                                    float* dM_in, const float* dz_out, float* dz_in, cudaStream_t st) {
  const int64_t nM4 = BH * D * D / 4, nz4 = BH * D / 4;
  const unsigned nb_z = (unsigned)((nz4 + 255) / 256), nb_m = (unsigned)((nM4 + 255) / 256);
  bwd_rscan_kernel<<<nb_z + nb_m, 256, 0, st>>>(G, Gz, BH, S, D, dM_out, dM_in, dz_out, dz_in, nb_z);
  return cudaGetLastError();
}

template <int D>
constexpr size_t bwd_keys_smem_bytes() {
  // own keys, values and sigma(k) rows, a query and a dA tile, lse, Delta, G, Gz.
  return sizeof(float) * ((size_t)5 * kBwdRows * bwd_stride<D>() + 2 * kBwdTile + (size_t)D * bwd_stride<D>() + D);
}

// grid (S * ceil(N / 32), H, B), 256 threads: 32 keys per CTA, 4 per warp.
// Writes dk and dv (fp32).
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32, D == 64 ? 2 : 1)
bwd_keys_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ beta, const T* __restrict__ dout, const float* __restrict__ lse_in,
                const float* __restrict__ delta_in, const float* __restrict__ G, const float* __restrict__ Gz,
                int64_t L, int N, int S, float* __restrict__ dk, float* __restrict__ dv) {
  constexpr int CPL = D / 32;
  constexpr int ST = bwd_stride<D>();
  constexpr int RW = kBwdRowsPerWarp;
  extern __shared__ __align__(16) float smem[];
  float* sk = smem;                      // [32][ST] own keys
  float* sv = sk + kBwdRows * ST;        // [32][ST] own values
  float* ssk = sv + kBwdRows * ST;       // [32][ST] sigma(own keys); later two score blocks
  float* sq = ssk + kBwdRows * ST;       // [32][ST] query tile
  float* sa = sq + kBwdTile * ST;        // [32][ST] dout tile
  float* sl = sa + kBwdTile * ST;        // [32] lse
  float* sdl = sl + kBwdTile;            // [32] Delta
  float* sG = sdl + kBwdTile;            // [D][ST]
  float* sGz = sG + D * ST;              // [D]
  const int blocks_per_seg = (N + kBwdRows - 1) / kBwdRows;
  const int s = blockIdx.x / blocks_per_seg, kb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int key_lo = kb * kBwdRows;
  const float g = gate_of(beta[h]);
  const float scale = rsqrtf((float)D);
  const int c0 = lane * CPL;
  const int r0 = warp * RW;

  load_tile_pair<T, D>(k, v, tok0 + key_lo, N - key_lo, sk, sv, tid);
  __syncthreads();
  for (int e = tid; e < kBwdRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    ssk[r * ST + c] = elu1(sk[r * ST + c]);
  }
  const float* Gs = G + (bh * S + s) * (int64_t)D * D;
  for (int e = tid; e < D * D; e += blockDim.x) sG[(e / D) * ST + e % D] = Gs[e];
  for (int e = tid; e < D; e += blockDim.x) sGz[e] = Gz[(bh * S + s) * D + e];
  __syncthreads();

  // Memory part: dv_j = G^T sigma(k_j) (lane's columns), dk_j = (G v_j + Gz)
  // * sigma'(k_j) (lane's rows of G).
  float dka[RW][CPL], dva[RW][CPL];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int r = r0 + i;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      dva[i][e] = 0.f;
      dka[i][e] = sGz[c0 + e];
    }
    if (key_lo + r >= N) continue;  // warp-uniform
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      const float4 sk4 = ld4(ssk + r * ST + c), v4 = ld4(sv + r * ST + c);
      const float skc[4] = {sk4.x, sk4.y, sk4.z, sk4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float gr[CPL];
        ldv<CPL>(sG + (c + u) * ST + c0, gr);
#pragma unroll
        for (int e = 0; e < CPL; ++e) dva[i][e] = fmaf(skc[u], gr[e], dva[i][e]);
      }
#pragma unroll
      for (int e = 0; e < CPL; ++e) dka[i][e] = dot4(ld4(sG + (c0 + e) * ST + c), v4, dka[i][e]);
    }
    float kv[CPL];
    ldv<CPL>(sk + r * ST + c0, kv);
#pragma unroll
    for (int e = 0; e < CPL; ++e) dka[i][e] *= dsigma(kv[e]);
  }

  // Local part over the query rows t >= key in the segment (lane = query row
  // of the tile for P and dS, lane's columns for the sums).
  const int first_qt = key_lo / kBwdTile;
  const int n_qt = (N + kBwdTile - 1) / kBwdTile;
  TilePair<T, D> qa_next;
  if (first_qt < n_qt) qa_next.issue(q, dout, tok0 + first_qt * kBwdTile, N - first_qt * kBwdTile, tid);
  if constexpr (kBwdTf32<T>) {
    // Tensor-core form: (1 - g) P and dS go through shared memory (G is no
    // longer needed) into accumulating MMAs; warp w owns keys 16 (w % 2)..
    // and columns (w / 2) D / 4 .. of dk and dv. Every warp takes part in
    // every barrier.
    constexpr int NTW = D / 32;
    const int mi = warp & 1, cb = (warp >> 1) * (D / 4);
    float* sp = sG;
    float* sds = sG + kBwdRows * kAccStride;
    float ck[NTW][4], cv[NTW][4];
#pragma unroll
    for (int n = 0; n < NTW; ++n)
#pragma unroll
      for (int x = 0; x < 4; ++x) ck[n][x] = cv[n][x] = 0.f;
    for (int qt = first_qt; qt < n_qt; ++qt) {
      __syncthreads();
      qa_next.store(sq, sa, tid);
      if (qt + 1 < n_qt) qa_next.issue(q, dout, tok0 + (qt + 1) * kBwdTile, N - (qt + 1) * kBwdTile, tid);
      for (int t = tid; t < kBwdTile; t += blockDim.x) {
        const int row = qt * kBwdTile + t;
        sl[t] = row < N ? lse_in[tok0 + row] : 0.f;
        sdl[t] = row < N ? delta_in[tok0 + row] : 0.f;
      }
      __syncthreads();
      // K Q^T and V dout^T (sigma(own keys) is no longer needed).
      score_block_tf32<D, ST>(sk, sq, ssk, warp, lane);
      score_block_tf32<D, ST>(sv, sa, ssk + kBwdRows * kScoreStride, warp, lane);
      __syncthreads();
      const int row = qt * kBwdTile + lane;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int key = key_lo + r0 + i;
        const bool vis = row < N && row >= key && key < N;
        const float sc = ssk[(r0 + i) * kScoreStride + lane];
        const float dp = (1.f - g) * ssk[kBwdRows * kScoreStride + (r0 + i) * kScoreStride + lane];
        const float pv = vis ? __expf(sc * scale - sl[lane]) : 0.f;
        sp[(r0 + i) * kAccStride + lane] = (1.f - g) * pv;
        sds[(r0 + i) * kAccStride + lane] = pv * (dp - sdl[lane]) * scale;
      }
      __syncthreads();
      mma_acc_split<NTW, ST>(cv, sp + 16 * mi * kAccStride, sa + cb, lane);
      mma_acc_split<NTW, ST>(ck, sds + 16 * mi * kAccStride, sq + cb, lane);
    }
    __syncthreads();
    store_acc<NTW, ST>(ck, sq + 16 * mi * ST + cb, lane);
    store_acc<NTW, ST>(cv, sa + 16 * mi * ST + cb, lane);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      float ak[CPL], av[CPL];
      ldv<CPL>(sq + (r0 + i) * ST + c0, ak);
      ldv<CPL>(sa + (r0 + i) * ST + c0, av);
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        dka[i][e] += ak[e];
        dva[i][e] += av[e];
      }
    }
  } else {
    for (int qt = first_qt; qt < n_qt; ++qt) {
      __syncthreads();
      qa_next.store(sq, sa, tid);
      if (qt + 1 < n_qt) qa_next.issue(q, dout, tok0 + (qt + 1) * kBwdTile, N - (qt + 1) * kBwdTile, tid);
      for (int t = tid; t < kBwdTile; t += blockDim.x) {
        const int row = qt * kBwdTile + t;
        sl[t] = row < N ? lse_in[tok0 + row] : 0.f;
        sdl[t] = row < N ? delta_in[tok0 + row] : 0.f;
      }
      __syncthreads();
      if (key_lo + r0 >= N) continue;
      float sc[RW], dp[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) sc[i] = dp[i] = 0.f;
#pragma unroll 2
      for (int c = 0; c < D; c += 4) {
        const float4 q4 = ld4(sq + lane * ST + c), a4 = ld4(sa + lane * ST + c);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          sc[i] = dot4(q4, ld4(sk + (r0 + i) * ST + c), sc[i]);
          dp[i] = dot4(a4, ld4(sv + (r0 + i) * ST + c), dp[i]);
        }
      }
      // dA = (1 - g) dout: into dP, and into P where it weighs dv.
#pragma unroll
      for (int i = 0; i < RW; ++i) dp[i] *= 1.f - g;
      const int row = qt * kBwdTile + lane;
      float p[RW], ds[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int key = key_lo + r0 + i;
        const bool vis = row < N && row >= key && key < N;
        p[i] = vis ? __expf(sc[i] * scale - sl[lane]) : 0.f;
        ds[i] = p[i] * (dp[i] - sdl[lane]) * scale;
      }
      for (int t = 0; t < kBwdTile; ++t) {
        float qr[CPL], ar[CPL];
        ldv<CPL>(sq + t * ST + c0, qr);
        ldv<CPL>(sa + t * ST + c0, ar);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          const float pt = (1.f - g) * __shfl_sync(0xffffffffu, p[i], t);
          const float dst = __shfl_sync(0xffffffffu, ds[i], t);
#pragma unroll
          for (int e = 0; e < CPL; ++e) {
            dva[i][e] = fmaf(pt, ar[e], dva[i][e]);
            dka[i][e] = fmaf(dst, qr[e], dka[i][e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int key = key_lo + r0 + i;
    if (key >= N) continue;
    stv<CPL>(dk + (tok0 + key) * D + c0, dka[i]);
    stv<CPL>(dv + (tok0 + key) * D + c0, dva[i]);
  }
}

}  // namespace infini
