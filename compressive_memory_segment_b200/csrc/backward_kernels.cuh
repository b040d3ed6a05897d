// Backward of the Infini-attention layer on CUDA cores (fp32 arithmetic, fp32
// gradients). The pages give no gradient; the formulas follow from the
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

#include "common.cuh"

namespace infini {

constexpr int kBwdWarps = 8;
constexpr int kBwdRowsPerWarp = 4;
constexpr int kBwdRows = kBwdWarps * kBwdRowsPerWarp;  // query rows (or keys) per CTA
constexpr int kBwdTile = 32;                            // keys (or query rows) per inner tile

__device__ __forceinline__ float dsigma(float x) { return x > 0.f ? 1.f : __expf(x); }

// Shared memory of bwd_rows_kernel: q rows, dout rows (scaled copies are made
// in registers), K tile (padded), V tile (padded), M_{s-1} (padded), z_{s-1}.
template <int D>
constexpr size_t bwd_rows_smem_bytes() {
  return sizeof(float) * ((size_t)kBwdRows * D * 2 + (size_t)kBwdTile * (D + 1) * 2 + (size_t)D * (D + 1) + D +
                          kBwdRows * D);
}

// grid (S * ceil(N / 32), H, B), 256 threads. Writes dq (fp32, [B,H,L,D]),
// lse and Delta ([BH, L]), dnum ([BH, L, D]) and dden ([BH, L]); adds this
// CTA's share of dbeta[h] with one atomic.
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ beta, const float* __restrict__ Mp, const float* __restrict__ zp,
                const T* __restrict__ dout, int64_t L, int N, int S, float* __restrict__ dq,
                float* __restrict__ lse_out, float* __restrict__ delta_out, float* __restrict__ dnum_out,
                float* __restrict__ dden_out, float* __restrict__ dbeta) {
  constexpr int C = D / 32;  // columns per lane: c = lane + 32 cc
  extern __shared__ float smem[];
  float* sq = smem;                                // [32][D]
  float* sdo = sq + kBwdRows * D;                  // [32][D] dout
  float* sk = sdo + kBwdRows * D;                  // [32][D+1]
  float* sv = sk + kBwdTile * (D + 1);             // [32][D+1]
  float* sM = sv + kBwdTile * (D + 1);             // [D][D+1]
  float* sz = sM + D * (D + 1);                    // [D]
  float* sx = sz + D;                              // [32][D] per-row scratch (dA, then dnum)
  const int blocks_per_seg = (N + kBwdRows - 1) / kBwdRows;
  const int s = blockIdx.x / blocks_per_seg, rb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int row_lo = rb * kBwdRows, row_hi = min(row_lo + kBwdRows, N);
  const float g = gate_of(beta[h]);
  const float scale = rsqrtf((float)D);

  for (int e = tid; e < kBwdRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    const bool in = row_lo + r < N;
    sq[e] = in ? to_f32(q[(tok0 + row_lo + r) * D + c]) : 0.f;
    sdo[e] = in ? to_f32(dout[(tok0 + row_lo + r) * D + c]) : 0.f;
  }
  const float* Ms = Mp + (bh * S + s) * (int64_t)D * D;
  for (int e = tid; e < D * D; e += blockDim.x) sM[(e / D) * (D + 1) + e % D] = Ms[e];
  for (int e = tid; e < D; e += blockDim.x) sz[e] = zp[(bh * S + s) * D + e];

  // Pass 1: the forward's online softmax per row (lane = key of the tile for
  // scores, lane + 32 cc = output column).
  float m[kBwdRowsPerWarp], l[kBwdRowsPerWarp], o[kBwdRowsPerWarp][C];
#pragma unroll
  for (int i = 0; i < kBwdRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) o[i][cc] = 0.f;
  }
  const int n_tiles = (row_hi + kBwdTile - 1) / kBwdTile;
  for (int kt = 0; kt < n_tiles; ++kt) {
    __syncthreads();
    for (int e = tid; e < kBwdTile * D; e += blockDim.x) {
      const int j = e / D, c = e % D, key = kt * kBwdTile + j;
      const bool in = key < N;
      sk[j * (D + 1) + c] = in ? to_f32(k[(tok0 + key) * D + c]) : 0.f;
      sv[j * (D + 1) + c] = in ? to_f32(v[(tok0 + key) * D + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kBwdRowsPerWarp; ++i) {
      const int r = warp * kBwdRowsPerWarp + i, row = row_lo + r;
      if (row >= N) continue;  // warp-uniform
      const int key = kt * kBwdTile + lane;
      float sc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) sc = fmaf(sq[r * D + c], sk[lane * (D + 1) + c], sc);
      sc = key <= row ? sc * scale : -INFINITY;
      const float mt = warp_max(sc);
      const float mn = fmaxf(m[i], mt);
      const float alpha = __expf(m[i] - mn);
      const float p = key <= row ? __expf(sc - mn) : 0.f;
      l[i] = l[i] * alpha + warp_sum(p);
#pragma unroll
      for (int cc = 0; cc < C; ++cc) o[i][cc] *= alpha;
      for (int j = 0; j < kBwdTile; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) o[i][cc] = fmaf(pj, sv[j * (D + 1) + lane + 32 * cc], o[i][cc]);
      }
      m[i] = mn;
    }
  }

  // Per row: A_dot, retrieval, gate gradient, Delta, dnum/dden and the
  // retrieval part of dq. dA = (1 - g) dout goes to sx for pass 2.
  float dbeta_acc = 0.f;
  float lse[kBwdRowsPerWarp], delta[kBwdRowsPerWarp], dqa[kBwdRowsPerWarp][C];
#pragma unroll
  for (int i = 0; i < kBwdRowsPerWarp; ++i) {
    const int r = warp * kBwdRowsPerWarp + i, row = row_lo + r;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dqa[i][cc] = 0.f;
    lse[i] = 0.f;
    delta[i] = 0.f;
    if (row >= N) continue;
    const int64_t tok = tok0 + row;
    float adot[C], sqv[C], num[C], gd[C];
    const float inv_l = 1.f / l[i];
#pragma unroll
    for (int cc = 0; cc < C; ++cc) adot[cc] = o[i][cc] * inv_l;
    lse[i] = m[i] + __logf(l[i]);
    float den = 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      sqv[cc] = elu1(sq[r * D + lane + 32 * cc]);
      den = fmaf(sqv[cc], sz[lane + 32 * cc], den);
    }
    den = warp_sum(den);
    // num_j = sum_c sigma(q)_c M[c][j]: sigma(q)_c broadcast from lane c % 32.
#pragma unroll
    for (int cc = 0; cc < C; ++cc) num[cc] = 0.f;
#pragma unroll
    for (int c2 = 0; c2 < C; ++c2)
      for (int src = 0; src < 32; ++src) {
        const int c = 32 * c2 + src;
        const float sc = __shfl_sync(0xffffffffu, sqv[c2], src);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) num[cc] = fmaf(sc, sM[c * (D + 1) + lane + 32 * cc], num[cc]);
      }
    float dl = 0.f, bsum = 0.f, dden = 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      const float go = sdo[r * D + lane + 32 * cc];
      const float amem = den != 0.f ? num[cc] / den : 0.f;
      bsum = fmaf(go, amem - adot[cc], bsum);
      const float dA = (1.f - g) * go;
      sx[r * D + lane + 32 * cc] = dA;
      dl = fmaf(dA, adot[cc], dl);
      const float dAm = g * go;
      gd[cc] = den != 0.f ? dAm / den : 0.f;  // dnum
      dden = fmaf(dAm, amem, dden);
    }
    dbeta_acc += g * (1.f - g) * warp_sum(bsum);
    delta[i] = warp_sum(dl);
    dden = den != 0.f ? -warp_sum(dden) / den : 0.f;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dnum_out[tok * D + lane + 32 * cc] = gd[cc];
    if (lane == 0) {
      dden_out[tok] = dden;
      lse_out[tok] = lse[i];
      delta_out[tok] = delta[i];
    }
    // dsigma(q)_c = sum_j M[c][j] dnum_j + z_c dden; dnum_j broadcast from lane j % 32.
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dqa[i][cc] = sz[lane + 32 * cc] * dden;
#pragma unroll
    for (int j2 = 0; j2 < C; ++j2)
      for (int src = 0; src < 32; ++src) {
        const int j = 32 * j2 + src;
        const float dn = __shfl_sync(0xffffffffu, gd[j2], src);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) dqa[i][cc] = fmaf(sM[(lane + 32 * cc) * (D + 1) + j], dn, dqa[i][cc]);
      }
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dqa[i][cc] *= dsigma(sq[r * D + lane + 32 * cc]);
  }

  // Pass 2: dq_t += sum_j dS_tj k_j / sqrt(d) over the causal keys.
  for (int kt = 0; kt < n_tiles; ++kt) {
    __syncthreads();
    for (int e = tid; e < kBwdTile * D; e += blockDim.x) {
      const int j = e / D, c = e % D, key = kt * kBwdTile + j;
      const bool in = key < N;
      sk[j * (D + 1) + c] = in ? to_f32(k[(tok0 + key) * D + c]) : 0.f;
      sv[j * (D + 1) + c] = in ? to_f32(v[(tok0 + key) * D + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kBwdRowsPerWarp; ++i) {
      const int r = warp * kBwdRowsPerWarp + i, row = row_lo + r;
      if (row >= N) continue;
      const int key = kt * kBwdTile + lane;
      float sc = 0.f, dp = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        sc = fmaf(sq[r * D + c], sk[lane * (D + 1) + c], sc);
        dp = fmaf(sx[r * D + c], sv[lane * (D + 1) + c], dp);
      }
      const float p = key <= row ? __expf(sc * scale - lse[i]) : 0.f;
      const float ds = p * (dp - delta[i]) * scale;
      for (int j = 0; j < kBwdTile; ++j) {
        const float dsj = __shfl_sync(0xffffffffu, ds, j);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) dqa[i][cc] = fmaf(dsj, sk[j * (D + 1) + lane + 32 * cc], dqa[i][cc]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kBwdRowsPerWarp; ++i) {
    const int row = row_lo + warp * kBwdRowsPerWarp + i;
    if (row >= N) continue;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dq[(tok0 + row) * D + lane + 32 * cc] = dqa[i][cc];
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
// One thread per element of a (b, h) matrix or vector; n = elements per
// (b, h) and segment.
__global__ void bwd_rscan_kernel(float* __restrict__ X, int64_t BH, int S, int64_t n, const float* __restrict__ g_out,
                                 float* __restrict__ g_in) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BH * n) return;
  const int64_t bh = idx / n, e = idx % n;
  float acc = g_out ? g_out[idx] : 0.f;
  for (int s = S - 1; s >= 0; --s) {
    float* x = X + (bh * S + s) * n + e;
    const float t = *x;
    *x = acc;
    acc += t;
  }
  g_in[idx] = acc;
}

template <int D>
constexpr size_t bwd_keys_smem_bytes() {
  // own keys and values, query tile (padded), dA tile (padded), lse, Delta, G (padded), Gz.
  return sizeof(float) * ((size_t)kBwdRows * D * 2 + (size_t)kBwdTile * (D + 1) * 2 + 2 * kBwdTile +
                          (size_t)D * (D + 1) + D);
}

// grid (S * ceil(N / 32), H, B), 256 threads: 32 keys per CTA, 4 per warp.
// Writes dk and dv (fp32).
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_keys_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ beta, const T* __restrict__ dout, const float* __restrict__ lse_in,
                const float* __restrict__ delta_in, const float* __restrict__ G, const float* __restrict__ Gz,
                int64_t L, int N, int S, float* __restrict__ dk, float* __restrict__ dv) {
  constexpr int C = D / 32;
  extern __shared__ float smem[];
  float* sk = smem;                               // [32][D] own keys
  float* sv = sk + kBwdRows * D;                  // [32][D] own values
  float* sq = sv + kBwdRows * D;                  // [32][D+1] query tile
  float* sa = sq + kBwdTile * (D + 1);            // [32][D+1] dA tile
  float* sl = sa + kBwdTile * (D + 1);            // [32] lse
  float* sdl = sl + kBwdTile;                     // [32] Delta
  float* sG = sdl + kBwdTile;                     // [D][D+1]
  float* sGz = sG + D * (D + 1);                  // [D]
  const int blocks_per_seg = (N + kBwdRows - 1) / kBwdRows;
  const int s = blockIdx.x / blocks_per_seg, kb = blockIdx.x % blocks_per_seg;
  const int h = blockIdx.y;
  const int64_t bh = (int64_t)blockIdx.z * gridDim.y + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tok0 = bh * L + (int64_t)s * N;
  const int key_lo = kb * kBwdRows;
  const float g = gate_of(beta[h]);
  const float scale = rsqrtf((float)D);

  for (int e = tid; e < kBwdRows * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    const bool in = key_lo + r < N;
    sk[e] = in ? to_f32(k[(tok0 + key_lo + r) * D + c]) : 0.f;
    sv[e] = in ? to_f32(v[(tok0 + key_lo + r) * D + c]) : 0.f;
  }
  const float* Gs = G + (bh * S + s) * (int64_t)D * D;
  for (int e = tid; e < D * D; e += blockDim.x) sG[(e / D) * (D + 1) + e % D] = Gs[e];
  for (int e = tid; e < D; e += blockDim.x) sGz[e] = Gz[(bh * S + s) * D + e];
  __syncthreads();

  // Memory part: dv_j = G^T sigma(k_j), dk_j = (G v_j + Gz) * sigma'(k_j).
  float dka[kBwdRowsPerWarp][C], dva[kBwdRowsPerWarp][C];
#pragma unroll
  for (int i = 0; i < kBwdRowsPerWarp; ++i) {
    const int r = warp * kBwdRowsPerWarp + i;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dka[i][cc] = dva[i][cc] = 0.f;
    if (key_lo + r >= N) continue;
    float skv[C], vv[C];
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      skv[cc] = elu1(sk[r * D + lane + 32 * cc]);
      vv[cc] = sv[r * D + lane + 32 * cc];
      dka[i][cc] = sGz[lane + 32 * cc];
    }
#pragma unroll
    for (int c2 = 0; c2 < C; ++c2)
      for (int src = 0; src < 32; ++src) {
        const int c = 32 * c2 + src;
        const float skc = __shfl_sync(0xffffffffu, skv[c2], src);
        const float vc = __shfl_sync(0xffffffffu, vv[c2], src);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) {
          dva[i][cc] = fmaf(skc, sG[c * (D + 1) + lane + 32 * cc], dva[i][cc]);   // sum_c sk_c G[c][j]
          dka[i][cc] = fmaf(sG[(lane + 32 * cc) * (D + 1) + c], vc, dka[i][cc]);  // sum_c G[i][c] v_c
        }
      }
#pragma unroll
    for (int cc = 0; cc < C; ++cc) dka[i][cc] *= dsigma(sk[r * D + lane + 32 * cc]);
  }

  // Local part over the query rows t >= key in the segment (lane = query row
  // of the tile for P and dS, lane + 32 cc = column for the sums).
  const int first_qt = key_lo / kBwdTile;
  const int n_qt = (N + kBwdTile - 1) / kBwdTile;
  for (int qt = first_qt; qt < n_qt; ++qt) {
    __syncthreads();
    for (int e = tid; e < kBwdTile * D; e += blockDim.x) {
      const int t = e / D, c = e % D, row = qt * kBwdTile + t;
      const bool in = row < N;
      sq[t * (D + 1) + c] = in ? to_f32(q[(tok0 + row) * D + c]) : 0.f;
      sa[t * (D + 1) + c] = in ? (1.f - g) * to_f32(dout[(tok0 + row) * D + c]) : 0.f;
    }
    for (int t = tid; t < kBwdTile; t += blockDim.x) {
      const int row = qt * kBwdTile + t;
      sl[t] = row < N ? lse_in[tok0 + row] : 0.f;
      sdl[t] = row < N ? delta_in[tok0 + row] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kBwdRowsPerWarp; ++i) {
      const int r = warp * kBwdRowsPerWarp + i, key = key_lo + r;
      if (key >= N) continue;
      const int row = qt * kBwdTile + lane;
      float sc = 0.f, dp = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        sc = fmaf(sq[lane * (D + 1) + c], sk[r * D + c], sc);
        dp = fmaf(sa[lane * (D + 1) + c], sv[r * D + c], dp);
      }
      const bool vis = row < N && row >= key;
      const float p = vis ? __expf(sc * scale - sl[lane]) : 0.f;
      const float ds = p * (dp - sdl[lane]) * scale;
      for (int t = 0; t < kBwdTile; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
        const float dst = __shfl_sync(0xffffffffu, ds, t);
#pragma unroll
        for (int cc = 0; cc < C; ++cc) {
          dva[i][cc] = fmaf(pt, sa[t * (D + 1) + lane + 32 * cc], dva[i][cc]);
          dka[i][cc] = fmaf(dst, sq[t * (D + 1) + lane + 32 * cc], dka[i][cc]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kBwdRowsPerWarp; ++i) {
    const int key = key_lo + warp * kBwdRowsPerWarp + i;
    if (key >= N) continue;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      dk[(tok0 + key) * D + lane + 32 * cc] = dka[i][cc];
      dv[(tok0 + key) * D + lane + 32 * cc] = dva[i][cc];
    }
  }
}

}  // namespace infini
