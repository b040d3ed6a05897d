// Tensor-core backward of the local attention for bf16 I/O, head dimension
// 128 and segments of whole 128-row tiles. The gradient formulas are the
// chain rule through the forward's steps ("Hugging Face Infini-Attention
// reproduction analysis", section "Infini-Attention mechanism": Local
// Attention, Memory Retrieval, Integration, Memory Update, State Transfer),
// as listed at the top of backward_kernels.cuh. With g = sigmoid(beta_h),
// dA = (1 - g) dout, P the causal softmax of the scaled scores (normalised
// through lse_t from the statistics pass) and Delta_t = dA_t . A_dot,t:
//
//   dS_tj = P_tj (dA_t . v_j - Delta_t)
//   dq_t  = sum_j dS_tj k_j / sqrt(d) + (M_{s-1} dnum_t + z_{s-1} dden_t) * sigma'(q_t)
//   dk_j  = sum_t dS_tj q_t / sqrt(d) + (G_s v_j + Gz_s) * sigma'(k_j)
//   dv_j  = (1 - g) sum_t P_tj dout_t + G_s^T sigma(k_j)
//
// where t runs over the queries of k_j's segment at or after it, G_s / Gz_s
// is the gradient reaching M_s / z_s (the dQ kernel's tail terms after the
// reverse scan, bwd_rscan_kernel) and dnum / dden come from the statistics
// pass.
//
// Two kernels, one CTA per (segment, 128-row tile), the CTAs of a segment
// consecutive (they share its tiles through L2), 320 threads: warp 0 issues
// the TMA copies, warp 1 owns TMEM and issues the MMAs (one elected lane of
// the converged warp), warps 2-9 run two threads per tile row (warps 2-5 the
// columns 0..63 of the score tiles, warps 6-9 the columns 64..127; warp w
// reaches TMEM lanes 32 (w % 4) .. + 31) and then the epilogue over the same
// column halves.
//
// The score-shaped tiles (S, dP and their transposes) are fp32 in TMEM; the
// threads turn them into bf16 P and dS and write them, packed in pairs, over
// the first 32 columns of their own 64-column half, so the MMA that consumes
// them reads A from TMEM (key or query k of a tile at packed column
// 64 (k / 64) + (k % 64) / 2) and no thread overwrites columns another thread
// has still to read.
#pragma once

namespace infini {
namespace tc {

constexpr int kBwdTcThreads = 320;
constexpr float kInvSqrtD = 0.08838834764831845f;                    // 1 / sqrt(128)
constexpr float kScoreScale2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
constexpr uint32_t kBColDP = 128;   // dP (dP^T), dS (dS^T) over its halves' first 32 columns
constexpr uint32_t kBColAcc = 256;  // dQ, or dV
constexpr uint32_t kBColAcc2 = 384; // dK

// sigma'(x) of ELU + 1: 1 for x > 0, e^x otherwise (as 2^(x log2 e)).
__device__ __forceinline__ float dsigma_tc(float x) { return x > 0.f ? 1.f : ex2(x * 1.4426950408889634f); }

// k-step kk (16 of the 128 contraction indices) of a K-major SW128 tile, and
// of an MN-major one (16 rows of 128 B), as descriptor address offsets.
__device__ __forceinline__ uint32_t kmaj_step(int kk) { return ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4; }
__device__ __forceinline__ uint32_t mnmaj_step(int kk) { return (kk * 2048) >> 4; }
// TMEM column of the packed bf16 A operand for k-step kk (see above).
__device__ __forceinline__ uint32_t packed_a_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }

// Eight bf16 values (one 16-byte chunk) to floats.
__device__ __forceinline__ void bf16x8_to_f32(uint4 x, float (&f)[8]) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    f[2 * t] = __uint_as_float(w[t] << 16);
    f[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
  }
}

// Byte offset of fp32 element (row, col) of a 128-row x 128-column tile
// stored as four 32-column blocks in the 128-byte swizzle (16-byte chunk index
// within a 128-byte row XORed with row % 8), the layout of a TMA box of
// 32 x 128 fp32 with CU_TENSOR_MAP_SWIZZLE_128B.
__device__ __forceinline__ uint32_t sw128_f32_offset(uint32_t row, uint32_t col) {
  return (col >> 5) * (128u * 128u) + row * 128u + ((((col & 31u) >> 2) ^ (row & 7u)) << 4) + (col & 3u) * 4u;
}

// ------------------------------------------------------------------ dQ
// CTA = (segment, query tile i). Shared memory: Q_i | dO_i | ring of two
// (A | B) tile pairs | dden^T tile (16 x 128 bf16, K-major) | barriers. Ring
// position j holds (K_j, V_j), j = 0..i, and position i + 1 (dnum16_i,
// M_{s-1}) for the retrieval and state terms.
// TMEM: S 0..127, dP 128..255 (dS over it), dQ 256..383; after the loop
// dnum M^T at 0..127, sigma(Q)^T dnum at 128..255, sigma(Q)^T dden at
// 384..399.
// MMA order: S_0, dP_0; per key tile j: S_{j+1} once every thread has read
// S_j, dQ += dS_j K_j once dS_j is written, dP_{j+1}; then the three tail
// MMAs once the threads have written sigma(Q_i) over dO_i (whose last reader
// is dP_i) and dden^T. The threads take P_j from S_j while the MMAs of
// dQ_{j-1} and dP_j run.
// The tail's sigma(Q_i)^T dnum_i and sigma(Q_i)^T dden_i are the query tile's
// share of the gradient reaching M_{s-1} and z_{s-1}; they are added into
// G[s] (by a TMA reduce-add of the staged 128 x 128 fp32 tile) and Gz[s]
// (fp32 atomics), both zeroed by the host, and the reverse scan over segments
// turns those into G_s, Gz_s. dq leaves through shared memory: each thread
// writes its row into an fp32 tile in the 128-byte swizzle over ring stage 0
// (free once the tail MMAs are done), the G share goes into stage 1 the same
// way (first, so that its reduce-add reads out while dq is formed), and one
// thread issues the TMA reduce-add and tensor store.
constexpr uint32_t kDqRing = 2 * kTileBytes;
constexpr uint32_t kDqDdenT = 16 * 128 * 2;  // 16 rows x 128 bf16: row 0 dden, rows 1..15 zero
constexpr uint32_t kDqZ = 2 * kTileBytes + 2 * kDqRing + kDqDdenT;  // z_{s-1} (bulk copy)
constexpr uint32_t kDqSmem = kDqZ + kD * 4 + 256;
static_assert(kDqSmem <= 232448, "dQ kernel shared memory");
constexpr uint32_t kBColGz = 384;

__global__ void __launch_bounds__(kBwdTcThreads, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmN, const __grid_constant__ CUtensorMap tmM,
                 const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmG,
                 const float* __restrict__ beta, const float* __restrict__ zp, const float* __restrict__ lse,
                 const float* __restrict__ delta, const float* __restrict__ dden, float* __restrict__ Gz, int L, int N,
                 int S, int H, int n_segs, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sO = smem_raw + kTileBytes;
  uint8_t* ring = smem_raw + 2 * kTileBytes;
  uint8_t* sDT = smem_raw + 2 * kTileBytes + 2 * kDqRing;
  const float* sz = reinterpret_cast<const float*>(smem_raw + kDqZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kDqZ + kD * 4);
  uint64_t* fix_full = bars + 0;     // Q_i and dO_i (TMA)
  uint64_t* ring_full = bars + 1;    // [2] TMA
  uint64_t* ring_empty = bars + 3;   // [2] MMAs done with the slot
  uint64_t* s_full = bars + 5;       // S_j done
  uint64_t* dp_full = bars + 6;      // dP_j done
  uint64_t* s_free = bars + 7;       // S_j read by all threads (8 warps)
  uint64_t* ds_full = bars + 8;      // dS_j written (8 warps)
  uint64_t* fin_ready = bars + 9;    // sigma(Q_i) and dden^T written, S and dP read (8 warps)
  uint64_t* fin_full = bars + 10;    // every MMA done
  uint64_t* drain = bars + 11;       // abort path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = N / kTile;
  const int seg = blockIdx.x / n_qt, rank = blockIdx.x - seg * n_qt;
  const int i = n_qt - 1 - rank, nk = i + 1;
  const int bh = seg / S, s = seg - bh * S, h = bh % H;
  const int row_seg = bh * L + s * N, row_q = row_seg + i * kTile;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 12; ++b) mbar_init(&bars[b], (b == 7 || b == 8 || b == 9) ? 8 : 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  uint32_t armed = 0;  // producer: barriers with a copy in flight (bit 0 fix, bits 1-2 ring), for the abort path

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (elect_one_lane()) {
      mbar_arrive_expect_tx(fix_full, 2 * kTileBytes + kD * 4);
      load_tile(sQ, &tmQ, row_q, fix_full);
      load_tile(sO, &tmO, row_q, fix_full);
      bulk_load(smem_raw + kDqZ, zp + (int64_t)seg * kD, kD * 4, fix_full);
    }
    __syncwarp();
    armed |= 1u;
    for (int p = 0; p <= nk && ok; ++p) {
      const int slot = p & 1, use = p >> 1;
      if (use > 0 && !(ok = mbar_wait_warp(&ring_empty[slot], (use - 1) & 1, epoch))) break;
      armed |= 2u << slot;
      if (elect_one_lane()) {
        uint8_t* st = ring + slot * kDqRing;
        mbar_arrive_expect_tx(&ring_full[slot], 2 * kTileBytes);
        if (p == nk) {
          load_tile(st, &tmN, row_q, &ring_full[slot]);
          load_tile(st + kTileBytes, &tmM, seg * kD, &ring_full[slot]);
        } else {
          load_tile(st, &tmK, row_seg + p * kTile, &ring_full[slot]);
          load_tile(st + kTileBytes, &tmV, row_seg + p * kTile, &ring_full[slot]);
        }
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    const uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
    const uint32_t id_kmn = idesc_bf16_f32(128, 128, false, true);
    const uint32_t id_mnmn = idesc_bf16_f32(128, 128, true, true);
    const uint32_t id_gz = idesc_bf16_f32(128, 16, true, false);
    const uint64_t dQ = desc_kmajor_sw128(smem_u32(sQ));
    const uint64_t dO = desc_kmajor_sw128(smem_u32(sO));
    const uint64_t dSigmn = desc_mnmajor_sw128(smem_u32(sO), kHalf);
    const uint64_t dDT = desc_kmajor_sw128(smem_u32(sDT));
    const uint64_t dA0 = desc_kmajor_sw128(smem_u32(ring));
    const uint64_t dB0 = desc_kmajor_sw128(smem_u32(ring + kTileBytes));
    const uint64_t dAmn0 = desc_mnmajor_sw128(smem_u32(ring), kHalf);
    constexpr uint32_t kSlotD = kDqRing >> 4;
    auto ring_wait = [&](int p) {
      return (ok = mbar_wait_warp(&ring_full[p & 1], (p >> 1) & 1, epoch));
    };
    // S_j (into S) from K_j at ring position p, or dP_j (into dP) from V_j.
    auto scores = [&](bool dp, int p) {
      const uint64_t a = dp ? dO : dQ, b = (dp ? dB0 : dA0) + (p & 1) * kSlotD;
      const uint32_t dst = tmem + (dp ? kBColDP : 0u);
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ss(dst, a + kmaj_step(kk), b + kmaj_step(kk), id_kk, kk != 0);
        mma_commit(dp ? dp_full : s_full);
      }
      __syncwarp();
    };
    do {
      if (!(ok = mbar_wait_warp(fix_full, 0, epoch)) || !ring_wait(0)) break;
      tc_fence_after();
      scores(false, 0);
      scores(true, 0);
      for (int j = 0; j < nk; ++j) {
        if (j + 1 < nk) {
          if (!(ok = mbar_wait_warp(s_free, j & 1, epoch)) || !ring_wait(j + 1)) break;
          tc_fence_after();
          scores(false, j + 1);
        }
        if (!(ok = mbar_wait_warp(ds_full, j & 1, epoch))) break;
        tc_fence_after();
        if (elect_one_lane()) {
          const uint64_t b = dAmn0 + (j & 1) * kSlotD;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + kBColAcc, tmem + kBColDP + packed_a_col(kk), b + mnmaj_step(kk), id_kmn,
                        (j | kk) != 0);
          mma_commit(&ring_empty[j & 1]);
        }
        __syncwarp();
        if (j + 1 < nk) scores(true, j + 1);
      }
      if (!ok) break;
      // Tail: dnum M^T (A = dnum16_i K-major, B = M_{s-1} read K-major: row
      // d_k, d_v contiguous) into S; sigma(Q)^T dnum (A = sigma(Q_i) and B =
      // dnum16_i, both MN-major) into dP; sigma(Q)^T dden (B = dden^T,
      // K-major, 16 rows) into 16 columns of its own.
      if (!ring_wait(nk) || !(ok = mbar_wait_warp(fin_ready, 0, epoch))) break;
      tc_fence_after();
      if (elect_one_lane()) {
        const uint32_t so = (nk & 1) * kSlotD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + 0, dA0 + so + kmaj_step(kk), dB0 + so + kmaj_step(kk), id_kk, kk != 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kBColDP, dSigmn + mnmaj_step(kk), dAmn0 + so + mnmaj_step(kk), id_mnmn, kk != 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kBColGz, dSigmn + mnmaj_step(kk), dDT + (((kk >> 2) * kDqDdenT / 2 + (kk & 3) * 32) >> 4),
                      id_gz, kk != 0);
        mma_commit(fin_full);
      }
      __syncwarp();
    } while (false);
  } else {
    // ------------------------------------------------ two threads per query row
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane, c0 = half * 64;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t row = (int64_t)row_q + r;
    const float lse2 = lse[row], dl = delta[row], ddn = dden[row];
    const float g = gate_of(beta[h]), omg = 1.f - g;
    const uint64_t sc2 = f32x2(kScoreScale2, kScoreScale2), nl2 = f32x2(-lse2, -lse2);
    uint32_t sr[64];
    for (int j = 0; j < nk; ++j) {
      const bool diag = j == i;  // key column c is visible to query row r iff c <= r
      if (!(ok = mbar_wait_warp(s_full, j & 1, epoch))) break;
      tc_fence_after();
      tmem_ld32(tl + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait_regs(sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // P = 2^(s log2(e)/sqrt(d) - lse), fp32, in place.
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float x0, x1;
        unpack_f32x2(fma_f32x2(f32x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nl2), x0, x1);
        const float p0 = (diag && c0 + c > r) ? 0.f : ex2(x0);
        const float p1 = (diag && c0 + c + 1 > r) ? 0.f : ex2(x1);
        sr[c] = __float_as_uint(p0);
        sr[c + 1] = __float_as_uint(p1);
      }
      if (!(ok = mbar_wait_warp(dp_full, j & 1, epoch))) break;
      tc_fence_after();
      uint32_t pk[32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dp[32];
        tmem_ld32(tl + kBColDP + c0 + ch * 32, dp);
        tmem_ld_wait_regs(dp);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float d0 = __uint_as_float(sr[ch * 32 + c]) * fmaf(omg, __uint_as_float(dp[c]), -dl);
          const float d1 = __uint_as_float(sr[ch * 32 + c + 1]) * fmaf(omg, __uint_as_float(dp[c + 1]), -dl);
          pk[(ch * 32 + c) >> 1] = pack_bf16x2(d0, d1);
        }
      }
      // dS over the first 32 columns of this half's dP (read above).
      tmem_st16(tl + kBColDP + c0, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(tl + kBColDP + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    // sigma(Q_i) over dO_i (every dP MMA, its only reader, has completed: this
    // thread saw dp_full of the last tile) and dden^T, for the tail MMAs.
    if (ok) ok = mbar_wait_warp(fix_full, 0, epoch);
    if (ok) {
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        const uint32_t off = sw128_offset(r, c0 + 8 * q8, 128);
        float qv[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + off), qv);
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) w[t] = pack_bf16x2(elu1(qv[2 * t]), elu1(qv[2 * t + 1]));
        *reinterpret_cast<uint4*>(sO + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      // dden^T: row 0 holds dden of the tile's 128 queries, rows 1..15 zero.
      const int tid = threadIdx.x - 64;  // 0..255
      if (tid < (int)(kDqDdenT / 16) - 16)
        *reinterpret_cast<uint4*>(sDT + sw128_offset(1 + tid / 16, (tid % 16) * 8, 16)) = make_uint4(0u, 0u, 0u, 0u);
      if (half == 0)
        *reinterpret_cast<__nv_bfloat16*>(sDT + sw128_offset(0, r, 16)) = __float2bfloat16_rn(ddn);
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(fin_ready);
    // Epilogue: dq = dQ / sqrt(d) + (dnum M^T + z dden) * sigma'(q); the
    // state terms added into G and Gz (TMEM lane = d_k index r). dq and this
    // tile's share of G are staged as fp32 in ring stages 0 and 1 (every MMA
    // is done with them) and leave by a TMA store and a TMA reduce-add.
    if (ok) ok = mbar_wait_warp(fin_full, 0, epoch);
    // The G share first (a copy out of TMEM): its reduce-add reads shared
    // memory out while the threads form and stage dq.
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        const int col = c0 + cb * 16;
        uint32_t gm[16];
        tmem_ld16(tl + kBColDP + col, gm);
        tmem_ld_wait_regs(gm);
#pragma unroll
        for (int t = 0; t < 16; t += 4)
          *reinterpret_cast<float4*>(ring + kDqRing + sw128_f32_offset(r, col + t)) =
              make_float4(__uint_as_float(gm[t]), __uint_as_float(gm[t + 1]), __uint_as_float(gm[t + 2]),
                          __uint_as_float(gm[t + 3]));
      }
      fence_proxy_async_smem();
    }
    // Every compute thread has written its rows of the G share (or none has:
    // it is skipped); one thread adds the tile (rows d_k of segment seg) into G.
    const bool g_ok = named_bar_and(1, 256, ok);
    if (g_ok && threadIdx.x == 64) {
      for (int b = 0; b < 4; ++b) tma_reduce_add_2d(&tmG, b * 32, seg * kD, ring + kDqRing + b * 16384);
      bulk_commit_group();
    }
    ok = g_ok;
    if (ok) {
      const float* z = sz;  // z_{s-1}, in shared memory since fix_full
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        const int col = c0 + cb * 16;
        uint32_t a[16], t2[16];
        tmem_ld16(tl + kBColAcc + col, a);
        tmem_ld16(tl + col, t2);
        tmem_ld_wait_regs(a);
        tmem_ld_wait_regs(t2);
        float qv[16];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + sw128_offset(r, col, 128)),
                      *reinterpret_cast<float(*)[8]>(&qv[0]));
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + sw128_offset(r, col + 8, 128)),
                      *reinterpret_cast<float(*)[8]>(&qv[8]));
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          const float4 zz = *reinterpret_cast<const float4*>(z + col + t);
          const float zv[4] = {zz.x, zz.y, zz.z, zz.w};
          float o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[e] = fmaf(__uint_as_float(a[t + e]), kInvSqrtD,
                        fmaf(zv[e], ddn, __uint_as_float(t2[t + e])) * dsigma_tc(qv[t + e]));
          *reinterpret_cast<float4*>(ring + sw128_f32_offset(r, col + t)) = make_float4(o[0], o[1], o[2], o[3]);
        }
      }
      if (half == 0) {
        uint32_t gzv[16];
        tmem_ld16(tl + kBColGz, gzv);
        tmem_ld_wait_regs(gzv);
        atomicAdd(Gz + (int64_t)seg * kD + r, __uint_as_float(gzv[0]));
      }
      fence_proxy_async_smem();
    }
    // The same for dq; then the storing thread waits until both tiles are read.
    const bool all_ok = named_bar_and(1, 256, ok);
    if (threadIdx.x == 64) {
      if (all_ok) {
        for (int b = 0; b < 4; ++b) tma_store_2d(&tmDQ, b * 32, row_q, ring + b * 16384);
        bulk_commit_group();
      }
      bulk_wait_read_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: this CTA's own copies (both parities of an armed barrier;
    // one of them is complete) and MMAs finish before exit.
    if (warp == 0 && lane == 0) {
      if (armed & 1u) mbar_drain(fix_full, 0);
      for (int b = 0; b < 2; ++b)
        if ((armed >> (1 + b)) & 1u) mbar_drain(&ring_full[b], 0), mbar_drain(&ring_full[b], 1);
    }
    if (warp == 1) {
      if (elect_one_lane()) {
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ dK, dV
// CTA = (segment, key tile j). Shared memory: K_j | V_j | ring of two stages
// (Q_i | dO_i | lse_i | Delta_i) | barriers, for the query tiles i = j ..
// n_qt - 1, then sigma(K_j) (bf16, written by the threads while they wait
// for the first S^T). TMEM: S^T 0..127 (P^T over it), dP^T 128..255 (dS^T
// over it), dV 256..383, dK 384..511; after the loop X = sigma(K_j) G_s at
// 0..127 and Y = V_j G_s^T at 128..255, with G_s (bf16) written by the
// threads into ring stage 0.
// MMA order per query tile: dV += P^T dO once P^T is written, S^T of the
// next tile, dK += dS^T Q once dS^T is written, dP^T of the next tile.
// The TMA warp copies G_s (fp32) into ring stage 1 as soon as the loop's
// last use of that stage ends; the threads turn it into bf16 from there. The
// outputs leave through shared memory: each thread writes its row of dk and
// dv into fp32 tiles in the 128-byte swizzle (dv over stage 0, dk over stage
// 1, both free once X and Y are done) and one thread stores them with TMA
// tensor stores, so the 2 x 64 KB per CTA reach global memory as whole
// coalesced rows.
constexpr uint32_t kKvStage = 2 * kTileBytes + 1024;
static_assert(kKvStage >= kD * kD * 4 + kD * 4, "ring stage 1 holds G_s and Gz_s (fp32)");
constexpr uint32_t kKvSig = 2 * kTileBytes + 2 * kKvStage;  // sigma(K_j)
constexpr uint32_t kKvSmem = kKvSig + kTileBytes + 256;
static_assert(kKvSmem <= 232448, "dK/dV kernel shared memory");
static_assert(kKvStage % 1024 == 0, "stages stay 1024-byte aligned for the swizzled tiles");

__global__ void __launch_bounds__(kBwdTcThreads, 1)
tc_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                 const float* __restrict__ beta, const float* __restrict__ lse, const float* __restrict__ delta,
                 const float* __restrict__ G, const float* __restrict__ Gz, int L, int N, int S, int H,
                 int n_segs, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sK = smem_raw;
  uint8_t* sV = smem_raw + kTileBytes;
  uint8_t* ring = smem_raw + 2 * kTileBytes;
  uint8_t* sSig = smem_raw + kKvSig;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kKvSig + kTileBytes);
  uint64_t* fix_full = bars + 0;     // K_j and V_j (TMA)
  uint64_t* ring_full = bars + 1;    // [2] TMA
  uint64_t* ring_empty = bars + 3;   // [2] MMAs done with the stage
  uint64_t* st_full = bars + 5;      // S^T done
  uint64_t* dpt_full = bars + 6;     // dP^T done
  uint64_t* p_full = bars + 7;       // P^T written (8 warps)
  uint64_t* ds_full = bars + 8;      // dS^T written (8 warps)
  uint64_t* loop_done = bars + 9;    // every MMA of the loop done: ring stages free
  uint64_t* fin_ready = bars + 10;   // sigma(K_j) and G_s written (8 warps)
  uint64_t* fin_full = bars + 11;    // X and Y done
  uint64_t* drain = bars + 12;       // abort path
  uint64_t* g_full = bars + 13;      // G_s in ring stage 1 (bulk copy)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = N / kTile;
  const int seg = blockIdx.x / n_qt, j = blockIdx.x - seg * n_qt;
  const int nq = n_qt - j;
  const int bh = seg / S, s = seg - bh * S, h = bh % H;
  const int row_seg = bh * L + s * N, row_k = row_seg + j * kTile;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 14; ++b) mbar_init(&bars[b], (b == 7 || b == 8 || b == 10) ? 8 : 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  uint32_t armed = 0;
  [[maybe_unused]] uint32_t trn = 0;  // tracing build: CTA 0 records channels 0 (TMA), 1 (MMA), 3 (warp 2)

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (elect_one_lane()) {
      mbar_arrive_expect_tx(fix_full, 2 * kTileBytes);
      load_tile(sK, &tmK, row_k, fix_full);
      load_tile(sV, &tmV, row_k, fix_full);
    }
    __syncwarp();
    armed |= 1u;
    for (int t = 0; t < nq && ok; ++t) {
      const int slot = t & 1, use = t >> 1;
      if (use > 0 && !(ok = mbar_wait_warp(&ring_empty[slot], (use - 1) & 1, epoch))) break;
      armed |= 2u << slot;
      if (elect_one_lane()) {
        uint8_t* st = ring + slot * kKvStage;
        const int row_i = row_seg + (j + t) * kTile;
        mbar_arrive_expect_tx(&ring_full[slot], 2 * kTileBytes + 1024);
        load_tile(st, &tmQ, row_i, &ring_full[slot]);
        load_tile(st + kTileBytes, &tmO, row_i, &ring_full[slot]);
        bulk_load(st + 2 * kTileBytes, lse + row_i, 512, &ring_full[slot]);
        bulk_load(st + 2 * kTileBytes + 512, delta + row_i, 512, &ring_full[slot]);
      }
      __syncwarp();
      TC_TRACE(trn, 0, 1, t);
    }
    // G_s (fp32, 64 KB) into stage 1 once the loop's last MMA reading it is done.
    const int uses1 = nq / 2;  // tiles t = 1, 3, ... use stage 1
    if (ok && uses1 > 0) ok = mbar_wait_warp(&ring_empty[1], (uses1 - 1) & 1, epoch);
    if (ok) {
      armed |= 8u;
      if (elect_one_lane()) {
        uint8_t* d = ring + kKvStage;
        const float* gsrc = G + (int64_t)seg * kD * kD;
        mbar_arrive_expect_tx(g_full, kD * kD * 4 + kD * 4);
        for (int c = 0; c < 4; ++c) bulk_load(d + c * 16384, gsrc + c * 4096, 16384, g_full);
        bulk_load(d + kD * kD * 4, Gz + (int64_t)seg * kD, kD * 4, g_full);  // Gz_s after G_s
      }
      __syncwarp();
      TC_TRACE(trn, 0, 2, 0);
    }
    TC_TRACE_END(trn, 0);
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    const uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
    const uint32_t id_kmn = idesc_bf16_f32(128, 128, false, true);
    const uint64_t dK = desc_kmajor_sw128(smem_u32(sK));
    const uint64_t dV = desc_kmajor_sw128(smem_u32(sV));
    const uint64_t dQ0 = desc_kmajor_sw128(smem_u32(ring));
    const uint64_t dO0 = desc_kmajor_sw128(smem_u32(ring + kTileBytes));
    const uint64_t dQmn0 = desc_mnmajor_sw128(smem_u32(ring), kHalf);
    const uint64_t dOmn0 = desc_mnmajor_sw128(smem_u32(ring + kTileBytes), kHalf);
    const uint64_t dSig = desc_kmajor_sw128(smem_u32(sSig));
    constexpr uint32_t kStageD = kKvStage >> 4;
    auto ring_wait = [&](int t) {
      return (ok = mbar_wait_warp(&ring_full[t & 1], (t >> 1) & 1, epoch));
    };
    // S^T = K_j Q_i^T, or dP^T = V_j dO_i^T, for the query tile in stage t & 1.
    auto scores = [&](bool dp, int t) {
      const uint64_t a = dp ? dV : dK, b = (dp ? dO0 : dQ0) + (t & 1) * kStageD;
      const uint32_t dst = tmem + (dp ? kBColDP : 0u);
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ss(dst, a + kmaj_step(kk), b + kmaj_step(kk), id_kk, kk != 0);
        mma_commit(dp ? dpt_full : st_full);
      }
      __syncwarp();
    };
    do {
      if (!(ok = mbar_wait_warp(fix_full, 0, epoch)) || !ring_wait(0)) break;
      TC_TRACE(trn, 1, 9, 0);
      tc_fence_after();
      scores(false, 0);
      scores(true, 0);
      for (int t = 0; t < nq; ++t) {
        const uint32_t so = (t & 1) * kStageD;
        TC_TRACE(trn, 1, 10, t);
        if (!(ok = mbar_wait_warp(p_full, t & 1, epoch))) break;
        TC_TRACE(trn, 1, 11, t);
        tc_fence_after();
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + kBColAcc, tmem + packed_a_col(kk), dOmn0 + so + mnmaj_step(kk), id_kmn,
                        (t | kk) != 0);
        }
        __syncwarp();
        if (t + 1 < nq) {
          if (!ring_wait(t + 1)) break;
          tc_fence_after();
          scores(false, t + 1);
        }
        TC_TRACE(trn, 1, 12, t);
        if (!(ok = mbar_wait_warp(ds_full, t & 1, epoch))) break;
        TC_TRACE(trn, 1, 13, t);
        tc_fence_after();
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + kBColAcc2, tmem + kBColDP + packed_a_col(kk), dQmn0 + so + mnmaj_step(kk), id_kmn,
                        (t | kk) != 0);
          mma_commit(&ring_empty[t & 1]);
        }
        __syncwarp();
        if (t + 1 < nq) scores(true, t + 1);
      }
      if (!ok) break;
      if (elect_one_lane()) mma_commit(loop_done);
      __syncwarp();
      TC_TRACE(trn, 1, 14, 0);
      // X = sigma(K_j) G_s (B = G_s MN-major: row d_k, d_v contiguous) and
      // Y = V_j G_s^T (B = G_s K-major, in ring stage 0).
      if (!(ok = mbar_wait_warp(fin_ready, 0, epoch))) break;
      tc_fence_after();
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + 0, dSig + kmaj_step(kk), dOmn0 + mnmaj_step(kk), id_kmn, kk != 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kBColDP, dV + kmaj_step(kk), dO0 + kmaj_step(kk), id_kk, kk != 0);
        mma_commit(fin_full);
      }
      __syncwarp();
      TC_TRACE(trn, 1, 15, 0);
    } while (false);
    TC_TRACE_END(trn, 1);
  } else {
    // ------------------------------------------------ two threads per key row
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane, c0 = half * 64;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float g = gate_of(beta[h]), omg = 1.f - g;
    const uint64_t sc2 = f32x2(kScoreScale2, kScoreScale2);
    [[maybe_unused]] const bool traced = warp == 2;
    // sigma(K_j), row r, this half's 64 columns, while the first S^T is computed.
    if ((ok = mbar_wait_warp(fix_full, 0, epoch))) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t off = sw128_offset(r, c0 + 8 * q, 128);
        float kv[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + off), kv);
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) w[t] = pack_bf16x2(elu1(kv[2 * t]), elu1(kv[2 * t + 1]));
        *reinterpret_cast<uint4*>(sSig + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    uint32_t sr[64];
    for (int t = 0; t < nq && ok; ++t) {
      if (traced) TC_TRACE(trn, 3, 20, t);
      const bool diag = t == 0;  // key row r is visible to query column c iff r <= c
      const float* sl = reinterpret_cast<const float*>(ring + (t & 1) * kKvStage + 2 * kTileBytes) + c0;
      const float* sd = sl + 128;
      if (!(ok = mbar_wait_warp(&ring_full[t & 1], (t >> 1) & 1, epoch) &&
                 mbar_wait_warp(st_full, t & 1, epoch)))
        break;
      if (traced) TC_TRACE(trn, 3, 21, t);
      tc_fence_after();
      tmem_ld32(tl + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait_regs(sr);
      // P^T = 2^(s log2(e)/sqrt(d) - lse_c), fp32 in place; bf16 pairs over
      // the first 32 columns of this half.
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(sl + c);
        float x0, x1, x2, x3;
        unpack_f32x2(fma_f32x2(f32x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, f32x2(-l4.x, -l4.y)),
                     x0, x1);
        unpack_f32x2(
            fma_f32x2(f32x2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sc2, f32x2(-l4.z, -l4.w)), x2,
            x3);
        const float p0 = (diag && r > c0 + c) ? 0.f : ex2(x0);
        const float p1 = (diag && r > c0 + c + 1) ? 0.f : ex2(x1);
        const float p2 = (diag && r > c0 + c + 2) ? 0.f : ex2(x2);
        const float p3 = (diag && r > c0 + c + 3) ? 0.f : ex2(x3);
        sr[c] = __float_as_uint(p0);
        sr[c + 1] = __float_as_uint(p1);
        sr[c + 2] = __float_as_uint(p2);
        sr[c + 3] = __float_as_uint(p3);
        pk[c >> 1] = pack_bf16x2(p0, p1);
        pk[(c >> 1) + 1] = pack_bf16x2(p2, p3);
      }
      tmem_st16(tl + c0, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(tl + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (traced) TC_TRACE(trn, 3, 22, t);
      if (!(ok = mbar_wait_warp(dpt_full, t & 1, epoch))) break;
      if (traced) TC_TRACE(trn, 3, 23, t);
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dp[32];
        tmem_ld32(tl + kBColDP + c0 + ch * 32, dp);
        tmem_ld_wait_regs(dp);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(sd + ch * 32 + c);
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
          float e[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            e[u] = __uint_as_float(sr[ch * 32 + c + u]) * fmaf(omg, __uint_as_float(dp[c + u]), -dd[u]);
          pk[(ch * 32 + c) >> 1] = pack_bf16x2(e[0], e[1]);
          pk[((ch * 32 + c) >> 1) + 1] = pack_bf16x2(e[2], e[3]);
        }
      }
      tmem_st16(tl + kBColDP + c0, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(tl + kBColDP + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
      if (traced) TC_TRACE(trn, 3, 24, t);
    }
    // G_s as bf16 into ring stage 0 (free once the loop's MMAs are done):
    // row r, this half's 64 columns, in the 128-row SW128 layout.
    if (ok)
      ok = mbar_wait_warp(fix_full, 0, epoch) && mbar_wait_warp(loop_done, 0, epoch) && mbar_wait_warp(g_full, 0, epoch);
    if (traced) TC_TRACE(trn, 3, 30, 0);
    if (ok) {
      uint8_t* sG = ring + kTileBytes;
      const float* grow = reinterpret_cast<const float*>(ring + kKvStage) + r * kD + c0;  // G_s row r (fp32)
#pragma unroll
      for (int q0 = 0; q0 < 8; ++q0) {
        const int q = (q0 + lane) & 7;  // rotated, so the lanes' rows spread over the banks
        const uint32_t off = sw128_offset(r, c0 + 8 * q, 128);
        const float4 g0 = *reinterpret_cast<const float4*>(grow + 8 * q);
        const float4 g1 = *reinterpret_cast<const float4*>(grow + 8 * q + 4);
        *reinterpret_cast<uint4*>(sG + off) = make_uint4(pack_bf16x2(g0.x, g0.y), pack_bf16x2(g0.z, g0.w),
                                                         pack_bf16x2(g1.x, g1.y), pack_bf16x2(g1.z, g1.w));
      }
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(fin_ready);
    if (traced) TC_TRACE(trn, 3, 31, 0);
    // Epilogue: dv = (1 - g) dV + X, dk = dK / sqrt(d) + (Y + Gz) * sigma'(k),
    // staged in shared memory (X and Y done: the ring is free) for the TMA
    // stores.
    if (ok) ok = mbar_wait_warp(fin_full, 0, epoch);
    if (traced) TC_TRACE(trn, 3, 32, 0);
    // dv first: its TMA stores read shared memory out while the threads
    // stage dk.
    uint8_t* sdv = ring;
    uint8_t* sdk = ring + kKvStage;
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        const int col = c0 + cb * 16;
        uint32_t av[16], x[16];
        tmem_ld16(tl + kBColAcc + col, av);
        tmem_ld16(tl + col, x);
        tmem_ld_wait_regs(av);
        tmem_ld_wait_regs(x);
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          float ov[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) ov[e] = fmaf(omg, __uint_as_float(av[t + e]), __uint_as_float(x[t + e]));
          *reinterpret_cast<float4*>(sdv + sw128_f32_offset(r, col + t)) = make_float4(ov[0], ov[1], ov[2], ov[3]);
        }
      }
      fence_proxy_async_smem();
    }
    // Every compute thread has written its rows of dv (or none has: the
    // stores are skipped); one thread stores the tile.
    const bool dv_ok = named_bar_and(1, 256, ok);
    if (dv_ok && threadIdx.x == 64) {
      for (int b = 0; b < 4; ++b) tma_store_2d(&tmDV, b * 32, row_k, sdv + b * 16384);
      bulk_commit_group();
    }
    ok = dv_ok;
    if (ok) {
      const float* gz = reinterpret_cast<const float*>(ring + kKvStage + kD * kD * 4);  // Gz_s (bulk copy)
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        const int col = c0 + cb * 16;
        uint32_t ak[16], y[16];
        tmem_ld16(tl + kBColAcc2 + col, ak);
        tmem_ld16(tl + kBColDP + col, y);
        tmem_ld_wait_regs(ak);
        tmem_ld_wait_regs(y);
        float kv[16];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + sw128_offset(r, col, 128)),
                      *reinterpret_cast<float(*)[8]>(&kv[0]));
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + sw128_offset(r, col + 8, 128)),
                      *reinterpret_cast<float(*)[8]>(&kv[8]));
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          const float4 z4 = *reinterpret_cast<const float4*>(gz + col + t);
          const float zv[4] = {z4.x, z4.y, z4.z, z4.w};
          float ok2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            ok2[e] = fmaf(__uint_as_float(ak[t + e]), kInvSqrtD,
                          (__uint_as_float(y[t + e]) + zv[e]) * dsigma_tc(kv[t + e]));
          *reinterpret_cast<float4*>(sdk + sw128_f32_offset(r, col + t)) = make_float4(ok2[0], ok2[1], ok2[2], ok2[3]);
        }
      }
      fence_proxy_async_smem();
    }
    if (traced) TC_TRACE(trn, 3, 34, 0);
    // The same for dk; then the storing thread waits until both tiles are read.
    const bool all_ok = named_bar_and(1, 256, ok);
    if (traced) TC_TRACE(trn, 3, 35, 0);
    if (threadIdx.x == 64) {
      if (all_ok) {
        for (int b = 0; b < 4; ++b) tma_store_2d(&tmDK, b * 32, row_k, sdk + b * 16384);
        bulk_commit_group();
      }
      bulk_wait_read_all();
    }
    if (traced) TC_TRACE(trn, 3, 33, 0);
    if (traced) TC_TRACE_END(trn, 3);
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    if (warp == 0 && lane == 0) {
      if (armed & 1u) mbar_drain(fix_full, 0);
      for (int b = 0; b < 2; ++b)
        if ((armed >> (1 + b)) & 1u) mbar_drain(&ring_full[b], 0), mbar_drain(&ring_full[b], 1);
      if (armed & 8u) mbar_drain(g_full, 0);
    }
    if (warp == 1) {
      if (elect_one_lane()) {
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace infini
