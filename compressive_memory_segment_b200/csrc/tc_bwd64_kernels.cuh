// Tensor-core backward for bf16 I/O with head dimension 64 and 64-token
// segments (the "Hugging Face Infini-Attention reproduction analysis" page's
// reproduction shape), an even number of segments per sequence. The
// gradients are the ones tc_bwd_kernels.cuh lists (the chain rule through
// Local Attention, Memory Retrieval, Integration, Memory Update and State
// Transfer on that page).
//
// As in the single-pass forward, a CTA takes a pair of segments (a = 2t,
// b = 2t + 1) as one 128-row tile: rows 0-63 are segment a's tokens, rows
// 64-127 segment b's. Operands that mix the two segments are block-diagonal
// 128 x 128 tiles (the other segment's block zero), so each MMA keeps the
// segments apart. Two launches:
//
//   tc_bwd64_pair_kernel, per pair: S = Q K^T and dP = dO V^T; each thread
//     (one row) takes the exact softmax of its row over the <= 64 keys it
//     sees, P into shared memory; sigma(Q) block-diagonal, then R = sigma(Q)
//     [M_{a-1}; M_{b-1}] and O = P V; per row den = sigma(q).z_{s-1}, Delta,
//     dnum = g dout / den, dden, dbeta and dS = P ((1 - g) dP - Delta); then
//     dQ = dS K, dnum [M_{a-1}^T; M_{b-1}^T] (block-diagonal dnum), dK =
//     dS^T Q, dV = P^T dO and sigma(Q)^T dnum (whose diagonal blocks are each
//     segment's share of the gradient reaching M_{s-1}). It writes dq, the
//     local parts of dk and dv, and G[s] of both segments by TMA stores from
//     shared memory, and Gz[s] (summed over the segment's rows in a fixed
//     order, so every output but dbeta is the same bits on every call).
//   (bwd_rscan_kernel turns G, Gz into G_s, Gz_s: the gradient reaching M_s.)
//   tc_bwd64_state_kernel, per pair: dv += sigma(K) G_s and
//     dk += (V G_s^T + Gz_s) sigma'(k), block-diagonal in the same way.
//
// Roles: warps 0-3 one row per thread (thread 0 also issues the pair
// kernel's TMA stores); warp 4 issues the TMA loads and the MMAs (one elected
// lane) and owns TMEM. Every wait is bounded; on a
// timeout the CTA drains its copies and MMAs and frees its TMEM.
#pragma once

namespace infini {
namespace tc {

constexpr int kB64Threads = 160;
constexpr float kB64Scale2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
constexpr float kB64InvSqrtD = 0.125f;

// Shared memory of the pair kernel (128-row x 64-column SW128 tiles of
// kBlk64 bytes; block-diagonal tiles are two of them, columns 0-63 | 64-127):
constexpr uint32_t kB64Q = 0, kB64K = kBlk64, kB64V = 2 * kBlk64, kB64O = 3 * kBlk64;  // Q, K, V, dO
constexpr uint32_t kB64SQ = 4 * kBlk64;   // sigma(Q), block-diagonal
constexpr uint32_t kB64P = 6 * kBlk64;    // P, block-diagonal
constexpr uint32_t kB64DS = 8 * kBlk64;   // dS, block-diagonal
constexpr uint32_t kB64DN = 10 * kBlk64;  // dnum, block-diagonal
constexpr uint32_t kB64MS = 12 * kBlk64;  // [M_{a-1}; M_{b-1}]: rows (segment, d_k), columns d_v
constexpr uint32_t kB64MC = 13 * kBlk64;  // [M_{a-1} | M_{b-1}]: rows d_k, columns (segment, d_v)
// (After the last MMAs, [kB64K, kB64K + 128 KB) holds the staged fp32 dq, dk,
// dv and G tiles, 32 KB each.)
constexpr uint32_t kB64GZ = 14 * kBlk64;  // dden of the pair's 128 rows, fp32
constexpr uint32_t kB64Z = kB64GZ + 512;    // z_{a-1}, z_{b-1} [2][64] fp32 (bulk copy)
constexpr uint32_t kB64Bars = kB64Z + 512;
constexpr uint32_t kB64Smem = kB64Bars + 128;
static_assert(kB64Smem <= 232448, "d = 64 backward pair kernel shared memory");

// TMEM columns. Before dS: S 0..127, dP 128..255, R 256..319, O 320..383.
// After: dQ 0..63, dnum M^T 64..127, dK 128..191, dV 192..255, sigma(Q)^T
// dnum 256..383.
constexpr uint32_t kB64ColR = 256, kB64ColO = 320;

// Row r (64 bf16 values) of a 128-row x 64-column SW128 tile as floats.
__device__ __forceinline__ void ld_row64(const uint8_t* tile, int r, float (&f)[64]) {
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const uint4 x = *reinterpret_cast<const uint4*>(tile + sw128_offset(r, c8 * 8, 128));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      f[c8 * 8 + 2 * t] = __uint_as_float(w[t] << 16);
      f[c8 * 8 + 2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
    }
  }
}

// Row r of a block-diagonal 128 x 128 tile: the 64 values v (rounded to bf16)
// in block `blk`, zeros in the other block.
__device__ __forceinline__ void st_row_bd(uint8_t* tile, int r, int blk, const float (&v)[64]) {
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const uint4 x = make_uint4(pack_bf16x2(v[c8 * 8], v[c8 * 8 + 1]), pack_bf16x2(v[c8 * 8 + 2], v[c8 * 8 + 3]),
                               pack_bf16x2(v[c8 * 8 + 4], v[c8 * 8 + 5]), pack_bf16x2(v[c8 * 8 + 6], v[c8 * 8 + 7]));
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, blk * 64 + c8 * 8, 128)) = x;
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, (blk ^ 1) * 64 + c8 * 8, 128)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Columns 32 hf .. 32 hf + 31 of row r of a 128-row SW128 tile as floats.
__device__ __forceinline__ void ld_half32(const uint8_t* tile, int r, int hf, float (&f)[32]) {
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    const uint4 x = *reinterpret_cast<const uint4*>(tile + sw128_offset(r, hf * 32 + c8 * 8, 128));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      f[c8 * 8 + 2 * t] = __uint_as_float(w[t] << 16);
      f[c8 * 8 + 2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
    }
  }
}

// Columns 32 hf .. + 31 of block `blk` of row r of a block-diagonal tile set
// to v (rounded to bf16), the same columns of the other block to zero.
__device__ __forceinline__ void st_half_bd(uint8_t* tile, int r, int blk, int hf, const float (&v)[32]) {
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    const uint4 x = make_uint4(pack_bf16x2(v[c8 * 8], v[c8 * 8 + 1]), pack_bf16x2(v[c8 * 8 + 2], v[c8 * 8 + 3]),
                               pack_bf16x2(v[c8 * 8 + 4], v[c8 * 8 + 5]), pack_bf16x2(v[c8 * 8 + 6], v[c8 * 8 + 7]));
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, blk * 64 + hf * 32 + c8 * 8, 128)) = x;
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, (blk ^ 1) * 64 + hf * 32 + c8 * 8, 128)) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

// grid: B * H * S / 2 pairs (blockIdx.x = bh * S / 2 + t), 160 threads.
__global__ void __launch_bounds__(kB64Threads, 1)
tc_bwd64_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const __grid_constant__ CUtensorMap tmM128, const __grid_constant__ CUtensorMap tmM64,
                     const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                     const __grid_constant__ CUtensorMap tmDV, const __grid_constant__ CUtensorMap tmG,
                     const float* __restrict__ beta, const float* __restrict__ zp, float* __restrict__ Gz,
                     float* __restrict__ dbeta, int L, int S, int H, int next_stride, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sm = smem_raw;
  float* dds = reinterpret_cast<float*>(sm + kB64GZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kB64Bars);
  uint64_t* tma_full = bars + 0;   // Q, K, V, dO, M tiles (TMA)
  uint64_t* s_ready = bars + 1;    // S, dP done
  uint64_t* sq_ready = bars + 2;   // sigma(Q) block-diagonal written (4 warps)
  uint64_t* p_ready = bars + 3;    // P written (4 warps)
  uint64_t* o_ready = bars + 4;    // R, O done
  uint64_t* ds_ready = bars + 5;   // dS, dnum written, S, dP, R, O read (4 warps)
  uint64_t* fin_ready = bars + 6;  // the last MMAs done
  uint64_t* drain = bars + 7;      // abort path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = S / 2;
  const int bh = blockIdx.x / pairs, t = blockIdx.x - bh * pairs;
  const int h = bh % H;
  const int64_t row0 = (int64_t)bh * L + (int64_t)t * 128;  // token row of the pair's first row
  const int seg0 = bh * S + 2 * t;                          // segment index of a

  if (threadIdx.x == 0) {
    for (int b = 0; b < 8; ++b) mbar_init(&bars[b], (b == 2 || b == 3 || b == 5) ? 4 : 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  bool armed = false;
  [[maybe_unused]] uint32_t n_tr = 0;  // tracing build: CTA 0 records channels 0 (TMA, MMA), 3 (warp 0)

  if (warp == 4) {
    // ------------------------------------------------ TMA and MMA issue
    TC_TRACE(n_tr, 0, 60, 0);
    do {
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(tma_full, 6 * kBlk64 + 512);
        bulk_load(sm + kB64Z, zp + (int64_t)seg0 * 64, 512, tma_full);
        tma_load_2d(sm + kB64Q, &tmQ, 0, (int)row0, tma_full);
        tma_load_2d(sm + kB64K, &tmK, 0, (int)row0, tma_full);
        tma_load_2d(sm + kB64V, &tmV, 0, (int)row0, tma_full);
        tma_load_2d(sm + kB64O, &tmO, 0, (int)row0, tma_full);
        tma_load_2d(sm + kB64MS, &tmM128, 0, seg0 * 64, tma_full);
        tma_load_2d(sm + kB64MC, &tmM64, 0, seg0 * 64, tma_full);
        tma_load_2d(sm + kB64MC + kBlk64 / 2, &tmM64, 0, (seg0 + 1) * 64, tma_full);
        // The pair that should run next on this SM (one CTA per SM, so about
        // next_stride CTAs later): its tiles into L2 while this one computes.
        const int nb = (int)blockIdx.x + next_stride;
        if (next_stride > 0 && nb < (int)gridDim.x) {
          const int nbh = nb / pairs, nt = nb - nbh * pairs;
          const int nrow0 = nbh * L + nt * 128, nseg0 = nbh * S + 2 * nt;
          tma_prefetch_l2_2d(&tmQ, 0, nrow0);
          tma_prefetch_l2_2d(&tmK, 0, nrow0);
          tma_prefetch_l2_2d(&tmV, 0, nrow0);
          tma_prefetch_l2_2d(&tmO, 0, nrow0);
          tma_prefetch_l2_2d(&tmM128, 0, nseg0 * 64);
        }
      }
      __syncwarp();
      armed = true;
      if (!(ok = mbar_wait_warp(tma_full, 0, epoch))) break;
      tc_fence_after();
      TC_TRACE(n_tr, 0, 61, 0);
      const uint32_t id_kk64 = idesc_bf16_f32(128, 128, false, false);  // N = 128
      const uint32_t id_n64_km = idesc_bf16_f32(128, 64, false, true);   // A K-major, B MN-major
      const uint32_t id_n64_kk = idesc_bf16_f32(128, 64, false, false);
      const uint32_t id_n64_mm = idesc_bf16_f32(128, 64, true, true);
      const uint32_t id_n128_mm = idesc_bf16_f32(128, 128, true, true);
      const uint64_t dQk = desc_kmajor_sw128(smem_u32(sm + kB64Q)), dKk = desc_kmajor_sw128(smem_u32(sm + kB64K));
      const uint64_t dVk = desc_kmajor_sw128(smem_u32(sm + kB64V)), dOk = desc_kmajor_sw128(smem_u32(sm + kB64O));
      if (elect_one_lane()) {
        // S = Q K^T and dP = dO V^T (contraction over d = 64: four k-steps in one block).
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tmem, dQk + ((kk * 32) >> 4), dKk + ((kk * 32) >> 4), id_kk64, kk != 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem + 128, dOk + ((kk * 32) >> 4), dVk + ((kk * 32) >> 4), id_kk64, kk != 0);
        mma_commit(s_ready);
      }
      __syncwarp();
      // R = sigma(Q)_bd [M_{a-1}; M_{b-1}] (B MN-major: rows (segment, d_k)).
      if (!(ok = mbar_wait_warp(sq_ready, 0, epoch))) break;
      tc_fence_after();
      TC_TRACE(n_tr, 0, 62, 0);
      if (elect_one_lane()) {
        const uint64_t da = desc_kmajor_sw128(smem_u32(sm + kB64SQ)), db = desc_mnmajor_sw128(smem_u32(sm + kB64MS), kBlk64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kB64ColR, da + (((kk >> 2) * kBlk64 + (kk & 3) * 32) >> 4), db + ((kk * 2048) >> 4),
                      id_n64_km, kk != 0);
      }
      __syncwarp();
      // O = P V (A = P K-major block-diagonal, B = V MN-major: rows keys).
      if (!(ok = mbar_wait_warp(p_ready, 0, epoch))) break;
      tc_fence_after();
      TC_TRACE(n_tr, 0, 63, 0);
      if (elect_one_lane()) {
        const uint64_t da = desc_kmajor_sw128(smem_u32(sm + kB64P)), db = desc_mnmajor_sw128(smem_u32(sm + kB64V), kBlk64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kB64ColO, da + (((kk >> 2) * kBlk64 + (kk & 3) * 32) >> 4), db + ((kk * 2048) >> 4),
                      id_n64_km, kk != 0);
        mma_commit(o_ready);
      }
      __syncwarp();
      if (!(ok = mbar_wait_warp(ds_ready, 0, epoch))) break;
      tc_fence_after();
      TC_TRACE(n_tr, 0, 64, 0);
      if (elect_one_lane()) {
        const uint64_t dS_k = desc_kmajor_sw128(smem_u32(sm + kB64DS)), dS_mn = desc_mnmajor_sw128(smem_u32(sm + kB64DS), kBlk64);
        const uint64_t dP_mn = desc_mnmajor_sw128(smem_u32(sm + kB64P), kBlk64);
        const uint64_t dN_k = desc_kmajor_sw128(smem_u32(sm + kB64DN)), dN_mn = desc_mnmajor_sw128(smem_u32(sm + kB64DN), kBlk64);
        const uint64_t dSQ_mn = desc_mnmajor_sw128(smem_u32(sm + kB64SQ), kBlk64);
        const uint64_t dMC = desc_kmajor_sw128(smem_u32(sm + kB64MC));
        const uint64_t dK_mn = desc_mnmajor_sw128(smem_u32(sm + kB64K), kBlk64);
        const uint64_t dQ_mn = desc_mnmajor_sw128(smem_u32(sm + kB64Q), kBlk64);
        const uint64_t dO_mn = desc_mnmajor_sw128(smem_u32(sm + kB64O), kBlk64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ka = ((kk >> 2) * kBlk64 + (kk & 3) * 32) >> 4, km = (kk * 2048) >> 4;
          // dQ = dS K (B = K MN-major: rows keys)
          mma_bf16_ss(tmem + 0, dS_k + ka, dK_mn + km, id_n64_km, kk != 0);
          // dnum [M_{a-1}^T; M_{b-1}^T] (B = [M_a | M_b] K-major: rows d_k, 64-row blocks)
          mma_bf16_ss(tmem + 64, dN_k + ka, dMC + (((kk >> 2) * (kBlk64 / 2) + (kk & 3) * 32) >> 4), id_n64_kk,
                      kk != 0);
          // dK = dS^T Q and dV = P^T dO (A MN-major: rows queries)
          mma_bf16_ss(tmem + 128, dS_mn + km, dQ_mn + km, id_n64_mm, kk != 0);
          mma_bf16_ss(tmem + 192, dP_mn + km, dO_mn + km, id_n64_mm, kk != 0);
          // sigma(Q)^T dnum (both MN-major: rows queries)
          mma_bf16_ss(tmem + 256, dSQ_mn + km, dN_mn + km, id_n128_mm, kk != 0);
        }
        mma_commit(fin_ready);
      }
      __syncwarp();
      TC_TRACE(n_tr, 0, 65, 0);
    } while (false);
    TC_TRACE_END(n_tr, 0);
  } else {
    // ------------------------------------------------ one row per thread
    const int r = threadIdx.x;   // 0..127, TMEM lane r (warp w reaches lanes 32 w..)
    const int seg = r >> 6, loc = r & 63;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const float g = gate_of(beta[h]), omg = 1.f - g;
    const float* z = reinterpret_cast<const float*>(sm + kB64Z) + seg * 64;  // after tma_full
    float den = 0.f;
    if (warp == 0) TC_TRACE(n_tr, 3, 70, 0);
    if ((ok = mbar_wait_warp(tma_full, 0, epoch))) {
      if (warp == 0) TC_TRACE(n_tr, 3, 71, 0);
      // sigma(q) of the row, block-diagonal, and den = sigma(q).z_{s-1}.
      float sq[64];
      ld_row64(sm + kB64Q, r, sq);
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        sq[c] = elu1(sq[c]);
        den = fmaf(sq[c], z[c], den);
      }
      st_row_bd(sm + kB64SQ, r, seg, sq);
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(sq_ready);
    if (warp == 0) TC_TRACE(n_tr, 3, 72, 0);
    // Exact softmax of the row over the keys of its segment at or before it.
    float p[64];
    if (ok) ok = mbar_wait_warp(s_ready, 0, epoch);
    if (ok) {
      tc_fence_after();
      if (warp == 0) TC_TRACE(n_tr, 3, 73, 0);
      uint32_t s[64];
      tmem_ld32(tl + seg * 64, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tl + seg * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait_regs(s);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) mx = c <= loc ? fmaxf(mx, __uint_as_float(s[c])) : mx;
      float l = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        p[c] = c <= loc ? ex2((__uint_as_float(s[c]) - mx) * kB64Scale2) : 0.f;
        l += p[c];
      }
      const float il = 1.f / l;
#pragma unroll
      for (int c = 0; c < 64; ++c) p[c] *= il;
      st_row_bd(sm + kB64P, r, seg, p);
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(p_ready);
    if (warp == 0) TC_TRACE(n_tr, 3, 74, 0);
    float ddn = 0.f, db = 0.f;
    if (ok) ok = mbar_wait_warp(o_ready, 0, epoch);
    if (ok) {
      tc_fence_after();
      if (warp == 0) TC_TRACE(n_tr, 3, 75, 0);
      const float inv_den = den != 0.f ? 1.f / den : 0.f;
      const float wm = den != 0.f ? g / den : 0.f;
      float sd = 0.f, smm = 0.f;  // dout . A_dot, dout . A_mem
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t o[32], rr[32];
        tmem_ld32(tl + kB64ColO + hf * 32, o);
        tmem_ld32(tl + kB64ColR + hf * 32, rr);
        tmem_ld_wait_regs(o);
        tmem_ld_wait_regs(rr);
        float go[32];
        ld_half32(sm + kB64O, r, hf, go);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sd = fmaf(go[c], __uint_as_float(o[c]), sd);
          smm = fmaf(go[c], __uint_as_float(rr[c]) * inv_den, smm);
        }
        // dnum = g dout / den, block-diagonal.
#pragma unroll
        for (int c = 0; c < 32; ++c) go[c] *= wm;
        st_half_bd(sm + kB64DN, r, seg, hf, go);
      }
      const float dl = omg * sd;
      ddn = -wm * smm;
      db = g * omg * (smm - sd);
      dds[r] = ddn;
      // dS = P ((1 - g) dP - Delta) over the segment's keys.
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t dp[32];
        tmem_ld32(tl + 128 + seg * 64 + hf * 32, dp);
        tmem_ld_wait_regs(dp);
        float ds[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) ds[c] = p[hf * 32 + c] * fmaf(omg, __uint_as_float(dp[c]), -dl);
        st_half_bd(sm + kB64DS, r, seg, hf, ds);
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(ds_ready);
    if (warp == 0) TC_TRACE(n_tr, 3, 76, 0);
    float dbw = db;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dbw += __shfl_xor_sync(0xffffffffu, dbw, o);
    if (ok && lane == 0 && dbw != 0.f) atomicAdd(&dbeta[h], dbw);
    // Gz_s[m] = sum_t sigma(q_t)[m] dden_t over the segment's rows, while the
    // last MMAs run (thread r: segment seg, m = loc). Every row's dden is in
    // shared memory once the four row warps have passed the barrier. The sum
    // takes a fixed order: four partial sums over rows q = u mod 4, then
    // combined.
    ok = named_bar_and(2, 128, ok);
    float gzs = 0.f;
    if (ok) {
      float gz4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int q = 0; q < 64; q += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rq = seg * 64 + q + u;
          const float x =
              __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kB64Q + sw128_offset(rq, loc, 128)));
          gz4[u] = fmaf(elu1(x), dds[rq], gz4[u]);
        }
      }
      gzs = (gz4[0] + gz4[1]) + (gz4[2] + gz4[3]);
      if (warp == 0) TC_TRACE(n_tr, 3, 79, 0);
    }
    // Epilogue: dq, the local dk and dv, G and Gz of the pair's segments.
    // dq, dk, dv and G (rows (segment, d_k)) are staged as fp32 in the tiles
    // the last MMAs have finished reading (K onwards; each 128 rows x 64
    // columns as two 32-column blocks in the 128-byte swizzle) and written by
    // TMA stores: one thread per row storing straight to global memory would
    // touch 32 rows per warp instruction.
    uint8_t* const sdq = sm + kB64K;
    uint8_t* const sdk = sdq + 2 * 16384;
    uint8_t* const sdv = sdk + 2 * 16384;
    uint8_t* const sg = sdv + 2 * 16384;
    if (ok) ok = mbar_wait_warp(fin_ready, 0, epoch);
    if (ok) {
      tc_fence_after();
      if (warp == 0) TC_TRACE(n_tr, 3, 77, 0);
      uint32_t a[32], b2[32];
      // dq and G first: their TMA stores read shared memory out while the
      // threads stage dk and dv.
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        float qv[32];
        ld_half32(sm + kB64Q, r, hf, qv);
        tmem_ld32(tl + hf * 32, a);
        tmem_ld32(tl + 64 + hf * 32, b2);
        tmem_ld_wait_regs(a);
        tmem_ld_wait_regs(b2);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          float o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o4[e] = fmaf(__uint_as_float(a[c + e]), kB64InvSqrtD,
                         fmaf(z[hf * 32 + c + e], ddn, __uint_as_float(b2[c + e])) * dsigma_tc(qv[c + e]));
          *reinterpret_cast<float4*>(sdq + sw128_f32_offset(r, hf * 32 + c)) = make_float4(o4[0], o4[1], o4[2], o4[3]);
        }
        // sigma(Q)^T dnum: lane r is (segment seg, d_k = loc); its segment's block.
        tmem_ld32(tl + 256 + seg * 64 + hf * 32, a);
        tmem_ld_wait_regs(a);
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(sg + sw128_f32_offset(r, hf * 32 + c)) =
              make_float4(__uint_as_float(a[c]), __uint_as_float(a[c + 1]), __uint_as_float(a[c + 2]),
                          __uint_as_float(a[c + 3]));
      }
      fence_proxy_async_smem();
    }
    // Every row thread has staged its rows of dq and G (or none stores: a
    // wait gave up); one thread stores them.
    const bool first_ok = named_bar_and(1, 128, ok);
    if (first_ok && threadIdx.x == 0) {
      for (int b = 0; b < 2; ++b) {
        tma_store_2d(&tmDQ, b * 32, (int)row0, sdq + b * 16384);
        tma_store_2d(&tmG, b * 32, seg0 * 64, sg + b * 16384);
      }
      bulk_commit_group();
    }
    ok = first_ok;
    if (ok) {
      uint32_t a[32], b2[32];
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        tmem_ld32(tl + 128 + hf * 32, a);
        tmem_ld32(tl + 192 + hf * 32, b2);
        tmem_ld_wait_regs(a);
        tmem_ld_wait_regs(b2);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const uint32_t off = sw128_f32_offset(r, hf * 32 + c);
          *reinterpret_cast<float4*>(sdk + off) =
              make_float4(__uint_as_float(a[c]) * kB64InvSqrtD, __uint_as_float(a[c + 1]) * kB64InvSqrtD,
                          __uint_as_float(a[c + 2]) * kB64InvSqrtD, __uint_as_float(a[c + 3]) * kB64InvSqrtD);
          *reinterpret_cast<float4*>(sdv + off) =
              make_float4(omg * __uint_as_float(b2[c]), omg * __uint_as_float(b2[c + 1]),
                          omg * __uint_as_float(b2[c + 2]), omg * __uint_as_float(b2[c + 3]));
        }
      }
      fence_proxy_async_smem();
      Gz[(int64_t)(seg0 + seg) * 64 + loc] = gzs;
      if (warp == 0) TC_TRACE(n_tr, 3, 78, 0);
    }
    // The same for dk and dv; then the storing thread waits until every tile
    // is read.
    const bool all_ok = named_bar_and(1, 128, ok);
    if (threadIdx.x == 0) {
      if (all_ok) {
        for (int b = 0; b < 2; ++b) {
          tma_store_2d(&tmDK, b * 32, (int)row0, sdk + b * 16384);
          tma_store_2d(&tmDV, b * 32, (int)row0, sdv + b * 16384);
        }
        bulk_commit_group();
      }
      bulk_wait_read_all();
    }
    if (warp == 0) TC_TRACE(n_tr, 3, 80, 0);
    if (warp == 0) TC_TRACE_END(n_tr, 3);
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    if (warp == 4) {
      if (elect_one_lane()) {
        if (armed) mbar_drain(tma_full, 0);
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 4) tmem_dealloc(tmem, 512);
}

// Shared memory of the state kernel (80 KB, so that two CTAs share an SM and
// one CTA's copies overlap the other's MMAs and epilogue): sigma(K)
// block-diagonal | V block-diagonal | G_s of both segments in bf16 | barriers.
// The diagonal blocks of K and V arrive by TMA as 64-row boxes straight into
// place (each lands at a multiple of 1024 bytes, so the swizzle matches the
// 128-row tile); the off-diagonal blocks are the contiguous byte range
// [8192, 24576) of each tile and are zeroed by the threads. The G_s tile
// serves both MMAs: as [G_a; G_b] (rows (segment, d_k), columns d_v) read
// MN-major, and as [G_a | G_b] (rows d_k, columns (segment, d_v)) read K-major
// with 64-row column blocks, the two layouts having the same bytes.
constexpr uint32_t kB64sSK = 0, kB64sVB = 2 * kBlk64, kB64sG = 4 * kBlk64;
constexpr uint32_t kB64sBars = kB64sG + kBlk64;
constexpr uint32_t kB64StateSmem = kB64sBars + 64;
static_assert(2 * (kB64StateSmem + 1024) <= 233472, "two d = 64 backward state CTAs per SM");

// grid: B * H * S / 2 pairs, 160 threads, two CTAs per SM: dv += sigma(K) G_s
// and dk += (V G_s^T + Gz_s) sigma'(k) for both segments of the pair. tmK and
// tmV are K and V with 64-row boxes; tmDK and tmDV the fp32 dk and dv with
// 32 x 128 boxes. The increments are staged as fp32 over the sigma(K) and V
// tiles once the MMAs are done with them and added by TMA reduce-adds (each
// element gets one add here), so the SM never reads dk or dv.
__global__ void __launch_bounds__(kB64Threads, 2)
tc_bwd64_state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                      const float* __restrict__ G, const float* __restrict__ Gz, int L, int S, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kB64sBars);
  uint64_t* tma_full = bars + 0;
  uint64_t* op_ready = bars + 1;   // block-diagonal operands written (4 warps)
  uint64_t* fin_ready = bars + 2;
  uint64_t* drain = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = S / 2;
  const int bh = blockIdx.x / pairs, t = blockIdx.x - bh * pairs;
  const int64_t row0 = (int64_t)bh * L + (int64_t)t * 128;
  const int seg0 = bh * S + 2 * t;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bars[b], b == 1 ? 4 : 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  bool armed = false;

  if (warp == 4) {
    do {
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(tma_full, kBlk64 * 2);
        for (int s = 0; s < 2; ++s) {  // segment s: rows 64 s .. 64 s + 63 of column block s
          const uint32_t off = (uint32_t)s * (kBlk64 + 64 * 128);
          tma_load_2d(sm + kB64sSK + off, &tmK, 0, (int)(row0 + 64 * s), tma_full);
          tma_load_2d(sm + kB64sVB + off, &tmV, 0, (int)(row0 + 64 * s), tma_full);
        }
      }
      __syncwarp();
      armed = true;
      if (!(ok = mbar_wait_warp(op_ready, 0, epoch))) break;
      tc_fence_after();
      if (elect_one_lane()) {
        const uint64_t dSK = desc_kmajor_sw128(smem_u32(sm + kB64sSK)), dVB = desc_kmajor_sw128(smem_u32(sm + kB64sVB));
        const uint64_t dGS = desc_mnmajor_sw128(smem_u32(sm + kB64sG), kBlk64);
        const uint64_t dGC = desc_kmajor_sw128(smem_u32(sm + kB64sG));
        const uint32_t id_km = idesc_bf16_f32(128, 64, false, true), id_kk = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ka = ((kk >> 2) * kBlk64 + (kk & 3) * 32) >> 4;
          // X = sigma(K)_bd [G_a; G_b] (B MN-major: rows (segment, d_k))
          mma_bf16_ss(tmem + 0, dSK + ka, dGS + ((kk * 2048) >> 4), id_km, kk != 0);
          // Y = V_bd [G_a^T; G_b^T] (B = [G_a | G_b] K-major: rows d_k, 64-row blocks)
          mma_bf16_ss(tmem + 64, dVB + ka, dGC + (((kk >> 2) * (kBlk64 / 2) + (kk & 3) * 32) >> 4), id_kk, kk != 0);
        }
        mma_commit(fin_ready);
      }
      __syncwarp();
    } while (false);
  } else {
    const int r = threadIdx.x;
    const int seg = r >> 6;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    // Off-diagonal blocks: zeros (16 KB per tile, 128 bytes per thread each).
    {
      const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t off = 8192u + (uint32_t)(j * 128 + r) * 16u;
        *reinterpret_cast<uint4*>(sm + kB64sSK + off) = z4;
        *reinterpret_cast<uint4*>(sm + kB64sVB + off) = z4;
      }
    }
    // G_s of the pair (128 rows (segment, d_k) x 64 columns d_v, 32 KB of
    // fp32, coalesced: piece q = r + 128 j is 8 values of row q / 8) to bf16.
    {
      const float4* g4 = reinterpret_cast<const float4*>(G + (int64_t)seg0 * 4096);
      float4 gv[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        gv[2 * j] = __ldg(g4 + 2 * (r + 128 * j));
        gv[2 * j + 1] = __ldg(g4 + 2 * (r + 128 * j) + 1);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = r + 128 * j;
        const float4 a = gv[2 * j], b = gv[2 * j + 1];
        *reinterpret_cast<uint4*>(sm + kB64sG + sw128_offset(q >> 3, (q & 7) * 8, 128)) =
            make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
      }
    }
    // Row r of K (in block seg of the sigma(K) tile) -> sigma(K) in place;
    // the raw bf16 row stays in registers for sigma'(k).
    uint32_t kraw[32];
    if ((ok = mbar_wait_warp(tma_full, 0, epoch))) {
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint4* p = reinterpret_cast<uint4*>(sm + kB64sSK + sw128_offset(r, seg * 64 + c8 * 8, 128));
        const uint4 x = *p;
        kraw[c8 * 4] = x.x; kraw[c8 * 4 + 1] = x.y; kraw[c8 * 4 + 2] = x.z; kraw[c8 * 4 + 3] = x.w;
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          w[u] = pack_bf16x2(elu1(__uint_as_float(w[u] << 16)), elu1(__uint_as_float(w[u] & 0xffff0000u)));
        *p = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(op_ready);
    uint8_t* const sdv = sm + kB64sSK;  // two 32-column fp32 blocks (32 KB) over sigma(K)
    uint8_t* const sdk = sm + kB64sVB;  // and over V, once the MMAs are done
    if (ok) ok = mbar_wait_warp(fin_ready, 0, epoch);
    if (ok) {
      tc_fence_after();
      const float4* gz4 = reinterpret_cast<const float4*>(Gz + (int64_t)(seg0 + seg) * 64);
      uint32_t x[32], y[32];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        tmem_ld32(tl + hf * 32, x);
        tmem_ld32(tl + 64 + hf * 32, y);
        tmem_ld_wait_regs(x);
        tmem_ld_wait_regs(y);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const int c = c4 * 4, cc = hf * 32 + c;
          const float4 g = __ldg(gz4 + (cc >> 2));
          const uint32_t k01 = kraw[cc >> 1], k23 = kraw[(cc >> 1) + 1];
          const uint32_t off = sw128_f32_offset(r, cc);
          *reinterpret_cast<float4*>(sdv + off) = make_float4(__uint_as_float(x[c]), __uint_as_float(x[c + 1]),
                                                              __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
          *reinterpret_cast<float4*>(sdk + off) =
              make_float4((__uint_as_float(y[c]) + g.x) * dsigma_tc(__uint_as_float(k01 << 16)),
                          (__uint_as_float(y[c + 1]) + g.y) * dsigma_tc(__uint_as_float(k01 & 0xffff0000u)),
                          (__uint_as_float(y[c + 2]) + g.z) * dsigma_tc(__uint_as_float(k23 << 16)),
                          (__uint_as_float(y[c + 3]) + g.w) * dsigma_tc(__uint_as_float(k23 & 0xffff0000u)));
        }
      }
      fence_proxy_async_smem();
    }
    // Every row thread has staged its increments (or none is added: a wait
    // gave up); one thread adds the tiles into dk and dv.
    const bool all_ok = named_bar_and(1, 128, ok);
    if (all_ok && threadIdx.x == 0) {
      for (int b = 0; b < 2; ++b) {
        tma_reduce_add_2d(&tmDV, b * 32, (int)row0, sdv + b * 16384);
        tma_reduce_add_2d(&tmDK, b * 32, (int)row0, sdk + b * 16384);
      }
      bulk_commit_group();
      bulk_wait_read_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    if (warp == 4) {
      if (elect_one_lane()) {
        if (armed) mbar_drain(tma_full, 0);
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 4) tmem_dealloc(tmem, 128);
}

}  // namespace tc
}  // namespace infini
