// Single-pass tensor-core forward for bf16 I/O with head dimension 64 and
// 64-token segments (the "Hugging Face Infini-Attention reproduction
// analysis" page's reproduction shape): one CTA per (b, h) walks that head's
// segments in order, two at a time, and keeps the compressive memory on chip,
// so the state, the prefix over segments and the attention are one launch with
// no workspace traffic:
//
//   per pair of segments (a = 2t, b = 2t + 1) of the CTA's (b, h):
//     S = Q K^T (both segments' 128 queries x 128 keys), block-diagonal
//         causal softmax per row (Infini-Attention mechanism: Local
//         Attention), P V into O;
//     dM = sigma(K)^T V of the two segments as one block-diagonal MMA (Memory
//         Update; sigma = ELU + 1 split in hi + lo bf16 parts, as in the
//         state kernels), dz = column sums of sigma(K);
//     M_{a-1} is the running prefix, M_{b-1} = M_{a-1} + dM_a (State
//         Transfer); both go into the retrieval's B operand as bf16, and the
//         retrieval sigma(Q) M_{s-1} / sigma(Q).z_{s-1} (Memory Retrieval) is
//         folded into O with the block-diagonal c sigma(Q) operand of
//         tc_attn64_kernel, held in TMEM (out = wd * O, or O when g == 1;
//         Integration);
//     the prefix moves on by dM_a + dM_b (fp32, in shared memory).
//   After the last pair the prefix is M_out, z_out (the final state).
//
// The prefix is the plain running sum in the segments' order, the same
// recurrence the scan kernel applies; keeping it in one CTA per (b, h) is what
// makes the pass single: no segment waits on another CTA. That needs B * H
// CTAs to fill the GPU, which the reproduction shape (8 x 12 heads of 16
// segments) has; longer sequences with few heads use the three-kernel path.
//
// Roles (288 threads), so that the state chain of one pair overlaps the
// attention of the pair before it:
//   warps 0-3  attention, one query row of the pair per thread: sigma(q),
//              softmax, den and the c sigma(q) row, the epilogue; thread 0
//              issues the QK^T, P V and retrieval MMAs.
//   warps 4-7  state: sigma(K) hi / lo and dz, the dM MMA (issued by thread
//              128), the prefix rows M_{a-1}^T, M_{b-1}^T as the retrieval's
//              B operand and z_{a-1}, z_{b-1} (double-buffered, so the state
//              group runs up to a pair ahead).
//   warp 8     TMA producer: the pairs' Q, K, V tiles into two stages.
// Every wait is bounded; on a timeout the CTA drains its own copies and MMAs
// and frees its TMEM. With an odd number of segments the last pair's second
// segment does not exist: its rows are computed on whatever the tiles hold
// (finite values: the V blocks start zeroed) and never written, and its dM,
// dz are not added.
#pragma once

namespace infini {
namespace tc {

constexpr int kF64Threads = 288;
// Shared memory, from the 1024-aligned base:
//   stage[2] = Q (16 KB) | K (16 KB) |
//              A0 (16 KB: V_a in token rows 0-63, zeros in 64-127) |
//              A1 (16 KB: zeros in rows 0-63, V_b in 64-127)
//   SG     = sigma_hi | sigma_lo of the pair's keys (16 KB each)
//   MR[2]  = the retrieval's B operand, K-major: rows d_v, block 0 =
//            M_{a-1}^T, block 1 = M_{b-1}^T (8 KB each)
//   PF     = the running prefix M^T in fp32, row d_v (68-float stride)
//   ZR     = the running z prefix [64]; ZS[2] = z_{a-1}, z_{b-1} of a pair
//            [2][2][64]; DZ = dz of the pair [2][64]; ZW = dz partial sums
//            [4 warps][8][8]; barriers.
constexpr uint32_t kF64Stage = 4 * kBlk64;
constexpr uint32_t kF64SG = 2 * kF64Stage;
constexpr uint32_t kF64MR = kF64SG + 2 * kBlk64;
constexpr uint32_t kF64PF = kF64MR + 2 * kBlk64;
constexpr int kF64PFStride = 68;
constexpr uint32_t kF64ZR = kF64PF + 64 * kF64PFStride * 4;
constexpr uint32_t kF64ZS = kF64ZR + 64 * 4;
constexpr uint32_t kF64DZ = kF64ZS + 2 * 2 * 64 * 4;
constexpr uint32_t kF64ZW = kF64DZ + 2 * 64 * 4;
constexpr uint32_t kF64Bars = kF64ZW + 4 * 8 * 8 * 4;
constexpr uint32_t kFused64Smem = kF64Bars + 128;
static_assert(kFused64Smem <= 232448, "fused d = 64 kernel shared memory");
static_assert((kF64MR % 1024) == 0 && (kF64PF % 16) == 0 && (kF64Bars % 8) == 0, "alignment");

// TMEM columns: S (P over its first 64), O, the retrieval's block-diagonal A
// operand (64 columns of bf16 pairs), the pair's dM (hi | lo).
constexpr uint32_t kF64ColO = 128, kF64ColA = 192, kF64ColST = 256;

__global__ void __launch_bounds__(kF64Threads, 1)
tc_fused64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const float* __restrict__ beta,
                  const float* __restrict__ M_in, const float* __restrict__ z_in, __nv_bfloat16* __restrict__ out,
                  float* __restrict__ M_out, float* __restrict__ z_out, int L, int S, int H, int out_v8,
                  uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sm = smem_raw;
  uint8_t* sSG = sm + kF64SG;
  float* PF = reinterpret_cast<float*>(sm + kF64PF);
  float* ZR = reinterpret_cast<float*>(sm + kF64ZR);
  float* ZS = reinterpret_cast<float*>(sm + kF64ZS);
  float* DZ = reinterpret_cast<float*>(sm + kF64DZ);
  float* ZW = reinterpret_cast<float*>(sm + kF64ZW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kF64Bars);
  uint64_t* full = bars + 0;       // [2] the stage's Q, K, V tiles landed
  uint64_t* empty = bars + 2;      // [2] both groups done with the stage (2 arrivals)
  uint64_t* mr_full = bars + 4;    // [2] MR / ZS buffer written (4 state warps)
  uint64_t* mr_empty = bars + 6;   // [2] MR buffer read by the retrieval MMA
  uint64_t* qk_done = bars + 8;    // S = Q K^T done
  uint64_t* st_done = bars + 9;    // dM of the pair done
  uint64_t* o_done = bars + 10;    // P V and the retrieval done
  uint64_t* drain = bars + 11;     // [2] abort path: each issuing thread's MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  constexpr int kNumBars = 13;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int pairs = (S + 1) / 2;
  const int64_t row_base = (int64_t)bh * L;
  [[maybe_unused]] const int64_t rows_total = (int64_t)gridDim.x * L;  // B * H * L: rows of q, k, v, out

  // Zero A0 / A1 of both stages (4 x 16 KB): the off-diagonal halves stay
  // zero, and the V_b rows of a pair without a second segment (never loaded)
  // hold zeros or an earlier pair's values, finite either way, so the zero P
  // columns of segment a's rows multiply finite numbers.
  {
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 4
    for (int w = tid; w < 4 * 1024; w += kF64Threads) {
      const int st = w >> 11, o = (w & 2047) * 16;
      *reinterpret_cast<uint4*>(sm + st * kF64Stage + 2 * kBlk64 + o) = zero;
    }
  }
  // Incoming state: PF row d_v = M_in[:, d_v], ZR = z_in (zeros without them).
  if (tid >= 128 && tid < 192) {
    const int dv = tid - 128;
    const float* mi = M_in ? M_in + (int64_t)bh * kD64 * kD64 : nullptr;
#pragma unroll 4
    for (int k = 0; k < kD64; ++k) PF[dv * kF64PFStride + k] = mi ? __ldg(mi + k * kD64 + dv) : 0.f;
    ZR[dv] = z_in ? __ldg(z_in + (int64_t)bh * kD64 + dv) : 0.f;
  }
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], (b == 2 || b == 3) ? 2u : ((b == 4 || b == 5) ? 4u : 1u));
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  uint32_t armed = 0;  // producer: stages with a copy phase in flight (bit st), for the abort path
  bool mma_issued = false;

  if (warp == 8) {
    // ------------------------------------------------ TMA producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    [[maybe_unused]] uint32_t trn = 0;
    for (int t = 0; t < pairs && ok; ++t) {
      const int st = t & 1;
      // The stage was last used by pair t - 2: both groups must be done with it.
      if (t >= 2 && !(ok = mbar_wait_warp(&empty[st], (uint32_t)((t - 2) >> 1) & 1u, epoch))) break;
      TC_TRACE(trn, 0, 1, t);
      if (elect_one_lane()) {
        uint8_t* base = sm + st * kF64Stage;
        const int row0 = (int)(row_base + 2 * t * kD64);
        const bool hb = 2 * t + 1 < S;
        mbar_arrive_expect_tx(&full[st], 2 * kBlk64 + (hb ? 2u : 1u) * (kBlk64 / 2));
        tma_load_2d(base, &tmQ, 0, row0, &full[st]);
        tma_load_2d(base + kBlk64, &tmK, 0, row0, &full[st]);
        tma_load_2d(base + 2 * kBlk64, &tmV, 0, row0, &full[st]);                           // V_a -> A0 rows 0-63
        if (hb) tma_load_2d(base + 3 * kBlk64 + 64 * 128, &tmV, 0, row0 + 64, &full[st]);  // V_b -> A1 rows 64-127
      }
      __syncwarp();
      armed |= 1u << st;
    }
    TC_TRACE_END(trn, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------ state group
    const int ts = tid - 128, sw = warp - 4;  // thread 0..127 and warp 0..3 of the group
    const int sseg = ts >> 6;
    const uint32_t tl = tmem + ((uint32_t)(sw * 32) << 16);
    [[maybe_unused]] uint32_t trn = 0;
    [[maybe_unused]] const bool traced = sw == 0;  // warp 4: channel 4
    for (int t = 0; t < pairs && ok; ++t) {
      const int st = t & 1, mb = t & 1;
      if (traced) TC_TRACE(trn, 4, 50, t);
      uint8_t* sK = sm + st * kF64Stage + kBlk64;
      uint8_t* sA0 = sm + st * kF64Stage + 2 * kBlk64;
      uint8_t* sMR = sm + kF64MR + mb * kBlk64;
      float* zs = ZS + mb * 128;
      const bool has_b = 2 * t + 1 < S;
      // A failed (bounded) wait does not leave the loop before the group's
      // next barrier: every warp arrives there and they leave together.
      bool w = mbar_wait_warp(&full[st], (uint32_t)(t >> 1) & 1u, epoch);
      if (traced) TC_TRACE(trn, 4, 51, t);
      // sigma(K) as hi + lo parts into SG, and per-column partial sums of
      // sigma for dz: thread ts takes the 16-byte column chunk c8 = ts & 7 of
      // rows 8 rg .. 8 rg + 7 of segment ts >> 6 (rg = (ts >> 3) & 7).
      if (w) {
        const int c8 = ts & 7, rg = (ts >> 3) & 7;
        float zacc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) zacc[q] = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t off = sw128_offset(sseg * 64 + rg * 8 + q, c8 * 8, 128);
          uint4 hi, lo;
          sigma8_split(*reinterpret_cast<const uint4*>(sK + off), hi, lo, zacc);
          *reinterpret_cast<uint4*>(sSG + off) = hi;
          *reinterpret_cast<uint4*>(sSG + kBlk64 + off) = lo;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 8);
          zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 16);
        }
        if (lane < 8) {
#pragma unroll
          for (int q = 0; q < 8; ++q) ZW[(sw * 8 + c8) * 8 + q] = zacc[q];
        }
      }
      fence_proxy_async_smem();
      if (traced) TC_TRACE(trn, 4, 52, t);
      if (!(ok = named_bar_and(1, 128, w))) break;
      if (traced) TC_TRACE(trn, 4, 53, t);
      if (ts == 0) {
        // dM^T of both segments: A = [V_a^T 0; 0 V_b^T] (A0 | A1, MN-major),
        // B = [sigma_hi | sigma_lo] (MN-major), D rows 0-63 segment a, 64-127 b.
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(128, 128, true, true);
        const uint64_t da = desc_mnmajor_sw128(smem_u32(sA0), kBlk64);
        const uint64_t dsg = desc_mnmajor_sw128(smem_u32(sSG), kBlk64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kF64ColST, da + ((kk * 2048) >> 4), dsg + ((kk * 2048) >> 4), id, kk != 0);
        mma_commit(st_done);
        mma_issued = true;
      }
      {
        const int rl = ts & 63;
        DZ[ts] = ZW[((2 * sseg) * 8 + (rl >> 3)) * 8 + (rl & 7)] + ZW[((2 * sseg + 1) * 8 + (rl >> 3)) * 8 + (rl & 7)];
      }
      // MR / ZS buffer mb was last read by the retrieval of pair t - 2.
      w = t < 2 || mbar_wait_warp(&mr_empty[mb], (uint32_t)((t - 2) >> 1) & 1u, epoch);
      w = w && mbar_wait_warp(st_done, (uint32_t)t & 1u, epoch);
      float dmr[64];
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < 4 && w; ++cb) {
        uint32_t rh[16], rlo[16];
        tmem_ld16(tl + kF64ColST + cb * 16, rh);
        tmem_ld16(tl + kF64ColST + 64 + cb * 16, rlo);
        tmem_ld_wait_regs(rh);
        tmem_ld_wait_regs(rlo);
#pragma unroll
        for (int q = 0; q < 16; ++q) dmr[cb * 16 + q] = __uint_as_float(rh[q]) + __uint_as_float(rlo[q]);
      }
      if (traced) TC_TRACE(trn, 4, 54, t);
      if (!(ok = named_bar_and(1, 128, w))) break;  // DZ complete
      if (ts < 64) {
        // Row d_v = ts of M_{a-1}^T (PF) and M_{b-1}^T = M_{a-1}^T + dM_a^T
        // as bf16 rows of MR; PF moves to M_{b-1}^T. z_{a-1} = ZR and
        // z_{b-1} = ZR + dz_a for the den of the pair's rows.
        float* prow = PF + ts * kF64PFStride;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {  // 8 d_k at a time: one 16-byte chunk of each MR block
          const float4 p0 = *reinterpret_cast<const float4*>(prow + cb * 8);
          const float4 p1 = *reinterpret_cast<const float4*>(prow + cb * 8 + 4);
          const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          float nb[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) nb[q] = pv[q] + dmr[cb * 8 + q];
          const uint32_t off = sw128_offset(ts, cb * 8, 64);
          *reinterpret_cast<uint4*>(sMR + off) = make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]),
                                                            pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
          *reinterpret_cast<uint4*>(sMR + kBlk64 / 2 + off) = make_uint4(
              pack_bf16x2(nb[0], nb[1]), pack_bf16x2(nb[2], nb[3]), pack_bf16x2(nb[4], nb[5]), pack_bf16x2(nb[6], nb[7]));
          *reinterpret_cast<float4*>(prow + cb * 8) = make_float4(nb[0], nb[1], nb[2], nb[3]);
          *reinterpret_cast<float4*>(prow + cb * 8 + 4) = make_float4(nb[4], nb[5], nb[6], nb[7]);
        }
        const float zr = ZR[ts];
        zs[ts] = zr;
        zs[64 + ts] = zr + DZ[ts];
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      // The prefix moves past segment b; z likewise.
      if (ts >= 64 && has_b) {
        float* prow = PF + (ts - 64) * kF64PFStride;
#pragma unroll
        for (int cb = 0; cb < 16; ++cb) {
          float4 p = *reinterpret_cast<const float4*>(prow + cb * 4);
          p.x += dmr[cb * 4];
          p.y += dmr[cb * 4 + 1];
          p.z += dmr[cb * 4 + 2];
          p.w += dmr[cb * 4 + 3];
          *reinterpret_cast<float4*>(prow + cb * 4) = p;
        }
      }
      if (ts < 64) ZR[ts] += DZ[ts] + (has_b ? DZ[64 + ts] : 0.f);
      __syncwarp();
      if (lane == 0) mbar_arrive(&mr_full[mb]);
      // The state group is done with the stage (its sigma(K) read K; its dM
      // MMA, complete, read V and SG).
      if (ts == 0) mbar_arrive(&empty[st]);
      if (traced) TC_TRACE(trn, 4, 55, t);
      tc_fence_before();
      named_bar_sync(1, 128);  // PF, ZR, DZ, ZW and the dM columns are the next pair's
    }
    if (traced) TC_TRACE_END(trn, 4);
    if (ok && ts < 64) {
      // The final state: M_out[:, d_v] = PF row d_v, z_out = ZR.
      float* mo = M_out + (int64_t)bh * kD64 * kD64;
      const float* prow = PF + ts * kF64PFStride;
#pragma unroll 4
      for (int k = 0; k < kD64; ++k) mo[k * kD64 + ts] = prow[k];
      z_out[(int64_t)bh * kD64 + ts] = ZR[ts];
    }
  } else {
    // ------------------------------------------------ attention group
    const int seg = tid >> 6, rl = tid & 63;  // this row's segment within the pair, and row within it
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const float g = gate_of(beta[bh % H]);
    const bool overwrite = g == 1.f;
    const float scale2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    constexpr float kLog2e = 1.4426950408889634f;
    [[maybe_unused]] uint32_t trn = 0;
    [[maybe_unused]] const bool traced = warp == 0;  // channel 3
    for (int t = 0; t < pairs && ok; ++t) {
      const int st = t & 1, mb = t & 1;
      if (traced) TC_TRACE(trn, 3, 40, t);
      uint8_t* sQ = sm + st * kF64Stage;
      uint8_t* sK = sQ + kBlk64;
      uint8_t* sA0 = sQ + 2 * kBlk64;
      const bool has_b = 2 * t + 1 < S;
      const uint32_t ph = (uint32_t)t & 1u;
      // A failed (bounded) wait does not leave the loop before the group's
      // next barrier: every warp arrives there and they leave together.
      bool w = mbar_wait_warp(&full[st], (uint32_t)(t >> 1) & 1u, epoch);
      if (traced) TC_TRACE(trn, 3, 41, t);
      if (w && tid == 0) {
        // S = Q K^T: 128 queries x 128 keys, K = 64. S (and P in it) was last
        // read by the previous pair's P V, complete (o_done) before this.
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(128, 128, false, false);
        const uint64_t da = desc_kmajor_sw128(smem_u32(sQ)), dk = desc_kmajor_sw128(smem_u32(sK));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tmem, da + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), id, kk != 0);
        mma_commit(qk_done);
        mma_issued = true;
      }
      // sigma(q) of this row, while the QK^T runs.
      float sg[64];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 x = *reinterpret_cast<const uint4*>(sQ + sw128_offset(tid, q * 8, 128));
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float f0 = __uint_as_float(w[e] << 16), f1 = __uint_as_float(w[e] & 0xffff0000u);
          sg[q * 8 + 2 * e] = f0 > 0.f ? f0 + 1.f : ex2(f0 * kLog2e);
          sg[q * 8 + 2 * e + 1] = f1 > 0.f ? f1 + 1.f : ex2(f1 * kLog2e);
        }
      }
      float l = 1.f, mult = 0.f;
      if (traced) TC_TRACE(trn, 3, 42, t);
      w = w && mbar_wait_warp(qk_done, ph, epoch);
      if (traced) TC_TRACE(trn, 3, 43, t);
      tc_fence_after();
      if (w) {
        // This row's 64 scores (its own segment's keys), causal within the segment.
        uint32_t sr[64];
        tmem_ld32(tl + seg * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tl + seg * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait_regs(sr);
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c > rl) sr[c] = __float_as_uint(-INFINITY);
        const float mx = row_max64(sr);
        uint64_t acc2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc2[q] = 0ull;
        const uint64_t sc2 = f32x2(scale2, scale2), nm2 = f32x2(-mx * scale2, -mx * scale2);
#pragma unroll
        for (int c = 0; c < 64; c += 2) exp2_pair(sr, c, sc2, nm2, acc2[(c >> 1) & 3]);
        l = sum_f32x2(acc2);
        // P over TMEM columns 0-63 (128 keys, 2 per column): this row's segment
        // half, zeros in the other.
        uint32_t zero16[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) zero16[q] = 0u;
        tmem_st16(tl + seg * 32, *reinterpret_cast<uint32_t(*)[16]>(&sr[0]));
        tmem_st16(tl + seg * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[16]));
        tmem_st16(tl + (seg ^ 1) * 32, zero16);
        tmem_st16(tl + (seg ^ 1) * 32 + 16, zero16);
      }
      // den = sigma(q) . z_{s-1} with z_{s-1} from the state group.
      if (traced) TC_TRACE(trn, 3, 44, t);
      w = w && mbar_wait_warp(&mr_full[mb], (uint32_t)(t >> 1) & 1u, epoch);
      if (traced) TC_TRACE(trn, 3, 45, t);
      if (w) {
        const float* zrow = ZS + mb * 128 + seg * 64;
        float den = 0.f;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 z4 = *reinterpret_cast<const float4*>(zrow + c);
          den = fmaf(sg[c], z4.x, den);
          den = fmaf(sg[c + 1], z4.y, den);
          den = fmaf(sg[c + 2], z4.z, den);
          den = fmaf(sg[c + 3], z4.w, den);
        }
        const float wm = den != 0.f ? g / den : 0.f;
        float c;
        if (overwrite) {
          c = wm;
          mult = 1.f;
        } else {
          mult = (1.f - g) / l;
          c = wm / mult;
        }
        // Row tid of the block-diagonal retrieval operand, in TMEM (the
        // retrieval reads its A operand from there): c sigma(q) in block
        // `seg` (K columns 64 seg .. 64 seg + 63, 32 TMEM columns), zeros in
        // the other.
        uint32_t pk[32], zero16[16];
#pragma unroll
        for (int q = 0; q < 32; ++q) pk[q] = pack_bf16x2(sg[2 * q] * c, sg[2 * q + 1] * c);
#pragma unroll
        for (int q = 0; q < 16; ++q) zero16[q] = 0u;
        tmem_st16(tl + kF64ColA + seg * 32, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
        tmem_st16(tl + kF64ColA + seg * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
        tmem_st16(tl + kF64ColA + (seg ^ 1) * 32, zero16);
        tmem_st16(tl + kF64ColA + (seg ^ 1) * 32 + 16, zero16);
      }
      tmem_st_wait();
      tc_fence_before();
      if (!(ok = named_bar_and(2, 128, w))) break;
      if (tid == 0) {
        tc_fence_after();
        // O = P V (P in TMEM columns 0-63; V from A0 rows 0-63 and A1 rows 64-127),
        // then O += (c sigma(Q) block diagonal) [M_{a-1}; M_{b-1}] (O = when g == 1).
        const uint32_t idv = idesc_bf16_f32(128, 64, false, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t dv = desc_mnmajor_sw128(smem_u32(sA0 + (kk >> 2) * kBlk64 + kk * 2048), kBlk64);
          mma_bf16_ts(tmem + kF64ColO, tmem + kk * 8, dv, idv, kk != 0);
        }
        const uint32_t idr = idesc_bf16_f32(128, 64, false, false);
        const uint64_t dm = desc_kmajor_sw128(smem_u32(sm + kF64MR + mb * kBlk64));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + kF64ColO, tmem + kF64ColA + kk * 8,
                      dm + (((kk >> 2) * (kBlk64 / 2) + (kk & 3) * 32) >> 4), idr, (overwrite && kk == 0) ? 0u : 1u);
        mma_commit(o_done);
        mma_commit(&mr_empty[mb]);
        mma_commit(&empty[st]);
      }
      if (traced) TC_TRACE(trn, 3, 46, t);
      w = mbar_wait_warp(o_done, ph, epoch);
      if (traced) TC_TRACE(trn, 3, 47, t);
      tc_fence_after();
      if (w) {
        uint32_t o[64];
        tmem_ld32(tl + kF64ColO, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld32(tl + kF64ColO + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        tmem_ld_wait_regs(o);
        const int64_t row = row_base + 2 * t * kD64 + tid;
        if ((seg == 0 || has_b) && INFINI_CHECK(row < rows_total)) {
          __nv_bfloat16* orow = out + row * kD64;
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t pk[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              pk[q] = pack_bf16x2(mult * __uint_as_float(o[cb * 16 + 2 * q]), mult * __uint_as_float(o[cb * 16 + 2 * q + 1]));
            if (out_v8) {
              st_global_v8(orow + cb * 16, pk);
            } else {
              uint4* o4 = reinterpret_cast<uint4*>(orow + cb * 16);
              o4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              o4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
      }
      if (traced) TC_TRACE(trn, 3, 48, t);
      tc_fence_before();
      if (!(ok = named_bar_and(2, 128, w))) break;  // S and O are the next pair's
    }
    if (traced) TC_TRACE_END(trn, 3);
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own copies and MMAs finish before exit (the
    // producer's armed stages: both parities, one of them is complete; each
    // issuing thread's MMAs through a commit of its own).
    if (warp == 8 && lane == 0) {
      for (int s = 0; s < 2; ++s)
        if ((armed >> s) & 1u) mbar_drain(&full[s], 0), mbar_drain(&full[s], 1);
    }
    if ((tid == 0 || tid == 128) && mma_issued) {
      uint64_t* d = &drain[tid == 0 ? 0 : 1];
      mma_commit(d);
      mbar_drain(d, 0);
    }
    __syncthreads();
  }
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace infini
