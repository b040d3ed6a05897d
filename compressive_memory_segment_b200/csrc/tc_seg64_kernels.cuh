// Tensor-core (tcgen05 / TMEM / TMA) kernels for bf16 I/O with head dimension
// 64 and 64-token segments -- the shape of the "Hugging Face Infini-Attention
// reproduction analysis" page's reproduction (segment length 64). A 128-row
// tensor-core tile holds two such segments, so both kernels work on pairs of
// consecutive segments of one (b, h), one CTA per pair:
//
//   tc_state64_kernel : dM_s = sigma(K_s)^T V_s and dz_s = sum_t sigma(K_t)
//                       for the pair's two segments (Infini-Attention
//                       mechanism: Memory Update) in one M128 x N128 x K128
//                       MMA: A = [V_a^T 0; 0 V_b^T] (block diagonal over the two
//                       segments' 64 tokens each), B = [sigma_hi | sigma_lo] of
//                       both segments' keys, so rows 0-63 of the accumulator
//                       are segment a's dM^T and rows 64-127 segment b's, each
//                       as a hi part plus a lo part (sigma split in two bf16
//                       values as in tc_state_kernel).
//   (scan_state_kernel<bf16> then forms M_{s-1} and z_{s-1}.)
//   tc_attn64_kernel  : the pair's 128 query rows against its 128 keys with a
//                       block-diagonal causal mask (a row sees the keys of its
//                       own segment up to itself: Local Attention), a
//                       single-pass softmax (all of a row's keys are in one
//                       tile), P V into O, and the retrieval folded into O:
//                       each row of sigma(Q) scaled by c = wm / wd goes into a
//                       block-diagonal operand [c sigma(Q_a) 0; 0 c sigma(Q_b)]
//                       against the stacked [M_a; M_b] (Memory Retrieval), so
//                       out = wd * O (or O with g == 1, when the retrieval
//                       overwrites O with c = wm); wd = (1 - g) / l,
//                       wm = g / den, den = sigma(q) . z_{s-1} (0 -> wm = 0).
//
// 128 threads per CTA, one row (token / query) per thread; thread 0 issues the
// TMA copies and the MMAs. Every mbarrier wait is bounded (sm100.cuh); on a
// timeout the CTA skips the rest of its work, drains its own copies and MMAs
// and frees its TMEM. With an odd number of segments per (b, h), the last
// pair's second segment does not exist: its rows are computed but never
// written.
#pragma once

namespace infini {
namespace tc {

constexpr int kD64 = 64;
constexpr int kSeg64Threads = 128;
constexpr uint32_t kBlk64 = 128 * 128;  // a 128-row x 64-column bf16 SW128 tile (16 KB)

// ------------------------------------------------------------------ state

// smem: Kh (K, then sigma_hi in place) | Kl (sigma_lo) | A block 0 | A block 1 |
// barriers. A = V^T block diagonal: block 0 holds segment a's V in rows 0-63
// and zeros in rows 64-127, block 1 zeros in rows 0-63 and segment b's V in
// rows 64-127 (rows = tokens, the MMA's K dimension).
constexpr uint32_t kState64Smem = 4 * kBlk64 + 64 + 4 * 64 * 4;

__global__ void __launch_bounds__(kSeg64Threads)
tc_state64_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int L, int S,
                  int pairs, float* __restrict__ dM, float* __restrict__ dz, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sKh = smem_raw;
  uint8_t* sKl = smem_raw + kBlk64;
  uint8_t* sA = smem_raw + 2 * kBlk64;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + 4 * kBlk64);
  uint64_t* k_full = bars + 0;
  uint64_t* v_full = bars + 1;
  uint64_t* mma_done = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  float* zred = reinterpret_cast<float*>(smem_raw + 4 * kBlk64 + 64);  // [4 warps][8 chunks][8]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / pairs, t = blockIdx.x % pairs;
  const int s_a = 2 * t;
  const bool has_b = s_a + 1 < S;
  const int row0 = bh * L + s_a * kD64;

  // Zero the off-diagonal halves of A: block 0 rows 64-127 and block 1 rows
  // 0-63, 16 KB as 1024 16-byte words, 8 per thread.
  {
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int w = tid * 8 + q;  // 0..1023
      uint8_t* dst = w < 512 ? sA + 64 * 128 + w * 16 : sA + kBlk64 + (w - 512) * 16;
      *reinterpret_cast<uint4*>(dst) = zero;
    }
  }
  if (tid == 0) {
    mbar_init(k_full, 1);
    mbar_init(v_full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(k_full, kBlk64);
    tma_load_2d(sKh, &tmK, 0, row0, k_full);
    mbar_arrive_expect_tx(v_full, kBlk64);
    tma_load_2d(sA, &tmV, 0, row0, v_full);                        // V_a -> block 0, rows 0-63
    tma_load_2d(sA + kBlk64 + 64 * 128, &tmV, 0, row0 + 64, v_full);  // V_b -> block 1, rows 64-127
  }
  bool ok = mbar_wait(k_full, 0, epoch);
  if (ok) {
    // sigma(K) as hi + lo bf16 parts (hi over K in place, lo beside it), and
    // dz. Thread t takes the 16-byte column chunk c8 = t & 7 of the 8 rows
    // 8 rg .. 8 rg + 7 of segment t >> 6 (rg = (t >> 3) & 7), summing sigma
    // per column; the sums over row groups then go through shuffles (within a
    // warp) and shared memory (the segment's two warps).
    const int c8 = tid & 7, rg = (tid >> 3) & 7, seg = tid >> 6;
    float zacc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) zacc[q] = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int row = seg * 64 + rg * 8 + q;
      uint4* pk = reinterpret_cast<uint4*>(sKh + sw128_offset(row, c8 * 8, 128));
      uint4* pl = reinterpret_cast<uint4*>(sKl + sw128_offset(row, c8 * 8, 128));
      uint4 hi, lo;
      sigma8_split(*pk, hi, lo, zacc);
      *pk = hi;
      *pl = lo;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 8);
      zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 16);
    }
    if (lane < 8) {
#pragma unroll
      for (int q = 0; q < 8; ++q) zred[(warp * 8 + c8) * 8 + q] = zacc[q];
    }
  }
  __syncthreads();
  if (ok) {
    const int seg = tid >> 6, c = tid & 63;
    const float zsum = zred[((2 * seg) * 8 + (c >> 3)) * 8 + (c & 7)] + zred[((2 * seg + 1) * 8 + (c >> 3)) * 8 + (c & 7)];
    if ((seg == 0 || has_b) && INFINI_CHECK((int64_t)bh * S + s_a + seg < (int64_t)(gridDim.x / pairs) * S))
      dz[((int64_t)bh * S + s_a + seg) * kD64 + c] = zsum;
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0 && ok) {
    if ((ok = mbar_wait(v_full, 0, epoch))) {
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(128, 128, true, true);
      const uint64_t da = desc_mnmajor_sw128(smem_u32(sA), kBlk64);
      const uint64_t db = desc_mnmajor_sw128(smem_u32(sKh), kBlk64);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) mma_bf16_ss(tmem, da + ((kk * 2048) >> 4), db + ((kk * 2048) >> 4), id, kk != 0);
      mma_commit(mma_done);
    }
  }
  ok = __syncthreads_and(ok);
  if (ok && mbar_wait_warp(mma_done, 0, epoch)) {
    tc_fence_after();
    // Lane tid: d_v index (tid & 63) of segment tid >> 6; columns: d_k hi | lo.
    const int seg = tid >> 6;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float* dst = dM + ((int64_t)bh * S + s_a + seg) * kD64 * kD64 + (tid & 63);
    const bool write = (seg == 0 || has_b) && INFINI_CHECK((int64_t)bh * S + s_a + seg < (int64_t)(gridDim.x / pairs) * S);
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t rh[16], rl[16];
      tmem_ld16(tl + cb * 16, rh);
      tmem_ld16(tl + 64 + cb * 16, rl);
      tmem_ld_wait_regs(rh);
      tmem_ld_wait_regs(rl);
      if (write) {
#pragma unroll
        for (int q = 0; q < 16; ++q) dst[(cb * 16 + q) * kD64] = __uint_as_float(rh[q]) + __uint_as_float(rl[q]);
      }
    }
  } else {
    ok = false;
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch && tid == 0) {
    // Abort path: let this CTA's own copies and MMAs finish before exit.
    mbar_drain(k_full, 0);
    mbar_drain(v_full, 0);
    mma_commit(mma_done);
    mbar_drain(mma_done, 0);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------ attention

// smem: Q (later block 0 of the retrieval operand) | K (later its block 1) |
// V | [M_a; M_b] | z of the two segments | barriers.
constexpr uint32_t kAttn64Smem = 4 * kBlk64 + 128 * 4 + 64;

__global__ void __launch_bounds__(kSeg64Threads)
tc_attn64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
                 const float* __restrict__ zp, const float* __restrict__ beta, __nv_bfloat16* __restrict__ out, int L,
                 int S, int H, int pairs, int out_v8, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sK = smem_raw + kBlk64;
  uint8_t* sV = smem_raw + 2 * kBlk64;
  uint8_t* sM = smem_raw + 3 * kBlk64;
  float* sZ = reinterpret_cast<float*>(smem_raw + 4 * kBlk64);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + 4 * kBlk64 + 128 * 4);
  uint64_t* qk_full = bars + 0;
  uint64_t* vm_full = bars + 1;
  uint64_t* s_full = bars + 2;
  uint64_t* o_full = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.x / pairs, t = blockIdx.x % pairs;
  const int s_a = 2 * t;
  const bool has_b = s_a + 1 < S;
  const int row0 = bh * L + s_a * kD64;
  const int seg = tid >> 6, rl = tid & 63;  // this row's segment (0 = a, 1 = b) and row within it

  if (tid == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  // z_{s-1} of the two segments (the second only when it exists).
  sZ[tid] = (seg == 0 || has_b) ? __ldg(zp + ((int64_t)bh * S + s_a) * kD64 + tid) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
  if (tid == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmM);
    mbar_arrive_expect_tx(qk_full, 2 * kBlk64);
    tma_load_2d(sQ, &tmQ, 0, row0, qk_full);
    tma_load_2d(sK, &tmK, 0, row0, qk_full);
    mbar_arrive_expect_tx(vm_full, 2 * kBlk64);
    tma_load_2d(sV, &tmV, 0, row0, vm_full);
    tma_load_2d(sM, &tmM, 0, ((int)bh * S + s_a) * kD64, vm_full);
  }
  bool ok = true;
  if (tid == 0) {
    // S = Q K^T: 128 queries x 128 keys (both segments), K = 64.
    if ((ok = mbar_wait(qk_full, 0, epoch))) {
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(128, 128, false, false);
      const uint64_t da = desc_kmajor_sw128(smem_u32(sQ)), db = desc_kmajor_sw128(smem_u32(sK));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tmem, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), id, kk != 0);
      mma_commit(s_full);
    }
  }
  const float scale2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
  constexpr float kLog2e = 1.4426950408889634f;
  float mult = 0.f;
  bool have_q = mbar_wait_warp(qk_full, 0, epoch);
  // sigma(q) and den = sigma(q) . z_{s-1} from this row of Q while the QK^T
  // MMA runs (the row is only read here; it is overwritten after S is ready).
  float sg[64];
  float den = 0.f;
  if (have_q) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 x = *reinterpret_cast<const uint4*>(sQ + sw128_offset(tid, q * 8, 128));
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float f0 = __uint_as_float(w[e] << 16), f1 = __uint_as_float(w[e] & 0xffff0000u);
        const float s0 = f0 > 0.f ? f0 + 1.f : ex2(f0 * kLog2e), s1 = f1 > 0.f ? f1 + 1.f : ex2(f1 * kLog2e);
        sg[q * 8 + 2 * e] = s0;
        sg[q * 8 + 2 * e + 1] = s1;
        den = fmaf(s0, sZ[seg * 64 + q * 8 + 2 * e], den);
        den = fmaf(s1, sZ[seg * 64 + q * 8 + 2 * e + 1], den);
      }
    }
  }
  if (have_q && mbar_wait_warp(s_full, 0, epoch)) {
    tc_fence_after();
    // This row's 64 scores (its own segment's keys), causal within the segment.
    uint32_t sr[64];
    tmem_ld32(tl + seg * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
    tmem_ld32(tl + seg * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
    tmem_ld_wait_regs(sr);
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (c > rl) sr[c] = __float_as_uint(-INFINITY);
    float mx = __uint_as_float(sr[0]);
#pragma unroll
    for (int c = 1; c < 64; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
    const float neg_m = -mx * scale2;
    float l = 0.f;
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
      const float p0 = ex2(fmaf(__uint_as_float(sr[c]), scale2, neg_m));
      const float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), scale2, neg_m));
      l += p0 + p1;
      sr[c >> 1] = pack_bf16x2(p0, p1);
    }
    // P over TMEM columns 0-63 (128 keys, 2 per column): this row's segment
    // half, zeros in the other.
    uint32_t zero16[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) zero16[q] = 0u;
    tmem_st16(tl + seg * 32, *reinterpret_cast<uint32_t(*)[16]>(&sr[0]));
    tmem_st16(tl + seg * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[16]));
    tmem_st16(tl + (seg ^ 1) * 32, zero16);
    tmem_st16(tl + (seg ^ 1) * 32 + 16, zero16);
    const float g = gate_of(beta[bh % H]);
    const float wm = den != 0.f ? g / den : 0.f;
    float c;
    if (g == 1.f) {
      c = wm;
      mult = 1.f;
    } else {
      mult = (1.f - g) / l;
      c = wm / mult;
    }
    // Row tid of the block-diagonal operand: c sigma(q) in block `seg`
    // (over Q for seg 0, over K for seg 1), zeros in the other block.
    uint8_t* own = seg == 0 ? sQ : sK;
    uint8_t* other = seg == 0 ? sK : sQ;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint4 v;
      v.x = pack_bf16x2(sg[q * 8 + 0] * c, sg[q * 8 + 1] * c);
      v.y = pack_bf16x2(sg[q * 8 + 2] * c, sg[q * 8 + 3] * c);
      v.z = pack_bf16x2(sg[q * 8 + 4] * c, sg[q * 8 + 5] * c);
      v.w = pack_bf16x2(sg[q * 8 + 6] * c, sg[q * 8 + 7] * c);
      *reinterpret_cast<uint4*>(own + sw128_offset(tid, q * 8, 128)) = v;
      *reinterpret_cast<uint4*>(other + sw128_offset(tid, q * 8, 128)) = make_uint4(0u, 0u, 0u, 0u);
    }
    tmem_st_wait();
  } else {
    ok = false;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (tid == 0 && ok) {
    if ((ok = mbar_wait(vm_full, 0, epoch))) {
      tc_fence_after();
      // O (TMEM columns 64-127, over the scores no longer needed) = P V, then
      // += (c sigma(Q) block diagonal) [M_a; M_b] (or = when g == 1).
      const uint32_t tO = tmem + 64;
      const uint32_t id = idesc_bf16_f32(128, 64, false, true);
      const uint64_t dv = desc_mnmajor_sw128(smem_u32(sV), kBlk64);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tO, tmem + kk * 8, dv + ((kk * 2048) >> 4), id, kk != 0);
      const bool overwrite = gate_of(beta[bh % H]) == 1.f;
      const uint64_t da = desc_kmajor_sw128(smem_u32(sQ)), dm = desc_mnmajor_sw128(smem_u32(sM), kBlk64);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tO, da + (((kk >> 2) * kBlk64 + (kk & 3) * 32) >> 4), dm + ((kk * 2048) >> 4), id,
                    (overwrite && kk == 0) ? 0u : 1u);
      mma_commit(o_full);
    }
  }
  ok = __syncthreads_and(ok);
  if (ok && mbar_wait_warp(o_full, 0, epoch)) {
    tc_fence_after();
    uint32_t o[64];
    tmem_ld32(tl + 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
    tmem_ld32(tl + 96, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
    tmem_ld_wait_regs(o);
    if ((seg == 0 || has_b) && INFINI_CHECK(row0 + tid < (int)(gridDim.x / pairs) * L)) {
      __nv_bfloat16* orow = out + (int64_t)(row0 + tid) * kD64;
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
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch && tid == 0) {
    // Abort path: let this CTA's own copies and MMAs finish before exit.
    mbar_drain(qk_full, 0);
    mbar_drain(vm_full, 0);
    mma_commit(o_full);
    mbar_drain(o_full, 0);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace tc
}  // namespace infini
