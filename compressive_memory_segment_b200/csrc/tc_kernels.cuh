// Tensor-core (tcgen05 / TMEM / TMA) path of the Infini-attention forward for
// bf16 I/O, head dimension 128 and segment lengths that are multiples of 128.
//
//   tc_state_kernel : per (b, h, segment): dM = sigma(K)^T V and dz = sum_t sigma(K_t)
//                     ("Hugging Face Infini-Attention reproduction analysis",
//                     Infini-Attention mechanism: Memory Update) as tcgen05 MMAs
//                     with fp32 accumulators in TMEM. K and V tiles arrive by TMA
//                     in the 128-byte-swizzled layout; sigma is applied in shared
//                     memory; sigma(K)^T and V are both read MN-major, so no
//                     transpose is materialised. dz comes from a second MMA
//                     against a block of ones.
//   scan_state_kernel<bf16> (scan_kernel.cuh): M_{s-1} as bf16 (the retrieval
//                     MMA operand) and z_{s-1} in fp32.
//   tc_attn_kernel  : per (b, h, segment, 128-row query tile): causal softmax
//                     attention inside the segment (Local Attention) with an
//                     online softmax over 128-key tiles (the running max /
//                     normaliser merge of the "Attention-State Memory" page,
//                     Methodology), then sigma(Q) M_{s-1} on the tensor cores and
//                     sigma(Q).z_{s-1} in fp32 (Memory Retrieval), the
//                     sigmoid(beta) blend (Integration) and the bf16 store.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs (one elected lane), warps 2-5 (128 threads, one query row /
// one d_k row each) run the softmax, the sigma transforms and the epilogues.
// Every mbarrier wait is bounded (sm100.cuh); on a timeout a thread stops
// issuing work, the device status word records it, and the CTA still frees
// its TMEM before exiting.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/infini_attn.h"
#include "common.cuh"
#include "scan_kernel.cuh"
#include "sm100.cuh"

namespace infini {

constexpr bool kTcPathBuilt = true;

struct TcArgs {
  int64_t B, H, L, N, S;
  const void *q, *k, *v;
  const float* beta;
  const float *M_in, *z_in;
  void* out;
  float *M_out, *z_out;
  float *dM, *dz;
  __nv_bfloat16* Mp;
  float* zp;
};

inline int tc_launch_count() { return 3; }

namespace tc {

using namespace sm100;

constexpr int kD = 128;                        // head dimension covered
constexpr int kTile = 128;                     // rows per query / key tile
constexpr uint32_t kHalf = kTile * 128;        // one 64-column SW128 block: 128 rows x 128 B
constexpr uint32_t kTileBytes = 2 * kHalf;     // a 128 x 128 bf16 tile
constexpr int kThreads = 192;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major SW128 operand, K step kk (16 bf16 = 32 B) of a 128 x 128 tile.
__device__ __forceinline__ uint64_t desc_k(const uint8_t* tile, int kk) {
  return desc_kmajor_sw128(smem_u32(tile) + (uint32_t)(kk >> 2) * kHalf + (uint32_t)(kk & 3) * 32u);
}
// MN-major SW128 operand, K step kk (16 rows = 2 KB) of a 128-row tile whose
// two 64-column blocks are kHalf apart.
__device__ __forceinline__ uint64_t desc_mn(const uint8_t* tile, int kk) {
  return desc_mnmajor_sw128(smem_u32(tile) + (uint32_t)kk * 2048u, kHalf);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* m, int row, uint64_t* bar) {
  tma_load_2d(dst, m, 0, row, bar);
  tma_load_2d(dst + kHalf, m, 64, row, bar);
}

// sigma(x) = ELU(x) + 1 on 8 packed bf16 values.
__device__ __forceinline__ uint4 sigma8(uint4 x) {
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&w[i]);
    float2 f = __bfloat1622float2(b);
    w[i] = pack_bf16x2(elu1(f.x), elu1(f.y));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// ------------------------------------------------------------------ state kernel

constexpr int kStateStages = 3;
constexpr uint32_t kStateSmem = 2 * kStateStages * kTileBytes + 2048 + 256 + 1024;
static_assert(14 * 8 + 4 <= 256, "state kernel barrier area");

// grid: B*H*S CTAs (unit = bh * S + s), 192 threads.
__global__ void __launch_bounds__(kThreads, 1)
tc_state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int L, int N,
                int S, float* __restrict__ dM, float* __restrict__ dz, uint32_t epoch) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sK = sm;                                   // kStateStages x 32 KB
  uint8_t* sV = sm + kStateStages * kTileBytes;       // kStateStages x 32 KB
  uint8_t* sOnes = sm + 2 * kStateStages * kTileBytes;  // 2 KB of bf16 1.0
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOnes + 2048);
  uint64_t* k_full = bars;                    // [3] TMA -> sigma warps
  uint64_t* v_full = bars + 3;                // [3] TMA -> MMA
  uint64_t* kt_ready = bars + 6;              // [3] sigma warps -> MMA (4 arrivals)
  uint64_t* empty = bars + 9;                 // [3] MMA commit -> TMA
  uint64_t* done = bars + 12;                 // MMA commit -> epilogue
  uint64_t* drain = bars + 13;                // abort path: in-flight MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x;
  const int bh = unit / S, s = unit % S;
  const int row0 = bh * L + s * N;
  const int nchunks = N / kTile;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStateStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kt_ready[i], 4);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  if (warp >= 2) {
    for (int i = threadIdx.x - 64; i < 512; i += 128) reinterpret_cast<uint32_t*>(sOnes)[i] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  int armed[kStateStages] = {-1, -1, -1};  // last phase armed per stage (producer lane)

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % kStateStages, use = c / kStateStages;
        if (use > 0 && !(ok = mbar_wait(&empty[st], (use - 1) & 1, epoch))) break;
        armed[st] = use;
        mbar_arrive_expect_tx(&k_full[st], kTileBytes);
        load_tile(sK + st * kTileBytes, &tmK, row0 + c * kTile, &k_full[st]);
        mbar_arrive_expect_tx(&v_full[st], kTileBytes);
        load_tile(sV + st * kTileBytes, &tmV, row0 + c * kTile, &v_full[st]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_m = idesc_bf16_f32(128, 128, true, true);
      const uint32_t id_z = idesc_bf16_f32(128, 16, true, true);
      const uint64_t d_ones = desc_mnmajor_sw128(smem_u32(sOnes), 1024);
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % kStateStages, use = c / kStateStages;
        if (!(ok = mbar_wait(&kt_ready[st], use & 1, epoch) && mbar_wait(&v_full[st], use & 1, epoch))) break;
        tc_fence_after();
        const uint8_t* k = sK + st * kTileBytes;
        const uint8_t* v = sV + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = desc_mn(k, kk);
          mma_bf16_ss(tmem, a, desc_mn(v, kk), id_m, (c | kk) != 0);
          mma_bf16_ss(tmem + 128, a, d_ones, id_z, (c | kk) != 0);
        }
        mma_commit(&empty[st]);
      }
      if (ok) mma_commit(done);
    }
  } else {
    // sigma(K) in place, elementwise (the swizzle does not matter here).
    const int t = threadIdx.x - 64;
    for (int c = 0; c < nchunks; ++c) {
      const int st = c % kStateStages, use = c / kStateStages;
      if (!(ok = mbar_wait_warp(&k_full[st], use & 1, epoch))) break;
      uint4* p = reinterpret_cast<uint4*>(sK + st * kTileBytes);
#pragma unroll 4
      for (int i = t; i < (int)(kTileBytes / 16); i += 128) p[i] = sigma8(p[i]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kt_ready[st]);
    }
    if (ok) ok = mbar_wait_warp(done, 0, epoch);
    tc_fence_after();
    if (ok) {
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;  // d_k index
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
      float4* dst = reinterpret_cast<float4*>(dM + ((int64_t)unit * kD + row) * kD);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t r[32];
        tmem_ld32(taddr + cb * 32, r);
        tmem_ld_wait_regs(r);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[cb * 8 + i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                        __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      }
      uint32_t rz[16];
      tmem_ld16(taddr + 128, rz);
      tmem_ld_wait_regs(rz);
      dz[(int64_t)unit * kD + row] = __uint_as_float(rz[0]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if (warp == 0 && lane == 0)
      for (int st = 0; st < kStateStages; ++st)
        if (armed[st] >= 0) {
          mbar_drain(&k_full[st], armed[st] & 1);
          mbar_drain(&v_full[st], armed[st] & 1);
        }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncthreads();
  }
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------ attention kernel

// Shared memory: Q | K[2] | V[2] | P[2] (32 KB each) | barriers.
constexpr uint32_t kAttnSmem = 7 * kTileBytes + 256 + 1024;
static_assert(17 * 8 + 4 <= 256, "attention kernel barrier area");

// TMEM columns: S[0] 0..127, S[1] 128..255, O 256..383, retrieval 384..511.
constexpr uint32_t kColO = 256, kColR = 384;

// Lazy rescaling: the running max used for the exponent is only raised when a
// row's new max exceeds it by more than 2^8 (so unnormalised P stays <= 256).
constexpr float kRescaleLog2 = 8.f;

// grid: B*H*S*(N/128) CTAs; unit u -> (segment unit u / n_qt, query tile
// n_qt - 1 - u % n_qt): the tiles of one segment run together (their K/V tiles
// are shared through L2) and the longest tile of each segment starts first.
__global__ void __launch_bounds__(kThreads, 1)
tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
               const float* __restrict__ zp, const float* __restrict__ beta, __nv_bfloat16* __restrict__ out,
               int L, int N, int S, int H, uint32_t epoch) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + kTileBytes;          // [2]
  uint8_t* sV = sm + 3 * kTileBytes;      // [2]
  uint8_t* sP = sm + 5 * kTileBytes;      // [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 7 * kTileBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* s_full = bars + 5;    // [2] QK^T done          (MMA commit)
  uint64_t* s_free = bars + 7;    // [2] S read by softmax   (4 warps)
  uint64_t* p_full = bars + 9;    // [2] P written           (4 warps)
  uint64_t* pv_done = bars + 11;  // [2] PV done: P, K, V buffers free (MMA commit)
  uint64_t* sq_full = bars + 13;  // sigma(Q) written        (4 warps)
  uint64_t* m_full = bars + 14;   // M_{s-1} tile loaded
  uint64_t* done = bars + 15;     // every MMA done          (MMA commit)
  uint64_t* drain = bars + 16;    // abort path: in-flight MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = N / kTile;
  const int seg_unit = blockIdx.x / n_qt;
  const int qt = n_qt - 1 - blockIdx.x % n_qt;
  const int bh = seg_unit / S, s = seg_unit % S;
  const int h = bh % H;
  const int n = qt + 1;                      // key tiles visible to this query tile
  const int row_seg = bh * L + s * N;        // first token row of the segment
  const int row_q = row_seg + qt * kTile;    // first token row of the query tile
  const int bm = n & 1;                      // K buffer that receives M_{s-1}

  if (threadIdx.x == 0) {
    for (int i = 0; i < 17; ++i) {
      const bool by_warps = (i >= 7 && i <= 10) || i == 13;  // s_free, p_full, sq_full
      mbar_init(&bars[i], by_warps ? 4 : 1);
    }
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
  int armed_kv[2] = {-1, -1};  // last phase armed per K/V buffer (producer lane)
  bool armed_m = false;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmM);
      mbar_arrive_expect_tx(q_full, kTileBytes);
      load_tile(sQ, &tmQ, row_q, q_full);
      for (int j = 0; j < n && ok; ++j) {
        const int b = j & 1;
        if (j >= 2 && !(ok = mbar_wait(&pv_done[b], ((j - 2) >> 1) & 1, epoch))) break;
        armed_kv[b] = j >> 1;
        mbar_arrive_expect_tx(&k_full[b], kTileBytes);
        load_tile(sK + b * kTileBytes, &tmK, row_seg + j * kTile, &k_full[b]);
        mbar_arrive_expect_tx(&v_full[b], kTileBytes);
        load_tile(sV + b * kTileBytes, &tmV, row_seg + j * kTile, &v_full[b]);
      }
      if (ok && n >= 2) ok = mbar_wait(&pv_done[bm], ((n - 2) >> 1) & 1, epoch);
      if (ok) {
        armed_m = true;
        mbar_arrive_expect_tx(m_full, kTileBytes);
        load_tile(sK + bm * kTileBytes, &tmM, seg_unit * kD, m_full);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
      auto issue_pv = [&](int i) {
        const int b = i & 1, ph = (i >> 1) & 1;
        if (!(ok = mbar_wait(&p_full[b], ph, epoch) && mbar_wait(&v_full[b], ph, epoch))) return;
        tc_fence_after();
        const uint8_t* p = sP + b * kTileBytes;
        const uint8_t* vv = sV + b * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ss(tmem + kColO, desc_k(p, kk), desc_mn(vv, kk), id_pv, (i | kk) != 0);
        mma_commit(&pv_done[b]);
      };
      ok = mbar_wait(q_full, 0, epoch);
      for (int j = 0; j < n && ok; ++j) {
        const int b = j & 1;
        if (!(ok = mbar_wait(&k_full[b], (j >> 1) & 1, epoch))) break;
        if (j >= 2 && !(ok = mbar_wait(&s_free[b], ((j - 2) >> 1) & 1, epoch))) break;
        tc_fence_after();
        const uint8_t* kk_tile = sK + b * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + b * 128, desc_k(sQ, kk), desc_k(kk_tile, kk), id_qk, kk != 0);
        mma_commit(&s_full[b]);
        if (j >= 1) issue_pv(j - 1);
      }
      if (ok) issue_pv(n - 1);
      // Retrieval: sigma(Q) (in the Q buffer) x M_{s-1} (MN-major, in K[bm]).
      if (ok) ok = mbar_wait(sq_full, 0, epoch) && mbar_wait(m_full, 0, epoch);
      if (ok) {
        tc_fence_after();
        const uint8_t* mt = sK + bm * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ss(tmem + kColR, desc_k(sQ, kk), desc_mn(mt, kk), id_pv, kk != 0);
        mma_commit(done);
      }
    }
  } else {
    // ------------------------------------------------ softmax + epilogue (one query row per thread)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float scale2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    float m_run = -INFINITY, l_run = 0.f, den = 0.f;
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (!(ok = mbar_wait_warp(&s_full[b], (j >> 1) & 1, epoch))) break;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) tmem_ld32(tl + b * 128 + cb * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[cb * 32]));
      tmem_ld_wait_regs(sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);

      float mx = -INFINITY;
      if (j == n - 1) {  // diagonal tile: key column c is visible to row r iff c <= r
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float x = c <= r ? __uint_as_float(sr[c]) : -INFINITY;
          sr[c] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      }
      const float m_new = mx * scale2;
      const bool need = m_new > m_run + kRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_tgt = need ? m_new : m_run;
        const float alpha = ex2(m_run - m_tgt);
        if (j > 0) {
          // O holds PV_0..PV_{j-1}; wait for the last one before rescaling it.
          if (!(ok = mbar_wait_warp(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, epoch))) break;
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t o[32];
            tmem_ld32(tl + kColO + cb * 32, o);
            tmem_ld_wait_regs(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + kColO + cb * 32, o);
          }
          tmem_st_wait();
        }
        l_run *= alpha;
        m_run = m_tgt;
      }
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2(fmaf(__uint_as_float(sr[c]), scale2, -m_run));
        const float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), scale2, -m_run));
        sum += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_run += sum;
      // P buffer b is free once PV_{j-2} has completed.
      if (j >= 2 && !(ok = mbar_wait_warp(&pv_done[b], ((j - 2) >> 1) & 1, epoch))) break;
      uint8_t* pb = sP + b * kTileBytes;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(pb + sw128_offset(r, c * 8, 128)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);

      if (j == n - 1) {
        // Q is no longer read by QK^T: replace it by sigma(Q) for the retrieval
        // MMA and form the fp32 denominator sigma(q) . z_{s-1}.
        const float4* zs = reinterpret_cast<const float4*>(zp + (int64_t)seg_unit * kD);
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          uint4* src = reinterpret_cast<uint4*>(sQ + sw128_offset(r, c * 8, 128));
          const uint4 x = *src;
          const float4 z0 = __ldg(&zs[2 * c]), z1 = __ldg(&zs[2 * c + 1]);
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
          const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            const float a = elu1_accurate(f.x), bq = elu1_accurate(f.y);
            den = fmaf(a, zz[2 * i], den);
            den = fmaf(bq, zz[2 * i + 1], den);
            o[i] = pack_bf16x2(a, bq);
          }
          *src = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(sq_full);
      }
    }
    if (ok) ok = mbar_wait_warp(done, 0, epoch);
    tc_fence_after();
    if (ok) {
      const float g = gate_of(beta[h]);
      const float wd = (1.f - g) / l_run;
      const float wm = den != 0.f ? g / den : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(out + (int64_t)(row_q + r) * kD);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t o[32], rr[32];
        tmem_ld32(tl + kColO + cb * 32, o);
        tmem_ld32(tl + kColR + cb * 32, rr);
        tmem_ld_wait_regs(o);
        asm volatile("" ::: "memory");
#pragma unroll
        for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(rr[i]));
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float y0 = wd * __uint_as_float(o[2 * i]) + wm * __uint_as_float(rr[2 * i]);
          const float y1 = wd * __uint_as_float(o[2 * i + 1]) + wm * __uint_as_float(rr[2 * i + 1]);
          pk[i] = pack_bf16x2(y0, y1);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) orow[cb * 4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if (warp == 0 && lane == 0) {
      mbar_drain(q_full, 0);
      for (int b = 0; b < 2; ++b)
        if (armed_kv[b] >= 0) {
          mbar_drain(&k_full[b], armed_kv[b] & 1);
          mbar_drain(&v_full[b], armed_kv[b] & 1);
        }
      if (armed_m) mbar_drain(m_full, 0);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncthreads();
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, []() {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [rows, 128] bf16 row-major matrix, loaded in 128-row x 64-column boxes
// with the 128-byte swizzle.
inline bool make_map(CUtensorMap* m, const void* base, int64_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

// Nonzero per-call epoch for the abort word of the bounded waits.
inline uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{0};
  uint32_t e = counter.fetch_add(1) + 1;
  while (e == 0) e = counter.fetch_add(1) + 1;
  return e;
}

inline int tc_forward(const TcArgs& a, cudaStream_t st, const Trace& tr) {
  using namespace tc;
  const uint32_t epoch = next_epoch();
  const int64_t BH = a.B * a.H, rows = BH * a.L;
  CUtensorMap mq, mk, mv, mm;
  if (!make_map(&mq, a.q, rows) || !make_map(&mk, a.k, rows) || !make_map(&mv, a.v, rows) ||
      !make_map(&mm, a.Mp, BH * a.S * kD))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem) != cudaSuccess ||
      cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem) != cudaSuccess)
    return INFINI_ERR_CUDA;
  const int L = (int)a.L, N = (int)a.N, S = (int)a.S, H = (int)a.H;

  if (!tr.mark(0, st)) return INFINI_ERR_CUDA;
  tc_state_kernel<<<(unsigned)(BH * S), kThreads, kStateSmem, st>>>(mk, mv, L, N, S, a.dM, a.dz, epoch);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(1, st)) return INFINI_ERR_CUDA;

  const int64_t flat = BH * ((int64_t)kD * kD + kD) / 4;
  scan_state_kernel<__nv_bfloat16><<<(unsigned)((flat + kScanThreads - 1) / kScanThreads), kScanThreads, 0, st>>>(
      a.dM, a.dz, a.M_in, a.z_in, a.Mp, a.zp, a.M_out, a.z_out, BH, S, kD);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(2, st)) return INFINI_ERR_CUDA;

  const int64_t units = BH * S * (N / kTile);
  tc_attn_kernel<<<(unsigned)units, kThreads, kAttnSmem, st>>>(mq, mk, mv, mm, a.zp, a.beta,
                                                             static_cast<__nv_bfloat16*>(a.out), L, N, S, H, epoch);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(3, st)) return INFINI_ERR_CUDA;
  return INFINI_OK;
}

}  // namespace infini
