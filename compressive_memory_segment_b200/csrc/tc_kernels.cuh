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

#include <algorithm>
#include <atomic>
#include <mutex>
#include <numeric>

#include "../../include/infini_attn.h"
#include "common.cuh"
#include "scan_kernel.cuh"
#include "sm100.cuh"

namespace infini {

constexpr bool kTcPathBuilt = true;

// Outputs of the backward's statistics pass (tc_attn_kernel<true>), one per
// query row t unless marked: lse_t = m_t + log2(l_t) in the base-2 domain of
// the scaled scores (P_tj = 2^(s_tj log2(e)/sqrt(d) - lse_t)); Delta_t =
// (1 - g) dout_t . A_dot,t; dnum_t = g dout_t / den_t (a bf16 row, the MMA
// operand of the backward's retrieval and state terms);
// dden_t = -g (dout_t . A_mem,t) / den_t (both 0 where den_t = 0); dbeta[h]
// accumulates g (1 - g) dout_t . (A_mem,t - A_dot,t) (one atomic per warp
// and unit).
struct BwdStats {
  const __nv_bfloat16* dout = nullptr;
  float* lse = nullptr;
  float* delta = nullptr;
  __nv_bfloat16* dnum16 = nullptr;
  float* dden = nullptr;
  float* dbeta = nullptr;
};

struct TcArgs {
  int64_t B, H, L, N, S, d = 128;
  const void *q, *k, *v;
  const float* beta;
  const float *M_in, *z_in;
  void* out;
  float *M_out, *z_out;
  float *dM, *dz;
  __nv_bfloat16* Mp;
  float* zp;
  bool state_only = false;  // launch the state and scan kernels only (q, out, beta unused)
  bool skip_state = false;  // dM, dz already in the workspace: scan and attention only
  bool paired = false;      // attention by tc_attn_pair_kernel (seg_len % 256 == 0) instead of tc_attn_kernel
  const BwdStats* bwd = nullptr;  // the backward's statistics pass instead of out (d = 128)
};

// Kernels one tensor-core forward launches: the single-pass kernel for d = 64
// with 64-token segments (a whole forward), else state, scan and attention.
inline bool tc_fused64_covers(int64_t d, int64_t N) { return d == 64 && N == 64; }
inline int tc_launch_count(int64_t d = 128, int64_t N = 128, bool full = true) {
  return full && tc_fused64_covers(d, N) ? 1 : 3;
}

namespace tc {

using namespace sm100;

constexpr int kD = 128;                        // head dimension covered
constexpr int kTile = 128;                     // rows per query / key tile
constexpr uint32_t kHalf = kTile * 128;        // one 64-column SW128 block: 128 rows x 128 B
constexpr uint32_t kTileBytes = 2 * kHalf;     // a 128 x 128 bf16 tile


__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

#ifdef INFINI_TRACE
// Trace channels of CTA 0 of an attention launch (tracing build only). The
// paired kernel: 0 K producer (warp 12), 1 / 2 MMA slot 0 / 1, 3 / 4 softmax
// slot 0 / 1 (warps 0 and 4), 5 / 6 retrieval warp 8 for slot 0 / 1, 7 V and Q
// producer (warp 15). The one-tile kernel: 0 producer (warp 0), 1 MMA issuer
// (warp 1), 3 / 4 softmax warps 4 / 8 (the two halves of rows 0-31), 5
// epilogue warp 10. Each channel has one writer thread (lane 0 of its warp),
// which counts its records in a register and stores the count at the end, so
// a record costs a clock read and one store. Record: clock64 (low 40 bits) |
// event code << 40 | index << 48.
constexpr int kTraceChannels = 8, kTraceCap = 1 << 15;
__device__ unsigned long long g_trace[kTraceChannels][kTraceCap];
__device__ unsigned int g_trace_n[kTraceChannels];
#define TC_TRACE(n, ch, code, idx)                                                                \
  do {                                                                                                \
    if (blockIdx.x == 0 && lane == 0) {                                                               \
      if ((n) < (unsigned)kTraceCap)                                                                  \
        g_trace[ch][(n)] = ((unsigned long long)clock64() & 0xFFFFFFFFFFull) |                        \
                           ((unsigned long long)(code) << 40) | ((unsigned long long)((idx) & 0xFFFF) << 48); \
      ++(n);                                                                                          \
    }                                                                                                 \
  } while (0)
#define TC_TRACE_END(n, ch)                                 \
  do {                                                        \
    if (blockIdx.x == 0 && lane == 0) g_trace_n[ch] = (n);    \
  } while (0)
#else
#define TC_TRACE(n, ch, code, idx) \
  do {                                 \
  } while (0)
#define TC_TRACE_END(n, ch) \
  do {                        \
  } while (0)
#endif

// Row max of 64 scores held as fp32 bit patterns: three-input max in eight
// independent chains, then across them.
__device__ __forceinline__ float row_max64(const uint32_t (&s)[64]) {
  float m[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) m[t] = __uint_as_float(s[t]);
#pragma unroll
  for (int c = 8; c < 64; c += 2) m[(c >> 1) & 7] = max3f(m[(c >> 1) & 7], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
  return fmaxf(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], max3f(m[5], m[6], m[7])));
}

// Scores s[c], s[c + 1] (fp32 bits) -> p = 2^(s * scale2 - m) for both, the
// scaling as one packed f32x2 FMA (sc2 = (scale2, scale2), nm2 = (-m, -m)),
// the pair's sum added into the packed accumulator acc and the two
// probabilities written back as one bf16 pair into s[c / 2].
template <int K>
__device__ __forceinline__ void exp2_pair(uint32_t (&s)[K], int c, uint64_t sc2, uint64_t nm2, uint64_t& acc) {
  float x0, x1;
  unpack_f32x2(fma_f32x2(f32x2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc2, nm2), x0, x1);
  const float p0 = ex2(x0), p1 = ex2(x1);
  acc = add_f32x2(acc, f32x2(p0, p1));
  s[c >> 1] = pack_bf16x2(p0, p1);
}

// The total of four packed pair accumulators.
__device__ __forceinline__ float sum_f32x2(const uint64_t (&acc)[4]) {
  float a, b;
  unpack_f32x2(add_f32x2(add_f32x2(acc[0], acc[1]), add_f32x2(acc[2], acc[3])), a, b);
  return a + b;
}

__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* m, int row, uint64_t* bar) {
  tma_load_2d(dst, m, 0, row, bar);
  tma_load_2d(dst + kHalf, m, 64, row, bar);
}

// ------------------------------------------------------------------ state kernel

// Persistent: one CTA per SM walks segments u = blockIdx.x, + gridDim.x, ...
// For each segment, 64-token chunks of K and V stream through a 4-stage TMA
// ring. sigma(K) is split as hi + lo (hi = bf16(sigma), lo = bf16(sigma - hi))
// so the bf16 MMAs reproduce sigma(K)^T V to ~2^-16 relative instead of the
// 2^-9 of a single bf16 rounding. One M128 x N256 MMA per 16 tokens computes
// V^T [hi | lo] (A = V^T, B = the hi and lo chunks side by side), i.e. both
// halves of (dM)^T; the epilogue adds them and writes dM transposed, which
// makes its stores coalesced. dz = sum_t sigma(K_t) is summed in fp32 by the
// transform threads. Two TMEM accumulator sets let the epilogue drain segment
// u while segment u + gridDim.x accumulates.
//   warp 0      TMA producer (elected lane)
//   warp 1      TMEM owner, MMA issuer (elected lane)
//   warps 2-9   sigma transform: K chunk -> hi in place, lo beside it; dz
//   warps 10-13 epilogue: TMEM -> dM (fp32 [d_k][d_v])
// TMEM: set b at columns 256 b + [0, 128) (hi part), 256 b + [128, 256) (lo).

constexpr int kSChunk = 64;                            // tokens per state chunk
constexpr uint32_t kSHalf = kSChunk * 128;             // one 64-column SW128 block of a chunk
constexpr uint32_t kSChunkBytes = 2 * kSHalf;          // a 64 x 128 bf16 chunk
constexpr int kStateStages = 4;
constexpr int kStateXform = 8;                         // transform warps
constexpr int kStateThreads = 32 * (2 + kStateXform + 4);
constexpr uint32_t kStateStage = 3 * kSChunkBytes;     // hi | lo | V
constexpr uint32_t kStateZBuf = kStateXform * 8 * 16 * 4;  // per-warp dz partials
constexpr uint32_t kStateSmem = kStateStages * kStateStage + 2 * kStateZBuf + 256;
static_assert(kStateSmem <= 232448, "state kernel shared memory");
static_assert(4 * kStateStages + 5 <= 30, "state kernel barrier area");
static_assert(kStateXform == 8 && kSChunkBytes / 16 == 8 * 128, "transform: two groups of 4 warps, 8 uint4 per thread");

// sigma(x) = ELU(x) + 1 on 8 packed bf16 values: hi + lo bf16 parts, and the
// fp32 values added into acc[0..7]. exp(x) = 2^(x log2 e) on the flush-to-zero
// ex2 unit (relative error ~2^-22; results below 2^-126 flush to 0, far under
// what the lo part resolves). NaN inputs give NaN as the x > 0 test fails.
__device__ __forceinline__ void sigma8_split(uint4 x, uint4& hi, uint4& lo, float* acc) {
  constexpr float kLog2e = 1.4426950408889634f;
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = __uint_as_float(w[i] << 16), x1 = __uint_as_float(w[i] & 0xffff0000u);
    const float e0 = ex2(x0 * kLog2e), e1 = ex2(x1 * kLog2e);
    const float s0 = x0 > 0.f ? x0 + 1.f : e0, s1 = x1 > 0.f ? x1 + 1.f : e1;
    h[i] = pack_bf16x2(s0, s1);
    l[i] = pack_bf16x2(s0 - __uint_as_float(h[i] << 16), s1 - __uint_as_float(h[i] & 0xffff0000u));
    acc[2 * i] += s0;
    acc[2 * i + 1] += s1;
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// grid: min(B*H*S, #SMs) persistent CTAs (segment u = bh * S + s).
__global__ void __launch_bounds__(kStateThreads, 1)
tc_state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int L, int N,
                int S, int units, float* __restrict__ dM, float* __restrict__ dz, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  constexpr int SS = kStateStages;
  // stage st: [hi block 0 | hi block 1 | lo block 0 | lo block 1 | V block 0 | V block 1]
  uint8_t* stages = smem_raw;
  float* zbuf = reinterpret_cast<float*>(smem_raw + SS * kStateStage);  // [2][8 warps][8][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + SS * kStateStage + 2 * kStateZBuf);
  uint64_t* k_full = bars;              // [SS] TMA
  uint64_t* v_full = bars + SS;         // [SS] TMA
  uint64_t* kt_ready = bars + 2 * SS;   // [SS] transform done (one group of 4 warps)
  uint64_t* empty = bars + 3 * SS;      // [SS] MMAs done with the stage
  uint64_t* acc_full = bars + 4 * SS;   // [2] segment accumulated
  uint64_t* acc_empty = acc_full + 2;   // [2] epilogue drained the set (4 warps)
  uint64_t* drain = acc_full + 4;       // abort path: in-flight MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = N / kSChunk;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4 * SS + 5; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < SS; ++i) mbar_init(&kt_ready[i], kStateXform / 2);
    for (int i = 0; i < 2; ++i) mbar_init(&acc_empty[i], 4);
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
  uint32_t armed = 0;  // producer: 2 bits per stage (armed, parity of the last armed phase)
  static_assert(2 * SS <= 32, "armed mask");

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    int gc = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int bh = u / S, s = u % S;
      const int row0 = bh * L + s * N;
      for (int c = 0; c < nch; ++c, ++gc) {
        const int st = gc % SS, use = gc / SS;
        if (use > 0 && !(ok = mbar_wait_warp(&empty[st], (use - 1) & 1, epoch))) break;
        armed = (armed & ~(3u << (2 * st))) | ((2u | (use & 1)) << (2 * st));
        if (elect_one_lane()) {
          const int row = row0 + c * kSChunk;
          uint8_t* sk = stages + st * kStateStage;
          uint8_t* sv = sk + 2 * kSChunkBytes;
          mbar_arrive_expect_tx(&k_full[st], kSChunkBytes);
          tma_load_2d(sk, &tmK, 0, row, &k_full[st]);
          tma_load_2d(sk + kSHalf, &tmK, 64, row, &k_full[st]);
          mbar_arrive_expect_tx(&v_full[st], kSChunkBytes);
          tma_load_2d(sv, &tmV, 0, row, &v_full[st]);
          tma_load_2d(sv + kSHalf, &tmV, 64, row, &v_full[st]);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    const uint32_t id = idesc_bf16_f32(128, 256, true, true);
    const uint64_t dkl0 = desc_mnmajor_sw128(smem_u32(stages), kSHalf);
    const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(stages + 2 * kSChunkBytes), kSHalf);
    constexpr uint32_t kStageD = kStateStage >> 4;
    int gc = 0, i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const int ab = i & 1;
      if (i >= 2 && !(ok = mbar_wait_warp(&acc_empty[ab], ((i - 2) >> 1) & 1, epoch))) break;
      tc_fence_after();
      const uint32_t dm = tmem + ab * 256;
      for (int c = 0; c < nch; ++c, ++gc) {
        const int st = gc % SS, use = gc / SS;
        if (!(ok = mbar_wait_warp(&kt_ready[st], use & 1, epoch) && mbar_wait_warp(&v_full[st], use & 1, epoch))) break;
        tc_fence_after();
        const uint64_t dkl = dkl0 + st * kStageD, dv = dv0 + st * kStageD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < kSChunk / 16; ++kk) {
            const uint32_t off = (kk * 2048) >> 4;
            mma_bf16_ss(dm, dv + off, dkl + off, id, (c | kk) != 0);
          }
          mma_commit(&empty[st]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one_lane()) mma_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else if (warp < 2 + kStateXform) {
    // ------------------------------------------------ sigma transform (elementwise) and dz
    // Two groups of four warps take alternate chunks, so one group's loads
    // and MUFU latency overlap the other's. Thread t of a group handles uint4
    // e = t + 128 q of its chunks: SW128 block q >> 2, row (t >> 3) + 16 (q & 3),
    // stored position t & 7, i.e. always the logical 8 columns
    // j = (t & 7) ^ ((t >> 3) & 7) of each block.
    const int grp = (warp - 2) >> 2, t = threadIdx.x - 64 - 128 * grp, xw = warp - 2;
    int gc = 0, i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      float zacc[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) zacc[q] = 0.f;
      for (int c = 0; c < nch; ++c, ++gc) {
        if ((c & 1) != grp) continue;
        const int st = gc % SS, use = gc / SS;
        if (!(ok = mbar_wait_warp(&k_full[st], use & 1, epoch))) break;
        uint4* pk = reinterpret_cast<uint4*>(stages + st * kStateStage);
        uint4* pl = reinterpret_cast<uint4*>(stages + st * kStateStage + kSChunkBytes);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = t + 128 * q;
          uint4 hi, lo;
          sigma8_split(pk[e], hi, lo, zacc + 8 * (q >> 2));
          pk[e] = hi;
          pl[e] = lo;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&kt_ready[st]);
      }
      // dz: lanes l, l^9, l^18, l^27 of a warp hold the same 8 columns; add
      // them, then add the eight warps' totals per column through shared memory.
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 9);
        zacc[q] += __shfl_xor_sync(0xffffffffu, zacc[q], 18);
      }
      float* zw = zbuf + (i & 1) * (kStateZBuf / 4);  // [8 warps][8 column groups][16]
      if (lane < 8) {
        const int j = lane ^ (4 * (xw & 1));
#pragma unroll
        for (int q = 0; q < 16; ++q) zw[(xw * 8 + j) * 16 + q] = zacc[q];
      }
      if (!(ok = named_bar_and(1, 32 * kStateXform, ok))) break;
      const int col = threadIdx.x - 64;
      if (col < kD) {
        const int blk = col >> 6, j = (col >> 3) & 7, w = col & 7;
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < kStateXform; ++r) sum += zw[(r * 8 + j) * 16 + blk * 8 + w];
        if (INFINI_CHECK(u < units)) dz[(int64_t)u * kD + col] = sum;
      }
    }
  } else {
    // ------------------------------------------------ epilogue: TMEM -> dM
    const int quarter = warp & 3;
    const int dv_row = quarter * 32 + lane;  // d_v index = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    int i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const int ab = i & 1;
      if (!(ok = mbar_wait_warp(&acc_full[ab], (i >> 1) & 1, epoch))) break;
      tc_fence_after();
      float* dst = dM + (int64_t)u * kD * kD + dv_row;
      const bool u_ok = INFINI_CHECK(u < units);
#pragma unroll 1
      for (int cb = 0; cb < 8; ++cb) {
        uint32_t rh[16], rl[16];
        tmem_ld16(tl + ab * 256 + cb * 16, rh);
        tmem_ld16(tl + ab * 256 + 128 + cb * 16, rl);
        tmem_ld_wait_regs(rh);
        tmem_ld_wait_regs(rl);
        if (u_ok) {
#pragma unroll
          for (int q = 0; q < 16; ++q) dst[(cb * 16 + q) * kD] = __uint_as_float(rh[q]) + __uint_as_float(rl[q]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if (warp == 0 && lane == 0)
      for (int st = 0; st < SS; ++st)
        if ((armed >> (2 * st)) & 2u) {
          mbar_drain(&k_full[st], (armed >> (2 * st)) & 1u);
          mbar_drain(&v_full[st], (armed >> (2 * st)) & 1u);
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

// ------------------------------------------------------------------ attention kernel

// Persistent fused attention. Each CTA walks work units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...; a unit is one (segment, query tile), and query
// tile t of a segment costs t + 1 key tiles. decode_unit() spreads that cost
// evenly over the CTAs (see there) while the segments in flight stay few
// enough for their K/V tiles to be shared through L2. Four roles run
// concurrently and meet only at mbarriers:
//
//   warp 0      TMA producer (one elected lane of a converged warp). Per unit:
//               Q (double-buffered), then K/V tiles in the order the MMA
//               consumes them (K_0, K_1, V_0, K_2, V_1, ..., V_{n-1}), then the
//               unit's M_{s-1} tile, which travels in the K ring. It runs ahead
//               into the next unit as buffers free up.
//   warp 1      TMEM owner and MMA issuer (one elected lane of a converged
//               warp). Per unit: S = Q K^T into one of two S buffers (QK^T runs
//               one tile ahead of PV), O (+)= P V with P read from TMEM (written
//               there by the softmax over the S columns), and the retrieval
//               R = sigma(Q) M_{s-1} into its own accumulator. The next unit's
//               QK^T of tile 0 goes right after this unit's second-to-last PV;
//               the retrieval as soon as its sigma(Q) and M tile are in (at the
//               latest before the next unit's first PV).
//   warps 2-9   softmax, two threads per query row (warps 2-5 own key
//               columns 0..63, warps 6-9 columns 64..127; warp w reaches TMEM
//               lanes 32*(w%4)..+31): causal mask on the diagonal tile, the
//               row max agreed through shared memory, lazy rescaling of O,
//               P = 2^(s - m) as packed bf16 into TMEM, partial row sums.
//   warps 10-13 epilogue, one row per thread: the denominator
//               den = sigma(q).z_{s-1} and sigma(q) while the unit's QK^Ts run
//               (sigma(q) parked in the row's lane of the R columns); sigma(Q)
//               copied over the unit's Q buffer as soon as its last QK^T is
//               done (so the retrieval never waits for the softmax); after the
//               retrieval, out = wd * O + wm * R as the bf16 output row, with
//               wd = (1 - g) / l and wm = g / den (0 when den = 0).
//
// O and R are single-buffered: the next unit's first PV overwrites O only
// after the epilogue has read both, and the next retrieval writes R only
// after that unit's sigma(Q) has been copied out of the R columns, which the
// epilogue does after reading R.
//
// TMEM (512 columns): S/P[0] 0..127, S/P[1] 128..255, O 256..383,
// R 384..511. Shared memory, from the (1024-aligned) base of the dynamic
// window: Q[2] | K ring[3] | V ring[2] (32 KB each) | barriers | row-max
// exchange [2][128] | partial row sums [2][128].

constexpr int kKRing = 3, kVRing = 2;
constexpr uint32_t kAttnTiles = (2 + kKRing + kVRing) * kTileBytes;
constexpr uint32_t kAttnSmem = kAttnTiles + 256 + 1024 + 1024;
static_assert(kAttnSmem <= 232448, "attention kernel shared memory");
constexpr int kAttnThreads = 448;
constexpr uint32_t kColO = 256;  // O: this unit's P V accumulator
constexpr uint32_t kColR = 384;  // R: sigma(Q) M_{s-1} of the unit

constexpr uint32_t kAttnSmemBwd = kAttnSmem + 512;  // + the rows' running maxima
static_assert(kAttnSmemBwd <= 232448, "attention kernel shared memory (statistics pass)");

// The backward's statistics of one query row (BwdStats), from the row's O and
// R accumulators once the unit's last P V and retrieval are done: A_dot =
// O / l, A_mem = R / den (0 where den = 0), with the row's dout read from
// global memory. O and R are released to the next unit after the last read.
__device__ __forceinline__ void bwd_stats_row(const BwdStats& bs, uint32_t tl, int row, bool row_ok, int h,
                                              float g, float l, float m_row, float den, float wm, int lane,
                                              uint64_t* o_empty) {
  const float inv_l = 1.f / l;
  const float inv_den = den != 0.f ? 1.f / den : 0.f;
  const uint4* drow = reinterpret_cast<const uint4*>(bs.dout + (int64_t)row * kD);
  uint4* n16 = reinterpret_cast<uint4*>(bs.dnum16 + (int64_t)row * kD);
  float sd = 0.f, sm = 0.f;  // dout . A_dot, dout . A_mem
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
    uint4 dv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) dv[q] = row_ok ? __ldg(&drow[hf * 8 + q]) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int cq = 0; cq < 4; ++cq) {
      const int cb = hf * 4 + cq;
      uint32_t o[16], rr[16];
      tmem_ld16(tl + kColO + cb * 16, o);
      tmem_ld16(tl + kColR + cb * 16, rr);
      tmem_ld_wait_regs(o);
      tmem_ld_wait_regs(rr);
      const uint32_t w[8] = {dv[2 * cq].x,     dv[2 * cq].y,     dv[2 * cq].z,     dv[2 * cq].w,
                             dv[2 * cq + 1].x, dv[2 * cq + 1].y, dv[2 * cq + 1].z, dv[2 * cq + 1].w};
      uint32_t dp[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        sd = fmaf(f.x, __uint_as_float(o[2 * t]) * inv_l, sd);
        sd = fmaf(f.y, __uint_as_float(o[2 * t + 1]) * inv_l, sd);
        sm = fmaf(f.x, __uint_as_float(rr[2 * t]) * inv_den, sm);
        sm = fmaf(f.y, __uint_as_float(rr[2 * t + 1]) * inv_den, sm);
        dp[t] = pack_bf16x2(wm * f.x, wm * f.y);
      }
      if (row_ok) {
        n16[cb * 2] = make_uint4(dp[0], dp[1], dp[2], dp[3]);
        n16[cb * 2 + 1] = make_uint4(dp[4], dp[5], dp[6], dp[7]);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(o_empty);
  if (row_ok) {
    bs.lse[row] = m_row + log2f(l);
    bs.delta[row] = (1.f - g) * sd;
    bs.dden[row] = -wm * sm;
  }
  float db = row_ok ? g * (1.f - g) * (sm - sd) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
  if (lane == 0 && db != 0.f) atomicAdd(&bs.dbeta[h], db);
}

// Lazy rescaling: the running max used for the exponent is only raised when a
// row's new max exceeds it by more than 2^8 (so unnormalised P stays <= 256).
constexpr float kRescaleLog2 = 8.f;

struct AttnUnit {
  int seg_unit, qt, n, h, row_seg, row_q;
};

// The balanced schedule. Segments go in groups of gs; a group's units are
// ordered longest first (rank = n_qt - 1 - query tile, then segment), and each
// pass of G = gridDim.x consecutive units is dealt to the CTAs in alternate
// directions. With gs dividing G and gs * n_qt a multiple of 2G (the host
// picks gs = G / gcd(G, n_qt / 2)), every pair of passes gives each CTA the same
// total number of key tiles. Plain u -> (u / n_qt, u % n_qt) would give CTA b
// only the query tiles congruent to b modulo gcd(G, n_qt): with 148 SMs and 16
// tiles per segment, a quarter of the CTAs would do 10 / 8.5 of the average work.
// The map is a bijection on [0, units) (the last group may hold fewer
// segments, and its last pass fewer units), and every role evaluates it alike.
// (Also compiled for the host, where infini_attn_schedule_check runs it.)
__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ AttnUnit decode_unit(int u, int n_qt, int S, int H, int L, int N, int G,
                                                         int gs, int n_seg) {
  AttnUnit a;
  const int group_units = gs * n_qt;
  const int grp = u / group_units, w = u - grp * group_units;
  const int R = imin(gs, n_seg - grp * gs);  // segments in this group
  const int pass = w / G, pos = w - pass * G;
  const int in_pass = imin(G, R * n_qt - pass * G);
  const int idx = pass * G + ((pass & 1) ? in_pass - 1 - pos : pos);
  const int rank = idx / R;
  a.seg_unit = grp * gs + (idx - rank * R);
  a.qt = n_qt - 1 - rank;
  a.n = a.qt + 1;
  const int bh = a.seg_unit / S, s = a.seg_unit % S;
  a.h = bh % H;
  a.row_seg = bh * L + s * N;
  a.row_q = a.row_seg + a.qt * kTile;
  return a;
}


// kBwd: the backward's statistics pass (BwdStats) instead of the output; the
// local attention, the retrieval and every role but the epilogue's last step
// are the forward's.
template <bool kBwd>
__global__ void __launch_bounds__(kAttnThreads, 1)
tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
               const float* __restrict__ zp, const float* __restrict__ beta, __nv_bfloat16* __restrict__ out,
               int L, int N, int S, int H, int units, int gs, uint32_t epoch, BwdStats bs) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled tiles need a 1024-byte aligned base; the dynamic window
  // starts there on sm_100. Should it ever not, do nothing and report.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kAttnTiles);
  float* xmax = reinterpret_cast<float*>(sm + kAttnTiles + 256);         // [2][128]
  float* lbuf = reinterpret_cast<float*>(sm + kAttnTiles + 256 + 1024);  // [2][128]
  [[maybe_unused]] float* mbuf = lbuf + 256;                              // [128] running max (kBwd)
  uint8_t* sQ = sm;                              // [2]
  uint8_t* sK = sm + 2 * kTileBytes;             // [kKRing]
  uint8_t* sV = sm + (2 + kKRing) * kTileBytes;  // [kVRing]

  uint64_t* q_full = bars + 0;     // [2]  TMA
  uint64_t* q_empty = bars + 2;    // [2]  retrieval MMA done with the Q buffer
  uint64_t* k_full = bars + 4;     // [3]  TMA
  uint64_t* k_empty = bars + 7;    // [3]  MMA done reading the slot
  uint64_t* v_full = bars + 10;    // [2]  TMA
  uint64_t* v_empty = bars + 12;   // [2]  MMA done reading the slot
  uint64_t* s_full = bars + 14;    // [2]  QK^T done
  uint64_t* p_full = bars + 16;    // [2]  P written to TMEM (8 softmax warps)
  uint64_t* pv_done = bars + 18;   //      one phase per PV
  uint64_t* l_full = bars + 19;    //      row sums handed to the epilogue (8 warps)
  uint64_t* l_empty = bars + 20;   //      row sums taken (4 epilogue warps)
  uint64_t* sq_full = bars + 21;   //      sigma(Q) written over the Q buffer (4 epilogue warps)
  uint64_t* o_full = bars + 22;    //      the unit's last PV and its retrieval done
  uint64_t* o_empty = bars + 24;   //      epilogue done reading O and R (4 epilogue warps)
  uint64_t* drain = bars + 26;     //      abort path: in-flight MMAs
  uint64_t* qk_last = bars + 27;   // [2]  the unit's last QK^T done: Q buffer free for sigma(Q)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 29);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = N / kTile;
  const int n_seg = units / n_qt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 29; ++i) {
      uint32_t count = 1;
      if ((i >= 16 && i <= 17) || i == 19) count = 8;                  // p_full, l_full
      if ((i >= 20 && i <= 21) || (i >= 24 && i <= 25)) count = 4;     // l_empty, sq_full, o_empty
      mbar_init(&bars[i], count);
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
  // Producer bookkeeping for the abort path, 2 bits per buffer (armed, parity
  // of the last armed phase): Q[2] at bits 0-3, K ring at 4-9, V ring at 10-13.
  uint32_t armed = 0;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    // The whole warp walks the units (uniform control flow keeps the
    // bookkeeping in uniform registers); one elected lane issues the copies.
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmM);
    int kc = 0, vc = 0;
    [[maybe_unused]] uint32_t trn = 0;
    auto load_k = [&](int row, const CUtensorMap* m) {
      const int slot = kc % kKRing, use = kc / kKRing;
      if (use > 0 && !(ok = mbar_wait_warp(&k_empty[slot], (use - 1) & 1, epoch))) return;
      armed = (armed & ~(3u << (4 + 2 * slot))) | ((2u | (use & 1)) << (4 + 2 * slot));
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(&k_full[slot], kTileBytes);
        load_tile(sK + slot * kTileBytes, m, row, &k_full[slot]);
      }
      __syncwarp();
      TC_TRACE(trn, 0, 1, kc);
      ++kc;
    };
    auto load_v = [&](int row) {
      const int slot = vc % kVRing, use = vc / kVRing;
      if (use > 0 && !(ok = mbar_wait_warp(&v_empty[slot], (use - 1) & 1, epoch))) return;
      armed = (armed & ~(3u << (10 + 2 * slot))) | ((2u | (use & 1)) << (10 + 2 * slot));
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(&v_full[slot], kTileBytes);
        load_tile(sV + slot * kTileBytes, &tmV, row, &v_full[slot]);
      }
      __syncwarp();
      TC_TRACE(trn, 0, 2, vc);
      ++vc;
    };
    // Loads go in the order the MMA warp first uses them: per unit K_1, V_0,
    // K_2, V_1, ..., K_{n-1}, V_{n-2}, then the unit's M tile, the next
    // unit's Q tile and K_0 (its QK^T(0) comes before this unit's last PV),
    // then V_{n-1}. The K ring order (K_0 .. K_{n-1}, M, next K_0, ...) is the
    // one the MMA warp's ring positions assume.
    auto load_q = [&](int i2, const AttnUnit& a2) {
      const int qb = i2 & 1;
      if (i2 >= 2 && !(ok = mbar_wait_warp(&q_empty[qb], ((i2 - 2) >> 1) & 1, epoch))) return;
      armed = (armed & ~(3u << (2 * qb))) | ((2u | ((i2 >> 1) & 1)) << (2 * qb));
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(&q_full[qb], kTileBytes);
        load_tile(sQ + qb * kTileBytes, &tmQ, a2.row_q, &q_full[qb]);
      }
      __syncwarp();
      TC_TRACE(trn, 0, 3, i2);
    };
    int i = 0;
    if (blockIdx.x < (unsigned)units) {
      const AttnUnit a0 = decode_unit(blockIdx.x, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
      load_q(0, a0);
      if (ok) load_k(a0.row_seg, &tmK);
    }
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const AttnUnit a = decode_unit(u, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
      for (int j = 1; j < a.n && ok; ++j) {
        load_k(a.row_seg + j * kTile, &tmK);
        if (ok) load_v(a.row_seg + (j - 1) * kTile);
      }
      if (ok) load_k(a.seg_unit * kD, &tmM);  // M_{s-1} of this unit
      const int u2 = u + (int)gridDim.x;
      if (ok && u2 < units) {
        const AttnUnit a2 = decode_unit(u2, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
        load_q(i + 1, a2);
        if (ok) load_k(a2.row_seg, &tmK);
      }
      if (ok) load_v(a.row_seg + (a.n - 1) * kTile);
    }
    TC_TRACE_END(trn, 0);
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    // The whole warp runs the loop and one elected lane issues every MMA and
    // commit (a commit tracks the MMAs issued by its own thread, and elect.sync
    // picks the same lane each time the warp is converged).
    const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
    const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
    const uint64_t dq0 = desc_kmajor_sw128(smem_u32(sQ));
    const uint64_t dk0 = desc_kmajor_sw128(smem_u32(sK));
    const uint64_t dkmn0 = desc_mnmajor_sw128(smem_u32(sK), kHalf);
    const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(sV), kHalf);
    constexpr uint32_t kTileD = kTileBytes >> 4;
    int kc = 0, vc = 0, sc = 0;
    [[maybe_unused]] uint32_t trn = 0;
    // The previous unit's retrieval, issued after the current unit's first QK^Ts.
    int prev_i = -1, prev_mpos = 0;
    // QK^T of the K-ring position `pos` into the next S buffer.
    auto qk_at = [&](int qb, bool last, int pos) {
      const int slot = pos % kKRing;
      if (!(ok = mbar_wait_warp(&k_full[slot], (pos / kKRing) & 1, epoch))) return;
      tc_fence_after();
      const int sb = sc & 1;
      const uint64_t da = dq0 + qb * kTileD, db = dk0 + slot * kTileD;
      const uint32_t dst = tmem + sb * 128;
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_bf16_ss(dst, da + off, db + off, id_qk, kk != 0);
        }
        mma_commit(&s_full[sb]);
        mma_commit(&k_empty[slot]);
        if (last) mma_commit(&qk_last[qb]);
      }
      __syncwarp();
      TC_TRACE(trn, 1, 14, sc);
      ++sc;
    };
    auto qk = [&](int qb, bool last) { qk_at(qb, last, kc++); };
    // PV for global tile `tile`; the first of a unit overwrites O once the
    // previous unit's epilogue has read O and R.
    auto pv = [&](int tile, bool first, int unit_i) {
      TC_TRACE(trn, 1, 12, tile);
      const int sb = tile & 1;
      const int vslot = vc % kVRing, vuse = vc / kVRing;
      ++vc;
      if (!(ok = mbar_wait_warp(&p_full[sb], (tile >> 1) & 1, epoch) && mbar_wait_warp(&v_full[vslot], vuse & 1, epoch))) return;
      if (first && unit_i >= 1 && !(ok = mbar_wait_warp(o_empty, (unit_i - 1) & 1, epoch))) return;
      tc_fence_after();
      const uint64_t db = dv0 + vslot * kTileD;
      const uint32_t dst = tmem + kColO, pa = tmem + sb * 128;
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(dst, pa + kk * 8, db + ((kk * 2048) >> 4), id_pv, (!first || kk != 0) ? 1u : 0u);
        mma_commit(&v_empty[vslot]);
        mma_commit(pv_done);
      }
      __syncwarp();
      TC_TRACE(trn, 1, 13, tile);
    };
    // o_full completes once per unit, after both its last PV and its
    // retrieval (issued in either order): the commit goes after whichever of
    // the two is issued second, and covers both.
    int last_pv_unit = -1, r_unit = -1;
    auto commit_o_if_done = [&](int unit) {
      if (last_pv_unit == unit && r_unit == unit) {
        if (elect_one_lane()) mma_commit(o_full);
        __syncwarp();
      }
    };
    auto retrieval = [&]() {
      if (prev_i < 0) return;
      const int qb = prev_i & 1;
      const int mslot = prev_mpos % kKRing;
      if (!(ok = mbar_wait_warp(sq_full, prev_i & 1, epoch) && mbar_wait_warp(&k_full[mslot], (prev_mpos / kKRing) & 1, epoch))) return;
      tc_fence_after();
      const uint64_t da = dq0 + qb * kTileD, db = dkmn0 + mslot * kTileD;
      const uint32_t dst = tmem + kColR;
      if (elect_one_lane()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_bf16_ss(dst, da + off, db + ((kk * 2048) >> 4), id_pv, kk != 0);
        }
        mma_commit(&k_empty[mslot]);
        mma_commit(&q_empty[qb]);
      }
      __syncwarp();
      TC_TRACE(trn, 1, 15, prev_i);
      r_unit = prev_i;
      commit_o_if_done(prev_i);
      prev_i = -1;
    };
    // The retrieval of the unit before is issued as soon as its sigma(Q) and
    // M tile are in (tested without waiting), so the epilogue can release O
    // and R early; the blocking form above is the fallback.
    auto try_retrieval = [&]() {
      if (prev_i < 0 || !ok) return;
      const int mslot = prev_mpos % kKRing;
      if (__all_sync(0xffffffffu, mbar_test_wait(sq_full, prev_i & 1) &&
                                      mbar_test_wait(&k_full[mslot], (prev_mpos / kKRing) & 1)))
        retrieval();
    };
    int i = 0;
    // A unit's QK^T of tile 0 is issued during the unit before it, right
    // after that unit's PV of its second-to-last tile (its S buffer is the one
    // that PV just read), so the softmax goes from one unit to the next
    // without waiting for a QK^T. Its K tile comes after the previous unit's
    // M tile in the K ring.
    bool early = false;  // this unit's QK^T(0) is already issued
    int tile0_next = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const AttnUnit a = decode_unit(u, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
      const int qb = i & 1;
      int tile0;
      if (early) {
        tile0 = tile0_next;
      } else {
        TC_TRACE(trn, 1, 10, i);
        if (!(ok = mbar_wait_warp(&q_full[qb], (i >> 1) & 1, epoch))) break;
        TC_TRACE(trn, 1, 11, i);
        tile0 = sc;
        qk(qb, a.n == 1);
      }
      early = false;
      if (ok && a.n >= 2) qk(qb, a.n == 2);
      // The previous unit's retrieval R = sigma(Q) M_{s-1}: its sigma(Q) was
      // written as soon as that unit's last QK^T completed, so this does not
      // wait on the previous unit's softmax. It goes before this unit's first
      // PV (which overwrites O after the epilogue has read O and R) and
      // before QK^T of tile 2, which needs the M tile's K-ring slot.
      if (ok) retrieval();
      // This unit's M tile takes the K-ring position after its last K tile;
      // the next unit's K_0 follows it.
      int mpos = -1;
      const int u2 = u + (int)gridDim.x;
      auto next_qk0 = [&]() {
        mpos = kc;  // every K tile of this unit has been issued
        if (!ok || u2 >= units) return;
        const AttnUnit a2 = decode_unit(u2, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
        TC_TRACE(trn, 1, 10, i + 1);
        if (!(ok = mbar_wait_warp(&q_full[qb ^ 1], ((i + 1) >> 1) & 1, epoch))) return;
        TC_TRACE(trn, 1, 11, i + 1);
        tile0_next = sc;
        qk_at(qb ^ 1, a2.n == 1, mpos + 1);
        early = ok;
      };
      if (a.n == 1) {
        next_qk0();
        prev_i = i;
        prev_mpos = mpos;
        try_retrieval();
        if (ok) pv(tile0, true, i);
        last_pv_unit = i;
        commit_o_if_done(i);
      } else {
        if (ok) pv(tile0, true, i);
        for (int j = 2; j < a.n && ok; ++j) {
          qk(qb, j == a.n - 1);
          if (ok) pv(tile0 + j - 1, false, i);
        }
        next_qk0();
        prev_i = i;
        prev_mpos = mpos;
        try_retrieval();
        if (ok) pv(tile0 + a.n - 1, false, i);
        last_pv_unit = i;
        commit_o_if_done(i);
      }
      try_retrieval();
      kc = mpos + (early ? 2 : 1);
    }
    if (ok) retrieval();
    TC_TRACE_END(trn, 1);
  } else if (warp < 10) {
    // ------------------------------------------------ softmax (two threads per query row)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int c0 = half * 64;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t pair_bar = 1 + quarter;  // the two warps holding rows 32*quarter..+31
    float* my_max = xmax + half * 128 + r;
    const float* other_max = xmax + (half ^ 1) * 128 + r;
    const float scale2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    [[maybe_unused]] const bool traced = quarter == 0;  // warps 4 and 8 (rows 0-31) record (channels 3, 4)
    [[maybe_unused]] uint32_t trn = 0;
    int sc = 0, i = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
      const AttnUnit a = decode_unit(u, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
      float m_run = -INFINITY, l_run = 0.f;
      // S of tile j + 1 is requested from TMEM at the end of tile j (while
      // tile j's P stores complete), within a unit: the next unit's first
      // QK^T is issued only after this unit's last P V, which needs this
      // unit's last P.
      uint32_t sr[64];
      bool pre = false;  // sr has a load of this tile's S in flight
      for (int j = 0; j < a.n; ++j, ++sc) {
        const int sb = sc & 1;
        const bool diag = j == a.n - 1;
        float mx = -INFINITY;
        if (traced) TC_TRACE(trn, 3 + half, 20, j);
        const bool w_ok = pre || (ok && mbar_wait_warp(&s_full[sb], (sc >> 1) & 1, epoch));
        if (traced) TC_TRACE(trn, 3 + half, 21, j);
        if (w_ok) {
          if (!pre) {
            tc_fence_after();
            tmem_ld32(tl + sb * 128 + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tl + sb * 128 + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          }
          tmem_ld_wait_regs(sr);
          if (diag) {  // key column c is visible to row r iff c <= r
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c0 + c > r) sr[c] = __float_as_uint(-INFINITY);
          }
          mx = row_max64(sr);
        }
        if (traced) TC_TRACE(trn, 3 + half, 22, j);
        // Both halves have their S in registers past this barrier, so either
        // may now overwrite the buffer's first 64 columns with P. The barrier
        // also counts the threads whose own 64 columns would raise the running
        // max (or whose wait failed): only then do the two halves of a row
        // exchange their maxima. With lazy rescaling that is rare after a
        // unit's first tile, and a row whose two halves both stay within
        // m_run + 2^8 keeps m_run.
        const bool flag = !w_ok || mx * scale2 > m_run + kRescaleLog2;
        if (named_bar_popc(pair_bar, 64, flag) == 0) {
          // fast path: no rescale anywhere in this pair of warps
        } else {
        if (w_ok) *my_max = mx;
        if (!(ok = named_bar_and(pair_bar, 64, w_ok))) break;
        const float m_new = fmaxf(mx, *other_max) * scale2;
        named_bar_sync(pair_bar, 64);  // both have read the exchange slots

        const bool need = m_new > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_tgt = need ? m_new : m_run;
          const float alpha = ex2(m_run - m_tgt);
          if (j > 0) {
            // O holds this unit's PVs so far; wait for the last one, then rescale this half.
            ok = mbar_wait_warp(pv_done, (sc - 1) & 1, epoch);
            if (ok) {
              tc_fence_after();
#pragma unroll 1
              for (int cb = 0; cb < 4; ++cb) {
                uint32_t o[16];
                tmem_ld16(tl + kColO + c0 + cb * 16, o);
                tmem_ld_wait_regs(o);
#pragma unroll
                for (int t = 0; t < 16; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                tmem_st16(tl + kColO + c0 + cb * 16, o);
              }
              tmem_st_wait();
            }
          }
          l_run *= alpha;
          m_run = m_tgt;
        }
        }
        if (!ok) continue;  // the next pair barrier takes both warps out
        if (traced) TC_TRACE(trn, 3 + half, 29, j);
        // p = 2^(s * log2(e)/sqrt(d) - m), packed as bf16 pairs in place (sr[c/2]).
        // On the diagonal tile a 32-column chunk that lies wholly right of
        // every row of this warp is all zeros and needs no exponentials.
        uint64_t acc2[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) acc2[t] = 0ull;
        const uint64_t sc2 = f32x2(scale2, scale2), nm2 = f32x2(-m_run, -m_run);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          if (diag && c0 + ch * 32 >= 32 * (quarter + 1)) {
#pragma unroll
            for (int c = ch * 32; c < ch * 32 + 32; c += 2) sr[c >> 1] = 0u;
          } else {
#pragma unroll
            for (int c = ch * 32; c < ch * 32 + 32; c += 2) exp2_pair(sr, c, sc2, nm2, acc2[(c >> 1) & 3]);
          }
          // P (128 bf16 = 64 columns) goes over the start of this S buffer;
          // this half writes its 32 columns, 16 per chunk, so the first store
          // overlaps the second chunk's exponentials.
          tmem_st16(tl + sb * 128 + half * 32 + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[ch * 16]));
        }
        l_run += sum_f32x2(acc2);
        if (traced) TC_TRACE(trn, 3 + half, 26, j);
        // Request the next tile's S now if its QK^T is already done (the
        // stores above have taken their registers); never wait for it here,
        // which would hold back this tile's P and with it the MMA order.
        pre = false;
        if (j + 1 < a.n && __all_sync(0xffffffffu, mbar_test_wait(&s_full[sb ^ 1], ((sc + 1) >> 1) & 1))) {
          tc_fence_after();
          tmem_ld32(tl + (sb ^ 1) * 128 + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(tl + (sb ^ 1) * 128 + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          pre = true;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
        if (traced) TC_TRACE(trn, 3 + half, 23, j);
      }
      // Hand the partial row sums to the epilogue warps. Both warps of the
      // pair agree on going on before either leaves the loop, so neither is
      // ever left waiting at a pair barrier.
      bool w_ok = ok;
      if (w_ok && i >= 1) w_ok = mbar_wait_warp(l_empty, (i - 1) & 1, epoch);
      if (w_ok) lbuf[half * 128 + r] = l_run;
      if constexpr (kBwd) {
        if (w_ok && half == 0) mbuf[r] = m_run;  // both halves of a row hold the same m_run
      }
      if (!(ok = named_bar_and(pair_bar, 64, w_ok))) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(l_full);
      if (traced) TC_TRACE(trn, 3 + half, 28, i);
    }
    if (traced) TC_TRACE_END(trn, 3 + half);
  } else {
    // ------------------------------------------------ epilogue (one row per thread)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    [[maybe_unused]] const bool traced = warp == 10;  // channel 5
    [[maybe_unused]] uint32_t trn = 0;
    int i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const AttnUnit a = decode_unit(u, n_qt, S, H, L, N, gridDim.x, gs, n_seg);
      const int qb = i & 1;
      if (traced) TC_TRACE(trn, 5, 30, i);
      // den = sigma(q) . z_{s-1} in fp32 from this row of the bf16 Q tile. The
      // tile is only read here, so this overlaps the unit's QK^T MMAs. Waiting on the Q buffer's barrier
      // (it cannot be a phase behind: the next load into the buffer needs this
      // unit's retrieval) makes the TMA-written tile visible to these threads.
      if (!(ok = mbar_wait_warp(&q_full[qb], (i >> 1) & 1, epoch))) break;
      const float g = gate_of(beta[a.h]);
      const float4* zs = reinterpret_cast<const float4*>(zp + (int64_t)a.seg_unit * kD);
      uint8_t* qrow = sQ + qb * kTileBytes;
      // sigma(q) of the row, packed as bf16 pairs, is parked in this row's
      // lane of the R columns (free from the previous unit's epilogue read
      // until this unit's retrieval) until the unit's last QK^T is done: then
      // it only has to be copied over the Q buffer, and the retrieval (and
      // with it the release of O for the next unit) waits for no sigma pass.
      float den = 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sqp[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = 4 * cc + k;
          const uint4 x = *reinterpret_cast<const uint4*>(qrow + sw128_offset(r, c * 8, 128));
          const float4 z0 = __ldg(&zs[2 * c]), z1 = __ldg(&zs[2 * c + 1]);
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
          const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
            const float s0 = elu1(f.x), s1 = elu1(f.y);
            den = fmaf(s0, zz[2 * t], den);
            den = fmaf(s1, zz[2 * t + 1], den);
            sqp[4 * k + t] = pack_bf16x2(s0, s1);
          }
        }
        tmem_st16(tl + kColR + cc * 16, sqp);
      }
      tmem_st_wait();
      if (traced) TC_TRACE(trn, 5, 31, i);
      // The unit's last QK^T has completed: sigma(Q) (unscaled) goes over the
      // Q buffer as the retrieval's A operand.
      if (!(ok = mbar_wait_warp(&qk_last[qb], (i >> 1) & 1, epoch))) break;
      if (traced) TC_TRACE(trn, 5, 34, i);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sqp[16];
        tmem_ld16(tl + kColR + cc * 16, sqp);
        tmem_ld_wait_regs(sqp);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(qrow + sw128_offset(r, (4 * cc + k) * 8, 128)) =
              make_uint4(sqp[4 * k], sqp[4 * k + 1], sqp[4 * k + 2], sqp[4 * k + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(sq_full);
      if (traced) TC_TRACE(trn, 5, 32, i);
      if (!(ok = mbar_wait_warp(l_full, i & 1, epoch))) break;
      if (traced) TC_TRACE(trn, 5, 33, i);
      const float l = lbuf[r] + lbuf[128 + r];
      [[maybe_unused]] float m_row = 0.f;
      if constexpr (kBwd) m_row = mbuf[r];
      __syncwarp();
      if (lane == 0) mbar_arrive(l_empty);
      const float wd = (1.f - g) / l;
      const float wm = den != 0.f ? g / den : 0.f;
      // After the retrieval: out = wd * O + wm * R.
      if (!(ok = mbar_wait_warp(o_full, i & 1, epoch))) break;
      tc_fence_after();
      if (traced) TC_TRACE(trn, 5, 24, i);
      const bool row_ok = INFINI_CHECK(a.row_q + r < n_seg * N);
      if constexpr (kBwd) {
        bwd_stats_row(bs, tl, a.row_q + r, row_ok, a.h, g, l, m_row, den, wm, lane, o_empty);
      } else {
        uint4* orow = reinterpret_cast<uint4*>(out + (int64_t)(a.row_q + r) * kD);
        // The row in two halves of 64 columns: the first half's stores go out
        // before the second half is read; O and R are released to the next
        // unit's first PV as soon as the second half is read, before its stores.
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
#pragma unroll
          for (int cq = 0; cq < 4; ++cq) {
            const int cb = hf * 4 + cq;
            uint32_t o[16], rr[16];
            tmem_ld16(tl + kColO + cb * 16, o);
            tmem_ld16(tl + kColR + cb * 16, rr);
            tmem_ld_wait_regs(o);
            tmem_ld_wait_regs(rr);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              pk[cq * 8 + t] = pack_bf16x2(fmaf(wm, __uint_as_float(rr[2 * t]), wd * __uint_as_float(o[2 * t])),
                                           fmaf(wm, __uint_as_float(rr[2 * t + 1]), wd * __uint_as_float(o[2 * t + 1])));
          }
          if (hf == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_empty);
          }
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              orow[hf * 8 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
      if (traced) TC_TRACE(trn, 5, 25, i);
    }
    if (traced) TC_TRACE_END(trn, 5);
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if (warp == 0 && lane == 0) {
      for (int b = 0; b < 2; ++b)
        if ((armed >> (2 * b)) & 2u) mbar_drain(&q_full[b], (armed >> (2 * b)) & 1u);
      for (int b = 0; b < kKRing; ++b)
        if ((armed >> (4 + 2 * b)) & 2u) mbar_drain(&k_full[b], (armed >> (4 + 2 * b)) & 1u);
      for (int b = 0; b < kVRing; ++b)
        if ((armed >> (10 + 2 * b)) & 2u) mbar_drain(&v_full[b], (armed >> (10 + 2 * b)) & 1u);
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

// A [rows, cols] bf16 row-major matrix (cols 128 or 64), loaded in
// box_rows x 64-column boxes with the 128-byte swizzle.
inline bool make_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows = kTile, int cols = kD) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace infini

#include "tc_pair_kernel.cuh"
#include "tc_seg64_kernels.cuh"
#include "tc_fused64_kernel.cuh"
#include "tc_bwd_kernels.cuh"

namespace infini {

// SMs of the current device (one persistent attention CTA per SM).
inline int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Nonzero per-call epoch for the abort word of the bounded waits.
inline uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{0};
  uint32_t e = counter.fetch_add(1) + 1;
  while (e == 0) e = counter.fetch_add(1) + 1;
  return e;
}

// Segments per group of the balanced attention schedule (decode_unit): the
// largest group size that divides the grid and makes a group an even number of
// passes; with an odd number of query tiles per segment, one group per grid.
inline int balance_group(int grid, int n_qt) {
  if (n_qt % 2 != 0) return grid;
  return grid / std::gcd(grid, n_qt / 2);
}

// True when tc_attn_pair_kernel launches with the per-thread register count
// its setmaxnreg split assumes (checked once per process).
inline bool pair_kernel_registers_ok() {
  static std::once_flag once;
  static bool good = false;
  std::call_once(once, []() {
    cudaFuncAttributes fa;
    good = cudaFuncGetAttributes(&fa, tc::tc_attn_pair_kernel) == cudaSuccess &&
           fa.numRegs == tc::kPairLaunchRegs;
  });
  return good;
}

// Head dimension 64 with 64-token segments: pairs of segments per CTA
// (tc_seg64_kernels.cuh), the same three launches.
inline int tc_forward64(const TcArgs& a, cudaStream_t st, const Trace& tr) {
  using namespace tc;
  const uint32_t epoch = next_epoch();
  const int64_t BH = a.B * a.H, rows = BH * a.L;
  const int L = (int)a.L, S = (int)a.S, H = (int)a.H;
  const int pairs = (S + 1) / 2;
  const int64_t units = BH * pairs;
  if (units >= (int64_t(1) << 31) || rows >= (int64_t(1) << 31)) return INFINI_ERR_SIZE;
  CUtensorMap mk128, mv64, mq, mm;
  if (!make_map(&mk128, a.k, rows, 128, kD64) || !make_map(&mv64, a.v, rows, 64, kD64)) return INFINI_ERR_CUDA;
  const int out_v8 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
  if (!a.state_only && !a.skip_state) {
    // A whole forward: the single-pass kernel, one CTA per (b, h).
    if (!make_map(&mq, a.q, rows, 128, kD64)) return INFINI_ERR_CUDA;
    if (cudaFuncSetAttribute(tc_fused64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFused64Smem) !=
        cudaSuccess)
      return INFINI_ERR_CUDA;
    if (!tr.mark(0, st)) return INFINI_ERR_CUDA;
    tc_fused64_kernel<<<(unsigned)BH, kF64Threads, kFused64Smem, st>>>(
        mq, mk128, mv64, a.beta, a.M_in, a.z_in, static_cast<__nv_bfloat16*>(a.out), a.M_out, a.z_out, L, S, H,
        out_v8, epoch);
    if (cudaGetLastError() != cudaSuccess || !tr.mark(1, st)) return INFINI_ERR_CUDA;
    return INFINI_OK;
  }
  if (!a.state_only && (!make_map(&mq, a.q, rows, 128, kD64) || !make_map(&mm, a.Mp, BH * a.S * kD64, 128, kD64)))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_state64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kState64Smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc_attn64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttn64Smem) !=
          cudaSuccess)
    return INFINI_ERR_CUDA;
  if (!tr.mark(0, st)) return INFINI_ERR_CUDA;
  if (!a.skip_state) {
    tc_state64_kernel<<<(unsigned)units, kSeg64Threads, kState64Smem, st>>>(mk128, mv64, L, S, pairs, a.dM, a.dz,
                                                                          epoch);
    if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  }
  if (!tr.mark(1, st)) return INFINI_ERR_CUDA;
  const int64_t flat = BH * ((int64_t)kD64 * kD64 + kD64) / 4;
  scan_state_kernel<__nv_bfloat16><<<(unsigned)((flat + kScanThreads - 1) / kScanThreads), kScanThreads, 0, st>>>(
      a.dM, a.dz, a.M_in, a.z_in, a.Mp, a.zp, a.M_out, a.z_out, BH, S, kD64);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(2, st)) return INFINI_ERR_CUDA;
  if (a.state_only) return INFINI_OK;
  CUtensorMap mk, mv;
  if (!make_map(&mk, a.k, rows, 128, kD64) || !make_map(&mv, a.v, rows, 128, kD64)) return INFINI_ERR_CUDA;
  tc_attn64_kernel<<<(unsigned)units, kSeg64Threads, kAttn64Smem, st>>>(
      mq, mk, mv, mm, a.zp, a.beta, static_cast<__nv_bfloat16*>(a.out), L, S, H, pairs, out_v8, epoch);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(3, st)) return INFINI_ERR_CUDA;
  return INFINI_OK;
}

inline int tc_forward(const TcArgs& a, cudaStream_t st, const Trace& tr) {
  using namespace tc;
  if (a.d == 64) return tc_forward64(a, st, tr);
  const uint32_t epoch = next_epoch();
  const int64_t BH = a.B * a.H, rows = BH * a.L;
  CUtensorMap mq, mk, mv, mm, mks, mvs, mm64;
  // 64-row boxes of k and v: the state kernel's chunks and the paired
  // attention kernel's key tiles.
  if (!make_map(&mks, a.k, rows, kSChunk) || !make_map(&mvs, a.v, rows, kSChunk)) return INFINI_ERR_CUDA;
  if (!a.state_only && (!make_map(&mq, a.q, rows) || !make_map(&mk, a.k, rows) || !make_map(&mv, a.v, rows) ||
                        !make_map(&mm, a.Mp, BH * a.S * kD) || !make_map(&mm64, a.Mp, BH * a.S * kD, kKT)))
    return INFINI_ERR_CUDA;
  if (cudaFuncSetAttribute(tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem) != cudaSuccess ||
      cudaFuncSetAttribute(tc_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmemBwd) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc_attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem) !=
          cudaSuccess)
    return INFINI_ERR_CUDA;
  // The paired kernel's setmaxnreg split draws on the registers it is launched
  // with; it is only correct when it launches with exactly kPairLaunchRegs.
  if (!pair_kernel_registers_ok()) return INFINI_ERR_CUDA;
  const int L = (int)a.L, N = (int)a.N, S = (int)a.S, H = (int)a.H;

  if (!tr.mark(0, st)) return INFINI_ERR_CUDA;
  if (!a.skip_state) {
    const int64_t seg_units = BH * S;
    const int sgrid = (int)std::min<int64_t>(seg_units, sm_count());
    tc_state_kernel<<<sgrid, kStateThreads, kStateSmem, st>>>(mks, mvs, L, N, S, (int)seg_units, a.dM, a.dz, epoch);
    if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  }
  if (!tr.mark(1, st)) return INFINI_ERR_CUDA;

  const int64_t flat = BH * ((int64_t)kD * kD + kD) / 4;
  scan_state_kernel<__nv_bfloat16><<<(unsigned)((flat + kScanThreads - 1) / kScanThreads), kScanThreads, 0, st>>>(
      a.dM, a.dz, a.M_in, a.z_in, a.Mp, a.zp, a.M_out, a.z_out, BH, S, kD);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(2, st)) return INFINI_ERR_CUDA;
  if (a.state_only) return INFINI_OK;

  const int n_qt = N / kTile;
  if (a.paired && n_qt % 2 == 0 && !a.bwd) {
    // Pairs of query tiles per work unit (tc_attn_pair_kernel).
    const int n_pairs = n_qt / 2;
    const int64_t units = BH * S * n_pairs;
    const int grid = (int)std::min<int64_t>(units, sm_count());
    const int gs = balance_group(grid, n_pairs);
    const int out_v8 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    tc_attn_pair_kernel<<<grid, kPairThreads, kPairSmem, st>>>(mq, mks, mvs, mm64, a.zp, a.beta,
                                                               static_cast<__nv_bfloat16*>(a.out), L, N, S, H,
                                                               (int)units, gs, out_v8, epoch);
  } else {
    const int64_t units = BH * S * n_qt;
    const int grid = (int)std::min<int64_t>(units, sm_count());
    const int gs = balance_group(grid, n_qt);
    if (a.bwd)
      tc_attn_kernel<true><<<grid, kAttnThreads, kAttnSmemBwd, st>>>(mq, mk, mv, mm, a.zp, a.beta, nullptr, L, N, S,
                                                                     H, (int)units, gs, epoch, *a.bwd);
    else
      tc_attn_kernel<false><<<grid, kAttnThreads, kAttnSmem, st>>>(mq, mk, mv, mm, a.zp, a.beta,
                                                                   static_cast<__nv_bfloat16*>(a.out), L, N, S, H,
                                                                   (int)units, gs, epoch, BwdStats{});
  }
  if (cudaGetLastError() != cudaSuccess || !tr.mark(3, st)) return INFINI_ERR_CUDA;
  return INFINI_OK;
}

}  // namespace infini
