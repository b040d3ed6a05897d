// Shared device helpers for the Infini-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infini {

// Device status word: bit 0 = a bounded wait gave up. Read and cleared by
// infini_attn_device_status(). The library is one translation unit, so the
// word is defined here.
__device__ unsigned int g_status = 0u;
constexpr unsigned int kStatusTimeout = 1u;

// Abort word for bounded waits: the host gives every call a fresh nonzero
// epoch; a wait that gives up stores the call's epoch here, and every other
// wait of the same call sees it and returns at once, so one stuck CTA does not
// make each later CTA wait out its own deadline. Stale values from earlier
// calls never match the current epoch.
__device__ unsigned int g_abort_epoch = 0u;

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_status, kStatusTimeout); }

// Bounds checks of the debug build. Compiled with INFINI_DEBUG, INFINI_CHECK(c)
// is c, and a false c sets bit 1 of the status word (the guarded access is
// then skipped by the caller); without it, INFINI_CHECK(c) is true and costs
// nothing. A failed check never traps: the kernel goes on, the host reads the
// bit through infini_attn_device_status (INFINI_ERR_BOUNDS).
constexpr unsigned int kStatusBounds = 2u;
#ifdef INFINI_DEBUG
__device__ __forceinline__ bool infini_check(bool c) {
  if (!c) atomicOr(&g_status, kStatusBounds);
  return c;
}
#define INFINI_CHECK(c) ::infini::infini_check(c)
#else
#define INFINI_CHECK(c) true
#endif

// Optional event trace of a forward call: events[i] is recorded on the stream
// after launch i (events[0] before the first launch). Host side only.
struct Trace {
  void* const* events;
  int n;
  bool mark(int i, cudaStream_t st) const {
    if (events == nullptr || i >= n) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
  }
};

// Load one I/O element as fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// sigma(x) = ELU(x) + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise.
__device__ __forceinline__ float elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float elu1_accurate(float x) { return x > 0.f ? x + 1.f : expf(x); }

// g = sigmoid(beta); beta = +inf -> 1, -inf -> 0 under IEEE arithmetic.
__device__ __forceinline__ float gate_of(float beta) { return 1.f / (1.f + expf(-beta)); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ROWS rows of a [*, D] tensor (rows tok_row0 .. ; rows >= valid read as
// zero) moved into shared memory as fp32 at row stride ST in two steps:
// issue() starts every 16-byte load of the calling thread (into registers),
// store() converts and writes them. A loop can put the work on the previous
// tile between the two, so the loads overlap it. NT threads take part.
template <typename T, int D, int ST, int ROWS, int NT>
struct RowTile {
  static constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte vector
  static constexpr int VPR = D / VE;              // vectors per row
  static_assert((ROWS * VPR) % NT == 0, "tile vectors per thread");
  static_assert(ST % 4 == 0, "16-byte aligned shared-memory rows");
  static constexpr int PER = ROWS * VPR / NT;
  uint4 r[PER];

  __device__ __forceinline__ void issue(const T* __restrict__ a, int64_t tok_row0, int valid, int tid) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int vec = tid + u * NT, row = vec / VPR, cv = vec % VPR;
      r[u] = row < valid ? *reinterpret_cast<const uint4*>(a + (tok_row0 + row) * D + cv * VE)
                         : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ __forceinline__ static void put(const uint4& x, float* d) {
    if constexpr (VE == 8) {  // bf16: the high half of an fp32 is the bf16 value
      *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u),
                                                  __uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u));
      *reinterpret_cast<float4*>(d + 4) = make_float4(__uint_as_float(x.z << 16), __uint_as_float(x.z & 0xffff0000u),
                                                      __uint_as_float(x.w << 16), __uint_as_float(x.w & 0xffff0000u));
    } else {
      *reinterpret_cast<uint4*>(d) = x;
    }
  }
  __device__ __forceinline__ void store(float* __restrict__ sa, int tid) const {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int vec = tid + u * NT, row = vec / VPR, cv = vec % VPR;
      put(r[u], sa + row * ST + cv * VE);
    }
  }
};

// The same for two tensors with the same rows (K and V, or Q and dout).
template <typename T, int D, int ST, int ROWS, int NT>
struct RowTilePair {
  RowTile<T, D, ST, ROWS, NT> ta, tb;
  __device__ __forceinline__ void issue(const T* __restrict__ a, const T* __restrict__ b, int64_t tok_row0,
                                        int valid, int tid) {
    ta.issue(a, tok_row0, valid, tid);
    tb.issue(b, tok_row0, valid, tid);
  }
  __device__ __forceinline__ void store(float* __restrict__ sa, float* __restrict__ sb, int tid) const {
    ta.store(sa, tid);
    tb.store(sb, tid);
  }
};

constexpr int kScoreStride = 33;  // [32][33] score blocks in shared memory

// The tensor-core tile helpers of the CUDA-core kernels (8 warps, 32-row
// tiles). All use mma.sync m16n8k8 with TF32 operands and fp32 accumulation:
// row r of the A fragment is lane / 4 (+ 8), its k index lane % 4 (+ 4), and B
// and C follow the same thread grouping.
//
// C[32][33] = A B^T for A, B of 32 fp32 rows at stride ST holding bf16 values
// (exact in TF32, so the products are exact): warp w computes the 16 x 8 block (rows 16 (w / 4).., columns
// 8 (w % 4)..) with mma.sync m16n8k8 TF32, fp32 accumulation. Row r of the
// m16n8k8 A fragment is lane / 4 (+ 8), its k index lane % 4 (+ 4); B and C
// follow the same thread grouping.
template <int D, int ST>
__device__ __forceinline__ void score_block_tf32(const float* __restrict__ A, const float* __restrict__ B,
                                                 float* __restrict__ C, int warp, int lane) {
  const int mi = warp >> 2, ni = warp & 3, gr = lane >> 2, tq = lane & 3;
  const float* a0p = A + (16 * mi + gr) * ST + tq;
  const float* a1p = a0p + 8 * ST;
  const float* bp = B + (8 * ni + gr) * ST + tq;
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int kk = 0; kk < D; kk += 8) {
    const uint32_t a0 = __float_as_uint(a0p[kk]), a1 = __float_as_uint(a1p[kk]);
    const uint32_t a2 = __float_as_uint(a0p[kk + 4]), a3 = __float_as_uint(a1p[kk + 4]);
    const uint32_t b0 = __float_as_uint(bp[kk]), b1 = __float_as_uint(bp[kk + 4]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  float* cp = C + (16 * mi + gr) * kScoreStride + 8 * ni + 2 * tq;
  cp[0] = c[0];
  cp[1] = c[1];
  cp[8 * kScoreStride] = c[2];
  cp[8 * kScoreStride + 1] = c[3];
}

// [32][kAccStride] fp32 blocks (P or dS) that feed the accumulating MMAs as
// the A operand: a stride of 36 makes the fragment reads conflict-free.
constexpr int kAccStride = 36;

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// c[n] (n < NTW, the 16 x 8 C fragments of columns 8 n ..) += A B over 32
// k: A = 16 rows of fp32 at stride kAccStride, taken as a TF32 high part plus
// the TF32 of the remainder (two MMAs, error ~2^-22 of |A|); B = 32 rows of
// bf16 values as fp32 at stride ST (exact in TF32), columns from B's start.
template <int NTW, int ST>
__device__ __forceinline__ void mma_acc_split(float (&c)[NTW][4], const float* __restrict__ A,
                                              const float* __restrict__ B, int lane) {
  const int gr = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int kk = 0; kk < 32; kk += 8) {
    const float af[4] = {A[gr * kAccStride + kk + tq], A[(gr + 8) * kAccStride + kk + tq],
                         A[gr * kAccStride + kk + tq + 4], A[(gr + 8) * kAccStride + kk + tq + 4]};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      hi[x] = tf32_rna(af[x]);
      lo[x] = __float_as_uint(af[x] - __uint_as_float(hi[x]));
    }
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      const uint32_t b0 = __float_as_uint(B[(kk + tq) * ST + 8 * n + gr]);
      const uint32_t b1 = __float_as_uint(B[(kk + tq + 4) * ST + 8 * n + gr]);
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
          "{%0, %1, %2, %3};"
          : "+f"(c[n][0]), "+f"(c[n][1]), "+f"(c[n][2]), "+f"(c[n][3])
          : "r"(hi[0]), "r"(hi[1]), "r"(hi[2]), "r"(hi[3]), "r"(b0), "r"(b1));
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
          "{%0, %1, %2, %3};"
          : "+f"(c[n][0]), "+f"(c[n][1]), "+f"(c[n][2]), "+f"(c[n][3])
          : "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3]), "r"(b0), "r"(b1));
    }
  }
}

// The C fragments of one warp's 16 x 8 NTW block into a [32][ST] fp32 array.
template <int NTW, int ST>
__device__ __forceinline__ void store_acc(const float (&c)[NTW][4], float* __restrict__ dst, int lane) {
  const int gr = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int n = 0; n < NTW; ++n) {
    *reinterpret_cast<float2*>(dst + gr * ST + 8 * n + 2 * tq) = make_float2(c[n][0], c[n][1]);
    *reinterpret_cast<float2*>(dst + (gr + 8) * ST + 8 * n + 2 * tq) = make_float2(c[n][2], c[n][3]);
  }
}

}  // namespace infini
