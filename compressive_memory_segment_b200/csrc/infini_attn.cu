// Host side of the C ABI declared in include/infini_attn.h: argument checks,
// workspace layout, path selection and kernel launches. No host
// synchronisation happens inside a forward call.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/infini_attn.h"
#include "common.cuh"
#include "scan_kernel.cuh"
#include "simt_kernels.cuh"
#include "tc_kernels.cuh"
#include "tc_bwd_host.cuh"
#include "decode_kernel.cuh"
#include "backward_kernels.cuh"

using namespace infini;

// Scratch for infini_attn_forward_noalloc: a fixed array in the library's
// device image, so that entry point never allocates. Host code may not use the
// array's name as a device address; it fetches the address per device with
// cudaGetSymbolAddress (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[INFINI_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kWsAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Plan {
  int64_t B, H, L, d, N, S, BH;
  int dtype;
  size_t off_dM, off_dz, off_Mp, off_zp, total;
};

// Validates the shape part of a call and fills the workspace layout.
int make_plan(const infini_shape* shp, int64_t seg_len, Plan* p) {
  if (!shp) return INFINI_ERR_NULL;
  if (shp->B < 1 || shp->H < 1 || shp->L < 1 || seg_len < 1) return INFINI_ERR_SHAPE;
  if (shp->L % seg_len != 0) return INFINI_ERR_SHAPE;
  if (shp->d != 64 && shp->d != 128) return INFINI_ERR_UNSUPPORTED;
  if (shp->dtype != INFINI_F32 && shp->dtype != INFINI_BF16) return INFINI_ERR_UNSUPPORTED;
  // Token rows are indexed with 32-bit TMA coordinates and int CTA indices.
  if (shp->B > (1 << 16) || shp->H > (1 << 16)) return INFINI_ERR_SIZE;
  const int64_t rows = shp->B * shp->H * shp->L;
  if (rows >= (int64_t(1) << 31) || seg_len >= (int64_t(1) << 30)) return INFINI_ERR_SIZE;
  p->B = shp->B; p->H = shp->H; p->L = shp->L; p->d = shp->d; p->N = seg_len;
  p->S = shp->L / seg_len; p->BH = shp->B * shp->H; p->dtype = shp->dtype;
  if (p->S * (p->N + 127) / 128 >= (int64_t(1) << 31)) return INFINI_ERR_SIZE;
  const size_t seg_units = (size_t)p->BH * (size_t)p->S;
  const size_t mat = seg_units * (size_t)p->d * (size_t)p->d * sizeof(float);
  const size_t vec = seg_units * (size_t)p->d * sizeof(float);
  p->off_dM = 0;
  p->off_dz = round_up(p->off_dM + mat, kWsAlign);
  p->off_Mp = round_up(p->off_dz + vec, kWsAlign);  // fp32 on the CUDA-core path, bf16 on tcgen05
  p->off_zp = round_up(p->off_Mp + mat, kWsAlign);
  p->total = round_up(p->off_zp + vec, kWsAlign);
  return INFINI_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// The tensor-core kernels cover bf16 with d = 128 and segments of whole
// 128-row tiles, and bf16 with d = 64 and 64-token segments (two per tile).
bool tc_covers(const Plan& p) {
  return kTcPathBuilt && p.dtype == INFINI_BF16 &&
         ((p.d == 128 && p.N % 128 == 0) || (p.d == 64 && p.N == 64));
}

int resolve_path(const Plan& p, int path) {
  if (path == INFINI_PATH_AUTO) return tc_covers(p) ? (int)INFINI_PATH_TC : (int)INFINI_PATH_SIMT;
  if (path == INFINI_PATH_SIMT) return INFINI_PATH_SIMT;
  if (path == INFINI_PATH_TC) return tc_covers(p) ? (int)INFINI_PATH_TC : (int)INFINI_ERR_UNSUPPORTED;
  if (path == INFINI_PATH_TC_PAIRED)
    return tc_covers(p) && p.d == 128 && p.N % 256 == 0 ? (int)INFINI_PATH_TC_PAIRED : (int)INFINI_ERR_UNSUPPORTED;
  return INFINI_ERR_UNSUPPORTED;
}

// Opt-in dynamic shared memory is a per-function, per-device attribute.
template <typename F>
cudaError_t allow_smem(F* fn, size_t bytes) {
  return cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D>
int launch_simt(const Plan& p, const T* q, const T* k, const T* v, const float* beta,
                const float* M_in, const float* z_in, T* out, float* M_out, float* z_out,
                char* ws, cudaStream_t st, const Trace& tr, bool state_only = false, bool skip_state = false) {
  float* dM = reinterpret_cast<float*>(ws + p.off_dM);
  float* dz = reinterpret_cast<float*>(ws + p.off_dz);
  float* Mp = reinterpret_cast<float*>(ws + p.off_Mp);
  float* zp = reinterpret_cast<float*>(ws + p.off_zp);
  const int N = (int)p.N, S = (int)p.S;

  if (!tr.mark(0, st)) return INFINI_ERR_CUDA;
  if (!skip_state) {
    simt_state_kernel<T, D><<<dim3(S, p.H, p.B), kSimtStateThreads, 0, st>>>(k, v, p.L, N, dM, dz);
    if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  }
  if (!tr.mark(1, st)) return INFINI_ERR_CUDA;

  const int64_t flat = p.BH * ((int64_t)D * D + D) / 4;
  scan_state_kernel<float><<<(unsigned)((flat + kScanThreads - 1) / kScanThreads), kScanThreads, 0, st>>>(
      dM, dz, M_in, z_in, Mp, zp, M_out, z_out, p.BH, S, D);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(2, st)) return INFINI_ERR_CUDA;
  if (state_only) return INFINI_OK;

  constexpr size_t smem = simt_attn_smem_bytes<D>();
  if (allow_smem(simt_attn_kernel<T, D>, smem) != cudaSuccess) return INFINI_ERR_CUDA;
  const int64_t blocks_x = (int64_t)S * ((N + kSimtAttnRows - 1) / kSimtAttnRows);
  simt_attn_kernel<T, D><<<dim3((unsigned)blocks_x, p.H, p.B), kSimtAttnWarps * 32, smem, st>>>(
      q, k, v, beta, Mp, zp, p.L, N, S, out);
  if (cudaGetLastError() != cudaSuccess || !tr.mark(3, st)) return INFINI_ERR_CUDA;
  return INFINI_OK;
}

template <typename T>
int dispatch_simt(const Plan& p, const void* q, const void* k, const void* v, const float* beta,
                  const float* M_in, const float* z_in, void* out, float* M_out, float* z_out,
                  char* ws, cudaStream_t st, const Trace& tr, bool state_only = false, bool skip_state = false) {
  const T* qq = static_cast<const T*>(q);
  const T* kk = static_cast<const T*>(k);
  const T* vv = static_cast<const T*>(v);
  T* oo = static_cast<T*>(out);
  if (p.d == 64)
    return launch_simt<T, 64>(p, qq, kk, vv, beta, M_in, z_in, oo, M_out, z_out, ws, st, tr, state_only, skip_state);
  return launch_simt<T, 128>(p, qq, kk, vv, beta, M_in, z_in, oo, M_out, z_out, ws, st, tr, state_only, skip_state);
}

int check_pointers(const Plan& p, const void* q, const void* k, const void* v, const float* beta,
                   const float* M_in, const float* z_in, const void* out, const float* M_out,
                   const float* z_out) {
  if (!q || !k || !v || !beta || !out || !M_out || !z_out) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  const void* ptrs[] = {q, k, v, out, beta, M_out, z_out, M_in, z_in};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return INFINI_ERR_ALIGN;
  const size_t elt = p.dtype == INFINI_F32 ? 4 : 2;
  const size_t act = (size_t)p.BH * (size_t)p.L * (size_t)p.d * elt;
  const size_t mbytes = (size_t)p.BH * (size_t)p.d * (size_t)p.d * sizeof(float);
  const size_t zbytes = (size_t)p.BH * (size_t)p.d * sizeof(float);
  const size_t bbytes = (size_t)p.H * sizeof(float);
  // out must not overlap any input.
  if (overlap(out, act, q, act) || overlap(out, act, k, act) || overlap(out, act, v, act) ||
      overlap(out, act, beta, bbytes) || overlap(out, act, M_out, mbytes) ||
      overlap(out, act, z_out, zbytes))
    return INFINI_ERR_ALIAS;
  if (M_in && (overlap(out, act, M_in, mbytes) || overlap(out, act, z_in, zbytes))) return INFINI_ERR_ALIAS;
  // M_out / z_out: equal to M_in / z_in is fine (in place); any other overlap is not.
  const void* ins[] = {q, k, v};
  for (const void* x : ins)
    if (overlap(M_out, mbytes, x, act) || overlap(z_out, zbytes, x, act)) return INFINI_ERR_ALIAS;
  if (overlap(M_out, mbytes, z_out, zbytes) || overlap(M_out, mbytes, beta, bbytes) ||
      overlap(z_out, zbytes, beta, bbytes))
    return INFINI_ERR_ALIAS;
  if (M_in) {
    if (M_out != M_in && overlap(M_out, mbytes, M_in, mbytes)) return INFINI_ERR_ALIAS;
    if (z_out != z_in && overlap(z_out, zbytes, z_in, zbytes)) return INFINI_ERR_ALIAS;
    if (overlap(M_out, mbytes, z_in, zbytes) || overlap(z_out, zbytes, M_in, mbytes)) return INFINI_ERR_ALIAS;
  }
  return INFINI_OK;
}

// The state phase reads k, v and writes the block totals (M_out, z_out).
int check_state_pointers(const Plan& p, const void* k, const void* v, const float* M_tot, const float* z_tot) {
  if (!k || !v || !M_tot || !z_tot) return INFINI_ERR_NULL;
  const void* ptrs[] = {k, v, M_tot, z_tot};
  for (const void* x : ptrs)
    if (!aligned16(x)) return INFINI_ERR_ALIGN;
  const size_t elt = p.dtype == INFINI_F32 ? 4 : 2;
  const size_t act = (size_t)p.BH * (size_t)p.L * (size_t)p.d * elt;
  const size_t mb = (size_t)p.BH * (size_t)p.d * (size_t)p.d * sizeof(float);
  const size_t zb = (size_t)p.BH * (size_t)p.d * sizeof(float);
  if (overlap(M_tot, mb, k, act) || overlap(M_tot, mb, v, act) || overlap(z_tot, zb, k, act) ||
      overlap(z_tot, zb, v, act) || overlap(M_tot, mb, z_tot, zb))
    return INFINI_ERR_ALIAS;
  return INFINI_OK;
}

// Device address of the built-in scratch array in the current device's
// context. It is looked up on every call (a host-side table lookup once the
// library's module is loaded on the device), so a context that was destroyed
// and created again (cudaDeviceReset) yields the array's new address rather
// than a stale one. The first call on a device may load the module there.
int noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return INFINI_ERR_CUDA;
  *out = p;
  return INFINI_OK;
}

// Largest segment length the decode step takes (the chunk grid dimension and
// the partials stay small).
constexpr int64_t kDecodeMaxN = 32768;

// Decode workspace: the fold's (the one-segment forward workspace) followed
// by the per-chunk partials of the step.
size_t decode_partials_offset(const Plan& p) { return round_up(p.total, kWsAlign); }
size_t decode_ws_total(const Plan& p) {
  const int max_chunks = (int)((p.N + kDecodeChunk - 1) / kDecodeChunk);
  const size_t per = p.d == 64 ? decode_partial_floats<64>(max_chunks) : decode_partial_floats<128>(max_chunks);
  return round_up(decode_partials_offset(p) + (size_t)p.BH * per * sizeof(float), kWsAlign);
}

template <typename T, int D>
int launch_decode(const Plan& p, const void* q, const void* k, const void* v, const float* beta,
                  void* k_cache, void* v_cache, int64_t pos, const float* M, const float* z, void* out,
                  char* ws, cudaStream_t st) {
  const int max_chunks = (int)((p.N + kDecodeChunk - 1) / kDecodeChunk);
  const int n_chunks = (int)((pos + kDecodeChunk) / kDecodeChunk);
  float* part = reinterpret_cast<float*>(ws + decode_partials_offset(p));
  decode_partial_kernel<T, D><<<dim3((unsigned)n_chunks + 1, (unsigned)p.BH), kDecodeThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(k_cache),
      static_cast<T*>(v_cache), (int)p.N, (int)pos, max_chunks, M, z, part);
  if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  decode_combine_kernel<T, D><<<(unsigned)p.BH, D, 0, st>>>(part, (int)pos, max_chunks, (int)p.H, beta,
                                                             static_cast<T*>(out));
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// Fold one full segment (the cache, as a [B,H,N,d] sequence with seg_len N)
// into (M, z) in place: the forward's state and scan kernels, no attention.
int fold_segment(const Plan& p, const void* k_cache, const void* v_cache, float* M, float* z, char* ws,
                 cudaStream_t st) {
  Trace tr{nullptr, 0};
  if (resolve_path(p, INFINI_PATH_AUTO) == INFINI_PATH_TC) {
    TcArgs a;
    a.B = p.B; a.H = p.H; a.L = p.L; a.N = p.N; a.S = p.S; a.d = p.d;
    a.q = nullptr; a.k = k_cache; a.v = v_cache; a.beta = nullptr; a.M_in = M; a.z_in = z;
    a.out = nullptr; a.M_out = M; a.z_out = z;
    a.dM = reinterpret_cast<float*>(ws + p.off_dM);
    a.dz = reinterpret_cast<float*>(ws + p.off_dz);
    a.Mp = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Mp);
    a.zp = reinterpret_cast<float*>(ws + p.off_zp);
    a.state_only = true;
    return tc_forward(a, st, tr);
  }
  if (p.dtype == INFINI_F32)
    return dispatch_simt<float>(p, nullptr, k_cache, v_cache, nullptr, M, z, nullptr, M, z, ws, st, tr, true);
  return dispatch_simt<__nv_bfloat16>(p, nullptr, k_cache, v_cache, nullptr, M, z, nullptr, M, z, ws, st, tr, true);
}

// Backward workspace: the forward's (dM, dz, M_{s-1}, z_{s-1}), then the
// per-row lse, Delta, dnum, dden, the per-segment state gradients G, Gz,
// scratch for the recomputed final state and dnum in bf16 (the tensor-core
// path's MMA operand).
struct BwdPlan {
  Plan p;
  size_t off_lse, off_delta, off_dnum, off_dden, off_G, off_Gz, off_Mo, off_zo, off_dnum16, total;
};

int make_bwd_plan(const infini_shape* shp, int64_t seg_len, BwdPlan* b) {
  int rc = make_plan(shp, seg_len, &b->p);
  if (rc != INFINI_OK) return rc;
  const Plan& p = b->p;
  const size_t rows = (size_t)p.BH * (size_t)p.L, D = (size_t)p.d, segs = (size_t)p.BH * (size_t)p.S;
  b->off_lse = round_up(p.total, kWsAlign);
  b->off_delta = round_up(b->off_lse + rows * 4, kWsAlign);
  b->off_dnum = round_up(b->off_delta + rows * 4, kWsAlign);
  b->off_dden = round_up(b->off_dnum + rows * D * 4, kWsAlign);
  b->off_G = round_up(b->off_dden + rows * 4, kWsAlign);
  b->off_Gz = round_up(b->off_G + segs * D * D * 4, kWsAlign);
  b->off_Mo = round_up(b->off_Gz + segs * D * 4, kWsAlign);
  b->off_zo = round_up(b->off_Mo + (size_t)p.BH * D * D * 4, kWsAlign);
  b->off_dnum16 = round_up(b->off_zo + (size_t)p.BH * D * 4, kWsAlign);
  b->total = round_up(b->off_dnum16 + rows * D * 2, kWsAlign);
  return INFINI_OK;
}

template <typename T, int D>
int launch_backward(const BwdPlan& b, const void* q, const void* k, const void* v, const float* beta,
                    const float* M_in, const float* z_in, const void* dout, const float* dM_out,
                    const float* dz_out, float* dq, float* dk, float* dv, float* dbeta, float* dM_in,
                    float* dz_in, char* ws, cudaStream_t st) {
  const Plan& p = b.p;
  const T* qq = static_cast<const T*>(q);
  const T* kk = static_cast<const T*>(k);
  const T* vv = static_cast<const T*>(v);
  const T* go = static_cast<const T*>(dout);
  float* Mo = reinterpret_cast<float*>(ws + b.off_Mo);
  float* zo = reinterpret_cast<float*>(ws + b.off_zo);
  Trace tr{nullptr, 0};
  if (cudaMemsetAsync(dbeta, 0, (size_t)p.H * sizeof(float), st) != cudaSuccess) return INFINI_ERR_CUDA;
  // M_{s-1}, z_{s-1} in fp32 (the forward's CUDA-core state and scan kernels).
  int rc = launch_simt<T, D>(p, qq, kk, vv, beta, M_in, z_in, nullptr, Mo, zo, ws, st, tr, true, false);
  if (rc != INFINI_OK) return rc;
  const float* Mp = reinterpret_cast<const float*>(ws + p.off_Mp);
  const float* zp = reinterpret_cast<const float*>(ws + p.off_zp);
  float* lse = reinterpret_cast<float*>(ws + b.off_lse);
  float* delta = reinterpret_cast<float*>(ws + b.off_delta);
  float* dnum = reinterpret_cast<float*>(ws + b.off_dnum);
  float* dden = reinterpret_cast<float*>(ws + b.off_dden);
  float* G = reinterpret_cast<float*>(ws + b.off_G);
  float* Gz = reinterpret_cast<float*>(ws + b.off_Gz);
  const int N = (int)p.N, S = (int)p.S;
  const dim3 grid((unsigned)((int64_t)S * ((N + kBwdRows - 1) / kBwdRows)), (unsigned)p.H, (unsigned)p.B);
  constexpr size_t smem_rows = bwd_rows_smem_bytes<D>();
  constexpr size_t smem_keys = bwd_keys_smem_bytes<D>();
  if (allow_smem(bwd_rows_kernel<T, D>, smem_rows) != cudaSuccess ||
      allow_smem(bwd_keys_kernel<T, D>, smem_keys) != cudaSuccess)
    return INFINI_ERR_CUDA;
  bwd_rows_kernel<T, D><<<grid, kBwdWarps * 32, smem_rows, st>>>(qq, kk, vv, beta, Mp, zp, go, p.L, N, S, dq, lse,
                                                                 delta, dnum, dden, dbeta);
  if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  bwd_state_grad_kernel<T, D><<<dim3(S, p.H, p.B), 256, 0, st>>>(qq, dnum, dden, p.L, N, G, Gz);
  if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
  if (launch_bwd_rscan(G, Gz, p.BH, S, D, dM_out, dM_in, dz_out, dz_in, st) != cudaSuccess) return INFINI_ERR_CUDA;
  bwd_keys_kernel<T, D><<<grid, kBwdWarps * 32, smem_keys, st>>>(qq, kk, vv, beta, go, lse, delta, G, Gz, p.L, N, S,
                                                                 dk, dv);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// The tensor-core backward (bf16, d = 128, seg_len % 128 == 0): the
// statistics pass is the forward's state, scan and attention kernels with
// the attention epilogue writing lse, Delta, dnum (bf16), dden and dbeta; the tcgen05 dQ kernel then writes dq and adds each query tile's
// sigma(Q)^T dnum and sigma(Q)^T dden into the zeroed G, Gz; the reverse scan
// over segments makes those the gradient reaching each M_s, z_s (and M_in,
// z_in); the tcgen05 dK/dV kernel last.
int launch_backward_tc(const BwdPlan& b, const void* q, const void* k, const void* v, const float* beta,
                       const float* M_in, const float* z_in, const void* dout, const float* dM_out,
                       const float* dz_out, float* dq, float* dk, float* dv, float* dbeta, float* dM_in,
                       float* dz_in, char* ws, cudaStream_t st) {
  const Plan& p = b.p;
  using T = __nv_bfloat16;
  constexpr int D = 128;
  if (cudaMemsetAsync(dbeta, 0, (size_t)p.H * sizeof(float), st) != cudaSuccess) return INFINI_ERR_CUDA;
  float* lse = reinterpret_cast<float*>(ws + b.off_lse);
  float* delta = reinterpret_cast<float*>(ws + b.off_delta);
  float* dden = reinterpret_cast<float*>(ws + b.off_dden);
  float* G = reinterpret_cast<float*>(ws + b.off_G);
  float* Gz = reinterpret_cast<float*>(ws + b.off_Gz);
  T* dnum16 = reinterpret_cast<T*>(ws + b.off_dnum16);
  BwdStats bs;
  bs.dout = static_cast<const T*>(dout);
  bs.lse = lse; bs.delta = delta; bs.dnum16 = dnum16; bs.dden = dden; bs.dbeta = dbeta;
  TcArgs a;
  a.B = p.B; a.H = p.H; a.L = p.L; a.N = p.N; a.S = p.S; a.d = p.d;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.M_in = M_in; a.z_in = z_in;
  a.out = nullptr;
  a.M_out = reinterpret_cast<float*>(ws + b.off_Mo);
  a.z_out = reinterpret_cast<float*>(ws + b.off_zo);
  a.dM = reinterpret_cast<float*>(ws + p.off_dM);
  a.dz = reinterpret_cast<float*>(ws + p.off_dz);
  a.Mp = reinterpret_cast<T*>(ws + p.off_Mp);
  a.zp = reinterpret_cast<float*>(ws + p.off_zp);
  a.bwd = &bs;
  Trace tr{nullptr, 0};
  int rc = tc_forward(a, st, tr);
  if (rc != INFINI_OK) return rc;
  const int S = (int)p.S;
  const size_t segs = (size_t)p.BH * (size_t)S;
  if (cudaMemsetAsync(G, 0, segs * D * D * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(Gz, 0, segs * D * sizeof(float), st) != cudaSuccess)
    return INFINI_ERR_CUDA;
  TcBwdArgs t;
  t.B = p.B; t.H = p.H; t.L = p.L; t.N = p.N; t.S = p.S;
  t.q = q; t.k = k; t.v = v; t.dout = dout;
  t.dnum16 = dnum16; t.Mp = a.Mp;
  t.beta = beta; t.zp = a.zp; t.lse = lse; t.delta = delta; t.dden = dden; t.G = G; t.Gz = Gz;
  t.dq = dq; t.dk = dk; t.dv = dv;
  if ((rc = tc_backward_local(t, st, false)) != INFINI_OK) return rc;
  if (launch_bwd_rscan(G, Gz, p.BH, S, D, dM_out, dM_in, dz_out, dz_in, st) != cudaSuccess) return INFINI_ERR_CUDA;
  return tc_backward_local(t, st, true);
}

// The tensor-core backward for d = 64 with 64-token segments: the state
// recompute (tcgen05 state kernel and scan), the pair kernel, the reverse
// scan of G and Gz, the state kernel.
int launch_backward_tc64(const BwdPlan& b, const void* q, const void* k, const void* v, const float* beta,
                         const float* M_in, const float* z_in, const void* dout, const float* dM_out,
                         const float* dz_out, float* dq, float* dk, float* dv, float* dbeta, float* dM_in,
                         float* dz_in, char* ws, cudaStream_t st) {
  const Plan& p = b.p;
  constexpr int D = 64;
  if (cudaMemsetAsync(dbeta, 0, (size_t)p.H * sizeof(float), st) != cudaSuccess) return INFINI_ERR_CUDA;
  TcArgs a;
  a.B = p.B; a.H = p.H; a.L = p.L; a.N = p.N; a.S = p.S; a.d = p.d;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.M_in = M_in; a.z_in = z_in;
  a.out = nullptr;
  a.M_out = reinterpret_cast<float*>(ws + b.off_Mo);
  a.z_out = reinterpret_cast<float*>(ws + b.off_zo);
  a.dM = reinterpret_cast<float*>(ws + p.off_dM);
  a.dz = reinterpret_cast<float*>(ws + p.off_dz);
  a.Mp = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Mp);
  a.zp = reinterpret_cast<float*>(ws + p.off_zp);
  a.state_only = true;
  Trace tr{nullptr, 0};
  int rc = tc_forward(a, st, tr);
  if (rc != INFINI_OK) return rc;
  float* G = reinterpret_cast<float*>(ws + b.off_G);
  float* Gz = reinterpret_cast<float*>(ws + b.off_Gz);
  TcBwd64Args t;
  t.B = p.B; t.H = p.H; t.L = p.L; t.S = p.S;
  t.q = q; t.k = k; t.v = v; t.dout = dout; t.Mp = a.Mp; t.beta = beta; t.zp = a.zp;
  t.G = G; t.Gz = Gz; t.dq = dq; t.dk = dk; t.dv = dv; t.dbeta = dbeta;
  if ((rc = tc_backward64(t, st, false)) != INFINI_OK) return rc;
  const int S = (int)p.S;
  if (launch_bwd_rscan(G, Gz, p.BH, S, D, dM_out, dM_in, dz_out, dz_in, st) != cudaSuccess) return INFINI_ERR_CUDA;
  return tc_backward64(t, st, true);
}

// One thread waits on an mbarrier that nothing arrives on, with a limit of
// limit_ns: the bounded wait gives up, records the timeout in the status word
// and returns, and the kernel exits normally.
__global__ void selftest_wait_kernel(uint64_t limit_ns, uint32_t epoch) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    (void)sm100::mbar_wait_for(&bar, 0, epoch, limit_ns);
  }
}

}  // namespace

extern "C" {

int infini_attn_version(void) { return 100; }

const char* infini_attn_strerror(int code) {
  switch (code) {
    case INFINI_OK: return "success";
    case INFINI_ERR_NULL: return "a required pointer is NULL (or only one of M_in/z_in given)";
    case INFINI_ERR_SHAPE: return "invalid shape: B, H, L, seg_len must be >= 1 and L % seg_len == 0";
    case INFINI_ERR_UNSUPPORTED: return "unsupported: d must be 64 or 128, dtype fp32 or bf16; forced path does not cover this shape";
    case INFINI_ERR_ALIGN: return "misaligned pointer: tensors need 16-byte, the workspace 256-byte alignment";
    case INFINI_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case INFINI_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case INFINI_ERR_WORKSPACE: return "workspace too small";
    case INFINI_ERR_ALIAS: return "overlapping buffers: out must not overlap inputs; M_out/z_out may only equal M_in/z_in exactly";
    case INFINI_ERR_SIZE: return "size too large for the kernels' indexing";
    case INFINI_ERR_SCRATCH: return "shape needs more scratch than the built-in buffer of infini_attn_forward_noalloc (INFINI_NOALLOC_SCRATCH_BYTES)";
    case INFINI_ERR_BOUNDS: return "a device-side index check of the debug build (INFINI_DEBUG) failed";
    default: return "unknown error code";
  }
}

size_t infini_attn_workspace_size(const infini_shape* shp, int64_t seg_len) {
  Plan p;
  if (make_plan(shp, seg_len, &p) != INFINI_OK) return 0;
  return p.total;
}

int infini_attn_select_path(const infini_shape* shp, int64_t seg_len) {
  Plan p;
  int rc = make_plan(shp, seg_len, &p);
  if (rc != INFINI_OK) return rc;
  return resolve_path(p, INFINI_PATH_AUTO);
}

int infini_attn_launch_count(const infini_shape* shp, int64_t seg_len, int path) {
  Plan p;
  int rc = make_plan(shp, seg_len, &p);
  if (rc != INFINI_OK) return rc;
  const int pth = resolve_path(p, path);
  if (pth < 0) return pth;
  return pth == INFINI_PATH_TC ? tc_launch_count(p.d, p.N) : 3;  // the paired path: state, scan, attention
}

enum Phase { kFull = 0, kStateOnly = 1, kSkipState = 2 };

static int forward_impl(const infini_shape* shp, const void* q, const void* k, const void* v,
                        const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                        void* out, float* M_out, float* z_out, void* workspace,
                        size_t workspace_bytes, int path, void* const* events, int n_events,
                        infini_stream_t stream, Phase phase = kFull) {
  Plan p;
  int rc = make_plan(shp, seg_len, &p);
  if (rc != INFINI_OK) return rc;
  if (phase == kStateOnly) {
    rc = check_state_pointers(p, k, v, M_out, z_out);
  } else {
    rc = check_pointers(p, q, k, v, beta, M_in, z_in, out, M_out, z_out);
  }
  if (rc != INFINI_OK) return rc;
  if (!workspace) return INFINI_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return INFINI_ERR_ALIGN;
  if (workspace_bytes < p.total) return INFINI_ERR_WORKSPACE;
  const int pth = resolve_path(p, path);
  if (pth < 0) return pth;
  const int launches = pth == INFINI_PATH_TC ? tc_launch_count(p.d, p.N, phase == kFull) : 3;
  if (events != nullptr && n_events != launches + 1) return INFINI_ERR_SHAPE;
  if (events == nullptr && n_events != 0) return INFINI_ERR_NULL;
  Trace tr{events, n_events};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (pth == INFINI_PATH_TC || pth == INFINI_PATH_TC_PAIRED) {
    TcArgs a;
    a.B = p.B; a.H = p.H; a.L = p.L; a.N = p.N; a.S = p.S; a.d = p.d;
    a.paired = pth == INFINI_PATH_TC_PAIRED;
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.M_in = M_in; a.z_in = z_in;
    a.out = out; a.M_out = M_out; a.z_out = z_out;
    a.dM = reinterpret_cast<float*>(ws + p.off_dM);
    a.dz = reinterpret_cast<float*>(ws + p.off_dz);
    a.Mp = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Mp);
    a.zp = reinterpret_cast<float*>(ws + p.off_zp);
    a.state_only = phase == kStateOnly;
    a.skip_state = phase == kSkipState;
    return tc_forward(a, st, tr);
  }
  if (p.dtype == INFINI_F32)
    return dispatch_simt<float>(p, q, k, v, beta, M_in, z_in, out, M_out, z_out, ws, st, tr, phase == kStateOnly,
                                phase == kSkipState);
  return dispatch_simt<__nv_bfloat16>(p, q, k, v, beta, M_in, z_in, out, M_out, z_out, ws, st, tr,
                                      phase == kStateOnly, phase == kSkipState);
}

int infini_attn_forward_ws(const infini_shape* shp, const void* q, const void* k, const void* v,
                           const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                           void* out, float* M_out, float* z_out, void* workspace,
                           size_t workspace_bytes, int path, infini_stream_t stream) {
  return forward_impl(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, workspace,
                      workspace_bytes, path, nullptr, 0, stream);
}

int infini_attn_state_ws(const infini_shape* shp, const void* k, const void* v, int64_t seg_len, float* M_tot,
                         float* z_tot, void* workspace, size_t workspace_bytes, int path, infini_stream_t stream) {
  return forward_impl(shp, nullptr, k, v, nullptr, nullptr, nullptr, seg_len, nullptr, M_tot, z_tot, workspace,
                      workspace_bytes, path, nullptr, 0, stream, kStateOnly);
}

int infini_attn_finish_ws(const infini_shape* shp, const void* q, const void* k, const void* v, const float* beta,
                          const float* M_in, const float* z_in, int64_t seg_len, void* out, float* M_out, float* z_out,
                          void* workspace, size_t workspace_bytes, int path, infini_stream_t stream) {
  return forward_impl(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, workspace, workspace_bytes, path,
                      nullptr, 0, stream, kSkipState);
}

int infini_attn_exscan_parts(int64_t n_M, int64_t n_z, int n_parts, int part, const float* totals_M,
                             const float* totals_z, const float* M_in, const float* z_in, float* off_M, float* off_z,
                             infini_stream_t stream) {
  if (n_M < 1 || n_z < 1 || n_parts < 1 || part < 0 || part >= n_parts) return INFINI_ERR_SHAPE;
  if (!totals_M || !totals_z || !off_M || !off_z) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if (n_M > (int64_t(1) << 40) || n_z > (int64_t(1) << 40)) return INFINI_ERR_SIZE;
  const void* ptrs[] = {totals_M, totals_z, off_M, off_z, M_in, z_in};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return INFINI_ERR_ALIGN;
  const size_t tm = (size_t)n_parts * n_M * 4, tz = (size_t)n_parts * n_z * 4, om = (size_t)n_M * 4, oz = (size_t)n_z * 4;
  if (overlap(off_M, om, totals_M, tm) || overlap(off_M, om, totals_z, tz) || overlap(off_z, oz, totals_M, tm) ||
      overlap(off_z, oz, totals_z, tz) || overlap(off_M, om, off_z, oz))
    return INFINI_ERR_ALIAS;
  if (M_in && ((M_in != off_M && overlap(off_M, om, M_in, om)) || (z_in != off_z && overlap(off_z, oz, z_in, oz)) ||
               overlap(off_M, om, z_in, oz) || overlap(off_z, oz, M_in, om)))
    return INFINI_ERR_ALIAS;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const unsigned gm = (unsigned)std::min<int64_t>((n_M + kScanThreads - 1) / kScanThreads, 65535);
  const unsigned gz = (unsigned)std::min<int64_t>((n_z + kScanThreads - 1) / kScanThreads, 65535);
  exscan_parts_kernel<<<gm, kScanThreads, 0, st>>>(totals_M, n_M, part, M_in, off_M);
  exscan_parts_kernel<<<gz, kScanThreads, 0, st>>>(totals_z, n_z, part, z_in, off_z);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_forward_traced(const infini_shape* shp, const void* q, const void* k, const void* v,
                               const float* beta, const float* M_in, const float* z_in,
                               int64_t seg_len, void* out, float* M_out, float* z_out,
                               void* workspace, size_t workspace_bytes, int path,
                               void* const* events, int n_events, infini_stream_t stream) {
  return forward_impl(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, workspace,
                      workspace_bytes, path, events, n_events, stream);
}

int infini_attn_forward(const infini_shape* shp, const void* q, const void* k, const void* v,
                        const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                        void* out, float* M_out, float* z_out, infini_stream_t stream) {
  Plan p;
  int rc = make_plan(shp, seg_len, &p);
  if (rc != INFINI_OK) return rc;
  rc = check_pointers(p, q, k, v, beta, M_in, z_in, out, M_out, z_out);
  if (rc != INFINI_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, p.total, st) != cudaSuccess) return INFINI_ERR_CUDA;
  rc = infini_attn_forward_ws(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, ws,
                              p.total, INFINI_PATH_AUTO, stream);
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_CUDA;
  return rc;
}

int infini_attn_forward_noalloc(const infini_shape* shp, const void* q, const void* k, const void* v,
                                const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                                void* out, float* M_out, float* z_out, infini_stream_t stream) {
  Plan p;
  int rc = make_plan(shp, seg_len, &p);
  if (rc != INFINI_OK) return rc;
  rc = check_pointers(p, q, k, v, beta, M_in, z_in, out, M_out, z_out);
  if (rc != INFINI_OK) return rc;
  if (p.total > INFINI_NOALLOC_SCRATCH_BYTES) return INFINI_ERR_SCRATCH;
  void* ws = nullptr;
  rc = noalloc_scratch(&ws);
  if (rc != INFINI_OK) return rc;
  return forward_impl(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, ws,
                      INFINI_NOALLOC_SCRATCH_BYTES, INFINI_PATH_AUTO, nullptr, 0, stream);
}

size_t infini_attn_decode_workspace_size(const infini_shape* shp) {
  Plan p;
  if (!shp || make_plan(shp, shp->L, &p) != INFINI_OK || p.N > kDecodeMaxN) return 0;
  return decode_ws_total(p);
}

int infini_attn_decode_step(const infini_shape* shp, const void* q, const void* k, const void* v,
                            const float* beta, void* k_cache, void* v_cache, int64_t pos, float* M, float* z,
                            void* out, void* workspace, size_t workspace_bytes, infini_stream_t stream) {
  if (!shp) return INFINI_ERR_NULL;
  Plan p;
  int rc = make_plan(shp, shp->L, &p);  // the cache holds one segment: L = N
  if (rc != INFINI_OK) return rc;
  if (p.N > kDecodeMaxN) return INFINI_ERR_SIZE;
  if (pos < 0 || pos >= p.N) return INFINI_ERR_SHAPE;
  if (!q || !k || !v || !beta || !k_cache || !v_cache || !M || !z || !out) return INFINI_ERR_NULL;
  const bool fold = pos == p.N - 1;
  if (!workspace) return INFINI_ERR_NULL;
  const void* ptrs[] = {q, k, v, beta, k_cache, v_cache, M, z, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return INFINI_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return INFINI_ERR_ALIGN;
  const size_t ws_need = decode_ws_total(p);
  if (workspace_bytes < ws_need) return INFINI_ERR_WORKSPACE;
  // No two of the buffers may overlap (the step writes out, a cache row and,
  // at a segment's end, M and z).
  const size_t elt = p.dtype == INFINI_F32 ? 4 : 2;
  const size_t row = (size_t)p.BH * (size_t)p.d * elt;
  const size_t cache = row * (size_t)p.N;
  const size_t mbytes = (size_t)p.BH * (size_t)p.d * (size_t)p.d * sizeof(float);
  const size_t zbytes = (size_t)p.BH * (size_t)p.d * sizeof(float);
  const void* bufs[] = {q, k, v, beta, k_cache, v_cache, M, z, out};
  const size_t sizes[] = {row, row, row, (size_t)p.H * sizeof(float), cache, cache, mbytes, zbytes, row};
  for (int a = 0; a < 9; ++a)
    for (int b = a + 1; b < 9; ++b)
      if (overlap(bufs[a], sizes[a], bufs[b], sizes[b])) return INFINI_ERR_ALIAS;
  for (int a = 0; a < 9; ++a)
    if (overlap(workspace, ws_need, bufs[a], sizes[a])) return INFINI_ERR_ALIAS;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* wsb = static_cast<char*>(workspace);
  if (p.dtype == INFINI_F32)
    rc = p.d == 64 ? launch_decode<float, 64>(p, q, k, v, beta, k_cache, v_cache, pos, M, z, out, wsb, st)
                   : launch_decode<float, 128>(p, q, k, v, beta, k_cache, v_cache, pos, M, z, out, wsb, st);
  else
    rc = p.d == 64 ? launch_decode<__nv_bfloat16, 64>(p, q, k, v, beta, k_cache, v_cache, pos, M, z, out, wsb, st)
                   : launch_decode<__nv_bfloat16, 128>(p, q, k, v, beta, k_cache, v_cache, pos, M, z, out, wsb, st);
  if (rc != INFINI_OK || !fold) return rc;
  return fold_segment(p, k_cache, v_cache, M, z, wsb, st);
}

size_t infini_attn_backward_workspace_size(const infini_shape* shp, int64_t seg_len) {
  BwdPlan b;
  if (make_bwd_plan(shp, seg_len, &b) != INFINI_OK) return 0;
  return b.total;
}

int infini_attn_backward(const infini_shape* shp, const void* q, const void* k, const void* v, const float* beta,
                         const float* M_in, const float* z_in, int64_t seg_len, const void* dout,
                         const float* dM_out, const float* dz_out, float* dq, float* dk, float* dv, float* dbeta,
                         float* dM_in, float* dz_in, void* workspace, size_t workspace_bytes,
                         infini_stream_t stream) {
  return infini_attn_backward_path(shp, q, k, v, beta, M_in, z_in, seg_len, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                                   dM_in, dz_in, workspace, workspace_bytes, INFINI_PATH_AUTO, stream);
}

// The tensor-core backward covers bf16 with d = 128 and segments of whole
// 128-row tiles, and bf16 with d = 64, 64-token segments and an even number
// of them per sequence (pairs of segments per 128-row tile).
bool tc_bwd_covers(const Plan& p) {
  return tc_covers(p) && (p.d == 128 || (p.d == 64 && p.N == 64 && p.S % 2 == 0));
}

int infini_attn_backward_path(const infini_shape* shp, const void* q, const void* k, const void* v,
                              const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                              const void* dout, const float* dM_out, const float* dz_out, float* dq, float* dk,
                              float* dv, float* dbeta, float* dM_in, float* dz_in, void* workspace,
                              size_t workspace_bytes, int path, infini_stream_t stream) {
  BwdPlan b;
  int rc = make_bwd_plan(shp, seg_len, &b);
  if (rc != INFINI_OK) return rc;
  const Plan& p = b.p;
  if (path == INFINI_PATH_AUTO) path = tc_bwd_covers(p) ? INFINI_PATH_TC : INFINI_PATH_SIMT;
  if (path != INFINI_PATH_SIMT && !(path == INFINI_PATH_TC && tc_bwd_covers(p))) return INFINI_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !dout || !dq || !dk || !dv || !dbeta || !dM_in || !dz_in || !workspace)
    return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr) || (dM_out == nullptr) != (dz_out == nullptr)) return INFINI_ERR_NULL;
  const size_t elt = p.dtype == INFINI_F32 ? 4 : 2;
  const size_t act = (size_t)p.BH * (size_t)p.L * (size_t)p.d * elt;
  const size_t grad = (size_t)p.BH * (size_t)p.L * (size_t)p.d * 4;
  const size_t mb = (size_t)p.BH * (size_t)p.d * (size_t)p.d * 4, zb = (size_t)p.BH * (size_t)p.d * 4;
  const size_t hb = (size_t)p.H * 4;
  const void* bufs[] = {q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta, dM_in, dz_in, workspace};
  const size_t sizes[] = {act, act, act, hb, mb, zb, act, mb, zb, grad, grad, grad, hb, mb, zb, b.total};
  const bool written[] = {false, false, false, false, false, false, false, false, false,
                          true,  true,  true,  true,  true,  true,  true};
  for (int i = 0; i < 16; ++i)
    if (bufs[i] && !aligned16(bufs[i])) return INFINI_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return INFINI_ERR_ALIGN;
  if (workspace_bytes < b.total) return INFINI_ERR_WORKSPACE;
  // Nothing the call writes may overlap any other buffer.
  for (int i = 0; i < 16; ++i)
    for (int j = i + 1; j < 16; ++j)
      if ((written[i] || written[j]) && bufs[i] && bufs[j] && overlap(bufs[i], sizes[i], bufs[j], sizes[j]))
        return INFINI_ERR_ALIAS;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (path == INFINI_PATH_TC)
    return p.d == 64 ? launch_backward_tc64(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                                            dM_in, dz_in, ws, st)
                     : launch_backward_tc(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                                          dM_in, dz_in, ws, st);
  if (p.dtype == INFINI_F32)
    return p.d == 64 ? launch_backward<float, 64>(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv,
                                                  dbeta, dM_in, dz_in, ws, st)
                     : launch_backward<float, 128>(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv,
                                                   dbeta, dM_in, dz_in, ws, st);
  return p.d == 64 ? launch_backward<__nv_bfloat16, 64>(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk,
                                                        dv, dbeta, dM_in, dz_in, ws, st)
                   : launch_backward<__nv_bfloat16, 128>(b, q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk,
                                                         dv, dbeta, dM_in, dz_in, ws, st);
}

int infini_attn_selftest_timeout(uint64_t limit_ns, infini_stream_t stream) {
  if (limit_ns < 1000u || limit_ns > 100000000u) return INFINI_ERR_SHAPE;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, next_epoch());
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_schedule_check(int64_t n_seg, int n_qt, int grid, double* max_over_mean) {
  if (n_seg <= 0 || n_qt <= 0 || grid <= 0 || n_seg * (int64_t)n_qt > (int64_t)1 << 24) return INFINI_ERR_SHAPE;
  const int units = (int)(n_seg * n_qt);
  const int G = grid < units ? grid : units;  // the launch's grid: min(units, SMs)
  const int gs = infini::balance_group(G, n_qt);
  std::vector<unsigned char> seen((size_t)units, 0);
  int64_t most = 0, total = 0;
  int rc = INFINI_OK;
  for (int b = 0; b < G; ++b) {
    int64_t tiles = 0;
    for (int u = b; u < units; u += G) {
      const infini::tc::AttnUnit a =
          infini::tc::decode_unit(u, n_qt, (int)n_seg, 1, (int)n_seg * n_qt * 128, n_qt * 128, G, gs, (int)n_seg);
      if (a.seg_unit < 0 || a.seg_unit >= n_seg || a.qt < 0 || a.qt >= n_qt) return 1;
      unsigned char& hit = seen[(size_t)a.seg_unit * n_qt + a.qt];
      if (hit) rc = 1;
      hit = 1;
      tiles += a.n;
    }
    most = tiles > most ? tiles : most;
    total += tiles;
  }
  for (unsigned char h : seen)
    if (!h) rc = 1;
  if (max_over_mean) *max_over_mean = total > 0 ? (double)most * G / (double)total : 0.0;
  return rc;
}

#ifdef INFINI_TRACE
#include "../../include/infini_attn_trace.h"

int infini_attn_trace_reset(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return INFINI_ERR_CUDA;
  unsigned int zero[infini::tc::kTraceChannels] = {};
  return cudaMemcpyToSymbol(infini::tc::g_trace_n, zero, sizeof zero) == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_trace_read(int channel, uint64_t* host, int cap) {
  if (channel < 0 || channel >= infini::tc::kTraceChannels || cap < 0) return INFINI_ERR_SHAPE;
  if (cap > 0 && host == nullptr) return INFINI_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return INFINI_ERR_CUDA;
  unsigned int n[infini::tc::kTraceChannels];
  if (cudaMemcpyFromSymbol(n, infini::tc::g_trace_n, sizeof n) != cudaSuccess) return INFINI_ERR_CUDA;
  const int have = (int)std::min<unsigned int>(n[channel], (unsigned int)infini::tc::kTraceCap);
  const int copy = std::min(have, cap);
  if (copy > 0 && cudaMemcpyFromSymbol(host, infini::tc::g_trace, (size_t)copy * sizeof(uint64_t),
                                       (size_t)channel * infini::tc::kTraceCap * sizeof(uint64_t)) != cudaSuccess)
    return INFINI_ERR_CUDA;
  return (int)std::min<unsigned int>(n[channel], 0x7fffffffu);
}
#endif

int infini_attn_device_status(infini_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return INFINI_ERR_CUDA;
  unsigned int st = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&st, infini::g_status, sizeof st) != cudaSuccess) return INFINI_ERR_CUDA;
  if (st != 0 && cudaMemcpyToSymbol(infini::g_status, &zero, sizeof zero) != cudaSuccess) return INFINI_ERR_CUDA;
  if (st & kStatusTimeout) return INFINI_ERR_TIMEOUT;
  return (st & kStatusBounds) ? INFINI_ERR_BOUNDS : INFINI_OK;
}

}  // extern "C"
