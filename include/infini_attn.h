/*
 * infini_attn.h -- C ABI of the B200 (sm_100a) Infini-attention layer forward.
 *
 * The operation (sources cited by page title and section):
 *   "Hugging Face Infini-Attention reproduction analysis", section
 *   "Infini-Attention mechanism": Segmentation, Local Attention, Memory
 *   Retrieval (sigma = ELU + 1 applied to Q against M_{s-1}), Integration (a
 *   learnable scalar beta through a sigmoid gate), Memory Update (add the
 *   segment's key-value states), State Transfer (only the memory crosses
 *   segments).
 *   "KV linear-addition Infini-attention": masked local attention plus
 *   long-term linear attention in one block; scaled dot-product attention;
 *   causal attention inside each segment; streaming inference.
 * With sigma(x) = ELU(x) + 1, g_h = sigmoid(beta_h), per (b, h) and segment s
 * of length N (rows t of the segment, keys j <= t of the same segment):
 *   A_dot = softmax(Q_s K_s^T / sqrt(d), causal) V_s
 *   A_mem = sigma(Q_s) M_{s-1} / (sigma(Q_s) z_{s-1})      (0 where the
 *                                                          denominator is 0)
 *   out_s = g_h A_mem + (1 - g_h) A_dot
 *   M_s   = M_{s-1} + sigma(K_s)^T V_s,   z_s = z_{s-1} + sum_t sigma(K_s,t)
 * M_{-1} = M_in, z_{-1} = z_in; M_out = M_{S-1}, z_out = z_{S-1}, so a long
 * sequence can be fed as consecutive calls that pass (M_out, z_out) on as the
 * next call's (M_in, z_in).
 *
 * Layout: q, k, v and out are [B, H, L, d] row-major and contiguous in the I/O
 * dtype (fp32 or bf16). M is [B, H, d_k, d_v] (d_k = d_v = d), M[i][j] =
 * sum_t sigma(k_t)_i v_t,j, and z is [B, H, d]; both are fp32. beta is fp32
 * [H], shared by every batch element.
 *
 * All pointers except `workspace` bookkeeping are DEVICE pointers. Calls are
 * asynchronous on `stream` (NULL = the legacy default stream); outputs are
 * valid once the stream has been synchronised. The caller owns every buffer;
 * the library keeps no state between calls apart from a device-side status
 * word that infini_attn_device_status() reads and clears.
 *
 * Errors: every int-returning call returns INFINI_OK (0) or a negative code.
 * Arguments are validated on the host before anything is launched; on an error
 * nothing is launched and no output is touched. No C++ exception crosses this
 * interface.
 */
#ifndef INFINI_ATTN_H
#define INFINI_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define INFINI_API __attribute__((visibility("default")))
#else
#define INFINI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; spelled out so this header needs no CUDA header. */
struct CUstream_st;
typedef struct CUstream_st* infini_stream_t;

typedef enum { INFINI_F32 = 0, INFINI_BF16 = 1 } infini_dtype;

typedef struct {
  int64_t B;      /* batch                                  >= 1            */
  int64_t H;      /* heads                                  >= 1            */
  int64_t L;      /* tokens in this call, a multiple of the segment length  */
  int64_t d;      /* head dimension d = d_k = d_v: 64 or 128                */
  int32_t dtype;  /* infini_dtype of q, k, v and out                        */
} infini_shape;

enum {
  INFINI_OK = 0,
  INFINI_ERR_NULL = -1,        /* a required pointer is NULL, or only one of M_in/z_in is */
  INFINI_ERR_SHAPE = -2,       /* B, H, L or seg_len < 1, or L % seg_len != 0             */
  INFINI_ERR_UNSUPPORTED = -3, /* d not in {64, 128}, unknown dtype, or a forced path that
                                  does not cover this shape                               */
  INFINI_ERR_ALIGN = -4,       /* a tensor pointer is not 16-byte aligned, or the
                                  workspace is not 256-byte aligned                       */
  INFINI_ERR_CUDA = -5,        /* a CUDA runtime call or kernel launch failed             */
  INFINI_ERR_TIMEOUT = -6,     /* a bounded device-side wait gave up (see device_status)  */
  INFINI_ERR_WORKSPACE = -7,   /* workspace smaller than infini_attn_workspace_size()     */
  INFINI_ERR_ALIAS = -8,       /* q/k/v/out overlap, or M_out/z_out partly overlap inputs */
  INFINI_ERR_SIZE = -9,        /* a size exceeds what the kernels index (B*H*L >= 2^31)   */
  INFINI_ERR_SCRATCH = -10,    /* the shape needs more scratch than the built-in buffer of
                                  infini_attn_forward_noalloc holds                       */
  INFINI_ERR_BOUNDS = -11      /* a device-side index check of the debug build (compiled with
                                  INFINI_DEBUG) failed; the regular build never reports it */
};

/* Kernel path selection for infini_attn_forward_ws. AUTO picks the tensor-core
 * (tcgen05) path for bf16 shapes it covers and the CUDA-core path otherwise. */
enum {
  INFINI_PATH_AUTO = 0,
  INFINI_PATH_SIMT = 1,   /* CUDA-core kernels; any supported shape, fp32 or bf16 I/O (fp32
                             arithmetic; with bf16 I/O the attention's score and P V tiles run
                             on TF32 mma.sync: exact products of the bf16 inputs, P split into
                             two TF32 parts)                                                  */
  INFINI_PATH_TC = 2,     /* tcgen05/TMEM/TMA kernels; bf16 with d = 128 and seg_len % 128
                             == 0 (state, prefix, attention: three launches), or bf16 with
                             d = 64 and seg_len == 64 (one single-pass launch per forward,
                             one CTA per (b, h) walking its segments in order; the phase
                             entry points below keep the three launches)                    */
  INFINI_PATH_TC_PAIRED = 3 /* the tensor-core path with the paired-query-tile attention
                             kernel (two 128-row query tiles of a segment per CTA sharing
                             their key / value tiles); bf16, d = 128, seg_len % 256 == 0.
                             Same results as INFINI_PATH_TC up to rounding order; AUTO never
                             picks it (the one-tile kernel is faster on B200)              */
};

/*
 * infini_attn_forward -- the layer forward for one call of L tokens.
 *   shp          shapes and I/O dtype (host pointer, read during the call only)
 *   q, k, v      [B,H,L,d] in shp->dtype, device, 16-byte aligned, read only
 *   beta         [H] fp32, device: the per-head gate parameter (g = sigmoid(beta));
 *                +/-inf are allowed and give g = 1 / 0 exactly
 *   M_in, z_in   [B,H,d,d] and [B,H,d] fp32, device; both NULL = zero state
 *   seg_len      N, the segment length; L % N must be 0
 *   out          [B,H,L,d] in shp->dtype, device; must not overlap q, k, v
 *   M_out, z_out [B,H,d,d] and [B,H,d] fp32, device; may be equal to M_in/z_in
 *                (updated in place) but must not partly overlap them
 *   stream       CUDA stream the work is ordered on
 * Allocates its scratch memory stream-ordered (cudaMallocAsync on `stream`)
 * and frees it the same way; use infini_attn_forward_ws to supply it instead.
 */
INFINI_API int infini_attn_forward(const infini_shape* shp,
                        const void* q, const void* k, const void* v,
                        const float* beta, const float* M_in, const float* z_in,
                        int64_t seg_len,
                        void* out, float* M_out, float* z_out,
                        infini_stream_t stream);

/* Bytes of device scratch memory infini_attn_forward_ws needs for this shape
 * (per-segment state increments and prefixes); 0 on invalid arguments. */
INFINI_API size_t infini_attn_workspace_size(const infini_shape* shp, int64_t seg_len);

/*
 * infini_attn_forward_ws -- as infini_attn_forward, with caller-owned scratch.
 *   workspace    device pointer, 256-byte aligned, at least
 *                infini_attn_workspace_size() bytes; its contents on entry are
 *                ignored and on return are unspecified. Two calls in flight at
 *                the same time must not share one workspace.
 *   path         INFINI_PATH_AUTO / _SIMT / _TC (see above)
 */
INFINI_API int infini_attn_forward_ws(const infini_shape* shp,
                           const void* q, const void* k, const void* v,
                           const float* beta, const float* M_in, const float* z_in,
                           int64_t seg_len,
                           void* out, float* M_out, float* z_out,
                           void* workspace, size_t workspace_bytes, int path,
                           infini_stream_t stream);

/*
 * infini_attn_forward_traced -- infini_attn_forward_ws that also records
 * caller-created CUDA events (cudaEvent_t handles) on `stream` around its
 * kernel launches: events[0] before the first launch and events[i] right after
 * launch i, for i = 1 .. n_events - 1. n_events must be
 * infini_attn_launch_count() + 1 (events = NULL and n_events = 0 record
 * nothing). Nothing is synchronised; read the elapsed times after the stream.
 */
INFINI_API int infini_attn_forward_traced(const infini_shape* shp,
                           const void* q, const void* k, const void* v,
                           const float* beta, const float* M_in, const float* z_in,
                           int64_t seg_len,
                           void* out, float* M_out, float* z_out,
                           void* workspace, size_t workspace_bytes, int path,
                           void* const* events, int n_events,
                           infini_stream_t stream);

/* Size of the scratch buffer built into the library for
 * infini_attn_forward_noalloc: 64 MiB of device memory per GPU. */
#define INFINI_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * infini_attn_forward_noalloc -- the same forward as infini_attn_forward, for
 * callers that cannot allocate device memory: code whose device memory is
 * already handed out in full by another allocator (a serving process that
 * reserves the GPU's memory up front), and code that must not enter the CUDA
 * allocator at all, because cudaMalloc/cudaFree can block or synchronise the
 * device. The paper has no counterpart to this entry point; it exists only
 * for such callers.
 *
 * Arguments, layout and errors are those of infini_attn_forward. It calls no
 * allocator: its scratch memory is one array of INFINI_NOALLOC_SCRATCH_BYTES
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits. Shapes whose scratch
 * (infini_attn_workspace_size()) exceeds that size are rejected with
 * INFINI_ERR_SCRATCH before anything is launched.
 *
 * Every call looks up the array's device address in the current device's
 * context (so it stays right after a context is destroyed and created again);
 * the first call on a device may load the library's device code there, so
 * make that first call before any stream capture begins. All calls share the
 * one array and it keeps the last call's
 * contents; every scratch element a call reads is written earlier in the same
 * call, so nothing needs clearing between calls. Calls that overlap on the GPU
 * (in flight on two streams at once) race on the array: order them on one
 * stream or synchronise between them.
 */
INFINI_API int infini_attn_forward_noalloc(const infini_shape* shp,
                           const void* q, const void* k, const void* v,
                           const float* beta, const float* M_in, const float* z_in,
                           int64_t seg_len,
                           void* out, float* M_out, float* z_out,
                           infini_stream_t stream);

/* Which path AUTO would take for this shape: INFINI_PATH_SIMT or _TC; a
 * negative error code for invalid arguments. Host only. */
INFINI_API int infini_attn_select_path(const infini_shape* shp, int64_t seg_len);

/* Number of kernel launches one forward call makes on `path` for this shape
 * (AUTO resolved first); a negative error code for invalid arguments. */
INFINI_API int infini_attn_launch_count(const infini_shape* shp, int64_t seg_len, int path);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: INFINI_ERR_TIMEOUT if a bounded wait inside a kernel gave up
 * since the last check, INFINI_ERR_BOUNDS if (debug build only) an index check
 * failed, INFINI_ERR_CUDA if the synchronisation failed, else INFINI_OK. */
INFINI_API int infini_attn_device_status(infini_stream_t stream);

/* ---------------------------------------------------------------- phases
 * The forward in two phases, for a sequence split into consecutive blocks of
 * segments (one block per GPU). Only (M, z) crosses segment boundaries
 * ("Hugging Face Infini-Attention reproduction analysis", section
 * "Infini-Attention mechanism", State Transfer), and M, z are sums over
 * segments, so block r's incoming state is the caller's state plus the totals
 * of blocks 0..r-1:
 *   1. infini_attn_state_ws on each block: the per-segment increments (kept in
 *      `workspace`) and the block totals M_tot = sum_s sigma(K_s)^T V_s,
 *      z_tot = sum_s sum_t sigma(K_s,t) (fp32 [B,H,d,d], [B,H,d], DEVICE).
 *   2. the totals of all blocks gathered (by the caller, e.g. an all-gather),
 *      then infini_attn_exscan_parts: off = M_in + sum_{r < part} totals[r].
 *   3. infini_attn_finish_ws on each block with M_in = off: the cross-segment
 *      prefix from off, then attention, retrieval and gate; its M_out is
 *      off + the block's total (the last block's M_out is the sequence's).
 * Phase 1 then phase 3 on one block with the same workspace equals
 * infini_attn_forward_ws. Arguments as for infini_attn_forward_ws; phase 3
 * requires the workspace written by phase 1 for the same shape and seg_len
 * (not modified in between). Errors as for the forward. */
INFINI_API int infini_attn_state_ws(const infini_shape* shp, const void* k, const void* v, int64_t seg_len,
                                    float* M_tot, float* z_tot, void* workspace, size_t workspace_bytes, int path,
                                    infini_stream_t stream);
INFINI_API int infini_attn_finish_ws(const infini_shape* shp, const void* q, const void* k, const void* v,
                                     const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                                     void* out, float* M_out, float* z_out, void* workspace, size_t workspace_bytes,
                                     int path, infini_stream_t stream);
/* off_M[e] = M_in[e] + sum_{r < part} totals_M[r * n_M + e] (and likewise for
 * z with n_z), summed in part order in fp32; M_in/z_in NULL = the zero state.
 * totals_M: [n_parts][n_M], totals_z: [n_parts][n_z] fp32 DEVICE; off_M may
 * equal M_in and off_z may equal z_in (in place). 0 <= part < n_parts.
 * Errors: INFINI_ERR_SHAPE, _NULL, _ALIGN (16 bytes), _ALIAS, _SIZE, _CUDA. */
INFINI_API int infini_attn_exscan_parts(int64_t n_M, int64_t n_z, int n_parts, int part, const float* totals_M,
                                        const float* totals_z, const float* M_in, const float* z_in, float* off_M,
                                        float* off_z, infini_stream_t stream);

/* ---------------------------------------------------------------- backward
 * Gradients of the forward (the pages give none; they follow from the
 * forward's steps by the chain rule: the gate, causal softmax attention, the
 * retrieval with A_mem = 0 where the denominator is 0 (no gradient there),
 * and the state chain M_s = M_{s-1} + sigma(K_s)^T V_s, z likewise).
 *
 * Inputs as for infini_attn_forward (DEVICE): q, k, v [B,H,L,d] in dtype,
 * beta [H], optional M_in, z_in, seg_len; dout [B,H,L,d] in dtype, the
 * gradient of out; dM_out [B,H,d,d], dz_out [B,H,d] fp32, the gradient of the
 * output state (both NULL = zero).
 * Outputs (DEVICE, fp32, overwritten): dq, dk, dv [B,H,L,d]; dbeta [H] (summed
 * over the batch); dM_in [B,H,d,d], dz_in [B,H,d] (the gradient of the
 * incoming state, also when M_in is NULL).
 * workspace: infini_attn_backward_workspace_size(shp, seg_len) bytes,
 * 256-byte aligned.
 * Arithmetic: bf16 with d = 128 and seg_len % 128 == 0, and bf16 with
 * d = 64, seg_len = 64 and an even number of segments, take the tensor-core
 * path (INFINI_PATH_TC): the state is recomputed on the tensor-core state
 * and scan kernels; at d = 128 the forward's attention kernel recomputes the
 * softmax statistics and tcgen05 kernels form dq, dk and dv; at d = 64 one
 * tcgen05 kernel per pair of segments recomputes the softmax exactly and
 * forms dq and the local dk, dv, and a second adds the state terms. P, dS,
 * sigma(Q), sigma(K), G_s, dnum and M_{s-1} are rounded to bf16 as MMA
 * operands (fp32 accumulation), about 2^-9 relative per product. Every other
 * shape takes the CUDA-core path (INFINI_PATH_SIMT): fp32 throughout for fp32
 * inputs; for bf16 inputs the products of the local attention (scores,
 * dout V^T, P V, dS K, dS^T Q, P^T dout) run on TF32 tensor cores with fp32
 * accumulation: products of two bf16 values are exact there, and the fp32
 * factors (P, dS) are split into a TF32 part and the TF32 of the remainder,
 * so the result differs from fp32 arithmetic by summation order and about
 * 2^-22 relative per product.
 * Errors: as for the forward; _ALIAS if an output overlaps any other buffer. */
INFINI_API size_t infini_attn_backward_workspace_size(const infini_shape* shp, int64_t seg_len);
INFINI_API int infini_attn_backward(const infini_shape* shp, const void* q, const void* k, const void* v,
                                    const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                                    const void* dout, const float* dM_out, const float* dz_out, float* dq,
                                    float* dk, float* dv, float* dbeta, float* dM_in, float* dz_in,
                                    void* workspace, size_t workspace_bytes, infini_stream_t stream);
/* The same with an explicit path: INFINI_PATH_AUTO (as infini_attn_backward),
 * INFINI_PATH_SIMT (the CUDA-core backward, any supported shape) or
 * INFINI_PATH_TC (bf16 with d = 128 and seg_len % 128 == 0, or d = 64,
 * seg_len = 64 and L / seg_len even; else INFINI_ERR_UNSUPPORTED). The
 * workspace size does not depend on the path. */
INFINI_API int infini_attn_backward_path(const infini_shape* shp, const void* q, const void* k, const void* v,
                                         const float* beta, const float* M_in, const float* z_in, int64_t seg_len,
                                         const void* dout, const float* dM_out, const float* dz_out, float* dq,
                                         float* dk, float* dv, float* dbeta, float* dM_in, float* dz_in,
                                         void* workspace, size_t workspace_bytes, int path, infini_stream_t stream);

/* ---------------------------------------------------------------- decode
 * Streaming decode: one new token per (b, h) at position `pos` of its segment
 * ("KV linear-addition Infini-attention": streaming inference with a bounded
 * local context; "Hugging Face Infini-Attention reproduction analysis",
 * section "Infini-Attention mechanism", State Transfer). Decoding a sequence
 * token by token gives the same outputs and final (M, z) as the forward over
 * it.
 *
 * shp: B, H, d, dtype as for the forward, L = N = the segment length (rows of
 *      the cache). 1 <= N <= 32768.
 * q, k, v: [B, H, d] in dtype, this token's query, key and value (DEVICE).
 * beta: [H] fp32.
 * k_cache, v_cache: [B, H, N, d] in dtype (DEVICE, read/write). Rows 0..pos-1
 *      hold the current segment's earlier keys and values; the call writes
 *      this token's key and value into row pos.
 * pos: 0 <= pos < N, the token's position inside its segment (the caller
 *      counts tokens; pos = t mod N).
 * M, z: [B, H, d, d] and [B, H, d] fp32 (DEVICE, read/write): the memory of
 *      the segments before the current one. Unchanged for pos < N - 1; when
 *      pos == N - 1 the whole cached segment is folded in after the output is
 *      formed (M += sigma(K)^T V, z += sum sigma(K)), ready for the next
 *      segment. Start a sequence with zeros (or a carried state).
 * out: [B, H, d] in dtype (DEVICE), the layer output for this token.
 * workspace: at least infini_attn_decode_workspace_size(shp) bytes, 256-byte
 *      aligned (per-chunk partial results of the step, and the fold's
 *      scratch at the segment's end).
 * Errors: INFINI_ERR_NULL, _SHAPE (bad shape or pos), _UNSUPPORTED (d, dtype),
 * _ALIGN (16-byte pointers, 256-byte workspace), _ALIAS (any two buffers
 * overlap), _SIZE (N > 32768), _WORKSPACE, _CUDA. Asynchronous on `stream`. */
INFINI_API size_t infini_attn_decode_workspace_size(const infini_shape* shp);
INFINI_API int infini_attn_decode_step(const infini_shape* shp, const void* q, const void* k, const void* v,
                                       const float* beta, void* k_cache, void* v_cache, int64_t pos, float* M,
                                       float* z, void* out, void* workspace, size_t workspace_bytes,
                                       infini_stream_t stream);

/* Self-test of the bounded device-side waits that every kernel of this
 * library uses (the pages define no API; this call has no counterpart there).
 * Launches one thread that waits on an mbarrier nothing ever arrives on. The
 * wait gives up after limit_ns nanoseconds of GPU time (1e3 <= limit_ns <= 1e8),
 * records INFINI_ERR_TIMEOUT in the device status word and the kernel exits
 * normally, so the CUDA context stays usable; the next
 * infini_attn_device_status(stream) returns INFINI_ERR_TIMEOUT and clears the
 * word. Asynchronous on `stream`. Returns INFINI_ERR_SHAPE (nothing launched)
 * for limit_ns out of range, INFINI_ERR_CUDA if the launch fails. */
INFINI_API int infini_attn_selftest_timeout(uint64_t limit_ns, infini_stream_t stream);

/* Self-check of the tensor-core attention kernel's unit schedule (the pages
 * define no API; this call has no counterpart there). The kernel runs one
 * CTA per SM (grid = min(units, SMs)) over units = n_seg * n_qt (segment,
 * query-tile) pairs and maps the CTA's k-th unit index to a pair with a
 * balanced map; this runs the same map on the host for n_seg segments of
 * n_qt query tiles and a grid of `grid` CTAs.
 * Returns 0 if every pair is taken exactly once, 1 if not, INFINI_ERR_SHAPE
 * for n_seg, n_qt or grid <= 0 or more than 2^24 units. If max_over_mean is
 * not NULL it receives the busiest CTA's key tiles (a unit of query tile t
 * costs t + 1) over the mean. Host only; no GPU needed. */
INFINI_API int infini_attn_schedule_check(int64_t n_seg, int n_qt, int grid, double* max_over_mean);

/* Static, human-readable text for a return code. */
INFINI_API const char* infini_attn_strerror(int code);

/* ABI version of this header (major * 100 + minor). */
INFINI_API int infini_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INFINI_ATTN_H */
