// Paired-query-tile tensor-core attention kernel (tcgen05 / TMEM / TMA) for
// bf16 I/O, head dimension 128 and segments of an even number of 128-row
// tiles (seg_len % 256 == 0).
//
// Per (b, h, segment, pair of 128-row query tiles): causal softmax attention
// inside the segment ("Hugging Face Infini-Attention reproduction analysis",
// Infini-Attention mechanism: Local Attention) by an online softmax over
// 128-key tiles (the running max / normaliser merge of the "Attention-State
// Memory" page, Methodology); the retrieval sigma(Q) M_{s-1} / sigma(Q).z_{s-1}
// (Memory Retrieval); the sigmoid(beta) blend (Integration); the bf16 store.
//
// Why pairs. With one query tile per CTA, the softmax of key tile j, the PV of
// tile j and the QK^T of tile j + 1 form one serial chain, and the tensor
// pipe waits for the softmax most of the time. Here each CTA holds two query
// tiles of the same segment (the "slots" 0 and 1), which share every K and V
// tile the TMA brings in, and each slot has its own softmax warpgroup, score
// buffer S and accumulator O in TMEM. While one slot's warpgroup turns its
// scores into probabilities, the MMA warp runs the other slot's PV and QK^T,
// so the two chains overlap on the tensor pipe.
//
// Work unit: (segment, pair p), query tiles 2p ("short": 2p + 1 key tiles)
// and 2p + 1 ("long": 2p + 2 key tiles). The units a CTA takes come from the
// balanced schedule (decode_unit, with the pairs of a segment in place of its
// tiles: a pair's cost, 4p + 3 key tiles, is linear in its rank like a tile's).
//
// Step sequence. Slot x walks its tiles as steps:
//   step 0           S = Q K_0^T
//   step s, 0<s<n    O (+)= P V_{s-1}, then S = Q K_s^T
//   step n           O += P V_{n-1}, then R = sigma(Q) M_{s-1} into S's columns
// Each slot has its own MMA-issuing warp, so one slot waiting (for its next
// Q tile, or for its softmax) never holds up the other; the two meet only at
// the K / V ring slots they share, whose release barriers count one arrival
// per slot (the slot that holds the long tile arrives twice for the key and
// value tile only it uses). The TMA warp loads every tile at its first use
// in one fixed interleaving of the two step sequences -- slot 0 step, slot 1
// step, slot 0 step, ... -- with the short tile in slot 0 in even units (per
// CTA) and in slot 1 in odd units: the slot with the short tile finishes its
// unit one step early and starts the next one step ahead, and the next unit
// gives it the long tile, so the two meet again at the end of every odd unit.
// In that interleaving the K ring receives unit by unit K_0 .. K_{2p}, then
// M, then K_{2p+1} (even units) or K_0 .. K_{2p+1}, then M (odd units), and
// the V ring V_0 .. V_{2p+1}, so ring positions follow from counts; every
// ring slot is refilled only after uses that come earlier in the
// interleaving, which is a valid order of the MMAs, so the loads never wait
// on work that needs a later load. MMAs issued by one thread execute in
// order, which orders every reuse of a TMEM column range after the MMA
// reading it (P of tile s-1 is read by the PV issued just before the QK^T
// that overwrites it; R goes after the slot's last PV).
//
// Roles (512 threads; register split per warpgroup with setmaxnreg):
//   warps 0-3   softmax of slot 0, one thread per query row: the 128 scores of
//               a key tile in registers, causal mask on the diagonal tile, row
//               max, lazy rescale of the row of O, P = 2^(s - m) as packed bf16
//               over the S columns, row sum; after the slot's last tile of a
//               unit, its epilogue: out = wd * O + wm * R as the bf16 row, with
//               wd = (1 - g) / l and wm = g / den (0 when den = 0).
//   warps 4-7   the same for slot 1.
//   warps 8-11  sigma(Q), one row per thread, slot 0 then slot 1 of every
//               unit: as soon as the slot's last QK^T of the unit is done,
//               its Q tile is replaced by sigma(Q) in place (the retrieval's
//               A operand) and den = sigma(q) . z_{s-1} is formed in fp32,
//               with z_{s-1} staged in shared memory once per tile.
//   warp 12     TMA producer (one elected lane of the converged warp).
//   warp 13     TMEM owner; MMA issuer of slot 0 (one elected lane).
//   warp 14     MMA issuer of slot 1.
//   warp 15     idle.
//
// TMEM (512 columns): S/P/R of slot 0 at 0..127, of slot 1 at 128..255; O of
// slot 0 at 256..383, of slot 1 at 384..511. Shared memory, from the
// 1024-aligned base: Q[2] | K ring[3] | V ring[2] (32 KB tiles) | barriers |
// den [2 slots][128] fp32 | z_{s-1} [128] fp32.
//
// Built with INFINI_TRACE defined, CTA 0 records clock64 timestamps of its
// pipeline events (infini_attn_trace.h); otherwise the trace points compile
// to nothing.
#pragma once

namespace infini {
namespace tc {

constexpr int kPairThreads = 512;
constexpr int kPairKRing = 3, kPairVRing = 2;
constexpr uint32_t kPairTiles = (2 + kPairKRing + kPairVRing) * kTileBytes;
constexpr uint32_t kPairBarBytes = 256;
constexpr uint32_t kPairSmem = kPairTiles + kPairBarBytes + 2 * 128 * 4 + 128 * 4;
static_assert(kPairSmem <= 232448, "paired attention kernel shared memory");
// setmaxnreg split: the kernel launches at 128 registers per thread (512 x 128
// = 65536, the SM's file); the softmax warpgroups take 176, the sigma(Q)
// warpgroup 64, the TMA / MMA warpgroup 96: 128 x (2 x 176 + 64 + 96) = 65536.
// (ptxas: no spills with this split.)
constexpr int kPairRegSoftmax = 176, kPairRegSigma = 64, kPairRegIssue = 96;
constexpr int kPairLaunchRegs = 128;
static_assert(2 * kPairRegSoftmax + kPairRegSigma + kPairRegIssue == 4 * kPairLaunchRegs, "register split");
static_assert(kPairThreads * kPairLaunchRegs == 65536, "launch registers");

#ifdef INFINI_TRACE
// Trace channels of CTA 0: producer, MMA slot 0 / 1, softmax slot 0 / 1
// (warps 0 and 4), sigma slot 0 / 1 (warps 8 and 10). Each record: clock64
// (low 40 bits) | event code << 40 | index << 48.
constexpr int kTraceChannels = 7, kTraceCap = 1 << 15;
__device__ unsigned long long g_trace[kTraceChannels][kTraceCap];
__device__ unsigned int g_trace_n[kTraceChannels];
#define PAIR_TRACE(ch, code, idx)                                                                     \
  do {                                                                                                \
    if (blockIdx.x == 0 && lane == 0) {                                                               \
      const unsigned int k_ = g_trace_n[ch]++;                                                        \
      if (k_ < kTraceCap)                                                                             \
        g_trace[ch][k_] = ((unsigned long long)clock64() & 0xFFFFFFFFFFull) |                         \
                          ((unsigned long long)(code) << 40) | ((unsigned long long)((idx) & 0xFFFF) << 48); \
    }                                                                                                 \
  } while (0)
#else
#define PAIR_TRACE(ch, code, idx) \
  do {                            \
  } while (0)
#endif

struct PairUnit {
  int seg_unit, p, h, row_seg;
};

// Unit u of the balanced schedule, with n_pairs units per segment.
__host__ __device__ __forceinline__ PairUnit decode_pair(int u, int n_pairs, int S, int H, int L, int N, int G,
                                                          int gs, int n_seg) {
  const AttnUnit a = decode_unit(u, n_pairs, S, H, L, N, G, gs, n_seg);
  PairUnit r;
  r.seg_unit = a.seg_unit;
  r.p = a.qt;
  r.h = a.h;
  r.row_seg = a.row_seg;
  return r;
}

// One slot's position in its step sequence.
struct PairCursor {
  int i;        // per-CTA unit index
  int u;        // unit id
  int step;     // step within the unit, 0 .. n
  int n;        // key tiles of this slot's tile in the unit
  int qt;       // this slot's query tile within the segment
  bool done;
  PairUnit a;
};

// Slot x holds the short tile (2p) in even units for x = 0, in odd units for x = 1.
__host__ __device__ __forceinline__ bool slot_is_short(int x, int i) { return ((i & 1) == 0) == (x == 0); }

__device__ __forceinline__ void cursor_load(PairCursor& c, int x, int units, int n_pairs, int S, int H, int L, int N,
                                            int gs, int n_seg) {
  c.done = c.u >= units;
  if (c.done) return;
  c.a = decode_pair(c.u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
  c.qt = 2 * c.a.p + (slot_is_short(x, c.i) ? 0 : 1);
  c.n = c.qt + 1;
  c.step = 0;
}
__device__ __forceinline__ void cursor_start(PairCursor& c, int x, int units, int n_pairs, int S, int H, int L, int N,
                                             int gs, int n_seg) {
  c.i = 0;
  c.u = blockIdx.x;
  cursor_load(c, x, units, n_pairs, S, H, L, N, gs, n_seg);
}
// Advances one step; returns true when the cursor entered a new unit.
__device__ __forceinline__ bool cursor_next(PairCursor& c, int x, int units, int n_pairs, int S, int H, int L, int N,
                                            int gs, int n_seg) {
  if (++c.step <= c.n) return false;
  ++c.i;
  c.u += gridDim.x;
  cursor_load(c, x, units, n_pairs, S, H, L, N, gs, n_seg);
  return true;
}

// Ring positions of the unit's tiles (see the interleaving above): the K ring
// receives 2p + 3 tiles per unit (its keys and the M tile), the V ring 2p + 2.
__device__ __forceinline__ int pair_kpos(int kbase, int i, int p, int j) {
  return kbase + j + (((i & 1) == 0 && j == 2 * p + 1) ? 1 : 0);
}
__device__ __forceinline__ int pair_mpos(int kbase, int i, int p) { return kbase + 2 * p + 1 + (i & 1); }

// 32 bytes to global memory in one 256-bit store (address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__global__ void __launch_bounds__(kPairThreads, 1)
tc_attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
                    const float* __restrict__ zp, const float* __restrict__ beta, __nv_bfloat16* __restrict__ out,
                    int L, int N, int S, int H, int units, int gs, int out_v8, uint32_t epoch) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) flag_timeout();
    return;
  }
  uint8_t* sm = smem_raw;
  uint8_t* sQ = sm;                                  // [2] one per slot
  uint8_t* sK = sm + 2 * kTileBytes;                 // [kPairKRing]
  uint8_t* sV = sm + (2 + kPairKRing) * kTileBytes;  // [kPairVRing]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kPairTiles);
  float* dbuf = reinterpret_cast<float*>(sm + kPairTiles + kPairBarBytes);  // den [slot][128]
  float* zbuf = dbuf + 2 * 128;                                               // z_{s-1} of the tile in work

  uint64_t* q_full = bars + 0;     // [2] TMA (per slot)
  uint64_t* q_empty = bars + 2;    // [2] retrieval done with the slot's Q buffer
  uint64_t* k_full = bars + 4;     // [3] TMA
  uint64_t* k_empty = bars + 7;    // [3] both slots done with the ring slot (2 arrivals)
  uint64_t* v_full = bars + 10;    // [2] TMA
  uint64_t* v_empty = bars + 12;   // [2] both slots done with the ring slot (2 arrivals)
  uint64_t* s_full = bars + 14;    // [2] QK^T done (per slot)
  uint64_t* p_full = bars + 16;    // [2] P written (4 softmax warps of the slot)
  uint64_t* qk_last = bars + 18;   // [2] the slot's last QK^T of the unit done
  uint64_t* sq_full = bars + 20;   // [2] sigma(Q) and den written (4 sigma warps)
  uint64_t* o_full = bars + 22;    // [2] retrieval done: O and R complete
  uint64_t* epi_done = bars + 24;  // [2] epilogue has read O and R (4 softmax warps)
  uint64_t* drain = bars + 26;     // [2] abort path: in-flight MMAs of each issuer
  constexpr int kNumBars = 28;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  static_assert(kNumBars * 8 + 4 <= kPairBarBytes, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = N / (2 * kTile);
  const int n_seg = units / n_pairs;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kNumBars; ++b) {
      uint32_t count = 1;
      if (b >= 7 && b <= 9) count = 2;                                  // k_empty
      if (b >= 12 && b <= 13) count = 2;                                // v_empty
      if ((b >= 16 && b <= 17) || (b >= 20 && b <= 21) || (b >= 24 && b <= 25)) count = 4;  // p_full, sq_full, epi_done
      mbar_init(&bars[b], count);
    }
    fence_mbar_init();
  }
  if (warp == 13) {
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

  if (warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegIssue));
    if (warp == 12) {
      // ------------------------------------------------ TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmM);
      auto load_k = [&](int pos, int row, const CUtensorMap* m) {
        const int slot = pos % kPairKRing, use = pos / kPairKRing;
        if (use > 0 && !(ok = mbar_wait_warp(&k_empty[slot], (use - 1) & 1, epoch))) return;
        armed = (armed & ~(3u << (4 + 2 * slot))) | ((2u | (use & 1)) << (4 + 2 * slot));
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(&k_full[slot], kTileBytes);
          load_tile(sK + slot * kTileBytes, m, row, &k_full[slot]);
        }
        __syncwarp();
        PAIR_TRACE(0, 1, pos);
      };
      auto load_v = [&](int pos, int row) {
        const int slot = pos % kPairVRing, use = pos / kPairVRing;
        if (use > 0 && !(ok = mbar_wait_warp(&v_empty[slot], (use - 1) & 1, epoch))) return;
        armed = (armed & ~(3u << (10 + 2 * slot))) | ((2u | (use & 1)) << (10 + 2 * slot));
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(&v_full[slot], kTileBytes);
          load_tile(sV + slot * kTileBytes, &tmV, row, &v_full[slot]);
        }
        __syncwarp();
        PAIR_TRACE(0, 2, pos);
      };
      // The fixed interleaving: slot 0 step, slot 1 step, ...; each tile is
      // loaded at its first use in it.
      // K / V ring base of the unit of each parity (the slots are at most one
      // unit apart) and the tile counts of the unit slot 0 entered last.
      int kb0 = 0, kb1 = 0, vb0 = 0, vb1 = 0, kc_prev = 0, vc_prev = 0;
      PairCursor c0, c1;
      cursor_start(c0, 0, units, n_pairs, S, H, L, N, gs, n_seg);
      cursor_start(c1, 1, units, n_pairs, S, H, L, N, gs, n_seg);
      auto step = [&](PairCursor& cx, const int x) {
        const int i = cx.i, p = cx.a.p, s = cx.step, n = cx.n;
        // Slot 0 uses every key / value tile j <= 2p of the unit, and
        // j = 2p + 1 as well when it holds the long tile.
        const bool slot0_long = !slot_is_short(0, i);
        if (s == 0) {
          if (x == 0) {  // slot 0 enters every unit first
            if (i & 1) {
              kb1 = kb0 + kc_prev;
              vb1 = vb0 + vc_prev;
            } else {
              kb0 = i == 0 ? 0 : kb1 + kc_prev;
              vb0 = i == 0 ? 0 : vb1 + vc_prev;
            }
            kc_prev = 2 * p + 3;
            vc_prev = 2 * p + 2;
          }
          if (i >= 1 && !(ok = mbar_wait_warp(&q_empty[x], (i - 1) & 1, epoch))) return;
          armed = (armed & ~(3u << (2 * x))) | ((2u | (i & 1)) << (2 * x));
          if (elect_one_lane()) {
            mbar_arrive_expect_tx(&q_full[x], kTileBytes);
            load_tile(sQ + x * kTileBytes, &tmQ, cx.a.row_seg + cx.qt * kTile, &q_full[x]);
          }
          __syncwarp();
          PAIR_TRACE(0, 3 + x, i);
          if (x == 0) load_k(pair_kpos(((i & 1) ? kb1 : kb0), i, p, 0), cx.a.row_seg, &tmK);
        } else {
          const int jv = s - 1;  // V tile of this step's PV
          const bool v_first = x == 0 || (jv == 2 * p + 1 && !slot0_long);
          if (v_first) load_v(((i & 1) ? vb1 : vb0) + jv, cx.a.row_seg + jv * kTile);
          if (!ok) return;
          if (s < n) {
            const bool k_first = x == 0 || (s == 2 * p + 1 && !slot0_long);
            if (k_first) load_k(pair_kpos(((i & 1) ? kb1 : kb0), i, p, s), cx.a.row_seg + s * kTile, &tmK);
          } else if (x == 0) {
            load_k(pair_mpos(((i & 1) ? kb1 : kb0), i, p), cx.a.seg_unit * kD, &tmM);  // M_{s-1} of the unit
          }
        }
      };
      while (ok && !(c0.done && c1.done)) {
        if (!c0.done) {
          step(c0, 0);
          cursor_next(c0, 0, units, n_pairs, S, H, L, N, gs, n_seg);
        }
        if (ok && !c1.done) {
          step(c1, 1);
          cursor_next(c1, 1, units, n_pairs, S, H, L, N, gs, n_seg);
        }
      }
    } else if (warp == 13 || warp == 14) {
      // ------------------------------------------------ MMA issuer of slot x
      const int x = warp - 13;
      const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
      const uint64_t dq = desc_kmajor_sw128(smem_u32(sQ + x * kTileBytes));
      const uint64_t dk0 = desc_kmajor_sw128(smem_u32(sK));
      const uint64_t dkmn0 = desc_mnmajor_sw128(smem_u32(sK), kHalf);
      const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(sV), kHalf);
      constexpr uint32_t kTileD = kTileBytes >> 4;
      const uint32_t tS = tmem + x * 128, tO = tmem + 256 + x * 128;
      int pcount = 0;
      // S = Q_x K^T from K-ring position kp; `arrivals` releases of the ring slot.
      auto qk = [&](int kp, int arrivals, bool last_qk) {
        const int slot = kp % kPairKRing;
        if (!(ok = mbar_wait_warp(&k_full[slot], (kp / kPairKRing) & 1, epoch))) return;
        tc_fence_after();
        const uint64_t db = dk0 + slot * kTileD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tS, dq + off, db + off, id_qk, kk != 0);
          }
          mma_commit(&s_full[x]);
          for (int a = 0; a < arrivals; ++a) mma_commit(&k_empty[slot]);
          if (last_qk) mma_commit(&qk_last[x]);
        }
        __syncwarp();
      };
      // O_x (+)= P_x V from V-ring position vp.
      auto pv = [&](int vp, int arrivals, bool first_pv) {
        const int slot = vp % kPairVRing;
        if (!(ok = mbar_wait_warp(&p_full[x], pcount & 1, epoch) &&
                   mbar_wait_warp(&v_full[slot], (vp / kPairVRing) & 1, epoch)))
          return;
        ++pcount;
        tc_fence_after();
        const uint64_t db = dv0 + slot * kTileD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tO, tS + kk * 8, db + ((kk * 2048) >> 4), id_pv, (!first_pv || kk != 0) ? 1u : 0u);
          for (int a = 0; a < arrivals; ++a) mma_commit(&v_empty[slot]);
        }
        __syncwarp();
      };
      // R_x = sigma(Q_x) M_{s-1} into slot x's S columns (M at K-ring position mp).
      auto retrieval = [&](int i, int mp) {
        const int slot = mp % kPairKRing;
        if (!(ok = mbar_wait_warp(&sq_full[x], i & 1, epoch) &&
                   mbar_wait_warp(&k_full[slot], (mp / kPairKRing) & 1, epoch)))
          return;
        tc_fence_after();
        const uint64_t db = dkmn0 + slot * kTileD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tS, dq + off, db + ((kk * 2048) >> 4), id_pv, kk != 0);
          }
          mma_commit(&o_full[x]);
          mma_commit(&q_empty[x]);
          mma_commit(&k_empty[slot]);
        }
        __syncwarp();
      };
      PairCursor c;
      cursor_start(c, x, units, n_pairs, S, H, L, N, gs, n_seg);
      int kbase = 0, vbase = 0;
      while (ok && !c.done) {
        const int i = c.i, p = c.a.p, s = c.step, n = c.n;
        if (s == 0) {
          PAIR_TRACE(1 + x, 10, i);
          if (!(ok = mbar_wait_warp(&q_full[x], i & 1, epoch))) break;
          if (i >= 1 && !(ok = mbar_wait_warp(&epi_done[x], (i - 1) & 1, epoch))) break;
          qk(pair_kpos(kbase, i, p, 0), 1, n == 1);
          PAIR_TRACE(1 + x, 11, i);
        } else {
          const int jv = s - 1;
          // The long tile's slot is the only user of K_{2p+1} and V_{2p+1}:
          // it gives both arrivals of their release.
          PAIR_TRACE(1 + x, 12, s);
          pv(vbase + jv, jv == 2 * p + 1 ? 2 : 1, jv == 0);
          if (!ok) break;
          PAIR_TRACE(1 + x, 13, s);
          if (s < n)
            qk(pair_kpos(kbase, i, p, s), s == 2 * p + 1 ? 2 : 1, s == n - 1);
          else
            retrieval(i, pair_mpos(kbase, i, p));
          PAIR_TRACE(1 + x, 14, s);
        }
        if (cursor_next(c, x, units, n_pairs, S, H, L, N, gs, n_seg)) {
          kbase += 2 * p + 3;
          vbase += 2 * p + 2;
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ sigma(Q) and den, one row per thread
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegSigma));
    const int r = (warp & 3) * 32 + lane;
    constexpr float kLog2e = 1.4426950408889634f;
    int i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const PairUnit a = decode_pair(u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
#pragma unroll 1
      for (int x = 0; x < 2; ++x) {
        // The TMA-written tile is visible to these threads once they have seen
        // its barrier complete; sigma(Q) may overwrite it once the slot's last
        // QK^T of the unit is done. The four warps agree before and after
        // staging z_{s-1} (a warp whose wait gave up still arrives, with its
        // predicate false, and then all four leave).
        bool w_ok = ok && mbar_wait_warp(&q_full[x], i & 1, epoch) && mbar_wait_warp(&qk_last[x], i & 1, epoch);
        if (!(ok = named_bar_and(1, 128, w_ok))) break;
        if (warp == 8) PAIR_TRACE(5 + x, 30, i);
        zbuf[r] = __ldg(zp + (int64_t)a.seg_unit * kD + r);
        named_bar_sync(1, 128);
        uint8_t* qt = sQ + x * kTileBytes;
        const float4* z4 = reinterpret_cast<const float4*>(zbuf);
        float den = 0.f;
#pragma unroll 4
        for (int cc = 0; cc < 16; ++cc) {
          uint4* px = reinterpret_cast<uint4*>(qt + sw128_offset(r, cc * 8, 128));
          const uint4 xq = *px;
          const float4 z0 = z4[2 * cc], z1 = z4[2 * cc + 1];
          const uint32_t w[4] = {xq.x, xq.y, xq.z, xq.w};
          const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
          uint32_t o4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float f0 = __uint_as_float(w[t] << 16), f1 = __uint_as_float(w[t] & 0xffff0000u);
            const float e0 = ex2(f0 * kLog2e), e1 = ex2(f1 * kLog2e);
            const float s0 = f0 > 0.f ? f0 + 1.f : e0, s1 = f1 > 0.f ? f1 + 1.f : e1;
            den = fmaf(s0, zz[2 * t], den);
            den = fmaf(s1, zz[2 * t + 1], den);
            o4[t] = pack_bf16x2(s0, s1);
          }
          *px = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        dbuf[x * 128 + r] = den;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sq_full[x]);
        if (warp == 8) PAIR_TRACE(5 + x, 31, i);
      }
    }
  } else {
    // ------------------------------------------------ softmax + epilogue of slot x (one row per thread)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairRegSoftmax));
    const int x = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t colS = x * 128, colO = 256 + x * 128;
    const float scale2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    int t = 0, i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const PairUnit a = decode_pair(u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
      const int qt = 2 * a.p + (slot_is_short(x, i) ? 0 : 1);
      const int n = qt + 1;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n; ++j, ++t) {
        if (quarter == 0) PAIR_TRACE(3 + x, 20, j);
        if (!(ok = mbar_wait_warp(&s_full[x], t & 1, epoch))) break;
        tc_fence_after();
        if (quarter == 0) PAIR_TRACE(3 + x, 21, j);
        uint32_t sr[128];
        tmem_ld32(tl + colS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tl + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(tl + colS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(tl + colS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait_regs(sr);
        const bool diag = j == n - 1;
        if (diag) {  // key column c is visible to row r iff c <= r
#pragma unroll
          for (int cc = 0; cc < 128; ++cc)
            if (cc > r) sr[cc] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mx8[q] = __uint_as_float(sr[q]);
#pragma unroll
        for (int cc = 8; cc < 128; ++cc) mx8[cc & 7] = fmaxf(mx8[cc & 7], __uint_as_float(sr[cc]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        if (quarter == 0) PAIR_TRACE(3 + x, 22, j);
        // Lazy rescaling: the exponent's max is raised only when the row's new
        // max exceeds it by more than 2^8 (unnormalised P stays <= 256).
        const bool need = mx * scale2 > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_tgt = need ? mx * scale2 : m_run;
          const float alpha = ex2(m_run - m_tgt);
          if (j > 0) {
            // PV of tile j - 1 was issued before this tile's QK^T, so it is
            // complete: rescale this row of O in place.
#pragma unroll 1
            for (int cb = 0; cb < 8; ++cb) {
              uint32_t o[16];
              tmem_ld16(tl + colO + cb * 16, o);
              tmem_ld_wait_regs(o);
#pragma unroll
              for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
              tmem_st16(tl + colO + cb * 16, o);
            }
          }
          l_run *= alpha;
          m_run = m_tgt;
        }
        // P = 2^(s log2(e)/sqrt(d) - m) as bf16 pairs over the S columns, in
        // four 32-key chunks (16 columns each); on the diagonal tile a chunk
        // wholly right of every row of this warp is all zeros.
        float sum8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) sum8[q] = 0.f;
        const float neg_m = -m_run;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if (diag && ch > quarter) {
#pragma unroll
            for (int cc = ch * 32; cc < ch * 32 + 32; cc += 2) sr[cc >> 1] = 0u;
          } else {
#pragma unroll
            for (int cc = ch * 32; cc < ch * 32 + 32; cc += 2) {
              const float p0 = ex2(fmaf(__uint_as_float(sr[cc]), scale2, neg_m));
              const float p1 = ex2(fmaf(__uint_as_float(sr[cc + 1]), scale2, neg_m));
              sum8[(cc >> 1) & 7] += p0 + p1;
              sr[cc >> 1] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st16(tl + colS + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[ch * 16]));
        }
        l_run += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
        if (quarter == 0) PAIR_TRACE(3 + x, 23, j);
      }
      if (!ok) break;
      // ---- epilogue of this slot's tile: out = wd * O + wm * R
      if (!(ok = mbar_wait_warp(&sq_full[x], i & 1, epoch))) break;
      // den of this unit: the sigma warps write the slot's next den only
      // after its next QK^Ts, which wait for this epilogue.
      const float den = dbuf[x * 128 + r];
      const float g = gate_of(beta[a.h]);
      const float wd = (1.f - g) / l_run;
      const float wm = den != 0.f ? g / den : 0.f;
      if (!(ok = mbar_wait_warp(&o_full[x], i & 1, epoch))) break;
      tc_fence_after();
      if (quarter == 0) PAIR_TRACE(3 + x, 24, i);
      __nv_bfloat16* orow = out + (int64_t)(a.row_seg + qt * kTile + r) * kD;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t o[32], rr[32];
        tmem_ld32(tl + colO + cb * 32, o);
        tmem_ld32(tl + colS + cb * 32, rr);
        tmem_ld_wait_regs(o);
        tmem_ld_wait_regs(rr);
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pk[q] = pack_bf16x2(fmaf(wm, __uint_as_float(rr[2 * q]), wd * __uint_as_float(o[2 * q])),
                              fmaf(wm, __uint_as_float(rr[2 * q + 1]), wd * __uint_as_float(o[2 * q + 1])));
        if (cb == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&epi_done[x]);
        }
        if (out_v8) {  // 32-byte stores: each lane writes whole sectors of its row
          st_global_v8(orow + cb * 32, pk);
          st_global_v8(orow + cb * 32 + 16, pk + 8);
        } else {
          uint4* o4 = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) o4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      if (quarter == 0) PAIR_TRACE(3 + x, 25, i);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if (warp == 12 && lane == 0) {
      for (int b = 0; b < 2; ++b)
        if ((armed >> (2 * b)) & 2u) mbar_drain(&q_full[b], (armed >> (2 * b)) & 1u);
      for (int b = 0; b < kPairKRing; ++b)
        if ((armed >> (4 + 2 * b)) & 2u) mbar_drain(&k_full[b], (armed >> (4 + 2 * b)) & 1u);
      for (int b = 0; b < kPairVRing; ++b)
        if ((armed >> (10 + 2 * b)) & 2u) mbar_drain(&v_full[b], (armed >> (10 + 2 * b)) & 1u);
    }
    if (warp == 13 || warp == 14) {
      if (elect_one_lane()) {
        mma_commit(&drain[warp - 13]);
        mbar_drain(&drain[warp - 13], 0);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 13) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace infini
