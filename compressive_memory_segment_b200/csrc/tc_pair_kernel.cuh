// Paired-query-tile tensor-core attention kernel (tcgen05 / TMEM / TMA) for
// bf16 I/O, head dimension 128 and segments of an even number of 128-row
// tiles (seg_len % 256 == 0).
//
// Per (b, h, segment, pair of 128-row query tiles): causal softmax attention
// inside the segment ("Hugging Face Infini-Attention reproduction analysis",
// Infini-Attention mechanism: Local Attention) by an online softmax over
// 64-key tiles (the running max / normaliser merge of the "Attention-State
// Memory" page, Methodology); the retrieval sigma(Q) M_{s-1} / sigma(Q).z_{s-1}
// (Memory Retrieval); the sigmoid(beta) blend (Integration); the bf16 store.
//
// Why pairs, and why 64-key tiles. With one query tile per CTA and one score
// buffer, the softmax of key tile j, the PV of tile j and the QK^T of tile
// j + 1 form one serial chain and the tensor pipe waits for the softmax most
// of the time. Here each CTA holds two query tiles of the same segment (the
// "slots" 0 and 1), which share every K and V tile the TMA brings in; each
// slot has its own softmax warpgroup, its own MMA-issuing warp, an
// accumulator O and two score buffers S^0, S^1 in TMEM. With 64-key tiles the
// two score buffers fit beside O (2 x 64 + 128 columns per slot), so QK^T of
// tile j + 1 runs while the softmax works on tile j, and the softmax goes from
// one tile to the next without waiting for the tensor pipe.
//
// Work unit: (segment, pair p), query tiles 2p ("short": n = 4p + 2 key
// tiles of 64) and 2p + 1 ("long": n = 4p + 4). The units a CTA takes come
// from the balanced schedule (decode_unit, with the pairs of a segment in
// place of its tiles: a pair's cost is linear in its rank like a tile's).
//
// Slot x issues, per unit: QK(0) -> S^0, QK(1) -> S^1, then PV(j) and
// QK(j + 2) -> S^{j&1} for j = 0 .. n - 3, PV(n - 2), PV(n - 1), and the
// retrieval R: O += (c sigma(Q)) M_{s-1}. The retrieval is folded into O: the
// softmax thread of row r scales its row of sigma(Q) (in shared memory) by
// c = wm / wd before R, with wd = (1 - g) / l and wm = g / den (0 when den =
// 0), so that out = wd * O; when g == 1 (wd = 0) R overwrites O with
// c = wm and out = O. MMAs issued by one thread execute in order, which
// orders every reuse of a TMEM column range after the MMA reading it (P of
// tile j in S^{j&1} is read by the PV issued just before the QK^T that
// overwrites it; R comes after the slot's last PV; the next unit's QK^Ts come
// after R, and its first PV waits for the epilogue to have read O).
//
// Steps and ring positions. As steps, slot x's unit is: 0: QK(0); 1: QK(1);
// s in 2 .. n-1: PV(s-2), QK(s); n: PV(n-2); n+1: PV(n-1), R. The TMA warp
// loads every tile at its first use in one fixed interleaving of the two
// slots' step sequences -- slot 0 step, slot 1 step, slot 0 step, ... -- with
// the short tile in slot 0 in even units (per CTA) and in slot 1 in odd units:
// the slot with the short tile finishes its unit two steps early and starts
// the next one ahead, and the next unit gives it the long tile, so the two
// meet again at the end of every odd unit. In that interleaving, slot 0
// issues the first use of every tile both slots use (K_j, V_j with
// j <= 4p + 1; the two 64-row halves of M_{s-1}) and slot 1 the last; K_j
// and V_j with j >= 4p + 2 belong to the long tile only. The K ring receives,
// unit by unit, K_0 .. K_{4p+2}, M, K_{4p+3} (even units) or K_0 .. K_{4p+3},
// M (odd units); the V ring V_0 .. V_{4p+3}; so every ring position follows
// from counts. Every ring slot (and Q buffer) is refilled only after uses
// that come earlier in the interleaving than the new tile's first use, which
// is a valid order of all the MMAs, so the loads never wait on work that needs
// a later load. Release barriers count one arrival per slot (the long tile's
// slot arrives twice for its own tiles). The Q tiles go through three
// buffers (pair_qbuf), so the slot that finishes a unit first finds its next
// Q tile already loaded.
//
// Roles (512 threads; register split per warpgroup with setmaxnreg):
//   warps 0-3   softmax of slot 0, one thread per query row: the 64 scores of
//               a key tile in registers, causal mask on the two diagonal
//               tiles, row max, lazy rescale of the row of O, P = 2^(s - m) as
//               packed bf16 over the tile's S columns, row sum; after the
//               slot's last tile of a unit, the c scaling of its sigma(Q) row
//               and the epilogue out = wd * O (or O) as the bf16 row.
//   warps 4-7   the same for slot 1.
//   warps 8-11  sigma(Q), one row per thread, slot 0 then slot 1 of every
//               unit: as soon as the slot's last QK^T of the unit is done,
//               its Q tile is replaced by sigma(Q) in place (the retrieval's
//               A operand) and den = sigma(q) . z_{s-1} is formed in fp32,
//               with z_{s-1} staged in shared memory once per tile.
//   warp 12     TMA producer of the K ring (keys, M halves).
//   warp 13     TMEM owner; MMA issuer of slot 0 (one elected lane).
//   warp 14     MMA issuer of slot 1.
//   warp 15     TMA producer of the V ring and the Q tiles.
//
// TMEM (512 columns): slot x has S^0 at 128x .. 128x+63, S^1 at 128x+64 ..
// 128x+127 and O at 256 + 128x .. 256 + 128x + 127. Shared memory, from the
// 1024-aligned base: Q[3] (32 KB) | K ring[5] | V ring[3] (16 KB tiles of 64
// keys) | barriers | den [2 slots][128] fp32 | z_{s-1} [128] fp32.
//
// Built with INFINI_TRACE defined, CTA 0 records clock64 timestamps of its
// pipeline events (infini_attn_trace.h); otherwise the trace points compile
// to nothing.
#pragma once

namespace infini {
namespace tc {

constexpr int kPairThreads = 512;
constexpr int kKT = 64;                               // keys per key tile
constexpr uint32_t kKTBytes = kKT * 256;              // a 64 x 128 bf16 tile
constexpr uint32_t kKTHalf = kKT * 128;               // one 64-column SW128 block of it
constexpr int kPairQBufs = 3, kPairKRing = 5, kPairVRing = 3;
constexpr uint32_t kPairTiles = kPairQBufs * kTileBytes + (kPairKRing + kPairVRing) * kKTBytes;
constexpr uint32_t kPairBarBytes = 512;
constexpr uint32_t kPairSmem = kPairTiles + kPairBarBytes + 2 * 2 * 128 * 4;
static_assert(kPairSmem <= 232448, "paired attention kernel shared memory");
// setmaxnreg split: the kernel launches at 128 registers per thread (512 x 128
// = 65536, the SM's file); the softmax warpgroups take 160, the retrieval /
// epilogue warpgroup 88, the TMA / MMA warpgroup 104: 128 x (2 x 160 + 88 +
// 104) = 65536 (ptxas: no spills with this split).
constexpr int kPairRegSoftmax = 160, kPairRegSigma = 88, kPairRegIssue = 104;
constexpr int kPairLaunchRegs = 128;
static_assert(2 * kPairRegSoftmax + kPairRegSigma + kPairRegIssue == 4 * kPairLaunchRegs, "register split");
static_assert(kPairThreads * kPairLaunchRegs == 65536, "launch registers");

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
  int step;     // step within the unit, 0 .. n + 1
  int n;        // 64-key tiles of this slot's query tile
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
  c.n = 2 * c.qt + 2;
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
  if (++c.step <= c.n + 1) return false;
  ++c.i;
  c.u += gridDim.x;
  cursor_load(c, x, units, n_pairs, S, H, L, N, gs, n_seg);
  return true;
}

// Ring positions of a unit's tiles (see the interleaving above).
__host__ __device__ __forceinline__ int pair_kpos(int kbase, int i, int p, int j) {
  return kbase + j + (((i & 1) == 0 && j == 4 * p + 3) ? 2 : 0);
}
__host__ __device__ __forceinline__ int pair_mpos(int kbase, int i, int p, int h) {
  return kbase + 4 * p + 3 + h + (i & 1);
}
__host__ __device__ __forceinline__ int pair_kcount(int p) { return 4 * p + 6; }
// Q buffer of slot x in unit i, and how many earlier units used that buffer.
// The slot that finishes unit i first (the short tile's: slot 0 in even
// units, slot 1 in odd ones) loads its next Q tile into the buffer nobody
// holds; the other slot then takes the buffer the first one's retrieval
// frees. That gives: slot 0 uses buffers 0, 2, 0, 2, ..., slot 1 uses 1, 0,
// 1, 0, ... (units 0, 1, 2, 3, ...).
__host__ __device__ __forceinline__ int pair_qbuf(int i, int x) {
  return x == 0 ? ((i & 1) ? 2 : 0) : ((i & 1) ? 0 : 1);
}
__host__ __device__ __forceinline__ int pair_quse(int i, int x) {
  return pair_qbuf(i, x) == 0 ? i : (i >> 1);
}
__host__ __device__ __forceinline__ int pair_vcount(int p) { return 4 * p + 4; }

__device__ __forceinline__ void load_ktile(uint8_t* dst, const CUtensorMap* m, int row, uint64_t* bar) {
  tma_load_2d(dst, m, 0, row, bar);
  tma_load_2d(dst + kKTHalf, m, 64, row, bar);
}

// 32 bytes to global memory in one 256-bit store (address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// tmQ: q as [rows, 128] in 128-row boxes; tmK, tmV: k, v in 64-row boxes;
// tmM: the bf16 M_{s-1} tiles as [rows, 128] in 64-row boxes.
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
  uint8_t* sQ = sm;                                          // [3]
  uint8_t* sK = sm + kPairQBufs * kTileBytes;                // [kPairKRing]
  uint8_t* sV = sK + kPairKRing * kKTBytes;                  // [kPairVRing]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kPairTiles);
  float* lbuf = reinterpret_cast<float*>(sm + kPairTiles + kPairBarBytes);  // row sums l [slot][unit parity][128]

  uint64_t* q_full = bars + 0;      // [3]    TMA
  uint64_t* q_empty = bars + 3;     // [3]    retrieval done with the buffer
  uint64_t* k_full = bars + 6;      // [5]    TMA
  uint64_t* k_empty = bars + 11;    // [5]    both slots done with the ring slot (2 arrivals)
  uint64_t* v_full = bars + 16;     // [3]    TMA
  uint64_t* v_empty = bars + 19;    // [3]    both slots done (2 arrivals)
  uint64_t* s_full = bars + 22;     // [2][2] QK^T into S^b of slot x done
  uint64_t* p_full = bars + 26;     // [2][2] P written into S^b (4 softmax warps)
  uint64_t* pv_done = bars + 30;    // [2][2] PV reading S^b done
  uint64_t* qk_last = bars + 34;    // [2][2] the slot's last QK^T of a unit done (by unit parity)
  uint64_t* l_full = bars + 38;     // [2][2] row sums of the slot's unit written, by unit parity (4 softmax warps)
  uint64_t* sc_full = bars + 42;    // [2]    c sigma(Q) in place (4 retrieval warps)
  uint64_t* o_full = bars + 44;     // [2]    retrieval done: O complete
  uint64_t* epi_done = bars + 46;   // [2]    epilogue has read O (4 retrieval warps)
  uint64_t* drain = bars + 48;      // [2]    abort path: in-flight MMAs of each issuer
  constexpr int kNumBars = 50;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  static_assert(kNumBars * 8 + 4 <= kPairBarBytes, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = N / (2 * kTile);
  const int n_seg = units / n_pairs;
  [[maybe_unused]] const int rows_total = n_seg * N;  // B * H * L: rows of q, k, v, out (index checks)

  if (threadIdx.x == 0) {
    for (int b = 0; b < kNumBars; ++b) {
      uint32_t count = 1;
      if ((b >= 11 && b <= 15) || (b >= 19 && b <= 21)) count = 2;                      // k_empty, v_empty
      if ((b >= 26 && b <= 29) || (b >= 38 && b <= 43) || (b >= 46 && b <= 47)) count = 4;  // p_full, l/sc_full, epi_done
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
  // of the last armed phase): Q[3] at bits 0-5, K ring at 6-15, V ring at 16-21.
  uint32_t armed = 0;
  static_assert(2 * (kPairQBufs + kPairKRing + kPairVRing) <= 32, "armed mask");

  if (warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegIssue));
    if (warp == 12 || warp == 15) {
      // ------------------------------------------------ TMA producers
      // Warp 12 loads the K ring (keys and M halves), warp 15 the V ring and
      // the Q tiles; both walk the same interleaving for their rings, so each
      // ring fills as soon as its own slots free up. The Q tiles wait only for
      // their buffers: warp 15 issues them whenever one frees up, also while
      // it waits for a V slot (a slot's next Q tile is needed before its
      // retrieval, which some later ring tiles wait for).
      const bool kq = warp == 12;
      [[maybe_unused]] const int chp = kq ? 0 : 7;  // trace channel
      [[maybe_unused]] uint32_t trn = 0;
      const int n_mine = (units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;  // units of this CTA
      int qk_next = 0;  // next Q load: unit qk_next >> 1, first or second of the unit's two
      // Issues the next Q load if its buffer is free; returns whether it did.
      auto service_q = [&]() -> bool {
        if (kq || qk_next >= 2 * n_mine) return false;
        const int i = qk_next >> 1;
        // Unit 0: slot 0 then 1; later units: the first finisher of the unit
        // before (slot 0 after an even unit, slot 1 after an odd one) first.
        const int f = i == 0 ? 0 : ((i - 1) & 1);
        const int x = (qk_next & 1) ? 1 - f : f;
        const int qb = pair_qbuf(i, x), quse = pair_quse(i, x);
        if (quse > 0 && !__any_sync(0xffffffffu, mbar_test_wait(&q_empty[qb], (quse - 1) & 1))) return false;
        if (quse > 0 && !(ok = mbar_wait_warp(&q_empty[qb], (quse - 1) & 1, epoch))) return false;
        const PairUnit a = decode_pair((int)blockIdx.x + i * (int)gridDim.x, n_pairs, S, H, L, N, gridDim.x, gs,
                                       n_seg);
        const int qt = 2 * a.p + (slot_is_short(x, i) ? 0 : 1);
        if (!INFINI_CHECK(a.row_seg + qt * kTile + kTile <= rows_total)) return false;
        armed = (armed & ~(3u << (2 * qb))) | ((2u | (quse & 1)) << (2 * qb));
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(&q_full[qb], kTileBytes);
          load_tile(sQ + qb * kTileBytes, &tmQ, a.row_seg + qt * kTile, &q_full[qb]);
        }
        __syncwarp();
        TC_TRACE(trn, chp, 3 + x, i);
        ++qk_next;
        return true;
      };
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmM);
      auto load_k = [&](int pos, int row, const CUtensorMap* m) {
        const int slot = pos % kPairKRing, use = pos / kPairKRing;
        if (!INFINI_CHECK(row >= 0 && row + kKT <= (m == &tmM ? n_seg * kD : rows_total))) return;
        if (use > 0 && !(ok = mbar_wait_warp(&k_empty[slot], (use - 1) & 1, epoch))) return;
        armed = (armed & ~(3u << (6 + 2 * slot))) | ((2u | (use & 1)) << (6 + 2 * slot));
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(&k_full[slot], kKTBytes);
          load_ktile(sK + slot * kKTBytes, m, row, &k_full[slot]);
        }
        __syncwarp();
        TC_TRACE(trn, chp, 1, pos);
      };
      auto load_v = [&](int pos, int row) {
        const int slot = pos % kPairVRing, use = pos / kPairVRing;
        if (!INFINI_CHECK(row >= 0 && row + kKT <= rows_total)) return;
        if (use > 0) {
          // Wait for the V slot (bounded), issuing Q loads meanwhile.
          uint64_t t0 = globaltimer_ns();
          uint32_t spins = 0;
          while (ok && !__any_sync(0xffffffffu, mbar_test_wait(&v_empty[slot], (use - 1) & 1))) {
            if (service_q()) {
              t0 = globaltimer_ns();
              continue;
            }
            if ((++spins & 31u) == 0) {
              if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
                ok = false;
              } else if (globaltimer_ns() - t0 > kWaitNs) {
                if (lane == 0) {
                  atomicExch(&g_abort_epoch, epoch);
                  flag_timeout();
                }
                ok = false;
              }
              ok = __all_sync(0xffffffffu, ok);
            }
          }
          if (!ok || !(ok = mbar_wait_warp(&v_empty[slot], (use - 1) & 1, epoch))) return;
        }
        armed = (armed & ~(3u << (16 + 2 * slot))) | ((2u | (use & 1)) << (16 + 2 * slot));
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(&v_full[slot], kKTBytes);
          load_ktile(sV + slot * kKTBytes, &tmV, row, &v_full[slot]);
        }
        __syncwarp();
        TC_TRACE(trn, chp, 2, pos);
      };
      // The fixed interleaving: slot 0 step, slot 1 step, ...; each tile is
      // loaded at its first use in it. K / V ring base of the unit of each
      // parity (the slots are at most one unit apart) and the tile counts of
      // the unit slot 0 entered last.
      int kb0 = 0, kb1 = 0, vb0 = 0, vb1 = 0, kc_prev = 0, vc_prev = 0;
      PairCursor c0, c1;
      cursor_start(c0, 0, units, n_pairs, S, H, L, N, gs, n_seg);
      cursor_start(c1, 1, units, n_pairs, S, H, L, N, gs, n_seg);
      auto step = [&](PairCursor& cx, const int x) {
        const int i = cx.i, p = cx.a.p, s = cx.step, n = cx.n;
        const bool slot0_long = !slot_is_short(0, i);
        // First use of tile j of this unit in the interleaving: slot 0's when
        // slot 0 uses it, else (j >= 4p + 2, short slot 0) slot 1's.
        auto first = [&](int j) { return x == 0 || (j >= 4 * p + 2 && !slot0_long); };
        if (s == 0) {
          if (x == 0) {  // slot 0 enters every unit first
            if (i & 1) {
              kb1 = kb0 + kc_prev;
              vb1 = vb0 + vc_prev;
            } else {
              kb0 = i == 0 ? 0 : kb1 + kc_prev;
              vb0 = i == 0 ? 0 : vb1 + vc_prev;
            }
            kc_prev = pair_kcount(p);
            vc_prev = pair_vcount(p);
          }
        }
        const int kb = (i & 1) ? kb1 : kb0, vb = (i & 1) ? vb1 : vb0;
        if (s <= 1) {
          if (kq && first(s)) load_k(pair_kpos(kb, i, p, s), cx.a.row_seg + s * kKT, &tmK);
        } else {
          const int jv = s - 2;  // V tile of this step's PV
          if (!kq && first(jv)) load_v(vb + jv, cx.a.row_seg + jv * kKT);
          if (!ok || !kq) return;
          if (s <= n - 1) {
            if (first(s)) load_k(pair_kpos(kb, i, p, s), cx.a.row_seg + s * kKT, &tmK);
          } else if (s == n + 1 && x == 0) {  // the two 64-row halves of M_{s-1}
            load_k(pair_mpos(kb, i, p, 0), cx.a.seg_unit * kD, &tmM);
            if (ok) load_k(pair_mpos(kb, i, p, 1), cx.a.seg_unit * kD + kKT, &tmM);
          }
        }
      };
      while (ok && service_q()) {
      }
      while (ok && !(c0.done && c1.done)) {
        if (!c0.done) {
          step(c0, 0);
          cursor_next(c0, 0, units, n_pairs, S, H, L, N, gs, n_seg);
        }
        if (ok && !c1.done) {
          step(c1, 1);
          cursor_next(c1, 1, units, n_pairs, S, H, L, N, gs, n_seg);
        }
        if (ok) service_q();
      }
      // The remaining Q loads (bounded wait for each buffer).
      while (ok && !kq && qk_next < 2 * n_mine) {
        const int i = qk_next >> 1;
        const int f = i == 0 ? 0 : ((i - 1) & 1);
        const int x = (qk_next & 1) ? 1 - f : f;
        const int quse = pair_quse(i, x);
        if (quse > 0 && !(ok = mbar_wait_warp(&q_empty[pair_qbuf(i, x)], (quse - 1) & 1, epoch))) break;
        service_q();
      }
      TC_TRACE_END(trn, chp);
    } else if (warp == 13 || warp == 14) {
      // ------------------------------------------------ MMA issuer of slot x
      const int x = warp - 13;
      const uint32_t id_qk = idesc_bf16_f32(128, kKT, false, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
      const uint64_t dq0 = desc_kmajor_sw128(smem_u32(sQ));
      const uint64_t dk0 = desc_kmajor_sw128(smem_u32(sK));
      const uint64_t dkmn0 = desc_mnmajor_sw128(smem_u32(sK), kKTHalf);
      const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(sV), kKTHalf);
      constexpr uint32_t kQD = kTileBytes >> 4, kKD = kKTBytes >> 4;
      const uint32_t tS = tmem + x * 128, tO = tmem + 256 + x * 128;
      int pv_count = 0;  // PVs issued by this slot (all units)
      [[maybe_unused]] uint32_t trn = 0;
      // S^b = Q K^T for the 64-key tile at K-ring position kp.
      auto qk = [&](int qb, int j, int kp, int arrivals, uint64_t* last_qk) {
        const int slot = kp % kPairKRing, b = j & 1;
        if (!(ok = mbar_wait_warp(&k_full[slot], (kp / kPairKRing) & 1, epoch))) return;
        tc_fence_after();
        const uint64_t da = dq0 + qb * kQD, db = dk0 + slot * kKD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tS + b * kKT, da + (((kk >> 2) * kHalf + (kk & 3) * 32) >> 4),
                        db + (((kk >> 2) * kKTHalf + (kk & 3) * 32) >> 4), id_qk, kk != 0);
          mma_commit(&s_full[x * 2 + b]);
          for (int a = 0; a < arrivals; ++a) mma_commit(&k_empty[slot]);
          if (last_qk) mma_commit(last_qk);
        }
        __syncwarp();
      };
      // O (+)= P_j V_j with P_j in S^{j&1}, V_j at V-ring position vp.
      auto pv = [&](int i, int j, int vp, int arrivals) {
        const int slot = vp % kPairVRing, b = j & 1;
        if (!(ok = mbar_wait_warp(&p_full[x * 2 + b], (pv_count >> 1) & 1, epoch) &&
                   mbar_wait_warp(&v_full[slot], (vp / kPairVRing) & 1, epoch)))
          return;
        // The unit's first PV overwrites O: the previous unit's epilogue must
        // have read it.
        if (j == 0 && i >= 1 && !(ok = mbar_wait_warp(&epi_done[x], (i - 1) & 1, epoch))) return;
        ++pv_count;
        tc_fence_after();
        const uint64_t db = dv0 + slot * kKD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tO, tS + b * kKT + kk * 8, db + ((kk * 2048) >> 4), id_pv, (j != 0 || kk != 0) ? 1u : 0u);
          for (int a = 0; a < arrivals; ++a) mma_commit(&v_empty[slot]);
          mma_commit(&pv_done[x * 2 + b]);
        }
        __syncwarp();
      };
      // O += (c sigma(Q)) M_{s-1} (or O = when g == 1), M halves at mp0, mp1.
      auto retrieval = [&](int i, int qb, int mp0, int mp1, bool overwrite) {
        const int s0 = mp0 % kPairKRing, s1 = mp1 % kPairKRing;
        if (!(ok = mbar_wait_warp(&sc_full[x], i & 1, epoch) &&
                   mbar_wait_warp(&k_full[s0], (mp0 / kPairKRing) & 1, epoch) &&
                   mbar_wait_warp(&k_full[s1], (mp1 / kPairKRing) & 1, epoch)))
          return;
        tc_fence_after();
        const uint64_t da = dq0 + qb * kQD;
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t db = dkmn0 + ((kk >> 2) ? s1 : s0) * kKD + (((kk & 3) * 2048) >> 4);
            mma_bf16_ss(tO, da + (((kk >> 2) * kHalf + (kk & 3) * 32) >> 4), db, id_pv,
                        (overwrite && kk == 0) ? 0u : 1u);
          }
          mma_commit(&o_full[x]);
          mma_commit(&q_empty[qb]);
          mma_commit(&k_empty[s0]);
          mma_commit(&k_empty[s1]);
        }
        __syncwarp();
      };
      // Per unit: PV(j) and QK^T(j + 2) for j = 0 .. n - 1, then the next
      // unit's QK^T(0), QK^T(1) (its Q tile was loaded ahead), then this
      // unit's retrieval; the first unit's QK^T(0), QK^T(1) come first.
      int u = blockIdx.x;
      if (u < units) {
        int i = 0, kbase = 0, vbase = 0;
        PairUnit a = decode_pair(u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
        int qt = 2 * a.p + (slot_is_short(x, 0) ? 0 : 1), n = 2 * qt + 2, qb = pair_qbuf(0, x);
        // Release arrivals: a unit's long-tile-only tiles (j >= 4p + 2) arrive twice.
        auto arr = [](int p, int j) { return j >= 4 * p + 2 ? 2 : 1; };
        TC_TRACE(trn, 1 + x, 10, 0);
        if ((ok = mbar_wait_warp(&q_full[qb], 0, epoch))) {
          qk(qb, 0, pair_kpos(0, 0, a.p, 0), arr(a.p, 0), nullptr);
          if (ok) qk(qb, 1, pair_kpos(0, 0, a.p, 1), arr(a.p, 1), n == 2 ? &qk_last[x * 2] : nullptr);
        }
        TC_TRACE(trn, 1 + x, 11, 0);
        while (ok) {
          for (int j = 0; j < n && ok; ++j) {
            TC_TRACE(trn, 1 + x, 12, j);
            pv(i, j, vbase + j, arr(a.p, j));
            TC_TRACE(trn, 1 + x, 13, j);
            if (ok && j + 2 < n)
              qk(qb, j + 2, pair_kpos(kbase, i, a.p, j + 2), arr(a.p, j + 2),
                 j + 2 == n - 1 ? &qk_last[x * 2 + (i & 1)] : nullptr);
            TC_TRACE(trn, 1 + x, 14, j);
          }
          if (!ok) break;
          const int u2 = u + gridDim.x;
          const bool has_next = u2 < units;
          const int kbase2 = kbase + pair_kcount(a.p), vbase2 = vbase + pair_vcount(a.p);
          PairUnit a2 = a;
          int qt2 = 0, n2 = 0, qb2 = 0;
          if (has_next) {
            a2 = decode_pair(u2, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
            qt2 = 2 * a2.p + (slot_is_short(x, i + 1) ? 0 : 1);
            n2 = 2 * qt2 + 2;
            qb2 = pair_qbuf(i + 1, x);
            TC_TRACE(trn, 1 + x, 10, i + 1);
            if (!(ok = mbar_wait_warp(&q_full[qb2], pair_quse(i + 1, x) & 1, epoch))) break;
            qk(qb2, 0, pair_kpos(kbase2, i + 1, a2.p, 0), arr(a2.p, 0), nullptr);
            if (ok)
              qk(qb2, 1, pair_kpos(kbase2, i + 1, a2.p, 1), arr(a2.p, 1),
                 n2 == 2 ? &qk_last[x * 2 + ((i + 1) & 1)] : nullptr);
            if (!ok) break;
            TC_TRACE(trn, 1 + x, 11, i + 1);
          }
          const bool overwrite = gate_of(beta[a.h]) == 1.f;
          retrieval(i, qb, pair_mpos(kbase, i, a.p, 0), pair_mpos(kbase, i, a.p, 1), overwrite);
          TC_TRACE(trn, 1 + x, 15, i);
          if (!ok || !has_next) break;
          ++i;
          u = u2;
          a = a2;
          qt = qt2;
          n = n2;
          qb = qb2;
          kbase = kbase2;
          vbase = vbase2;
        }
      }
      TC_TRACE_END(trn, 1 + x);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ retrieval operand and epilogue, one row per thread
    // Per slot and unit, three tasks in order: sigma(Q) and den (once the
    // slot's last QK^T of the unit is done); the c scaling of the sigma(Q)
    // row (once the softmax has handed over the row sums); the epilogue
    // out = mult * O (once the retrieval is done). Each warp runs the next
    // task of whichever slot is ready; the warps do not wait for each other.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegSigma));
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    constexpr float kLog2e = 1.4426950408889634f;
    // One slot's progress: unit index and id, next task, den and the output
    // multiplier of its current unit.
    struct SlotWork {
      int i, u, task;
      float den, mult;
    };
    SlotWork w0{0, (int)blockIdx.x, 0, 0.f, 0.f}, w1{0, (int)blockIdx.x, 0, 0.f, 0.f};
    [[maybe_unused]] uint32_t trn5 = 0, trn6 = 0;
    auto run_task = [&](SlotWork& w, const int x) -> bool {
      if (w.u >= units) return false;
      const int i = w.i, qb = pair_qbuf(i, x);
      uint8_t* qtile = sQ + qb * kTileBytes;
      if (w.task == 0) {
        // sigma(Q) in place over the slot's Q tile, den = sigma(q) . z_{s-1}.
        uint64_t* bar = &qk_last[x * 2 + (i & 1)];
        if (!__any_sync(0xffffffffu, mbar_test_wait(bar, (i >> 1) & 1))) return false;
        // The TMA-written tile becomes visible to this thread through its own barrier.
        if (!(ok = mbar_wait_warp(bar, (i >> 1) & 1, epoch) &&
                   mbar_wait_warp(&q_full[qb], pair_quse(i, x) & 1, epoch)))
          return false;
        if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 30, i);
        const PairUnit a = decode_pair(w.u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
        // Lane l holds z[4l .. 4l + 3]; column c's value comes from lane c / 4.
        const float4 zl = __ldg(reinterpret_cast<const float4*>(zp + (int64_t)a.seg_unit * kD) + lane);
        float den = 0.f;
#pragma unroll 2
        for (int cc = 0; cc < 16; ++cc) {
          uint4* px = reinterpret_cast<uint4*>(qtile + sw128_offset(r, cc * 8, 128));
          const uint4 xq = *px;
          float zz[8];
          zz[0] = __shfl_sync(0xffffffffu, zl.x, 2 * cc);
          zz[1] = __shfl_sync(0xffffffffu, zl.y, 2 * cc);
          zz[2] = __shfl_sync(0xffffffffu, zl.z, 2 * cc);
          zz[3] = __shfl_sync(0xffffffffu, zl.w, 2 * cc);
          zz[4] = __shfl_sync(0xffffffffu, zl.x, 2 * cc + 1);
          zz[5] = __shfl_sync(0xffffffffu, zl.y, 2 * cc + 1);
          zz[6] = __shfl_sync(0xffffffffu, zl.z, 2 * cc + 1);
          zz[7] = __shfl_sync(0xffffffffu, zl.w, 2 * cc + 1);
          const uint32_t wq[4] = {xq.x, xq.y, xq.z, xq.w};
          uint32_t o4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float f0 = __uint_as_float(wq[t] << 16), f1 = __uint_as_float(wq[t] & 0xffff0000u);
            const float e0 = ex2(f0 * kLog2e), e1 = ex2(f1 * kLog2e);
            const float s0 = f0 > 0.f ? f0 + 1.f : e0, s1 = f1 > 0.f ? f1 + 1.f : e1;
            den = fmaf(s0, zz[2 * t], den);
            den = fmaf(s1, zz[2 * t + 1], den);
            o4[t] = pack_bf16x2(s0, s1);
          }
          *px = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        w.den = den;
        w.task = 1;
        if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 31, i);
        return true;
      }
      if (w.task == 1) {
        // c = wm / wd scales the row (wd = (1 - g) / l, wm = g / den, 0 when
        // den = 0); with g == 1 the retrieval overwrites O and c = wm.
        uint64_t* lbar = &l_full[x * 2 + (i & 1)];
        if (!__any_sync(0xffffffffu, mbar_test_wait(lbar, (i >> 1) & 1))) return false;
        if (!(ok = mbar_wait_warp(lbar, (i >> 1) & 1, epoch))) return false;
        if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 33, i);
        const PairUnit a = decode_pair(w.u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
        const float l = lbuf[(x * 2 + (i & 1)) * 128 + r];
        const float g = gate_of(beta[a.h]);
        const float wm = w.den != 0.f ? g / w.den : 0.f;
        float c;
        if (g == 1.f) {
          c = wm;
          w.mult = 1.f;
        } else {
          w.mult = (1.f - g) / l;
          c = wm / w.mult;
        }
#pragma unroll 4
        for (int cc = 0; cc < 16; ++cc) {
          uint4* px = reinterpret_cast<uint4*>(qtile + sw128_offset(r, cc * 8, 128));
          const uint4 v = *px;
          const uint32_t wq[4] = {v.x, v.y, v.z, v.w};
          uint32_t o4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t)
            o4[t] = pack_bf16x2(__uint_as_float(wq[t] << 16) * c, __uint_as_float(wq[t] & 0xffff0000u) * c);
          *px = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sc_full[x]);
        w.task = 2;
        if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 27, i);
        return true;
      }
      // The epilogue: out = mult * O as this row of the output tile.
      if (!__any_sync(0xffffffffu, mbar_test_wait(&o_full[x], i & 1))) return false;
      if (!(ok = mbar_wait_warp(&o_full[x], i & 1, epoch))) return false;
      tc_fence_after();
      if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 24, i);
      const PairUnit a = decode_pair(w.u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
      const int qt = 2 * a.p + (slot_is_short(x, i) ? 0 : 1);
      const bool row_ok = INFINI_CHECK(a.row_seg + qt * kTile + r < rows_total);
      __nv_bfloat16* orow = out + (int64_t)(a.row_seg + qt * kTile + r) * kD;
      const uint32_t colO = 256 + x * 128;
#pragma unroll 1
      for (int cb = 0; cb < 8; ++cb) {
        uint32_t o[16];
        tmem_ld16(tl + colO + cb * 16, o);
        tmem_ld_wait_regs(o);
        uint32_t pk[8];
#pragma unroll
        for (int t = 0; t < 8; ++t)
          pk[t] = pack_bf16x2(w.mult * __uint_as_float(o[2 * t]), w.mult * __uint_as_float(o[2 * t + 1]));
        if (cb == 7) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&epi_done[x]);
        }
        if (!row_ok) continue;
        if (out_v8) {  // 32-byte stores: each lane writes whole sectors of its row
          st_global_v8(orow + cb * 16, pk);
        } else {
          uint4* o4 = reinterpret_cast<uint4*>(orow + cb * 16);
          o4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          o4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (warp == 8) TC_TRACE(x ? trn6 : trn5, 5 + x, 25, i);
      w.task = 0;
      ++w.i;
      w.u += gridDim.x;
      return true;
    };
    uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (ok && (w0.u < units || w1.u < units)) {
      bool did = run_task(w0, 0);
      if (ok) did = run_task(w1, 1) || did;
      if (did) {
        t0 = globaltimer_ns();
        spins = 0;
      } else if ((++spins & 31u) == 0) {
        // Bounded like every other wait: give up after kWaitNs without progress.
        if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
          ok = false;
        } else if (globaltimer_ns() - t0 > kWaitNs) {
          if (lane == 0) {
            atomicExch(&g_abort_epoch, epoch);
            flag_timeout();
          }
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
      }
    }
    if (warp == 8) {
      TC_TRACE_END(trn5, 5);
      TC_TRACE_END(trn6, 6);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue of slot x (one row per thread)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairRegSoftmax));
    const int x = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t colS = x * 128, colO = 256 + x * 128;
    const float scale2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    int t = 0, i = 0;  // tiles of this slot so far (all units); unit index
    [[maybe_unused]] uint32_t trn = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      const PairUnit a = decode_pair(u, n_pairs, S, H, L, N, gridDim.x, gs, n_seg);
      const int qt = 2 * a.p + (slot_is_short(x, i) ? 0 : 1);
      const int n = 2 * qt + 2;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n; ++j, ++t) {
        const int b = j & 1;
        if (quarter == 0) TC_TRACE(trn, 3 + x, 20, j);
        if (!(ok = mbar_wait_warp(&s_full[x * 2 + b], (t >> 1) & 1, epoch))) break;
        tc_fence_after();
        if (quarter == 0) TC_TRACE(trn, 3 + x, 21, j);
        uint32_t sr[64];
        tmem_ld32(tl + colS + b * kKT, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tl + colS + b * kKT + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait_regs(sr);
        // Tiles 2qt and 2qt + 1 hold the segment's keys of this query tile:
        // key 64 (j - 2qt) + c is visible to row r iff it is <= r.
        const int dj = j - 2 * qt;
        const bool diag = dj >= 0;
        if (diag) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (64 * dj + cc > r) sr[cc] = __float_as_uint(-INFINITY);
        }
        const float mx = row_max64(sr);
        if (quarter == 0) TC_TRACE(trn, 3 + x, 22, j);
        // Lazy rescaling: the exponent's max is raised only when the row's new
        // max exceeds it by more than 2^8 (unnormalised P stays <= 256).
        const bool need = mx * scale2 > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_tgt = need ? mx * scale2 : m_run;
          const float alpha = ex2(m_run - m_tgt);
          if (j > 0) {
            // Rescale this row of O once the PV of tile j - 1 is done (PV j - 2
            // is: it came before QK^T j - 1 in issue order).
            if (!(ok = mbar_wait_warp(&pv_done[x * 2 + (b ^ 1)], ((t - 1) >> 1) & 1, epoch))) break;
            tc_fence_after();
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
        // P = 2^(s log2(e)/sqrt(d) - m) as bf16 pairs over the tile's S
        // columns, in two 32-key chunks (16 columns each); on a diagonal tile a
        // chunk wholly right of every row of this warp is all zeros.
        uint64_t acc2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc2[q] = 0ull;
        const uint64_t sc2 = f32x2(scale2, scale2), nm2 = f32x2(-m_run, -m_run);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          if (diag && 2 * dj + ch > quarter) {
#pragma unroll
            for (int cc = ch * 32; cc < ch * 32 + 32; cc += 2) sr[cc >> 1] = 0u;
          } else {
#pragma unroll
            for (int cc = ch * 32; cc < ch * 32 + 32; cc += 2) exp2_pair(sr, cc, sc2, nm2, acc2[(cc >> 1) & 3]);
          }
          tmem_st16(tl + colS + b * kKT + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[ch * 16]));
        }
        l_run += sum_f32x2(acc2);
        if (quarter == 0) TC_TRACE(trn, 3 + x, 26, j);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x * 2 + b]);
        if (quarter == 0) TC_TRACE(trn, 3 + x, 23, j);
      }
      if (!ok) break;
      // Hand the row sums to the retrieval / epilogue warps and go on to the
      // next unit. Buffers alternate by unit: the next unit may have only two
      // key tiles (both QK^Ts issued before this unit's retrieval) and end
      // before these sums are read, but the unit after it cannot start
      // before this unit's epilogue, which comes after the read.
      lbuf[(x * 2 + (i & 1)) * 128 + r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&l_full[x * 2 + (i & 1)]);
      if (quarter == 0) TC_TRACE(trn, 3 + x, 28, i);
    }
    if (quarter == 0) TC_TRACE_END(trn, 3 + x);
  }
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch) {
    // Abort path: let this CTA's own TMA copies and MMAs finish before exit.
    if ((warp == 12 || warp == 15) && lane == 0) {  // each producer's own armed buffers
      for (int b = 0; b < kPairQBufs; ++b)
        if ((armed >> (2 * b)) & 2u) mbar_drain(&q_full[b], (armed >> (2 * b)) & 1u);
      for (int b = 0; b < kPairKRing; ++b)
        if ((armed >> (6 + 2 * b)) & 2u) mbar_drain(&k_full[b], (armed >> (6 + 2 * b)) & 1u);
      for (int b = 0; b < kPairVRing; ++b)
        if ((armed >> (16 + 2 * b)) & 2u) mbar_drain(&v_full[b], (armed >> (16 + 2 * b)) & 1u);
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
