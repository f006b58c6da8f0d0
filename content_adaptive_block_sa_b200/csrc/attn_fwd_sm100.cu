// Block-sparse attention forward on the 5th-generation tensor cores (sm_100a).
//
// A work item is one (128-query tile, head, sequence); its listed 128-key
// tiles are visited in order and everything else is skipped ("UniGist ...",
// Approach: skipping non-visible blocks is what makes the sparse layout fast;
// "Gzip-guided sparse attention ...", Scope: dense-then-mask gives no
// speed-up). With gzip blocks of 64 tokens ("pair mode") an item is a pair of
// 64-row query blocks and a visit a pair of 64-key blocks, so that a 128 x 128
// tensor-core tile holds only block pairs of the mask (see gzip_pair_kernel).
// The kernel is persistent: one CTA per SM walks the items blockIdx.x,
// blockIdx.x + gridDim.x, ... (the longest lists first). Ring slots and
// mbarrier phases run on across items, so the loads and the first Q K^T of the
// next item overlap the softmax and epilogue of the current one.
//
// Roles (480 threads):
//   warp 0      TMA producer: Q per item (d = 64: two Q stages, so the next
//               item's Q loads early); K and V per visit (d = 64: one stage
//               and one barrier for both; d = 128: separate rings, K one tile
//               ahead of V); TMEM allocation.
//   warp 1      one thread issues tcgen05.mma: S_j = Q K_j^T into one of two
//               TMEM S buffers, then O_h += P_j[:, h-half] V_j[h-half, :] for
//               the two column halves h = 0, 1, each into its own TMEM
//               accumulator, with P_j read from TMEM (A operand) and V_j from
//               shared memory. Completion is signalled with tcgen05.commit.
//               (d = 64: two O buffers, items alternate.)
//   warps 2-9   softmax, two groups of four warps: group h owns key columns
//               [64h, 64h + 64) of every S tile; thread (h, r) owns query row
//               r (TMEM lane r) within that half. Each half keeps its own
//               running max (log2 domain) and row sum, so the two halves never
//               synchronise per tile; O_h is rescaled lazily, only when the
//               half's max grew by more than 2^8 (P <= 256 otherwise). At the
//               end of an item each half leaves its (max, sum) in shared memory.
//   warp 10     mask: for each visited tile, ahead of the softmax, the
//               visibility of its 128 x 128 (row, key) pairs as 4 x 128 bit
//               words in a shared-memory ring, so that no global load or
//               mask arithmetic sits on the softmax's path.
//   warps 11-14 epilogue: thread r merges row r of the two halves,
//               O = (2^(m_0-m) O_0 + 2^(m_1-m) O_1) / (2^(m_0-m) l_0 + 2^(m_1-m) l_1),
//               and stores O and LSE while the softmax works on the next item.
// S is double-buffered (Q K^T of tile j+1 runs while tile j's softmax runs).
// Each half writes its bf16 P over the first 32 of its own 64 S columns, so P
// never passes through shared memory; Q K^T(j+2) may overwrite that buffer
// right after P V(j) is issued, as tcgen05.mma ops of one thread execute in
// issue order. Every wait is bounded; on timeout the device status word
// is set and all roles leave after draining their copies and MMAs, freeing
// TMEM.
#include <cuda.h>

#include "attn_mask.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

struct FwdTcParams {
  CUtensorMap tmq, tmk, tmv;
  CUtensorMap tmq64, tmk64, tmv64;  // pair mode: 64-row boxes
  CUtensorMap tmkc, tmvc;  // gist mode: sinks + gists compacted in logical order
  AttnArgs a;
  MaskArgs m;
  // gist mode: element masks of (query tile I, near key tile J), [T][near_nt][4][128]
  // words, pair index I * near_nt + (J - I + near_nt - 1)
  const uint32_t* near;
  int near_nt;
};

// Item -> (query tile, head, sequence): late query tiles of every head and
// sequence first.
struct Item {
  int I, h, bt;
  __device__ Item(int idx, int T, int Hq, int Bt) {
    const int hb = Hq * Bt;
    I = T - 1 - idx / hb;
    h = (idx % hb) % Hq;
    bt = (idx % hb) / Hq;
  }
};


constexpr int kMaskSlots = 8;              // mask ring depth (tiles)
constexpr uint32_t kMaskSlotBytes = 2048;  // [4 words][128 rows] uint32
constexpr int kRowCacheWords = 1024;       // gzip: the item's block-row bits

// exponential pairs i with i % 8 >= the threshold take the FMA-pipe polynomial,
// the rest the exp unit: d = 64 is bound by the exp unit's 16 results per clock
// and SM, d = 128 is not (measured fastest with no polynomial at all)
#ifndef SA_FWD64_POLY_FROM
#define SA_FWD64_POLY_FROM 5
#endif
#ifndef SA_FWD128_POLY_FROM
#define SA_FWD128_POLY_FROM 8
#endif
#ifndef SA_FWD64_QSTAGES
#define SA_FWD64_QSTAGES 2
#endif
static_assert(SA_FWD64_QSTAGES >= 1 && SA_FWD64_QSTAGES <= 4, "Q stages at d = 64: 1..4");

template <int D>
struct FwdLayout {
  static constexpr int kKStages = D == 64 ? 4 : 3;  // K ring depth
  static constexpr int kVStages = D == 64 ? 4 : 2;  // V ring depth
  // Q tiles: d = 64 keeps several, so that an item's Q is requested kQAhead
  // items before it starts (its stage was last read by the item kQStages
  // earlier, whose Q K^T is long done by then)
  static constexpr int kQStages = D == 64 ? SA_FWD64_QSTAGES : 1;
  static constexpr int kQAhead = kQStages >= 3 ? kQStages - 2 : 0;
  // d = 64: K and V of a tile share a stage and one full / free barrier pair,
  // so the MMA thread waits once per tile for both (every mbarrier wait on
  // that thread leaves the tensor core idle for its latency, as tcgen05.mma
  // issue blocks until the previous MMA has started)
  static constexpr bool kMergedKV = D == 64;
  // d = 64: two O accumulators in TMEM (items alternate), so the next item's
  // P V never waits for the epilogue warps to read the previous O
  static constexpr int kOBufs = D == 64 ? 2 : 1;
  static constexpr uint32_t kQ = 128 * D * 2;        // Q tile
  static constexpr uint32_t kKV = 128 * D * 2;       // one K or V tile
  static constexpr uint32_t kAtom = 128 * 128;       // [128 rows][64 bf16] swizzle atom
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k0 = kQStages * kQ;
  static constexpr uint32_t v0 = k0 + kKStages * kKV;
  static constexpr uint32_t mask = v0 + kVStages * kKV;
  static constexpr uint32_t rows = mask + kMaskSlots * kMaskSlotBytes;
  static constexpr uint32_t ml = rows + kRowCacheWords * 4;  // [2 items][2 halves][128] (max, sum)
  static constexpr uint32_t bars = ml + 2 * 2 * 128 * 8;
  static constexpr uint32_t bytes = bars + 512 + 1024;  // + alignment slack
};

// mbarriers. QF/QE: Q stage full / consumed (per item). KF/KE, VF/VE: K or V
// stage full / free (d = 64: KF/KE cover K and V). SF: S buffer written. PF:
// P written to TMEM by both halves, one barrier per S buffer: the softmax can
// finish tile j + 1 before the MMA thread has seen tile j's P, but not tile
// j + 2 (its S needs P V(j) issued), so a barrier per S buffer is never two
// phases ahead of its waiter. OD: P V done, one barrier per S buffer (waited
// for only before an O rescale). MF/ME: mask slot
// written / read. OI: every MMA of the item done. OF: both halves have read O
// (per item). OI/OF/ML, one barrier per item parity: OI every MMA of the item
// done; OF the epilogue warps have read O and (max, sum); ML the softmax
// halves have written (max, sum). DRAIN: all MMAs done before exit.
enum {
  B_QF = 0, B_QE = 4, B_KF = 8, B_KE = 12, B_VF = 16, B_VE = 20, B_SF = 24, B_PF = 26,
  B_OD = 28, B_MF = 30, B_ME = B_MF + kMaskSlots, B_OI = B_ME + kMaskSlots, B_OF = B_OI + 2,
  B_ML = B_OF + 2, B_DRAIN = B_ML + 2, kNumBars
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;  // O_0 at 256, O_1 at 256 + D
constexpr int kSoftmaxThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kThreads = 64 + kSoftmaxThreads + 32 + kEpiThreads;
constexpr int kMaskWarp = 10;
constexpr int kEpiWarp0 = 11;  // warps 11-14: epilogue (one per TMEM lane quarter)

// Pair mode: visibility words of one visit (v = j1 | j2 << 12 | vis << 24)
// for rows lane + 32 i: rows 0-63 belong to query block qa, 64-127 to qb
// (qb < 0: none). Key columns 0-63 are block j1, 64-127 block j2. A visited
// block is either below the row's block (fully visible) or the row's own
// block (causal: columns up to the row).
__device__ __forceinline__ void pair_tile_words(uint32_t v, int qa, int qb, int lane,
                                                uint32_t* out) {
  const int j1 = v & 0xfff, j2 = (v >> 12) & 0xfff;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int blk = i < 2 ? qa : qb, rr = lane + 32 * (i & 1);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = w < 2 ? j1 : j2;
      const uint32_t seen = (v >> (24 + 2 * (w >> 1) + (i >> 1))) & 1u;
      uint32_t word = 0u;
      if (blk >= 0 && seen) word = j < blk ? 0xffffffffu : prefix_bits(rr - 32 * (w & 1) + 1);
      out[w * 128 + lane + 32 * i] = word;
    }
  }
}

// Number of visited tiles of item idx.
__device__ __forceinline__ int item_tiles(const MaskArgs& m, int idx, int T, int Hq, int Bt) {
  const Item itm(idx, T, Hq, Bt);
  WorkList wl;
  wl.init(m, list_of(m, itm.bt, itm.h), itm.I);
  return wl.n;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) fwd_tc_kernel(const __grid_constant__ FwdTcParams P) {
  using L = FwdLayout<D>;
  constexpr int KS = L::kKStages, VS = L::kVStages, QS = L::kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + kNumBars) + 1;
  float2* ml = reinterpret_cast<float2*>(smem + L::ml);
  uint32_t* mwords = reinterpret_cast<uint32_t*>(smem + L::mask);

  const AttnArgs& a = P.a;
  const MaskArgs& m = P.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = m.pair ? m.P : m.T;  // items per (head, sequence)
  const int n_items = T * a.Hq * a.Bt;
  DeviceStatus* st = a.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QS; ++s) {
      mbar_init(&bar[B_QF + s], 1);
      mbar_init(&bar[B_QE + s], 1);
    }
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bar[B_KF + s], 1);
      mbar_init(&bar[B_KE + s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bar[B_VF + s], 1);
      mbar_init(&bar[B_VE + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_SF + s], 1);
      mbar_init(&bar[B_PF + s], kSoftmaxThreads);
    }
    mbar_init(&bar[B_OD], 1);
    mbar_init(&bar[B_OD + 1], 1);
    for (int s = 0; s < kMaskSlots; ++s) {
      mbar_init(&bar[B_MF + s], 32);
      mbar_init(&bar[B_ME + s], kSoftmaxThreads);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_OI + s], 1);
      mbar_init(&bar[B_OF + s], kEpiThreads);
      mbar_init(&bar[B_ML + s], kSoftmaxThreads);
    }
    mbar_init(&bar[B_DRAIN], 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      prefetch_tmap(&P.tmq);
      prefetch_tmap(&P.tmk);
      prefetch_tmap(&P.tmv);
      if (m.kind == SA_MASK_GIST) {
        prefetch_tmap(&P.tmkc);
        prefetch_tmap(&P.tmvc);
      }
      int g = 0, k = 0, last_k = -1, last_v = -1, last_q = -1;
      bool ok = true;
      WorkList wl_next;  // the next item's list, read one item ahead
      if (blockIdx.x < n_items) {
        const Item f(blockIdx.x, T, a.Hq, a.Bt);
        wl_next.init(m, list_of(m, f.bt, f.h), f.I);
      }
      // Q of this CTA's item kq (global index iq) into stage kq % QS, whose
      // last occupant, item kq - QS, must have finished its Q K^T
      auto load_q = [&](int kq, int iq) -> bool {
        const Item itq(iq, T, a.Hq, a.Bt);
        const int qs = kq % QS;
        if (kq >= QS && !mbar_wait(&bar[B_QE + qs], ((kq / QS) - 1) & 1, abort, st, 1))
          return false;
        mbar_arrive_expect_tx(&bar[B_QF + qs], L::kQ);
        if (m.pair) {
          // rows 0-63: query block qa, rows 64-127: qb (qa again when there is none)
          const uint32_t pq = (uint32_t)m.pair_q[list_of(m, itq.bt, itq.h) * m.P + itq.I];
          const int qa = pq & 0xffff, qb = (pq >> 16) == 0xffff ? qa : (int)(pq >> 16);
          for (int at = 0; at < D / 64; ++at) {
            uint8_t* dst = smem + L::q + qs * L::kQ + at * L::kAtom;
            tma_load_4d(dst, &P.tmq64, &bar[B_QF + qs], at * 64, itq.h, qa * 64, itq.bt);
            tma_load_4d(dst + 64 * 128, &P.tmq64, &bar[B_QF + qs], at * 64, itq.h, qb * 64, itq.bt);
          }
        } else {
          for (int at = 0; at < D / 64; ++at)
            tma_load_4d(smem + L::q + qs * L::kQ + at * L::kAtom, &P.tmq, &bar[B_QF + qs], at * 64,
                        itq.h, itq.I * kTile, itq.bt);
        }
        last_q = kq;
        return true;
      };
      constexpr int QA = L::kQAhead;
      for (int j = 0; ok && j < QA && blockIdx.x + j * (int)gridDim.x < n_items; ++j)
        ok = load_q(j, blockIdx.x + j * gridDim.x);
      for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x, ++k) {
        const Item itm(idx, T, a.Hq, a.Bt);
        const WorkList wl = wl_next;
        const bool more = idx + (int)gridDim.x < n_items;
        if (more) {
          const Item nx(idx + gridDim.x, T, a.Hq, a.Bt);
          wl_next.init(m, list_of(m, nx.bt, nx.h), nx.I);
        }
        const int hk = itm.h / (a.Hq / a.Hkv);
        if (QA == 0) {
          if (!load_q(k, idx)) break;
        } else if (idx + QA * (int)gridDim.x < n_items) {
          if (!load_q(k + QA, idx + QA * gridDim.x)) break;
        }
        // K of tile it + 1 is requested before V of tile it
        auto load = [&](bool is_k, int it) -> bool {
          const int ns = is_k ? KS : VS;
          const int gt = g + it, s = gt % ns;
          uint64_t* full = &bar[(is_k ? B_KF : B_VF) + s];
          if (!mbar_wait(&bar[(is_k ? B_KE : B_VE) + s], ((gt / ns) & 1) ^ 1, abort, st, 2))
            return false;
          const uint32_t dst = (is_k ? L::k0 : L::v0) + s * L::kKV;
          mbar_arrive_expect_tx(full, L::kKV);
          if (m.pair) {
            int ka, kb;
            wl.pair_entry(m, it, ka, kb);
            const CUtensorMap* map = is_k ? &P.tmk64 : &P.tmv64;
            for (int at = 0; at < D / 64; ++at) {
              tma_load_4d(smem + dst + at * L::kAtom, map, full, at * 64, hk, ka, itm.bt);
              tma_load_4d(smem + dst + at * L::kAtom + 64 * 128, map, full, at * 64, hk, kb, itm.bt);
            }
          } else {
            int src, k0, kind, cnt;
            wl.entry(m, it, src, k0, kind, cnt);
            const CUtensorMap* map = is_k ? (src ? &P.tmkc : &P.tmk) : (src ? &P.tmvc : &P.tmv);
            for (int at = 0; at < D / 64; ++at)
              tma_load_4d(smem + dst + at * L::kAtom, map, full, at * 64, hk, k0, itm.bt);
          }
          if (is_k) last_k = gt; else last_v = gt;
          return true;
        };
        // d = 64: K and V of tile it on one barrier of stage (g + it) % KS
        auto load_kv = [&](int it) -> bool {
          const int gt = g + it, s = gt % KS;
          if (!mbar_wait(&bar[B_KE + s], ((gt / KS) & 1) ^ 1, abort, st, 2)) return false;
          mbar_arrive_expect_tx(&bar[B_KF + s], 2 * L::kKV);
          if (m.pair) {
            int ka, kb;
            wl.pair_entry(m, it, ka, kb);
            for (int at = 0; at < D / 64; ++at) {
              const uint32_t ko = L::k0 + s * L::kKV + at * L::kAtom;
              const uint32_t vo = L::v0 + s * L::kKV + at * L::kAtom;
              tma_load_4d(smem + ko, &P.tmk64, &bar[B_KF + s], at * 64, hk, ka, itm.bt);
              tma_load_4d(smem + ko + 64 * 128, &P.tmk64, &bar[B_KF + s], at * 64, hk, kb, itm.bt);
              tma_load_4d(smem + vo, &P.tmv64, &bar[B_KF + s], at * 64, hk, ka, itm.bt);
              tma_load_4d(smem + vo + 64 * 128, &P.tmv64, &bar[B_KF + s], at * 64, hk, kb, itm.bt);
            }
          } else {
            int src, k0, kind, cnt;
            wl.entry(m, it, src, k0, kind, cnt);
            for (int at = 0; at < D / 64; ++at) {
              tma_load_4d(smem + L::k0 + s * L::kKV + at * L::kAtom, src ? &P.tmkc : &P.tmk,
                          &bar[B_KF + s], at * 64, hk, k0, itm.bt);
              tma_load_4d(smem + L::v0 + s * L::kKV + at * L::kAtom, src ? &P.tmvc : &P.tmv,
                          &bar[B_KF + s], at * 64, hk, k0, itm.bt);
            }
          }
          last_k = gt;
          return true;
        };
        if (L::kMergedKV) {
          for (int it = 0; ok && it < wl.n; ++it) ok = load_kv(it);
        } else {
          if (wl.n > 0) ok = load(true, 0);
          for (int it = 0; ok && it < wl.n; ++it) {
            if (it + 1 < wl.n) ok = load(true, it + 1);
            if (ok) ok = load(false, it);
          }
        }
#ifdef SA_COUNT_TILES
        if (ok) {
          count_tiles(st, CNT_FWD_VISITS, wl.n);
          if (m.pair) {
            const uint32_t pq = (uint32_t)m.pair_q[list_of(m, itm.bt, itm.h) * m.P + itm.I];
            const int qa = pq & 0xffff, qb = (pq >> 16) == 0xffff ? -1 : (int)(pq >> 16);
            int blocks = 0;
            for (int it = 0; it < wl.n; ++it) blocks += __popc(((uint32_t)m.visits[wl.e0 + it] >> 24) & 0xfu);
            count_tiles(st, CNT_PAIR_BLOCKS, blocks);
            count_tiles(st, CNT_PAIR_DENSE, (qa + 1) + (qb + 1));
          } else {
            count_tiles(st, CNT_FWD_DENSE, itm.I + 1);
          }
        }
#endif
        if (more && m.kind == SA_MASK_GZIP) {
          // the next item's first entries, so that its first K load is not
          // held up by a list lookup
          if (m.pair) {
            prefetch_l1(m.visits + wl_next.e0);
          } else {
            prefetch_l1(m.tcol + wl_next.e0);
            prefetch_l1(m.tkind + wl_next.e0);
          }
        }
        g += wl.n;
      }
      // every copy this CTA started must land before the CTA may exit
      volatile int no_abort = 0;
      for (int q = last_q; q >= 0 && q > last_q - QS; --q)
        mbar_wait(&bar[B_QF + q % QS], (q / QS) & 1, &no_abort, nullptr, 3);
      for (int s = 0; s < KS; ++s) {
        if (last_k >= s) {
          const int gs = last_k - ((last_k - s) % KS);
          mbar_wait(&bar[B_KF + s], (gs / KS) & 1, &no_abort, nullptr, 4);
        }
      }
      for (int s = 0; s < VS; ++s) {
        if (last_v >= s) {
          const int gs = last_v - ((last_v - s) % VS);
          mbar_wait(&bar[B_VF + s], (gs / VS) & 1, &no_abort, nullptr, 5);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      // One thread issues S_j = Q K_j^T and then O += P_{j-1} V_{j-1}: tcgen05
      // ops of one thread run in issue order, so Q K^T(j + 1) may reuse the S
      // buffer of P(j - 1) right after P V(j - 1) is issued. tcgen05.mma issue
      // blocks until the tensor core has taken the previous MMA and a barrier
      // wait after it waits for the queued MMAs, so the waits are kept to two
      // per tile (K/V landed, P written).
      constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);
      int g = 0, k = 0;
      bool ok = true;
      int n_next = blockIdx.x < n_items ? item_tiles(m, blockIdx.x, T, a.Hq, a.Bt) : 0;
      for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x, ++k) {
        const int n = n_next;
        n_next = idx + (int)gridDim.x < n_items ? item_tiles(m, idx + gridDim.x, T, a.Hq, a.Bt) : 0;
        const int qs = k % QS;
        const uint32_t qa = sb + L::q + qs * L::kQ;
        if (!mbar_wait(&bar[B_QF + qs], (k / QS) & 1, abort, st, 10)) break;
        // O buffer k % kOBufs last held item k - kOBufs: its epilogue must have
        // read it (waited for once per item, in order, so the per-parity
        // barrier is never two phases ahead)
        const int kp = k - L::kOBufs;
        const uint32_t ob = kTmemO + (uint32_t)((k % L::kOBufs) * 2 * D);
        bool o_free = kp < 0;
        for (int it = 0; it <= n; ++it) {
          if (it < n) {
            const int gq = g + it, s = gq % KS, sb2 = gq & 1;
            if (!mbar_wait(&bar[B_KF + s], (gq / KS) & 1, abort, st, 11)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kb = sb + L::k0 + s * L::kKV;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
              mma_bf16(tmem + sb2 * 128, smem_desc_sw128(qa + off, 16, 1024),
                       smem_desc_sw128(kb + off, 16, 1024), kIdQK, kk > 0);
            }
            mma_commit(&bar[B_SF + sb2]);
            if (!L::kMergedKV) mma_commit(&bar[B_KE + s]);
            if (it == n - 1) mma_commit(&bar[B_QE + qs]);
          }
          if (it >= 1) {
            const int gp = g + it - 1, s = gp % (L::kMergedKV ? KS : VS);
            if (!o_free) {
              if (!mbar_wait(&bar[B_OF + (kp & 1)], (kp >> 1) & 1, abort, st, 13)) {
                ok = false;
                break;
              }
              o_free = true;
            }
            if (!L::kMergedKV && !mbar_wait(&bar[B_VF + s], (gp / VS) & 1, abort, st, 14)) {
              ok = false;
              break;
            }
            if (!mbar_wait(&bar[B_PF + (gp & 1)], (gp >> 1) & 1, abort, st, 15)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vb = sb + L::v0 + s * L::kKV;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              // P of this half: bf16 pairs in the first 32 columns of its S columns
              const uint32_t pa = tmem + (gp & 1) * 128 + hf * 64;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = smem_desc_sw128(vb + (hf * 4 + kk) * 2048, L::kAtom, 1024);
                mma_bf16_ts(tmem + ob + hf * D, pa + kk * 8, bd, kIdPV,
                            (it > 1 || kk > 0) ? 1u : 0u);
              }
            }
            mma_commit(&bar[B_OD + (gp & 1)]);
            mma_commit(&bar[L::kMergedKV ? B_KE + s : B_VE + s]);
          }
        }
        if (!ok) break;
        if (n == 0) {
          mma_commit(&bar[B_QE + qs]);
          if (!o_free && !mbar_wait(&bar[B_OF + (kp & 1)], (kp >> 1) & 1, abort, st, 13)) break;
        }
        mma_commit(&bar[B_OI + (k & 1)]);
        g += n;
      }
      // drain: every MMA issued above has completed
      mma_commit(&bar[B_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[B_DRAIN], 0, &no_abort, nullptr, 17);
    }
  } else if (warp == kMaskWarp) {
    // -------------------------------------------------------------- mask
    // Lane l writes rows l, l + 32, l + 64, l + 96 of every slot:
    // word w of row r at mwords[slot][w][r].
    const int gzip = m.kind == SA_MASK_GZIP;
    const int lb = (gzip && m.b < kTile) ? __ffs(m.b) - 1 : 0;  // b < 128 is a power of two
    uint32_t* rcache = reinterpret_cast<uint32_t*>(smem + L::rows);
    // gzip: the block rows of a query tile (first and last block row)
    auto row_span = [&](int I, int& rb0, int& rb1) {
      rb0 = I * kTile / (gzip ? m.b : 1);
      rb1 = gzip ? min(m.B - 1, (I * kTile + kTile - 1) / m.b) : rb0;
    };
    // The next item's list, its first 32 block-row words and its first 32
    // tile entries are read one item ahead, into registers, so that no
    // global round trip sits between two items.
    WorkList wl_next;
    uint32_t row_next = 0u, pq_next = 0u;
    int col_next = 0, kind_next = 0;
    auto fetch_head = [&](int idx) {
      const Item nx(idx, T, a.Hq, a.Bt);
      const int list = list_of(m, nx.bt, nx.h);
      wl_next.init(m, list, nx.I);
      if (m.pair) {
        pq_next = (uint32_t)m.pair_q[list * m.P + nx.I];
      } else if (gzip) {
        int rb0, rb1;
        row_span(nx.I, rb0, rb1);
        const int nw = (rb1 - rb0 + 1) * m.words;
        row_next = lane < nw ? m.bits[((int64_t)list * m.B + rb0) * m.words + lane] : 0u;
      }
    };
    auto fetch_entries = [&]() {
      if (m.pair) {
        col_next = lane < wl_next.n ? m.visits[wl_next.e0 + lane] : 0;
      } else if (gzip) {
        col_next = lane < wl_next.n ? m.tcol[wl_next.e0 + lane] : 0;
        kind_next = lane < wl_next.n ? m.tkind[wl_next.e0 + lane] : 0;
      }
    };
    if (blockIdx.x < n_items) {
      fetch_head(blockIdx.x);
      fetch_entries();
    }
    int g = 0;
    for (int idx = blockIdx.x; idx < n_items; idx += gridDim.x) {
      const Item itm(idx, T, a.Hq, a.Bt);
      const int list = list_of(m, itm.bt, itm.h);
      const WorkList wl = wl_next;
      const uint32_t row_pre = row_next, pq = pq_next;
      const int pqa = pq & 0xffff, pqb = (pq >> 16) == 0xffff ? -1 : (int)(pq >> 16);
      int col_reg = col_next, kind_reg = kind_next;  // gzip: tile list entries it0 + lane
      const bool more = idx + (int)gridDim.x < n_items;
      if (more) fetch_head(idx + gridDim.x);  // in flight during this item
      // gzip: the block rows of this query tile, copied once per item when they fit
      int rb0, rb1;
      row_span(itm.I, rb0, rb1);
      const int nw = (rb1 - rb0 + 1) * m.words;
      const bool cached = gzip && !m.pair && nw <= kRowCacheWords;
      __syncwarp();  // the previous item's lookups are done
      if (cached) {
        const uint32_t* src = m.bits + ((int64_t)list * m.B + rb0) * m.words;
        if (lane < nw) rcache[lane] = row_pre;
        for (int x = lane + 32; x < nw; x += 32) rcache[x] = src[x];
      }
      __syncwarp();
      RowCtx rc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        rc[i].p = itm.I * kTile + lane + 32 * i;
        rc[i].ok = rc[i].p < a.N;
        rc[i].bits = nullptr;
        if (gzip) {  // rows past N point at the first row of the tile (cleared later)
          const int rb = rc[i].ok ? rc[i].p / m.b : rb0;
          rc[i].bits = cached ? rcache + (rb - rb0) * m.words
                              : m.bits + ((int64_t)list * m.B + rb) * m.words;
        }
        rc[i].li = 0;
      }
      bool ok = true;
      for (int it = 0; it < wl.n; ++it) {
        if (gzip && it > 0 && (it & 31) == 0) {
          const int e = it + lane;
          if (m.pair) {
            col_reg = e < wl.n ? m.visits[wl.e0 + e] : 0;
          } else {
            col_reg = e < wl.n ? m.tcol[wl.e0 + e] : 0;
            kind_reg = e < wl.n ? m.tkind[wl.e0 + e] : 0;
          }
        }
        const int gq = g + it, slot = gq % kMaskSlots;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_ME + slot], ((gq / kMaskSlots) & 1) ^ 1,
                                                abort, st, 30))) {
          ok = false;
          break;
        }
        int src, kbase, kind, cnt;
        if (gzip) {
          src = 0;
          cnt = kTile;
          kbase = __shfl_sync(0xffffffffu, col_reg, it & 31) * kTile;
          kind = __shfl_sync(0xffffffffu, kind_reg, it & 31) == SA_TILE_FULL ? SA_TILE_FULL
                                                                              : SA_TILE_MASKED;
        } else {
          wl.entry(m, it, src, kbase, kind, cnt);
        }
        uint32_t* words = mwords + slot * (kMaskSlotBytes / 4);
        if (m.pair) {
          pair_tile_words((uint32_t)__shfl_sync(0xffffffffu, col_reg, it & 31), pqa, pqb, lane,
                          words);
        } else if (!gzip && src == 0) {
          // gist near tile: the element rule was evaluated once for every head
          const uint4* from = reinterpret_cast<const uint4*>(
              P.near + ((int64_t)itm.I * P.near_nt + (kbase / kTile - itm.I + P.near_nt - 1)) * 512);
          uint4 v[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) v[q4] = from[lane + 32 * q4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) reinterpret_cast<uint4*>(words)[lane + 32 * q4] = v[q4];
        } else if (gzip) {
          gzip_tile_words(m, lb, a.N, rc, kbase, kind, lane, words);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int w = 0; w < 4; ++w)
              words[w * 128 + lane + 32 * i] = tile_word(m, gzip, lb, a.N, rc[i], kbase, kind, cnt, w);
        }
        mbar_arrive(&bar[B_MF + slot]);  // release: the words above are visible to the waiter
      }
      if (!ok) break;
      if (more) fetch_entries();  // the next list's head has arrived by now
      g += wl.n;
    }
  } else if (warp >= 2 && warp < 2 + kSoftmaxThreads / 32) {
    // --------------------------------------------------------------- softmax
    const int half = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;
    int g = 0, k = 0;
    bool ok = true;
    int n_next = blockIdx.x < n_items ? item_tiles(m, blockIdx.x, T, a.Hq, a.Bt) : 0;
    // Every tcgen05.ld/st below is warp-collective: the branches around them
    // are made warp-uniform with __all_sync / __any_sync.
    for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x, ++k) {
      const Item itm(idx, T, a.Hq, a.Bt);
      const int n = n_next;
      n_next = idx + (int)gridDim.x < n_items ? item_tiles(m, idx + gridDim.x, T, a.Hq, a.Bt) : 0;
      const uint32_t ob = kTmemO + (uint32_t)((k % L::kOBufs) * 2 * D);  // this item's O
      float m_run = -INFINITY, l_run = 0.f;
      for (int it = 0; it < n; ++it) {
        const int gq = g + it, s = gq & 1, slot = gq % kMaskSlots;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bar[B_SF + s], (gq >> 1) & 1, abort, st, 20) &&
                            mbar_wait(&bar[B_MF + slot], (gq / kMaskSlots) & 1, abort, st, 24))) {
          ok = false;
          break;
        }
        tc_fence_after();
        __syncwarp();  // tcgen05.ld is warp-collective (.sync.aligned)
        float x[64];
        tmem_ld32(lane_addr + s * 128 + half * 64, x);
        tmem_ld32(lane_addr + s * 128 + half * 64 + 32, x + 32);
        const uint32_t* words = mwords + slot * (kMaskSlotBytes / 4);
        const uint32_t mw0 = words[(2 * half) * 128 + r], mw1 = words[(2 * half + 1) * 128 + r];
        mbar_arrive(&bar[B_ME + slot]);
        tmem_wait_ld();
        // scores stay unscaled here; the scale is folded into the exponent
        if ((mw0 & mw1) != 0xffffffffu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = ((mw0 >> i) & 1u) ? x[i] : -INFINITY;
            x[32 + i] = ((mw1 >> i) & 1u) ? x[32 + i] : -INFINITY;
          }
        }
        // row max of the 64 scores with three-input max: 21 + 7 + 3 + 1
        float t[21], u[7];
#pragma unroll
        for (int i = 0; i < 21; ++i) t[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
#pragma unroll
        for (int i = 0; i < 7; ++i) u[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
        const float tmax = fmax3(fmax3(u[0], u[1], u[2]), fmax3(u[3], u[4], u[5]),
                                 fmaxf(u[6], x[63]));
        const float m_new = fmaxf(m_run, tmax * sl2);  // scale > 0 keeps the order
        const bool resc = m_new > m_run + 8.f;          // true on the first finite max
        const float m_use = resc ? m_new : m_run;
        uint32_t pk[32];
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // a warp whose 32 rows see none of this half's keys (pair mode: a query
        // block that does not list a visited key block) skips the exponentials
        const bool warp_masked = __all_sync(0xffffffffu, (mw0 | mw1) == 0u);
        if (m_use == -INFINITY || warp_masked) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        } else {
          // pairs in packed fp32 arithmetic; three of every eight pairs take
          // 2^x on the FMA pipe (polynomial), the rest on the special-function
          // unit, whose 16 results per clock and SM bound this loop otherwise
          const float2 sc = make_float2(sl2, sl2), nm = make_float2(-m_use, -m_use);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 e = ffma2(make_float2(x[2 * i], x[2 * i + 1]), sc, nm);
            float2 p;
            if ((i & 7) >= (D == 64 ? SA_FWD64_POLY_FROM : SA_FWD128_POLY_FROM)) {
              p = exp2_poly2(e);
            } else {
              p.x = ex2(e.x);
              p.y = ex2(e.y);
            }
            sum2[i & 1] = fadd2(sum2[i & 1], p);
            pk[i] = pack_bf16(p.x, p.y);
          }
        }
        const float rowsum = (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
        const float alpha = !resc ? 1.f : (m_run == -INFINITY ? 0.f : ex2(m_run - m_use));
        if (it >= 1 && __any_sync(0xffffffffu, resc)) {
          // O_h was last accumulated by P V of tile gq - 1, which must be done
          // before O_h is rescaled. Only then is it waited for: the OD barrier
          // of that S buffer has completed P V(gq - 3) (issued before Q K^T(gq
          // - 1), whose S this softmax has read) and cannot have completed
          // P V(gq + 1) (no P yet), so the parity of P V(gq - 1)'s phase is
          // unambiguous. Without a rescale, P(gq) goes to the other S buffer
          // while P V(gq - 1) may still run.
          if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_OD + ((gq - 1) & 1)], ((gq - 1) >> 1) & 1,
                                                  abort, st, 21))) {
            ok = false;
            break;
          }
          // the whole warp takes part; rows that keep their max use alpha = 1
          tc_fence_after();
          __syncwarp();
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            tmem_ld32(lane_addr + ob + half * D + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(lane_addr + ob + half * D + cc * 32, o);
          }
        }
        l_run = l_run * alpha + rowsum;
        m_run = m_use;
        // P (bf16 pairs) over the first 32 of this half's S columns, already read
        __syncwarp();
        tmem_st32(lane_addr + s * 128 + half * 64, reinterpret_cast<const float*>(pk));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[B_PF + s]);
      }
      if (!ok) break;
      // hand (max, sum) to the epilogue warps; the slot of this item's parity
      // was last read by the epilogue of item k - 2
      if (k >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar[B_OF + (k & 1)], ((k - 2) >> 1) & 1,
                                                        abort, st, 23)))
        break;
      ml[((k & 1) * 2 + half) * 128 + r] = make_float2(m_run, l_run);
      mbar_arrive(&bar[B_ML + (k & 1)]);
      g += n;
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiThreads / 32) {
    // ------------------------------------------------------------ epilogue
    // Thread r owns output row r (TMEM lane r): once every MMA of the item is
    // done and both softmax halves have left (max, sum), it merges
    // O = (2^(m_0-m) O_0 + 2^(m_1-m) O_1) / (2^(m_0-m) l_0 + 2^(m_1-m) l_1)
    // and stores O and LSE, while the softmax warps already work on the next
    // item.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    int k = 0;
    int n_next = blockIdx.x < n_items ? item_tiles(m, blockIdx.x, T, a.Hq, a.Bt) : 0;
    for (int idx = blockIdx.x; idx < n_items; idx += gridDim.x, ++k) {
      const Item itm(idx, T, a.Hq, a.Bt);
      const int n = n_next;
      n_next = idx + (int)gridDim.x < n_items ? item_tiles(m, idx + gridDim.x, T, a.Hq, a.Bt) : 0;
      // query position of this row (pair mode: rows 0-63 are query block qa,
      // rows 64-127 block qb, which may not exist)
      int p = itm.I * kTile + r;
      bool row_in = true;
      if (m.pair) {
        const uint32_t pq = (uint32_t)m.pair_q[list_of(m, itm.bt, itm.h) * m.P + itm.I];
        const int qb = (int)(pq >> 16);
        p = r < 64 ? (int)(pq & 0xffff) * 64 + r : qb * 64 + (r - 64);
        row_in = r < 64 || qb != 0xffff;
      }
      const bool row_ok = row_in && p < a.N;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_ML + (k & 1)], (k >> 1) & 1, abort, st, 25) &&
                                       mbar_wait(&bar[B_OI + (k & 1)], (k >> 1) & 1, abort, st, 22)))
        break;
      const float2 h0 = ml[((k & 1) * 2 + 0) * 128 + r], h1 = ml[((k & 1) * 2 + 1) * 128 + r];
      const float mm = fmaxf(h0.x, h1.x);
      const float a0 = h0.x == -INFINITY ? 0.f : ex2(h0.x - mm);
      const float a1 = h1.x == -INFINITY ? 0.f : ex2(h1.x - mm);
      const float l = h0.y * a0 + h1.y * a1;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float c0 = a0 * inv, c1 = a1 * inv;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + itm.bt * a.os[0] +
                            (int64_t)p * a.os[1] + (int64_t)itm.h * a.os[2];
      if (n > 0) {
        const uint32_t ob = kTmemO + (uint32_t)((k % L::kOBufs) * 2 * D);
        tc_fence_after();
        __syncwarp();
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          float o0[32], o1[32];
          tmem_ld32(lane_addr + ob + cc * 32, o0);  // all lanes: collective
          tmem_ld32(lane_addr + ob + D + cc * 32, o1);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 wv;
              wv.x = pack_bf16(o0[v * 8 + 0] * c0 + o1[v * 8 + 0] * c1,
                               o0[v * 8 + 1] * c0 + o1[v * 8 + 1] * c1);
              wv.y = pack_bf16(o0[v * 8 + 2] * c0 + o1[v * 8 + 2] * c1,
                               o0[v * 8 + 3] * c0 + o1[v * 8 + 3] * c1);
              wv.z = pack_bf16(o0[v * 8 + 4] * c0 + o1[v * 8 + 4] * c1,
                               o0[v * 8 + 5] * c0 + o1[v * 8 + 5] * c1);
              wv.w = pack_bf16(o0[v * 8 + 6] * c0 + o1[v * 8 + 6] * c1,
                               o0[v * 8 + 7] * c0 + o1[v * 8 + 7] * c1);
              *reinterpret_cast<uint4*>(orow + cc * 32 + v * 8) = wv;
            }
          }
        }
      } else if (row_ok) {
        for (int cc = 0; cc < D; cc += 8)
          *reinterpret_cast<uint4*>(orow + cc) = make_uint4(0u, 0u, 0u, 0u);
      }
      tc_fence_before();
      mbar_arrive(&bar[B_OF + (k & 1)]);  // O and (max, sum) of this parity may be reused
      if (row_ok)
        a.lse[((int64_t)itm.bt * a.Hq + itm.h) * a.N + p] =
            l > 0.f ? (mm + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// -------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [Bt, N, H, d] of `ebytes`-byte elements with element strides {batch, seq,
// head}; box box_d x 1 x rows x 1, 128-byte swizzle (box_d * ebytes <= 128).
bool make_map_4d(CUtensorMap* map, CUtensorMapDataType dtype, int ebytes, const void* base, int d,
                 int H, int N, int Bt, const int64_t* s, int box_d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t sh = s[2] > 0 ? s[2] : d, sn = s[1];
  const int64_t sbat = (Bt > 1) ? s[0] : sn * N;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)Bt};
  cuuint64_t strides[3] = {(cuuint64_t)(sh * ebytes), (cuuint64_t)(sn * ebytes),
                           (cuuint64_t)(sbat * ebytes)};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 with a box of 64 x 1 x rows x 1.
bool make_tile_map_box(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                       const int64_t* s, int rows) {
  return make_map_4d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d, H, N, Bt, s, 64, rows);
}

bool make_tile_map(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                   const int64_t* s) {
  return make_tile_map_box(map, base, d, H, N, Bt, s, kTile);
}

// Gist mode: copies the K and V rows of every sink / gist (far_idx, logical
// order) into dense [Bt, N, Hkv, D] buffers, and zero-fills the rest of the
// last 128-row tile so that masked columns multiply finite values.
template <int D>
__global__ void __launch_bounds__(256) gist_gather_kernel(AttnArgs a, MaskArgs m,
                                                          __nv_bfloat16* kc, __nv_bfloat16* vc) {
  const int f = blockIdx.x * 8 + (threadIdx.x >> 5), bt = blockIdx.y, lane = threadIdx.x & 31;
  const int nf = m.far_ptr[m.T];
  const int nf_pad = (nf + kTile - 1) / kTile * kTile;
  if (f >= nf_pad || f >= a.N) return;
  const int64_t row = (int64_t)a.Hkv * D;  // elements per compacted row
  __nv_bfloat16* dk = kc + ((int64_t)bt * a.N + f) * row;
  __nv_bfloat16* dv = vc + ((int64_t)bt * a.N + f) * row;
  for (int x = lane * 8; x < row; x += 32 * 8) {
    const int hh = x / D, c = x % D;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (f < nf) {
      const int src = m.far_idx[f];
      kv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.k) +
                                           bt * a.ks[0] + (int64_t)src * a.ks[1] + hh * a.ks[2] + c);
      vv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.v) +
                                           bt * a.vs[0] + (int64_t)src * a.vs[1] + hh * a.vs[2] + c);
    }
    *reinterpret_cast<uint4*>(dk + x) = kv;
    *reinterpret_cast<uint4*>(dv + x) = vv;
  }
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Gist mode: the element masks of every (query tile I, near key tile J) pair,
// the same for every head ("UniGist ...", Approach: a query sees the sinks and
// the gists that are not in its future, and the raw tokens of its window; in
// the coarse layout of "A Silver Bullet or a Compromise ...", sections 2 and
// 6, the raw tokens of its segment instead). Block (I, J - I + nt - 1),
// thread r = query row; bit c of word w tells whether key 128 J + 32 w + c is
// visible from row 128 I + r. With d = li - lj (logical positions) the rule is
// (unsigned)d < lim, lim = gist_reach(lj).
__global__ void __launch_bounds__(128) gist_near_mask_kernel(MaskArgs m, int N, int nt_count,
                                                             uint32_t* near) {
  const int I = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int J = I - (nt_count - 1) + nt;
  if (J < 0) return;  // not a key tile of this query tile
  __shared__ int lj_s[kTile];
  __shared__ uint32_t lim_s[kTile];
  const int kq = J * kTile + r;
  int lj = 0;
  uint32_t lim = 0u;  // no key: never visible
  if (kq < N) {
    lj = m.perm[kq];
    const bool always = lj < m.sinks || ((m.gist_bits[lj >> 5] >> (lj & 31)) & 1u);
    lim = gist_reach(always, lj, m.sinks, m.window, m.period);
  }
  lj_s[r] = lj;
  lim_s[r] = lim;
  __syncthreads();
  const int p = I * kTile + r;
  const int li = p < N ? m.perm[p] : 0;
  uint32_t* out = near + ((int64_t)I * nt_count + nt) * 512;
#pragma unroll 1
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0u;
#pragma unroll 8
    for (int j = 0; j < 32; ++j)
      word |= ((uint32_t)(li - lj_s[32 * w + j]) < lim_s[32 * w + j] ? 1u : 0u) << j;
    out[w * 128 + r] = p < N ? word : 0u;
  }
}

// Pair mode (gzip, b = 64): the query blocks of each (sequence, class) list
// are paired and every pair gets the ascending union of its two key-block
// lists, two key blocks per visit ("Gzip-guided sparse attention ...", Core
// equations: a query block sees exactly the key blocks of its mask row).
// Blocks whose row holds more than the diagonal (literal class) or more than
// the local window (hybrid class) are "long"; short blocks are paired first
// and long ones after, both ascending, so that two long rows, which share
// most of their literal key blocks, are merged with each other. Local lists
// pair neighbours. The pairing only schedules work: every (query block, key
// block) pair of the mask is visited exactly once whatever it is. One CTA per
// list; pair k is handled by thread k.
constexpr int kPairStageWords = 8192;  // bit rows staged in shared memory up to 32 KB

__global__ void __launch_bounds__(512) gzip_pair_kernel(MaskArgs m, int32_t* pair_q,
                                                        int32_t* pair_ptr, int32_t* visits) {
  extern __shared__ int32_t psh[];
  const int l = blockIdx.x, cls = l % 3;
  const int B = m.B, W = m.words, P = (B + 1) / 2;
  int32_t* order = psh;           // [B]   pair order of the query blocks
  int32_t* longs = psh + B;       // [B]   inclusive count of long rows
  int32_t* vis = psh + 2 * B;     // [P]   inclusive count of visits
  // the list's bit rows, staged in shared memory when the launch gave room
  const uint32_t* bits = m.bits + (int64_t)l * B * W;
  if (kPairStageWords > 0 && B * W <= kPairStageWords) {
    uint32_t* staged = reinterpret_cast<uint32_t*>(psh + 2 * B + P);
    for (int x = threadIdx.x; x < B * W; x += blockDim.x) staged[x] = bits[x];
    bits = staged;
    __syncthreads();
  }
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    int len = 0;
    for (int w = 0; w < W; ++w) len += __popc(bits[(int64_t)i * W + w]);
    const int base = cls == SA_CLASS_LOCAL ? len : cls == SA_CLASS_LITERAL ? 1 : min(i, m.wb) + 1;
    longs[i] = len > base ? 1 : 0;
  }
  __syncthreads();
  block_inclusive_scan(longs, B, 0);
  const int n_long = longs[B - 1], n_short = B - n_long;
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const int before = i > 0 ? longs[i - 1] : 0, is_long = longs[i] - before;
    order[is_long ? n_short + before : i - before] = i;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < P; k += blockDim.x) {
    const uint32_t* ra = bits + (int64_t)order[2 * k] * W;
    const uint32_t* rb = 2 * k + 1 < B ? bits + (int64_t)order[2 * k + 1] * W : ra;
    int c = 0;
    for (int w = 0; w < W; ++w) c += __popc(ra[w] | rb[w]);
    vis[k] = (c + 1) / 2;
  }
  __syncthreads();
  const int64_t region = (int64_t)B * (B + 1) / 2;
  block_inclusive_scan(vis, P, (int32_t)(l * region));
  if (threadIdx.x == 0) pair_ptr[(int64_t)l * (P + 1)] = (int32_t)(l * region);
  for (int k = threadIdx.x; k < P; k += blockDim.x) {
    pair_ptr[(int64_t)l * (P + 1) + k + 1] = vis[k];
    const int qa = order[2 * k], qb = 2 * k + 1 < B ? order[2 * k + 1] : -1;
    pair_q[(int64_t)l * P + k] = qa | ((qb < 0 ? 0xffff : qb) << 16);
    const uint32_t* ra = bits + (int64_t)qa * W;
    const uint32_t* rb = qb >= 0 ? bits + (int64_t)qb * W : nullptr;
    int32_t* out = visits + (k > 0 ? vis[k - 1] : l * region);
    uint32_t cur = 0u;
    bool second = false;
    for (int w = 0; w < W; ++w) {
      const uint32_t a = ra[w], b = rb ? rb[w] : 0u;
      uint32_t u = a | b;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        const uint32_t j = (uint32_t)(32 * w + bit);
        const uint32_t sa = (a >> bit) & 1u, sb2 = (b >> bit) & 1u;
        if (!second) {
          cur = j | (sa << 24) | (sb2 << 25);
        } else {
          *out++ = (int32_t)(cur | (j << 12) | (sa << 26) | (sb2 << 27));
        }
        second = !second;
      }
    }
    if (second) *out = (int32_t)(cur | (0xfffu << 12));
  }
}

// Workspace of pair mode: pair_q, pair_ptr and visits of every list.
size_t fwd_pair_workspace(int Bt, int B) {
  const size_t lists = (size_t)Bt * 3, P = (size_t)(B + 1) / 2;
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  return r256(lists * P * 4) + r256(lists * (P + 1) * 4) + r256(lists * ((size_t)B * (B + 1) / 2) * 4);
}

// The same masks transposed for the key-major backward: block (I, J - I + nt
// - 1), thread r = key row; bit c of word w tells whether key 128 J + r is
// visible from query 128 I + 32 w + c.
__global__ void __launch_bounds__(128) gist_near_mask_t_kernel(MaskArgs m, int N, int nt_count,
                                                               uint32_t* near_t) {
  const int I = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int J = I - (nt_count - 1) + nt;
  if (J < 0) return;  // not a key tile of this query tile
  __shared__ int li_s[kTile];
  __shared__ int ok_s[kTile];
  const int p = I * kTile + r;
  li_s[r] = p < N ? m.perm[p] : 0;
  ok_s[r] = p < N;
  __syncthreads();
  const int kq = J * kTile + r;
  int lj = 0;
  uint32_t lim = 0u;  // no key: never visible
  if (kq < N) {
    lj = m.perm[kq];
    const bool always = lj < m.sinks || ((m.gist_bits[lj >> 5] >> (lj & 31)) & 1u);
    lim = gist_reach(always, lj, m.sinks, m.window, m.period);
  }
  uint32_t* out = near_t + ((int64_t)I * nt_count + nt) * 512;
#pragma unroll 1
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0u;
#pragma unroll 8
    for (int c = 0; c < 32; ++c)
      word |= (ok_s[32 * w + c] && (uint32_t)(li_s[32 * w + c] - lj) < lim ? 1u : 0u) << c;
    out[w * 128 + r] = word;
  }
}

// Gist pre-passes shared by the forward and the backward: the compacted sink /
// gist K and V (`compact`, 2 * Bt * N * Hkv * d bf16), the near-tile masks
// (`near`, T * gist_near_tiles(window, period) * 2048 bytes) and, for the key-major
// backward, their transpose (`near_t`, same size, or null).
template <int D>
static cudaError_t gist_prepass(const AttnArgs& a, const MaskArgs& m, void* compact, void* near,
                                void* near_t, cudaStream_t s) {
  const int64_t row = (int64_t)a.Hkv * D;
  __nv_bfloat16* kc = static_cast<__nv_bfloat16*>(compact);
  __nv_bfloat16* vc = kc + (int64_t)a.Bt * a.N * row;
  gist_gather_kernel<D><<<dim3((a.N + 7) / 8, a.Bt), 256, 0, s>>>(a, m, kc, vc);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nt = gist_near_tiles(m.window, m.period);
  gist_near_mask_kernel<<<dim3(m.T, nt), kTile, 0, s>>>(m, a.N, nt, static_cast<uint32_t*>(near));
  e = cudaGetLastError();
  if (e != cudaSuccess || near_t == nullptr) return e;
  gist_near_mask_t_kernel<<<dim3(m.T, nt), kTile, 0, s>>>(m, a.N, nt, static_cast<uint32_t*>(near_t));
  return cudaGetLastError();
}

cudaError_t launch_gist_prepass(int d, const AttnArgs& a, const MaskArgs& m, void* compact,
                                void* near, void* near_t, cudaStream_t s) {
  if (d == 64) return gist_prepass<64>(a, m, compact, near, near_t, s);
  if (d == 128) return gist_prepass<128>(a, m, compact, near, near_t, s);
  return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t fwd_tc_launch(const AttnArgs& a, const MaskArgs& m_in, void* compact,
                                 void* near, void* pair_ws, cudaStream_t s) {
  FwdTcParams P;
  memset(&P, 0, sizeof(P));
  MaskArgs m = m_in;
  if (pair_ws != nullptr) {
    // pair mode (gzip, b = 64): pairs and merged visit lists, then 64-row boxes
    const int lists = a.Bt * 3, np = (m.B + 1) / 2;
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    char* w = static_cast<char*>(pair_ws);
    int32_t* pair_q = reinterpret_cast<int32_t*>(w);
    int32_t* pair_ptr = reinterpret_cast<int32_t*>(w + r256((size_t)lists * np * 4));
    int32_t* visits = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(pair_ptr) +
                                                 r256((size_t)lists * (np + 1) * 4));
    const int stage = m.B * m.words <= kPairStageWords ? m.B * m.words : 0;
    gzip_pair_kernel<<<lists, 512, (size_t)(2 * m.B + np + stage) * 4, s>>>(m, pair_q, pair_ptr,
                                                                         visits);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    m.pair = 1;
    m.P = np;
    m.pair_q = pair_q;
    m.pair_ptr = pair_ptr;
    m.visits = visits;
    if (!make_tile_map_box(&P.tmq64, a.q, D, a.Hq, a.N, a.Bt, a.qs, 64) ||
        !make_tile_map_box(&P.tmk64, a.k, D, a.Hkv, a.N, a.Bt, a.ks, 64) ||
        !make_tile_map_box(&P.tmv64, a.v, D, a.Hkv, a.N, a.Bt, a.vs, 64))
      return cudaErrorInvalidValue;
  }
  if (!make_tile_map(&P.tmq, a.q, D, a.Hq, a.N, a.Bt, a.qs) ||
      !make_tile_map(&P.tmk, a.k, D, a.Hkv, a.N, a.Bt, a.ks) ||
      !make_tile_map(&P.tmv, a.v, D, a.Hkv, a.N, a.Bt, a.vs))
    return cudaErrorInvalidValue;
  P.tmkc = P.tmk;
  P.tmvc = P.tmv;
  if (m.kind == SA_MASK_GIST) {
    const int64_t row = (int64_t)a.Hkv * D;
    __nv_bfloat16* kc = static_cast<__nv_bfloat16*>(compact);
    __nv_bfloat16* vc = kc + (int64_t)a.Bt * a.N * row;
    const int64_t cs[3] = {(int64_t)a.N * row, row, D};
    if (!make_tile_map(&P.tmkc, kc, D, a.Hkv, a.N, a.Bt, cs) ||
        !make_tile_map(&P.tmvc, vc, D, a.Hkv, a.N, a.Bt, cs))
      return cudaErrorInvalidValue;
    cudaError_t e = gist_prepass<D>(a, m, compact, near, nullptr, s);
    if (e != cudaSuccess) return e;
    P.near = static_cast<const uint32_t*>(near);
    P.near_nt = gist_near_tiles(m.window, m.period);
  }
  P.a = a;
  P.m = m;
  const int bytes = (int)FwdLayout<D>::bytes;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (TMEM and shared memory admit one per SM)
  const int items = (m.pair ? m.P : m.T) * a.Hq * a.Bt;
  const int grid = items < sm_count() ? items : sm_count();
  fwd_tc_kernel<D><<<dim3(grid), kThreads, bytes, s>>>(P);
  return cudaGetLastError();
}

// Gist mode only: `compact`, 2 * Bt * N * Hkv * d bf16 of workspace; `near`,
// T * gist_near_tiles(window, period) * 2048 bytes. Gzip with b = 64: `pair_ws`,
// fwd_pair_workspace(Bt, B) bytes, selects pair mode (null: 128-row tiles).
cudaError_t launch_fwd_tc(int d, const AttnArgs& a, const MaskArgs& m, void* compact, void* near,
                          void* pair_ws, cudaStream_t s) {
  if (d == 64) return fwd_tc_launch<64>(a, m, compact, near, pair_ws, s);
  if (d == 128) return fwd_tc_launch<128>(a, m, compact, near, pair_ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace sa
