// Block-sparse attention backward on the 5th-generation tensor cores (sm_100a).
//
// Gradients of the masked softmax attention for an upstream dO:
//   P = exp(s - LSE), dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
//   dS = P * (dP - D), dQ = dS K * scale, dK = dS^T Q * scale
// (the training use of the method: "UniGist ...", Approach, one-pass training;
// forward/backward latency is a metric that page names).
//
// This key-major pass computes dK and dV; dQ comes from the query-major pass
// (attn_dq_sm100.cu), which recomputes S and dP instead of adding partial dQ
// tiles into global memory. A work item is one (128-key tile J, KV head,
// sequence); its visits are every query tile I that lists J, for every query
// head of the KV group (the transposed tile lists). The kernel is persistent:
// one CTA per SM takes items from a run-time queue in (sequence, KV head)
// order, early key tiles (the longest lists) first within a head, so that the
// CTAs running together read the query tiles of one head through L2. TMEM lanes are key rows:
//   S^T = K_J Q_I^T (columns 0-127); each half h of the compute warps writes
//     its bf16 P^T over the first 32 of its 64 S columns
//   dP^T = V_J dO_I^T (columns 128-255)
//   dV += P^T dO_I (A = P^T from TMEM), dK += dS^T Q_I (TMEM accumulators)
// dS^T goes to shared memory: it is the A operand of dK.
//
// Roles (352 threads): warp 0 TMA (K, V per item; Q, LSE, D double-buffered;
// dO single-buffered), warp 1 one thread issuing tcgen05.mma, warps 2-9 two
// groups of four compute warps (group h owns query columns [64h, 64h + 64) of
// every tile; the backward needs no cross-column reduction since P comes from
// the stored LSE), warp 10 the visit list and the visibility of each tile's
// (key, query) pairs as 4 x 128 bit words in a shared-memory ring. Every wait
// is bounded; on timeout the device status word is set and all roles leave
// after draining their copies and MMAs.
#include <cuda.h>

#include "attn_mask.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

struct BwdTcParams {
  CUtensorMap tmq, tmk, tmv, tmdo;
  CUtensorMap tmkc, tmvc;  // gist mode: sinks + gists compacted in logical order
  const uint32_t* near_t;  // gist mode: transposed near-tile masks
  int near_nt;
  float* dkf;              // gist mode: dK, dV of the compacted keys from far queries
  float* dvf;
  AttnArgs a;
  MaskArgs m;
  const float* lse2;   // [Bt, Hq, Tpad] LSE * log2(e), +inf past N
  const float* delta;  // [Bt, Hq, Tpad] rowsum(dO * O), 0 past N
  int Tpad;            // T * 128
};

namespace bwd {

constexpr int kSlots = 8;             // mask ring depth (visits the mask warp may run ahead)
constexpr uint32_t kSlotBytes = 2048;  // [4 words][128 key rows]
constexpr int kCompute = 256;          // compute threads
constexpr int kThreads = 64 + kCompute + 32;
constexpr int kMaskWarp = 10;

template <int D>
struct Layout {
  static constexpr uint32_t kT = 128 * D * 2;     // a 128 x D bf16 tile
  static constexpr uint32_t kP = 128 * 128 * 2;   // a 128 x 128 bf16 tile
  static constexpr uint32_t kAtom = 128 * 128;    // [128 rows][64 bf16] swizzle atom
  static constexpr uint32_t k = 0;
  static constexpr uint32_t v = kT;
  static constexpr uint32_t q = 2 * kT;           // 2 stages
  static constexpr uint32_t dO = 4 * kT;          // 2 stages
  static constexpr uint32_t rowv = 6 * kT;        // [2 stages][lse2 128 | delta 128] fp32
  static constexpr uint32_t mask = rowv + 2 * 1024;
  static constexpr uint32_t hdr = mask + kSlots * kSlotBytes;  // the item ring's slots
  static constexpr uint32_t bars = hdr + 64;
  static constexpr uint32_t bytes = bars + 512 + 1024;
};

// mbarriers. KVF/KVE: K, V of the item loaded / no longer read. QF/QE: Q
// stage (with its LSE and D rows) full / free. DOF/DOE: dO stage full / free.
// SF, DPF: S^T, dP^T in TMEM. PF1: P^T written to TMEM over S^T; PF2: dS^T
// written to TMEM over dP^T. MF/ME: mask slot full / read. OI: every MMA of
// the item done. OF: dV and dK of the item read out. DRAIN: all MMAs done.
enum {
  B_KVF = 0, B_KVE = 1, B_QF = 2, B_QE = 4, B_DOF = 6, B_DOE = 8, B_SF = 10, B_DPF = 11,
  B_PF1 = 12, B_PF2 = 13, B_OI = 14, B_MF = 16, B_ME = B_MF + kSlots, B_OF = B_ME + kSlots,
  B_DRAIN = B_OF + 1, B_IQF = B_DRAIN + 1, B_IQE = B_IQF + kItemRing, kNumBars = B_IQE + kItemRing
};
// consumers of each item of the run-time queue: the MMA thread, the mask warp
// and the eight compute warps
constexpr int kQueueConsumers = 1 + 1 + kCompute / 32;

constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256;  // dK at 256 + D

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Item -> (key tile J, KV head, sequence): early key tiles first. The gist
// layout has two kinds of items: "far" items (tile J of the sinks and gists
// compacted in logical order, visited by every query tile whose near tiles
// start past them) first, then "near" items (physical key tile J, visited by
// the query tiles that hold it among their near tiles).
struct Item {
  int J, hk, bt, far;
  __device__ Item(int idx, int Hkv, int Bt, int T, bool gist) {
    // (sequence, KV head) outermost, so that the CTAs running together share the
    // query tiles of one head through L2; then the far items, then the key tiles
    const int per = (gist ? 2 : 1) * T;
    const int hb = idx / per, local = idx % per;
    hk = hb % Hkv;
    bt = hb / Hkv;
    far = gist && local < T;
    J = far || !gist ? local : local - T;
  }
};

// The visits of one item, for every query head of the KV group: gzip, the
// transposed tile list; gist near items, the query tiles I >= J whose near
// tiles start at or below J (I = J .. J + c - 1: the start is non-decreasing
// in I and at most nt - 1 tiles below it); gist far items, the query tiles
// whose far-key prefix reaches past 128 J (a suffix of the query tiles, found
// by bisection: far_ptr and the near start are non-decreasing), visited from
// the last tile down.
struct Visits {
  int n, cnt, i0;
  __device__ void init(const MaskArgs& m, const Item& itm, int rep, int nt) {
    if (m.kind == SA_MASK_GIST) {
      if (itm.far) {
        int lo = 0, hi = m.T;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (m.far_ptr[gist_near_lo(mid, m.sinks, m.window, m.period)] > itm.J * kTile) hi = mid;
          else lo = mid + 1;
        }
        i0 = lo;
        cnt = m.T - lo;
      } else {
        i0 = itm.J;
        const int last = min(m.T - 1, itm.J + nt - 1);
        cnt = 1;
        while (itm.J + cnt <= last && gist_near_lo(itm.J + cnt, m.sinks, m.window, m.period) <= itm.J)
          ++cnt;
      }
      n = rep * cnt;
      return;
    }
    n = 0;
    for (int r = 0; r < rep; ++r) {
      const int list = list_of(m, itm.bt, itm.hk * rep + r);
      n += m.tcp[list * (m.T + 1) + itm.J + 1] - m.tcp[list * (m.T + 1) + itm.J];
    }
  }
  __device__ void entry(const MaskArgs& m, const Item& itm, int rep, int it, int& h, int& I,
                        int& kind) const {
    if (m.kind == SA_MASK_GIST) {
      if (itm.far) {
        // far items: query tiles from the last one down, the group's heads
        // per tile. Every far item's suffix ends at the last query tile, so
        // the far items that run together start on the same tiles and read
        // their Q and dO rows from L2 while they stay in step.
        I = m.T - 1 - it / rep;
        h = itm.hk * rep + it % rep;
      } else {
        h = itm.hk * rep + it / cnt;
        I = i0 + it % cnt;
      }
      kind = SA_TILE_MASKED;
      return;
    }
    for (int r = 0; r < rep; ++r) {
      const int list = list_of(m, itm.bt, itm.hk * rep + r);
      const int e0 = m.tcp[list * (m.T + 1) + itm.J];
      const int c = m.tcp[list * (m.T + 1) + itm.J + 1] - e0;
      if (it < c) {
        h = itm.hk * rep + r;
        I = m.trow[e0 + it];
        kind = m.tkind_t[e0 + it];
        return;
      }
      it -= c;
    }
    h = itm.hk * rep;
    I = 0;
    kind = SA_TILE_MASKED;
  }
};

// Visibility of query columns [32w, 32w + 32) of tile (I, J) from key row kq
// ("Gzip-guided sparse attention ...", Core equations: the block mask, then the
// causal cut q >= kq), with the key and query ranges cut at N.
__device__ __forceinline__ uint32_t key_word(const MaskArgs& m, int list, int lb, int N, int kq,
                                             int q0, int kind, int w) {
  if (kq >= N) return 0u;
  const int c0 = q0 + 32 * w;
  const uint32_t in_range = prefix_bits(N - c0);
  const uint32_t causal = ~prefix_bits(kq - c0);  // columns with q >= kq
  if (kind == SA_TILE_FULL) return in_range & causal;
  const int kb = kq / m.b;
  const uint32_t* rows = m.bits + (int64_t)list * m.B * m.words;
  uint32_t blk;
  if (m.b >= kTile || lb >= 5) {
    const int qb = min(m.B - 1, m.b >= kTile ? q0 / m.b : c0 >> lb);
    blk = ((rows[(int64_t)qb * m.words + (kb >> 5)] >> (kb & 31)) & 1u) ? 0xffffffffu : 0u;
  } else {
    // 32 >> lb query blocks per word: one bit of each block row
    const int nb = 32 >> lb, run = 1 << lb;
    blk = 0u;
    for (int t = 0; t < nb; ++t) {
      const int qb = min(m.B - 1, (c0 >> lb) + t);
      if ((rows[(int64_t)qb * m.words + (kb >> 5)] >> (kb & 31)) & 1u)
        blk |= (uint32_t)((1ull << run) - 1ull) << (t * run);
    }
  }
  return blk & in_range & causal;
}

}  // namespace bwd

using namespace bwd;

template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_tc_kernel(const __grid_constant__ BwdTcParams P) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + kNumBars) + 1;
  float* rowv = reinterpret_cast<float*>(smem + L::rowv);
  uint32_t* mwords = reinterpret_cast<uint32_t*>(smem + L::mask);
  int* hdr = reinterpret_cast<int*>(smem + L::hdr);

  const AttnArgs& a = P.a;
  const MaskArgs& m = P.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = m.T;
  const int rep = a.Hq / a.Hkv;
  const bool gist = m.kind == SA_MASK_GIST;
  const int n_items = (gist ? 2 : 1) * T * a.Hkv * a.Bt;
  DeviceStatus* st = a.status;

  if (threadIdx.x == 0) {
    mbar_init(&bar[B_KVF], 1);
    mbar_init(&bar[B_KVE], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_QF + s], 1);
      mbar_init(&bar[B_QE + s], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar[B_MF + s], 32);
      mbar_init(&bar[B_ME + s], kCompute);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_DOF + s], 1);
      mbar_init(&bar[B_DOE + s], 1);
    }
    mbar_init(&bar[B_SF], 1);
    mbar_init(&bar[B_DPF], 1);
    mbar_init(&bar[B_PF1], kCompute);
    mbar_init(&bar[B_PF2], kCompute);
    mbar_init(&bar[B_OF], kCompute);
    mbar_init(&bar[B_OI], 1);
    mbar_init(&bar[B_DRAIN], 1);
    for (int s = 0; s < kItemRing; ++s) {
      mbar_init(&bar[B_IQF + s], 1);
      mbar_init(&bar[B_IQE + s], kQueueConsumers);
    }
    *abort = 0;
    fence_barrier_init();
  }
  ItemQueue queue{hdr + 8, &bar[B_IQF], &bar[B_IQE],
                  reinterpret_cast<unsigned int*>(st->aux + kQueueWordDkdv)};
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------- TMA producer
      prefetch_tmap(&P.tmq);
      prefetch_tmap(&P.tmk);
      prefetch_tmap(&P.tmv);
      prefetch_tmap(&P.tmdo);
      if (gist) {
        prefetch_tmap(&P.tmkc);
        prefetch_tmap(&P.tmvc);
      }
      int g = 0, k = 0, last_q = -1, last_do = -1, last_kv = -1;
      bool ok = true;
      for (;; ++k) {
        int idx;
        if (!queue.publish(k, idx, abort, st, 106) || idx >= n_items) break;
        const Item itm(idx, a.Hkv, a.Bt, T, gist);
        Visits vis;
        vis.init(m, itm, rep, P.near_nt);
        // K and V of the previous item are no longer read
        if (k > 0 && !mbar_wait(&bar[B_KVE], (k - 1) & 1, abort, st, 100)) break;
        if (vis.n == 0) {
          // nothing to load (a far tile no query tile reaches): the phase of
          // this item completes at once, so that no load of the next item can
          // fall into it
          mbar_arrive(&bar[B_KVF]);
        } else {
          mbar_arrive_expect_tx(&bar[B_KVF], 2 * L::kT);
          for (int at = 0; at < D / 64; ++at) {
            tma_load_4d(smem + L::k + at * L::kAtom, itm.far ? &P.tmkc : &P.tmk, &bar[B_KVF],
                        at * 64, itm.hk, itm.J * kTile, itm.bt);
            tma_load_4d(smem + L::v + at * L::kAtom, itm.far ? &P.tmvc : &P.tmv, &bar[B_KVF],
                        at * 64, itm.hk, itm.J * kTile, itm.bt);
          }
        }
        last_kv = k;
        for (int it = 0; it < vis.n; ++it) {
          const int gt = g + it, s = gt & 1;
          int h, I, kind;
          vis.entry(m, itm, rep, it, h, I, kind);
          if (!mbar_wait(&bar[B_QE + s], ((gt >> 1) & 1) ^ 1, abort, st, 101)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar[B_QF + s], L::kT + 2 * 512);
          for (int at = 0; at < D / 64; ++at)
            tma_load_4d(smem + L::q + s * L::kT + at * L::kAtom, &P.tmq, &bar[B_QF + s], at * 64,
                        h, I * kTile, itm.bt);
          const int64_t ro = ((int64_t)itm.bt * a.Hq + h) * P.Tpad + (int64_t)I * kTile;
          bulk_load(rowv + s * 256, P.lse2 + ro, 512, &bar[B_QF + s]);
          bulk_load(rowv + s * 256 + 128, P.delta + ro, 512, &bar[B_QF + s]);
          last_q = gt;
          if (!mbar_wait(&bar[B_DOE + s], ((gt >> 1) & 1) ^ 1, abort, st, 102)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar[B_DOF + s], L::kT);
          for (int at = 0; at < D / 64; ++at)
            tma_load_4d(smem + L::dO + s * L::kT + at * L::kAtom, &P.tmdo, &bar[B_DOF + s], at * 64, h,
                        I * kTile, itm.bt);
          last_do = gt;
        }
        if (ok) count_tiles(st, CNT_DKDV_VISITS, vis.n);
        g += vis.n;
        if (!ok) break;
      }
      // every copy this CTA started must land before the CTA may exit
      volatile int no_abort = 0;
      if (last_kv >= 0) mbar_wait(&bar[B_KVF], last_kv & 1, &no_abort, nullptr, 103);
      for (int s = 0; s < 2; ++s)
        if (last_q >= s) {
          const int gs = last_q - ((last_q - s) & 1);
          mbar_wait(&bar[B_QF + s], (gs >> 1) & 1, &no_abort, nullptr, 104);
        }
      for (int s = 0; s < 2; ++s)
        if (last_do >= s) {
          const int gs = last_do - ((last_do - s) & 1);
          mbar_wait(&bar[B_DOF + s], (gs >> 1) & 1, &no_abort, nullptr, 105);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdAcc = idesc_bf16_f32(128, D, false, true);  // P^T dO, dS^T Q
      int g = 0, k = 0;
      bool ok = true;
      // Per visit gt the order is: dV(gt) once P^T is written, then S^T(gt + 1)
      // (its S columns held P^T(gt), read by the dV just issued: tcgen05.mma ops
      // of one thread run in order), dK(gt) once dS^T is written, then
      // dP^T(gt + 1) (its columns held dS^T(gt), read by the dK just issued).
      // dO has two stages, so dO(gt + 1) loads while visit gt runs.
      auto issue_s = [&](int gt) -> bool {  // S^T = K Q^T
        const int s = gt & 1;
        if (!mbar_wait(&bar[B_QF + s], (gt >> 1) & 1, abort, st, 111)) return false;
        tc_fence_after();
        const uint32_t qb = sb + L::q + s * L::kT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + kColS, smem_desc_sw128(sb + L::k + off, 16, 1024),
                   smem_desc_sw128(qb + off, 16, 1024), kIdS, kk > 0);
        }
        mma_commit(&bar[B_SF]);
        return true;
      };
      auto issue_dp = [&](int gt) -> bool {  // dP^T = V dO^T
        const int d = gt & 1;
        if (!mbar_wait(&bar[B_DOF + d], (gt >> 1) & 1, abort, st, 112)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + kColDP, smem_desc_sw128(sb + L::v + off, 16, 1024),
                   smem_desc_sw128(sb + L::dO + d * L::kT + off, 16, 1024), kIdS, kk > 0);
        }
        mma_commit(&bar[B_DPF]);
        return true;
      };
      for (;; ++k) {
        int idx;
        if (!queue.take(k, idx, abort, st, 118)) break;
        queue.release(k);
        if (idx >= n_items) break;
        const Item itm(idx, a.Hkv, a.Bt, T, gist);
        Visits vis;
        vis.init(m, itm, rep, P.near_nt);
        // every item's K/V phase is waited for, empty items included, so that the
        // phases of the producer and this thread never drift apart
        if (!mbar_wait(&bar[B_KVF], k & 1, abort, st, 110)) break;
        if (vis.n > 0 && (!issue_s(g) || !issue_dp(g))) break;
        for (int it = 0; it < vis.n; ++it) {
          const int gt = g + it, s = gt & 1;
          const bool more = it + 1 < vis.n;
          // P^T in TMEM: dV += P^T dO (the previous item's dV, dK read out first)
          if (!mbar_wait(&bar[B_PF1], gt & 1, abort, st, 114) ||
              (it == 0 && k > 0 && !mbar_wait(&bar[B_OF], (k - 1) & 1, abort, st, 115))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // K = 128 queries
            const uint32_t pa = tmem + kColS + (kk >> 2) * 64 + (kk & 3) * 8;
            mma_bf16_ts(tmem + kColDV, pa,
                        smem_desc_sw128(sb + L::dO + s * L::kT + kk * 2048, L::kAtom, 1024), kIdAcc,
                        (it > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_DOE + s]);
          if (more && !issue_s(gt + 1)) {
            ok = false;
            break;
          }
          // dS^T in TMEM (over dP^T): dK += dS^T Q
          if (!mbar_wait(&bar[B_PF2], gt & 1, abort, st, 117)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qb = sb + L::q + s * L::kT;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // K = 128 queries
            const uint32_t da = tmem + kColDP + (kk >> 2) * 64 + (kk & 3) * 8;
            mma_bf16_ts(tmem + kColDV + D, da, smem_desc_sw128(qb + kk * 2048, L::kAtom, 1024),
                        kIdAcc, (it > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_QE + s]);
          if (more && !issue_dp(gt + 1)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        // an item without visits still takes its turn of OF and OI, so that
        // OI never runs two phases ahead of the compute warps
        if (vis.n == 0 && k > 0 && !mbar_wait(&bar[B_OF], (k - 1) & 1, abort, st, 115)) break;
        mma_commit(&bar[B_KVE]);  // every MMA of this item reading K and V is issued
        mma_commit(&bar[B_OI]);   // dK and dV of the item complete
        g += vis.n;
      }
      mma_commit(&bar[B_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[B_DRAIN], 0, &no_abort, nullptr, 116);
    }
  } else if (warp == kMaskWarp) {
    // ------------------------------------------------- visits and their masks
    const int lb = !gist && m.b < kTile ? __ffs(m.b) - 1 : 0;  // b < 128 is a power of two
    int g = 0;
    for (int k = 0;; ++k) {
      int idx;
      if (!__all_sync(0xffffffffu, queue.take(k, idx, abort, st, 131))) break;
      __syncwarp();
      if (lane == 0) queue.release(k);
      if (idx >= n_items) break;
      const Item itm(idx, a.Hkv, a.Bt, T, gist);
      Visits vis;
      vis.init(m, itm, rep, P.near_nt);
      bool ok = true;
      for (int it = 0; it < vis.n; ++it) {
        const int gt = g + it, s = gt % kSlots;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bar[B_ME + s], ((gt / kSlots) & 1) ^ 1, abort, st, 130))) {
          ok = false;
          break;
        }
        int h, I, kind;
        vis.entry(m, itm, rep, it, h, I, kind);
        const int list = list_of(m, itm.bt, h);
        uint32_t* words = mwords + s * (kSlotBytes / 4);
        const int q0 = I * kTile;
        if (gist && !itm.far) {
          // near tile: the transposed element masks of the pre-pass
          const uint4* from = reinterpret_cast<const uint4*>(
              P.near_t + ((int64_t)I * P.near_nt + (itm.J - I + P.near_nt - 1)) * 512);
          uint4 v[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) v[q4] = from[lane + 32 * q4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) reinterpret_cast<uint4*>(words)[lane + 32 * q4] = v[q4];
        } else if (gist) {
          // far tile: compacted keys below this query tile's far prefix are seen
          // by every query row of the tile
          const int nf = m.far_ptr[gist_near_lo(I, m.sinks, m.window, m.period)];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const bool seen = itm.J * kTile + lane + 32 * i < nf;
#pragma unroll
            for (int w = 0; w < 4; ++w)
              words[w * 128 + lane + 32 * i] = seen ? prefix_bits(a.N - (q0 + 32 * w)) : 0u;
          }
        } else if (kind != SA_TILE_FULL && (m.b >= kTile || lb >= 5)) {
          // one block bit per (key row, word): every load first, then the words
          uint32_t u[4][4];
          int qb[4];
#pragma unroll
          for (int w = 0; w < 4; ++w)
            qb[w] = min(m.B - 1, m.b >= kTile ? q0 / m.b : (q0 + 32 * w) >> lb);
          const uint32_t* rows = m.bits + (int64_t)list * m.B * m.words;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int kb = min(a.N - 1, itm.J * kTile + lane + 32 * i) / m.b;
#pragma unroll
            for (int w = 0; w < 4; ++w) u[i][w] = rows[(int64_t)qb[w] * m.words + (kb >> 5)];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int kq = itm.J * kTile + lane + 32 * i;
            const int kb = min(a.N - 1, kq) / m.b;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int c0 = q0 + 32 * w;
              const uint32_t v = kq < a.N ? prefix_bits(a.N - c0) & ~prefix_bits(kq - c0) : 0u;
              words[w * 128 + lane + 32 * i] = ((u[i][w] >> (kb & 31)) & 1u) ? v : 0u;
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int w = 0; w < 4; ++w)
              words[w * 128 + lane + 32 * i] =
                  key_word(m, list, lb, a.N, itm.J * kTile + lane + 32 * i, q0, kind, w);
        }
        mbar_arrive(&bar[B_MF + s]);  // release: header and words are visible to the waiter
      }
      if (!ok) break;
      g += vis.n;
    }
  } else if (warp >= 2 && warp < 2 + kCompute / 32) {
    // -------------------------------------------------------- compute warps
    const int half = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;
    int g = 0, k = 0;
    bool ok = true;
    for (; ok; ++k) {
      int idx;
      if (!__all_sync(0xffffffffu, queue.take(k, idx, abort, st, 125))) break;
      __syncwarp();
      if (lane == 0) queue.release(k);
      if (idx >= n_items) break;
      const Item itm(idx, a.Hkv, a.Bt, T, gist);
      Visits vis;
      vis.init(m, itm, rep, P.near_nt);
      const int kq = itm.J * kTile + r;  // this thread's key row
      for (int it = 0; it < vis.n; ++it) {
        const int gt = g + it, s = gt & 1, ms = gt % kSlots;
        // phase 1: P from S^T (needs only S^T and the stored LSE)
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bar[B_SF], gt & 1, abort, st, 120) &&
                            mbar_wait(&bar[B_MF + ms], (gt / kSlots) & 1, abort, st, 121))) {
          ok = false;
          break;
        }
        const uint32_t* words = mwords + ms * (kSlotBytes / 4);
        const uint32_t mw[2] = {words[(2 * half) * 128 + r], words[(2 * half + 1) * 128 + r]};
        mbar_arrive(&bar[B_ME + ms]);
        const float* lse2 = rowv + s * 256 + half * 64;
        const float* dlt = lse2 + 128;
        tc_fence_after();
        __syncwarp();  // the TMEM loads below are warp-collective (.sync.aligned)
        float pv[64];
        tmem_ld32(lane_addr + kColS + half * 64, pv);
        tmem_ld32(lane_addr + kColS + half * 64 + 32, pv + 32);
        tmem_wait_ld();
        // P = 2^(s * scale * log2 e - LSE * log2 e) on visible pairs: the
        // per-column LSE four at a time (the whole warp reads the same words),
        // packed fp32 pairs, three of every eight exponentials on the FMA pipe
        uint32_t pk[32];
        const float2 sc = make_float2(sl2, sl2);
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          const float4 l4 = reinterpret_cast<const float4*>(lse2)[i4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int i = 4 * i4 + 2 * u;
            const float2 nl = u == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w);
            const float2 e = ffma2(make_float2(pv[i], pv[i + 1]), sc, nl);
            float2 p;
            if (((i >> 1) & 7) >= 5) {
              p = exp2_poly2(e);
            } else {
              p.x = ex2(e.x);
              p.y = ex2(e.y);
            }
            const uint32_t w = mw[i >> 5];
            pv[i] = ((w >> (i & 31)) & 1u) ? p.x : 0.f;
            pv[i + 1] = ((w >> ((i + 1) & 31)) & 1u) ? p.y : 0.f;
            pk[i >> 1] = pack_bf16(pv[i], pv[i + 1]);
          }
        }
        // P^T (bf16 pairs) over the first 32 of this half's S columns, all read
        __syncwarp();
        tmem_st32(lane_addr + kColS + half * 64, reinterpret_cast<const float*>(pk));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[B_PF1]);
        // phase 2: dS = P (dP - D) into dS^T (key row r, this half's 64 query
        // columns), bf16 pairs over the first 32 of this half's dP^T columns
        // once all 64 are read
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_DPF], gt & 1, abort, st, 122))) {
          ok = false;
          break;
        }
        tc_fence_after();
        __syncwarp();
        uint32_t dsk[32];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {  // 32 query columns at a time
          float dv[32];
          tmem_ld32(lane_addr + kColDP + half * 64 + c2 * 32, dv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int i = c2 * 32 + c;
            const float4 d4 = reinterpret_cast<const float4*>(dlt)[i >> 2];
            const float2 s0 = fmul2(make_float2(pv[i], pv[i + 1]),
                                    fadd2(make_float2(dv[c], dv[c + 1]), make_float2(-d4.x, -d4.y)));
            const float2 s1 = fmul2(make_float2(pv[i + 2], pv[i + 3]),
                                    fadd2(make_float2(dv[c + 2], dv[c + 3]), make_float2(-d4.z, -d4.w)));
            dsk[i >> 1] = pack_bf16(s0.x, s0.y);
            dsk[(i >> 1) + 1] = pack_bf16(s1.x, s1.y);
          }
        }
        __syncwarp();
        tmem_st32(lane_addr + kColDP + half * 64, reinterpret_cast<const float*>(dsk));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[B_PF2]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      // dK and dV of this key tile and KV head once every MMA of the item is
      // done (the next item's first dV / dK wait for OF); fp32, this half's
      // D / 2 columns
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_OI], k & 1, abort, st, 125))) break;
      // far items write the compacted keys' far contributions (added to their
      // rows by gist_far_scatter_kernel)
      float* dkr = (itm.far ? P.dkf : a.dk) + (((int64_t)itm.bt * a.N + kq) * a.Hkv + itm.hk) * D +
                   half * (D / 2);
      float* dvr = (itm.far ? P.dvf : a.dv) + (((int64_t)itm.bt * a.N + kq) * a.Hkv + itm.hk) * D +
                   half * (D / 2);
      if (vis.n > 0) {
        tc_fence_after();
        __syncwarp();
#pragma unroll
        for (int c4 = 0; c4 < D / 64; ++c4) {
          float x[32], y[32];
          tmem_ld32(lane_addr + kColDV + D + half * (D / 2) + c4 * 32, x);
          tmem_ld32(lane_addr + kColDV + half * (D / 2) + c4 * 32, y);
          tmem_wait_ld();
          if (kq < a.N) {
#pragma unroll
            for (int v = 0; v < 32; v += 4) {
              *reinterpret_cast<float4*>(dkr + c4 * 32 + v) =
                  make_float4(x[v] * a.scale, x[v + 1] * a.scale, x[v + 2] * a.scale, x[v + 3] * a.scale);
              *reinterpret_cast<float4*>(dvr + c4 * 32 + v) = make_float4(y[v], y[v + 1], y[v + 2], y[v + 3]);
            }
          }
        }
      } else if (kq < a.N) {  // no query tile visits this key tile: zero gradients
        for (int c = 0; c < D / 2; c += 4) {
          *reinterpret_cast<float4*>(dkr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(dvr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[B_OF]);  // dV and dK may be overwritten by the next item
      g += vis.n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Gist mode: adds the far contributions of every sink and gist (compacted
// index f, key far_idx[f]) to its dK and dV row; each key appears once in the
// compacted list, so no two threads add to the same element.
template <int D>
__global__ void __launch_bounds__(256) gist_far_scatter_kernel(AttnArgs a, MaskArgs m,
                                                               const float* dkf, const float* dvf) {
  const int f = blockIdx.x * 8 + (threadIdx.x >> 5), bt = blockIdx.y, lane = threadIdx.x & 31;
  if (f >= m.far_ptr[m.T]) return;
  const int64_t row = (int64_t)a.Hkv * D;
  const int64_t src = ((int64_t)bt * a.N + f) * row, dst = ((int64_t)bt * a.N + m.far_idx[f]) * row;
  for (int x = lane * 4; x < row; x += 32 * 4) {
    const float4 k4 = *reinterpret_cast<const float4*>(dkf + src + x);
    const float4 v4 = *reinterpret_cast<const float4*>(dvf + src + x);
    float4* pk = reinterpret_cast<float4*>(a.dk + dst + x);
    float4* pv = reinterpret_cast<float4*>(a.dv + dst + x);
    float4 ok = *pk, ov = *pv;
    ok.x += k4.x; ok.y += k4.y; ok.z += k4.z; ok.w += k4.w;
    ov.x += v4.x; ov.y += v4.y; ov.z += v4.z; ov.w += v4.w;
    *pk = ok;
    *pv = ov;
  }
}

// D = rowsum(dO * O) and LSE * log2(e), into padded [Bt, Hq, T*128] rows
// (+inf LSE and zero D past the end of the sequence). D / 8 lanes per row,
// one 16-byte load of O and of dO each.
template <int D>
__global__ void __launch_bounds__(256) bwd_tc_prep_kernel(AttnArgs a, float* lse2, float* delta,
                                                          int Tpad) {
  constexpr int kLanes = D / 8, kRowsPerWarp = 32 / kLanes;
  const int lane = threadIdx.x & 31, sub = lane / kLanes, l = lane % kLanes;
  const int64_t row = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kRowsPerWarp + sub;
  const int64_t rows = (int64_t)a.Bt * a.Hq * Tpad;
  const bool live = row < rows;
  const int p = live ? (int)(row % Tpad) : 0;
  const int h = live ? (int)((row / Tpad) % a.Hq) : 0;
  const int bt = live ? (int)(row / ((int64_t)Tpad * a.Hq)) : 0;
  float s = 0.f;
  if (live && p < a.N) {
    const int64_t off = bt * a.os[0] + (int64_t)p * a.os[1] + (int64_t)h * a.os[2] + l * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.o) + off);
    const uint4 dv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.dout) + off);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(o2[i]), y = __bfloat1622float2(d2[i]);
      s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (live && l == 0) {
    delta[row] = s;
    lse2[row] = p < a.N ? a.lse[((int64_t)bt * a.Hq + h) * a.N + p] * 1.4426950408889634f
                        : INFINITY;
  }
}

// [Bt, N, H, d] bf16 with element strides {batch, seq, head}; box 64 x 1 x 128 x 1.
bool make_tile_map(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                   const int64_t* s);
bool make_map_4d(CUtensorMap* map, CUtensorMapDataType dtype, int ebytes, const void* base, int d,
                 int H, int N, int Bt, const int64_t* s, int box_d, int rows);
int sm_count();
cudaError_t launch_dq_tc(int d, const AttnArgs& a, const MaskArgs& m, const float* lse2,
                         const float* delta, int Tpad, const void* compact, const void* near,
                         cudaStream_t s);
cudaError_t launch_gist_prepass(int d, const AttnArgs& a, const MaskArgs& m, void* compact,
                                void* near, void* near_t, cudaStream_t s);

// Workspace bytes after the status header: lse2 and delta, [Bt, Hq, T*128]
// fp32 each; gist mode also the compacted sink / gist K and V (bf16), the
// near-tile masks and their transpose, and the far dK and dV of the compacted
// keys (fp32, [Bt, N, Hkv, d] each).
struct BwdWs {
  size_t rows, compact, near, far;
};
static size_t r256b(size_t x) { return (x + 255) / 256 * 256; }
static BwdWs bwd_ws_parts(int Bt, int Hq, int Hkv, int64_t N, int d, int T, int near_nt, bool gist) {
  BwdWs w{};
  w.rows = r256b((size_t)2 * Bt * Hq * T * kTile * 4);
  if (gist) {
    w.compact = 2 * r256b((size_t)Bt * N * Hkv * d * 2);
    w.near = r256b((size_t)T * near_nt * 2048);
    w.far = 2 * r256b((size_t)Bt * N * Hkv * d * 4);
  }
  return w;
}
size_t bwd_tc_workspace(int Bt, int Hq, int Hkv, int64_t N, int d, int T, int near_nt, bool gist) {
  const BwdWs w = bwd_ws_parts(Bt, Hq, Hkv, N, d, T, near_nt, gist);
  return w.rows + w.compact + 2 * w.near + w.far;
}

template <int D>
static cudaError_t bwd_tc_launch(const AttnArgs& a, const MaskArgs& m, void* ws, cudaStream_t s) {
  BwdTcParams P;
  memset(&P, 0, sizeof(P));
  if (!make_tile_map(&P.tmq, a.q, D, a.Hq, a.N, a.Bt, a.qs) ||
      !make_tile_map(&P.tmk, a.k, D, a.Hkv, a.N, a.Bt, a.ks) ||
      !make_tile_map(&P.tmv, a.v, D, a.Hkv, a.N, a.Bt, a.vs) ||
      !make_tile_map(&P.tmdo, a.dout, D, a.Hq, a.N, a.Bt, a.os))
    return cudaErrorInvalidValue;
  P.tmkc = P.tmk;
  P.tmvc = P.tmv;
  P.a = a;
  P.m = m;
  P.Tpad = m.T * kTile;
  const bool gist = m.kind == SA_MASK_GIST;
  const BwdWs parts = bwd_ws_parts(a.Bt, a.Hq, a.Hkv, a.N, D, m.T, gist_near_tiles(m.window, m.period), gist);
  char* base = static_cast<char*>(ws);
  float* lse2 = reinterpret_cast<float*>(base);
  float* delta = lse2 + (size_t)a.Bt * a.Hq * P.Tpad;
  P.lse2 = lse2;
  P.delta = delta;
  const int64_t rows = (int64_t)a.Bt * a.Hq * P.Tpad;
  const int64_t rows_per_block = 8 * (32 / (D / 8));
  bwd_tc_prep_kernel<D><<<(unsigned)((rows + rows_per_block - 1) / rows_per_block), 256, 0, s>>>(
      a, lse2, delta, P.Tpad);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  void *compact = nullptr, *near = nullptr;
  if (gist) {
    // the forward's pre-passes (compacted sinks / gists, near-tile masks) and
    // the transposed masks the key-major pass reads
    compact = base + parts.rows;
    near = base + parts.rows + parts.compact;
    void* near_t = static_cast<char*>(near) + parts.near;
    float* far = reinterpret_cast<float*>(static_cast<char*>(near_t) + parts.near);
    e = launch_gist_prepass(D, a, m, compact, near, near_t, s);
    if (e != cudaSuccess) return e;
    const int64_t row = (int64_t)a.Hkv * D;
    const __nv_bfloat16* kc = static_cast<const __nv_bfloat16*>(compact);
    const __nv_bfloat16* vc = kc + (int64_t)a.Bt * a.N * row;
    const int64_t cs[3] = {(int64_t)a.N * row, row, D};
    if (!make_tile_map(&P.tmkc, kc, D, a.Hkv, a.N, a.Bt, cs) ||
        !make_tile_map(&P.tmvc, vc, D, a.Hkv, a.N, a.Bt, cs))
      return cudaErrorInvalidValue;
    P.near_t = static_cast<const uint32_t*>(near_t);
    P.near_nt = gist_near_tiles(m.window, m.period);
    P.dkf = far;
    P.dvf = reinterpret_cast<float*>(reinterpret_cast<char*>(far) + parts.far / 2);
  }
  // dQ: the query-major pass
  e = launch_dq_tc(D, a, m, lse2, delta, P.Tpad, compact, near, s);
  if (e != cudaSuccess) return e;
  const int bytes = (int)Layout<D>::bytes;
  e = cudaFuncSetAttribute(bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (TMEM and shared memory admit one)
  const int items = (gist ? 2 : 1) * m.T * a.Hkv * a.Bt;
  const int grid = items < sm_count() ? items : sm_count();
  bwd_tc_kernel<D><<<dim3(grid), kThreads, bytes, s>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess || !gist) return e;
  gist_far_scatter_kernel<D><<<dim3((a.N + 7) / 8, a.Bt), 256, 0, s>>>(a, m, P.dkf, P.dvf);
  return cudaGetLastError();
}

cudaError_t launch_bwd_tc(int d, const AttnArgs& a, const MaskArgs& m, void* ws, cudaStream_t s) {
  if (d == 64) return bwd_tc_launch<64>(a, m, ws, s);
  if (d == 128) return bwd_tc_launch<128>(a, m, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace sa
