// Query-major dQ pass of the block-sparse backward (5th-generation tensor
// cores, sm_100a).
//
//   dQ_I = scale * sum_J dS_IJ K_J,  dS = P * (dP - D),  P = exp(s - LSE),
//   dP = dO V^T,  D = rowsum(dO * O)
// (the gradient of the masked softmax attention; "UniGist ...", Approach:
// one-pass training needs the backward). A work item is one (128-query tile
// I, head, sequence) and visits the key tiles J of I's tile list, as the
// forward does, the items taken from a run-time queue in (sequence, KV head)
// order so that the CTAs running together read one KV head's K/V tiles
// through L2. S and dP are recomputed per visit and dQ accumulates in TMEM,
// so every dQ row is written once, with no reductions in global memory; the
// key-major pass (attn_bwd_sm100.cu) computes dK and dV only.
//
// Roles (352 threads):
//   warp 0     TMA: Q and dO per item (d = 64: two stages), K and V per visit
//              on one barrier per stage.
//   warp 1     one thread issues tcgen05.mma: S_j = Q K_j^T into one of two S
//              buffers, dP_j = dO V_j^T into one dP buffer, and dQ += dS_j K_j
//              with dS_j read from TMEM (A operand) and K_j from shared memory.
//   warps 2-9  compute: half h owns key columns [64h, 64h + 64) of a visit and
//              thread (h, r) query row r (TMEM lane r): P = 2^(s log2(e) scale
//              - LSE log2(e)) on visible pairs, dS = P (dP - D), written as
//              bf16 over the first 32 of its S columns. At the end of an item
//              each half stores D / 2 columns of its dQ row.
//   warp 10    visibility words of each visited tile (the forward's gzip rule).
// Every wait is bounded; on timeout the device status word is set and all
// roles leave after draining their copies and MMAs, freeing TMEM.
#include <cuda.h>

#include "attn_mask.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

struct DqTcParams {
  CUtensorMap tmq, tmk, tmv, tmdo;
  CUtensorMap tmkc, tmvc;  // gist mode: sinks + gists compacted in logical order
  const uint32_t* near;    // gist mode: element masks of (query tile, near key tile)
  int near_nt;
  AttnArgs a;
  MaskArgs m;
  const float* lse2;   // [Bt, Hq, Tpad] LSE * log2(e), +inf past N
  const float* delta;  // [Bt, Hq, Tpad] rowsum(dO * O), 0 past N
  int Tpad;
};

namespace dqk {

constexpr int kSlots = 8;              // mask ring depth
constexpr uint32_t kSlotBytes = 2048;  // [4 words][128 rows]
constexpr int kRowWords = 1024;        // the item's block-row bits
constexpr int kCompute = 256;
constexpr int kThreads = 64 + kCompute + 32;
constexpr int kMaskWarp = 10;
constexpr uint32_t kColS = 0, kColDP = 256, kColDQ = 384;

template <int D>
struct Layout {
  static constexpr int kQStages = D == 64 ? 2 : 1;
  static constexpr int kKVStages = D == 64 ? 3 : 2;
  static constexpr uint32_t kT = 128 * D * 2;   // a 128 x D bf16 tile
  static constexpr uint32_t kAtom = 128 * 128;  // [128 rows][64 bf16] swizzle atom
  static constexpr uint32_t q = 0;              // [stage] Q, then dO
  static constexpr uint32_t k = 2 * kQStages * kT;
  static constexpr uint32_t v = k + kKVStages * kT;
  static constexpr uint32_t mask = v + kKVStages * kT;
  static constexpr uint32_t rows = mask + kSlots * kSlotBytes;
  static constexpr uint32_t bars = rows + kRowWords * 4;
  static constexpr uint32_t bytes = bars + 512 + 1024;
};

// QF/QE: Q and dO of a stage loaded / read. KVF/KVE: K and V of a stage
// loaded / read. SF: S buffer written. DPF: dP written. DS: dS written by both
// halves. MF/ME: mask slot written / read. OI: every MMA of the item done. OF:
// both halves have read dQ. DRAIN: all MMAs done.
enum {
  B_QF = 0, B_QE = 2, B_KVF = 4, B_KVE = 8, B_SF = 12, B_DPF = 14, B_DS = 15, B_MF = 16,
  B_ME = B_MF + kSlots, B_OI = B_ME + kSlots, B_OF, B_DRAIN, B_IQF,
  B_IQE = B_IQF + kItemRing, kNumBars = B_IQE + kItemRing
};
// consumers of each item of the run-time queue: the MMA thread, the mask warp
// and the eight compute warps
constexpr int kQueueConsumers = 1 + 1 + kCompute / 32;

struct Item {
  int I, h, bt;
  __device__ Item(int idx, int T, int Hq, int Hkv, int Bt) {
    // (sequence, KV head) outermost, so that the CTAs running together share the
    // K/V tiles of one KV head through L2; then late query tiles (long lists)
    // first, the group's query heads of one tile next to each other
    const int rep = Hq / Hkv, per = T * rep;
    const int hb = idx / per, local = idx % per;
    bt = hb / Hkv;
    h = (hb % Hkv) * rep + local % rep;
    I = T - 1 - local / rep;
  }
};


}  // namespace dqk

using namespace dqk;

template <int D>
__global__ void __launch_bounds__(kThreads, 1) dq_tc_kernel(const __grid_constant__ DqTcParams P) {
  using L = Layout<D>;
  constexpr int QS = L::kQStages, KS = L::kKVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + kNumBars) + 1;
  uint32_t* mwords = reinterpret_cast<uint32_t*>(smem + L::mask);

  const AttnArgs& a = P.a;
  const MaskArgs& m = P.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = m.T;
  const int n_items = T * a.Hq * a.Bt;
  DeviceStatus* st = a.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_QF + s], 1);
      mbar_init(&bar[B_QE + s], 1);
      mbar_init(&bar[B_SF + s], 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bar[B_KVF + s], 1);
      mbar_init(&bar[B_KVE + s], 1);
    }
    mbar_init(&bar[B_DPF], 1);
    mbar_init(&bar[B_DS], kCompute);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar[B_MF + s], 32);
      mbar_init(&bar[B_ME + s], kCompute);
    }
    mbar_init(&bar[B_OI], 1);
    mbar_init(&bar[B_OF], kCompute);
    mbar_init(&bar[B_DRAIN], 1);
    for (int s = 0; s < kItemRing; ++s) {
      mbar_init(&bar[B_IQF + s], 1);
      mbar_init(&bar[B_IQE + s], kQueueConsumers);
    }
    *abort = 0;
    fence_barrier_init();
  }
  ItemQueue queue{reinterpret_cast<int*>(bar + kNumBars) + 2, &bar[B_IQF], &bar[B_IQE],
                  reinterpret_cast<unsigned int*>(st->aux + kQueueWordDq)};
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
      // ------------------------------------------------------ TMA producer
      prefetch_tmap(&P.tmq);
      prefetch_tmap(&P.tmk);
      prefetch_tmap(&P.tmv);
      prefetch_tmap(&P.tmdo);
      if (m.kind == SA_MASK_GIST) {
        prefetch_tmap(&P.tmkc);
        prefetch_tmap(&P.tmvc);
      }
      int g = 0, k = 0, last_q = -1, last_kv = -1;
      bool ok = true;
      for (; ok; ++k) {
        int idx;
        if (!queue.publish(k, idx, abort, st, 204) || idx >= n_items) break;
        const Item itm(idx, T, a.Hq, a.Hkv, a.Bt);
        const int list = list_of(m, itm.bt, itm.h), hk = itm.h / (a.Hq / a.Hkv);
        WorkList wl;
        wl.init(m, list, itm.I);
        const int n = wl.n;
        const int qs = k % QS;
        if (k >= QS && !mbar_wait(&bar[B_QE + qs], ((k / QS) - 1) & 1, abort, st, 200)) break;
        mbar_arrive_expect_tx(&bar[B_QF + qs], 2 * L::kT);
        for (int at = 0; at < D / 64; ++at) {
          uint8_t* dq = smem + L::q + 2 * qs * L::kT + at * L::kAtom;
          tma_load_4d(dq, &P.tmq, &bar[B_QF + qs], at * 64, itm.h, itm.I * kTile, itm.bt);
          tma_load_4d(dq + L::kT, &P.tmdo, &bar[B_QF + qs], at * 64, itm.h, itm.I * kTile, itm.bt);
        }
        last_q = k;
        for (int it = 0; it < n; ++it) {
          const int gt = g + it, s = gt % KS;
          if (!mbar_wait(&bar[B_KVE + s], ((gt / KS) & 1) ^ 1, abort, st, 201)) {
            ok = false;
            break;
          }
          int src, k0, kind, cnt;
          wl.entry(m, it, src, k0, kind, cnt);
          const CUtensorMap* mk = src ? &P.tmkc : &P.tmk;
          const CUtensorMap* mv = src ? &P.tmvc : &P.tmv;
          mbar_arrive_expect_tx(&bar[B_KVF + s], 2 * L::kT);
          for (int at = 0; at < D / 64; ++at) {
            tma_load_4d(smem + L::k + s * L::kT + at * L::kAtom, mk, &bar[B_KVF + s], at * 64, hk, k0,
                        itm.bt);
            tma_load_4d(smem + L::v + s * L::kT + at * L::kAtom, mv, &bar[B_KVF + s], at * 64, hk, k0,
                        itm.bt);
          }
          last_kv = gt;
        }
        if (ok) count_tiles(st, CNT_DQ_VISITS, n);
        g += n;
      }
      // every copy this CTA started must land before the CTA may exit
      volatile int no_abort = 0;
      for (int q = last_q; q >= 0 && q > last_q - QS; --q)
        mbar_wait(&bar[B_QF + q % QS], (q / QS) & 1, &no_abort, nullptr, 202);
      for (int s = 0; s < KS; ++s)
        if (last_kv >= s) {
          const int gs = last_kv - ((last_kv - s) % KS);
          mbar_wait(&bar[B_KVF + s], (gs / KS) & 1, &no_abort, nullptr, 203);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      // Per visit g: S(g + 1) (its buffer held dS(g - 1), read by dQ(g - 1),
      // issued before: one thread's tcgen05 ops run in order), dQ(g) once
      // dS(g) is written (which also means dP(g) has been read), then
      // dP(g + 1) into the one dP buffer.
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdDq = idesc_bf16_f32(128, D, false, true);  // B = K, MN-major
      int g = 0, k = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t qa, int gt) -> bool {
        const int s = gt % KS;
        if (!mbar_wait(&bar[B_KVF + s], (gt / KS) & 1, abort, st, 210)) return false;
        tc_fence_after();
        const uint32_t kb = sb + L::k + s * L::kT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + kColS + (gt & 1) * 128, smem_desc_sw128(qa + off, 16, 1024),
                   smem_desc_sw128(kb + off, 16, 1024), kIdS, kk > 0);
        }
        mma_commit(&bar[B_SF + (gt & 1)]);
        return true;
      };
      auto issue_dp = [&](uint32_t da, int gt) {  // V of visit gt landed with its K
        const uint32_t vb = sb + L::v + (gt % KS) * L::kT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + kColDP, smem_desc_sw128(da + off, 16, 1024),
                   smem_desc_sw128(vb + off, 16, 1024), kIdS, kk > 0);
        }
        mma_commit(&bar[B_DPF]);
      };
      for (; ok; ++k) {
        int idx;
        if (!queue.take(k, idx, abort, st, 215)) break;
        queue.release(k);
        if (idx >= n_items) break;
        const Item itm(idx, T, a.Hq, a.Hkv, a.Bt);
        WorkList wl;
        wl.init(m, list_of(m, itm.bt, itm.h), itm.I);
        const int n = wl.n;
        const int qs = k % QS;
        const uint32_t qa = sb + L::q + 2 * qs * L::kT, da = qa + L::kT;
        if (!mbar_wait(&bar[B_QF + qs], (k / QS) & 1, abort, st, 211)) break;
        if (n > 0) {
          if (!issue_s(qa, g)) break;
          issue_dp(da, g);
        }
        for (int it = 0; it < n; ++it) {
          const int gt = g + it;
          if (it + 1 < n && !issue_s(qa, gt + 1)) {
            ok = false;
            break;
          }
          // dS(gt) written (both halves); the previous item's dQ read out
          if (!mbar_wait(&bar[B_DS], gt & 1, abort, st, 212) ||
              (it == 0 && k > 0 && !mbar_wait(&bar[B_OF], (k - 1) & 1, abort, st, 213))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = sb + L::k + (gt % KS) * L::kT;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            // dS of this half: bf16 pairs in the first 32 columns of its S columns
            const uint32_t pa = tmem + kColS + (gt & 1) * 128 + hf * 64;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = smem_desc_sw128(kb + (hf * 4 + kk) * 2048, L::kAtom, 1024);
              mma_bf16_ts(tmem + kColDQ, pa + kk * 8, bd, kIdDq, (it > 0 || hf > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bar[B_KVE + gt % KS]);
          if (it + 1 < n) issue_dp(da, gt + 1);
        }
        if (!ok) break;
        if (n == 0 && k > 0 && !mbar_wait(&bar[B_OF], (k - 1) & 1, abort, st, 213)) break;
        mma_commit(&bar[B_QE + qs]);
        mma_commit(&bar[B_OI]);
        g += n;
      }
      mma_commit(&bar[B_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[B_DRAIN], 0, &no_abort, nullptr, 214);
    }
  } else if (warp == kMaskWarp) {
    // -------------------------------------------------------------- mask
    const int gzip = m.kind == SA_MASK_GZIP;
    const int lb = gzip && m.b < kTile ? __ffs(m.b) - 1 : 0;  // b < 128 is a power of two
    uint32_t* rcache = reinterpret_cast<uint32_t*>(smem + L::rows);
    int g = 0;
    for (int k = 0;; ++k) {
      int idx;
      if (!__all_sync(0xffffffffu, queue.take(k, idx, abort, st, 231))) break;
      __syncwarp();
      if (lane == 0) queue.release(k);
      if (idx >= n_items) break;
      const Item itm(idx, T, a.Hq, a.Hkv, a.Bt);
      const int list = list_of(m, itm.bt, itm.h);
      WorkList wl;
      wl.init(m, list, itm.I);
      const int n = wl.n;
      // gzip: the block rows of this query tile, copied once per item when they fit
      const int rb0 = gzip ? itm.I * kTile / m.b : 0;
      const int rb1 = gzip ? min(m.B - 1, (itm.I * kTile + kTile - 1) / m.b) : 0;
      const int nw = (rb1 - rb0 + 1) * m.words;
      const bool cached = gzip && nw <= kRowWords;
      __syncwarp();
      if (cached) {
        const uint32_t* src = m.bits + ((int64_t)list * m.B + rb0) * m.words;
        for (int x = lane; x < nw; x += 32) rcache[x] = src[x];
      }
      __syncwarp();
      RowCtx rc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        rc[i].p = itm.I * kTile + lane + 32 * i;
        rc[i].ok = rc[i].p < a.N;
        rc[i].bits = nullptr;
        if (gzip) {
          const int rb = rc[i].ok ? rc[i].p / m.b : rb0;
          rc[i].bits = cached ? rcache + (rb - rb0) * m.words
                              : m.bits + ((int64_t)list * m.B + rb) * m.words;
        }
        rc[i].li = 0;
      }
      bool ok = true;
      int col_reg = 0, kind_reg = 0;
      for (int it = 0; it < n; ++it) {
        if (gzip && (it & 31) == 0) {
          const int e = it + lane;
          col_reg = e < n ? m.tcol[wl.e0 + e] : 0;
          kind_reg = e < n ? m.tkind[wl.e0 + e] : 0;
        }
        const int gq = g + it, slot = gq % kSlots;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_ME + slot], ((gq / kSlots) & 1) ^ 1, abort,
                                                st, 230))) {
          ok = false;
          break;
        }
        uint32_t* words = mwords + slot * (kSlotBytes / 4);
        if (gzip) {
          const int kbase = __shfl_sync(0xffffffffu, col_reg, it & 31) * kTile;
          const int kind = __shfl_sync(0xffffffffu, kind_reg, it & 31) == SA_TILE_FULL
                               ? SA_TILE_FULL : SA_TILE_MASKED;
          gzip_tile_words(m, lb, a.N, rc, kbase, kind, lane, words);
        } else {
          int src, kbase, kind, cnt;
          wl.entry(m, it, src, kbase, kind, cnt);
          if (src == 0) {
            // gist near tile: the element rule, evaluated once for every head
            const uint4* from = reinterpret_cast<const uint4*>(
                P.near + ((int64_t)itm.I * P.near_nt + (kbase / kTile - itm.I + P.near_nt - 1)) * 512);
            uint4 v[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) v[q4] = from[lane + 32 * q4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) reinterpret_cast<uint4*>(words)[lane + 32 * q4] = v[q4];
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int w = 0; w < 4; ++w)
                words[w * 128 + lane + 32 * i] = tile_word(m, 0, lb, a.N, rc[i], kbase, kind, cnt, w);
          }
        }
        mbar_arrive(&bar[B_MF + slot]);  // release: the words above are visible to the waiter
      }
      if (!ok) break;
      g += n;
    }
  } else if (warp >= 2 && warp < 2 + kCompute / 32) {
    // ----------------------------------------------------------- compute
    const int half = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;
    int g = 0, k = 0;
    bool ok = true;
    for (; ok; ++k) {
      int idx;
      if (!__all_sync(0xffffffffu, queue.take(k, idx, abort, st, 225))) break;
      __syncwarp();
      if (lane == 0) queue.release(k);
      if (idx >= n_items) break;
      const Item itm(idx, T, a.Hq, a.Hkv, a.Bt);
      WorkList wl;
      wl.init(m, list_of(m, itm.bt, itm.h), itm.I);
      const int n = wl.n;
      const int p = itm.I * kTile + r;
      const int64_t ro = ((int64_t)itm.bt * a.Hq + itm.h) * P.Tpad + p;
      const float lse2 = P.lse2[ro], dlt = P.delta[ro];
      for (int it = 0; it < n; ++it) {
        const int gq = g + it, slot = gq % kSlots;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bar[B_SF + (gq & 1)], (gq >> 1) & 1, abort, st, 220) &&
                            mbar_wait(&bar[B_DPF], gq & 1, abort, st, 221) &&
                            mbar_wait(&bar[B_MF + slot], (gq / kSlots) & 1, abort, st, 222))) {
          ok = false;
          break;
        }
        tc_fence_after();
        __syncwarp();  // tcgen05.ld is warp-collective (.sync.aligned)
        const uint32_t scol = kColS + (gq & 1) * 128 + half * 64;
        const uint32_t* words = mwords + slot * (kSlotBytes / 4);
        const uint32_t mw[2] = {words[(2 * half) * 128 + r], words[(2 * half + 1) * 128 + r]};
        // P = 2^(s * scale * log2 e - LSE * log2 e) on visible pairs and
        // dS = P (dP - D), 32 key columns at a time, in packed fp32 pairs;
        // three of every eight exponentials on the FMA pipe (as in the forward)
        uint32_t pk[32];
        const float2 sc = make_float2(sl2, sl2), nl = make_float2(-lse2, -lse2);
        const float2 nd = make_float2(-dlt, -dlt);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float x[32], y[32];
          tmem_ld32(lane_addr + scol + c * 32, x);
          tmem_ld32(lane_addr + kColDP + half * 64 + c * 32, y);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 e = ffma2(make_float2(x[2 * i], x[2 * i + 1]), sc, nl);
            float2 pr;
            if ((i & 7) >= 5) {
              pr = exp2_poly2(e);
            } else {
              pr.x = ex2(e.x);
              pr.y = ex2(e.y);
            }
            pr.x = ((mw[c] >> (2 * i)) & 1u) ? pr.x : 0.f;
            pr.y = ((mw[c] >> (2 * i + 1)) & 1u) ? pr.y : 0.f;
            const float2 ds = fmul2(pr, fadd2(make_float2(y[2 * i], y[2 * i + 1]), nd));
            pk[c * 16 + i] = pack_bf16(ds.x, ds.y);
          }
        }
        mbar_arrive(&bar[B_ME + slot]);
        // dS (bf16 pairs) over the first 32 of this half's S columns, all read
        __syncwarp();
        tmem_st32(lane_addr + scol, reinterpret_cast<const float*>(pk));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[B_DS]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_OI], k & 1, abort, st, 223))) break;
      float* dqr = a.dq + (((int64_t)itm.bt * a.N + p) * a.Hq + itm.h) * D + half * (D / 2);
      if (n > 0) {
        tc_fence_after();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          float o[32];
          tmem_ld32(lane_addr + kColDQ + half * (D / 2) + c * 32, o);
          tmem_wait_ld();
          if (p < a.N) {
#pragma unroll
            for (int v = 0; v < 32; v += 4)
              *reinterpret_cast<float4*>(dqr + c * 32 + v) =
                  make_float4(o[v] * a.scale, o[v + 1] * a.scale, o[v + 2] * a.scale, o[v + 3] * a.scale);
          }
        }
      } else if (p < a.N) {
        for (int c = 0; c < D / 2; c += 4)
          *reinterpret_cast<float4*>(dqr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      tc_fence_before();
      mbar_arrive(&bar[B_OF]);  // dQ may be overwritten by the next item
      g += n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

bool make_tile_map(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                   const int64_t* s);
int sm_count();

template <int D>
static cudaError_t dq_tc_launch(const AttnArgs& a, const MaskArgs& m, const float* lse2,
                                const float* delta, int Tpad, const void* compact, const void* near,
                                cudaStream_t s) {
  DqTcParams P;
  memset(&P, 0, sizeof(P));
  if (!make_tile_map(&P.tmq, a.q, D, a.Hq, a.N, a.Bt, a.qs) ||
      !make_tile_map(&P.tmk, a.k, D, a.Hkv, a.N, a.Bt, a.ks) ||
      !make_tile_map(&P.tmv, a.v, D, a.Hkv, a.N, a.Bt, a.vs) ||
      !make_tile_map(&P.tmdo, a.dout, D, a.Hq, a.N, a.Bt, a.os))
    return cudaErrorInvalidValue;
  P.tmkc = P.tmk;
  P.tmvc = P.tmv;
  if (m.kind == SA_MASK_GIST) {
    // the compacted sink / gist K and V and the near-tile masks of the forward's pre-passes
    const int64_t row = (int64_t)a.Hkv * D;
    const __nv_bfloat16* kc = static_cast<const __nv_bfloat16*>(compact);
    const __nv_bfloat16* vc = kc + (int64_t)a.Bt * a.N * row;
    const int64_t cs[3] = {(int64_t)a.N * row, row, D};
    if (!make_tile_map(&P.tmkc, kc, D, a.Hkv, a.N, a.Bt, cs) ||
        !make_tile_map(&P.tmvc, vc, D, a.Hkv, a.N, a.Bt, cs))
      return cudaErrorInvalidValue;
    P.near = static_cast<const uint32_t*>(near);
    P.near_nt = gist_near_tiles(m.window, m.period);
  }
  P.a = a;
  P.m = m;
  P.lse2 = lse2;
  P.delta = delta;
  P.Tpad = Tpad;
  const int bytes = (int)Layout<D>::bytes;
  cudaError_t e = cudaFuncSetAttribute(dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes);
  if (e != cudaSuccess) return e;
  const int items = m.T * a.Hq * a.Bt;
  const int grid = items < sm_count() ? items : sm_count();
  dq_tc_kernel<D><<<dim3(grid), kThreads, bytes, s>>>(P);
  return cudaGetLastError();
}

// dQ of every query row (fp32, dense [Bt, N, Hq, d]), from the padded
// LSE * log2(e) and D rows the backward's preparation kernel wrote. Gist mode:
// `compact` and `near` as the forward's pre-passes leave them.
cudaError_t launch_dq_tc(int d, const AttnArgs& a, const MaskArgs& m, const float* lse2,
                         const float* delta, int Tpad, const void* compact, const void* near,
                         cudaStream_t s) {
  if (d == 64) return dq_tc_launch<64>(a, m, lse2, delta, Tpad, compact, near, s);
  if (d == 128) return dq_tc_launch<128>(a, m, lse2, delta, Tpad, compact, near, s);
  return cudaErrorInvalidValue;
}

}  // namespace sa
