// Gist-scored selective unfolding at decode, one CTA per (sequence, KV head),
// on the 5th-generation tensor cores.
//
// "Simplified Sparse Attention via Gist Tokens" (abstract) and "Forget, Then
// Recall: ... Gist Sparse Attention" (abstract): the new query is scored
// against the gist keys, the top-k chunks are unfolded into their raw tokens,
// and attention runs over the gists, the unfolded chunks and the recent
// window. Everything of one (sequence, KV head g) happens in one CTA, in one
// online softmax over 128-key blocks:
//   1. gist blocks: S^T = K_blk Q_g^T (keys on TMEM lanes, the group's query
//      heads on columns); the selection score of gist j, sum_h s_hj, goes to
//      shared memory; O^T += V_blk^T P with the same logits.
//   2. window blocks: the last `window` positions of the raw cache (these are
//      loaded while step 3 runs).
//   3. top-k selection over the eligible chunks (wholly before the window) by
//      a 4-pass radix select on the order-preserving 32-bit key of the score,
//      ties to the lower chunk index, written ascending (-1 padded). The
//      sum-of-probabilities rule stores each head's logits during step 1 and
//      scores gist j by sum_h 2^(s_hj - m_h) / l_h with the heads' gist-only
//      softmax state; the top-p rule then keeps the shortest score-ordered
//      prefix of the top_k whose softmax over the eligible chunks reaches p.
//   4. chunk blocks: 128 / chunk selected chunks per block, each brought in
//      by its own TMA box.
// The output O = O^T / l and LSE follow from the single softmax state; no
// partial results leave the CTA.
//
// Gist of gists ("Forget, Then Recall: ...", abstract: recursive gist-of-gist
// construction with logarithmic per-step cost), the HIER instantiation: the
// same CTA streams the level-2 gists, selects the top groups after them, then
// half the window, the kept groups' level-1 gists (one TMA box of `fanout`
// rows per group), selects the top chunks among those candidates, then the
// rest of the window and the chunks, all in the one online softmax.
//
// Roles (192 threads): warp 0 issues the TMA loads (K blocks into a 3-stage
// ring, up to two blocks ahead, freed once Q K^T has read them; V blocks into
// a 2-stage ring, freed after P V) and owns the TMEM allocation; one thread of warp 1 issues
// tcgen05.mma (S^T = K Q^T, M = 128 keys, N = 16 head columns; O^T += V^T P,
// M = 128 dims, N = 16) with completion on mbarriers; warps 2-5 (thread = key
// row of the block for the softmax, = output dimension for O^T) run the
// softmax, the selection and the epilogue. The block maximum per head is
// exchanged between the four softmax warps through shared memory; O^T is
// rescaled only when a head's maximum grew by more than 2^8. Every wait is
// bounded; on timeout the device status word is set and all roles leave
// after draining their copies and MMAs.
#include <cuda.h>

#include "sa_common.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

bool make_tile_map_box(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                       const int64_t* s, int rows);

namespace dec {

constexpr int kD = 128;        // head dim
constexpr int kBlk = 128;      // keys per block
constexpr int kN = 16;         // MMA N: query-head columns (rep <= 8 used)
constexpr int kMaxG = 8192;    // gists held in shared memory for the selection
constexpr int kMaxTopK = 256;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 softmax

struct Params {
  CUtensorMap gk, gv;    // gists (gist of gists: the level-2 gists), box 128 rows
  CUtensorMap ck, cv;    // raw cache, box 128 rows (window)
  CUtensorMap ckc, cvc;  // raw cache, box `chunk` rows (unfolded chunks)
  CUtensorMap g1k, g1v;  // gist of gists: level-1 gists, box `fanout` rows (kept groups)
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  float* lse;
  int32_t* sel;
  float* logits;         // [n_seq, Hq, G] raw dot products (sum-of-probabilities rule)
  DeviceStatus* status;
  int rule;
  float top_p;
  int n_seq, Hkv, rep, G, cache_len, chunk, top_k, window;
  int n_slots;           // unfolded chunk slots: top_k, or rep * top_k (per-head rule)
  int nG, nW, nC;        // gist, window and chunk blocks
  // gist of gists: G and nG describe the level-2 gists; the blocks run
  // [level-2][first nW1 window][nB1 level-1 of the kept groups][other window][chunks]
  int fanout, top_k2, nW1, nB1;
  int32_t* sel2;         // [n_seq, Hkv, top_k2] kept groups
  float scale;
  int64_t qs[2], os[2];
};

// Gist of gists: kind and index (within its kind; window blocks 0..nW-1) of
// block b in stream order.
enum { BK_GIST = 0, BK_WIN, BK_L1, BK_CHUNK };
struct BlockOf {
  int kind, idx;
  __device__ BlockOf(const Params& P, int b) {
    if (b < P.nG) { kind = BK_GIST; idx = b; return; }
    b -= P.nG;
    if (b < P.nW1) { kind = BK_WIN; idx = b; return; }
    b -= P.nW1;
    if (b < P.nB1) { kind = BK_L1; idx = b; return; }
    b -= P.nB1;
    if (b < P.nW - P.nW1) { kind = BK_WIN; idx = P.nW1 + b; return; }
    kind = BK_CHUNK;
    idx = b - (P.nW - P.nW1);
  }
};

// Shared memory (offsets from a 1024-aligned base).
constexpr uint32_t kAtom = kBlk * 128;          // [128 rows][64 bf16]
constexpr uint32_t kTileBytes = 2 * kAtom;      // one K or V block, 2 atoms
constexpr int kKStages = 3, kVStages = 2;
constexpr int kKAhead = 2;                      // K blocks requested ahead of V
constexpr uint32_t kQtAtom = kN * 128;          // [16 rows][64 bf16]
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t OFF_QT = OFF_V + kVStages * kTileBytes;  // Q^T [16][128], 2 atoms
constexpr uint32_t OFF_PT = OFF_QT + 2 * kQtAtom;  // P^T [2 buffers][16][128], 2 atoms each
constexpr uint32_t OFF_SCORE = OFF_PT + 2 * 2 * kQtAtom;  // float [kMaxG]
constexpr uint32_t OFF_HIST = OFF_SCORE + kMaxG * 4;     // uint32 [256]
constexpr uint32_t OFF_SEL = OFF_HIST + 256 * 4;         // int32 [kMaxTopK]
constexpr uint32_t OFF_RED = OFF_SEL + kMaxTopK * 4;     // float [2][4 warps][kN]
constexpr uint32_t OFF_SCAN = OFF_RED + 2 * 4 * kN * 4;  // uint32 [8] + misc
constexpr uint32_t OFF_HMASK = OFF_SCAN + 64;            // uint8 [kMaxTopK]: heads per slot
constexpr uint32_t OFF_SEL2 = OFF_HMASK + kMaxTopK;      // int32 [kMaxTopK]: kept groups
constexpr uint32_t OFF_SIDX = OFF_SEL2 + kMaxTopK * 4;    // uint8 [256]: sorted candidate indices
constexpr uint32_t OFF_BARS = OFF_SIDX + 256;
constexpr uint32_t kSmemBytes = OFF_BARS + 256 + 1024;

enum {
  B_KF = 0, B_KE = 3, B_VF = 6, B_VE = 8, B_SF = 10, B_SE = 12, B_PF = 14, B_PD = 16, B_MX = 17,
  B_GS = 18, B_QR = 19, B_SELD = 20, B_DRAIN = 21, B_SEL2 = 22, kNumBars = 23
};

constexpr uint32_t kTmemCols = 64;  // S^T buffers at 0 and 16, O^T at 32
constexpr uint32_t kTmemO = 32;

// Order-preserving map of a float to an unsigned key (0 is below every float).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Arrive-and-wait of the 128 softmax threads on one mbarrier (bounded).
struct GroupSync {
  uint64_t* bar;
  uint32_t phase;
  volatile int* abort;
  DeviceStatus* st;
  __device__ bool operator()(int where) {
    mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase & 1u, abort, st, where);
    ++phase;
    return ok;
  }
};

// Block-wide exclusive prefix sum over the 128 softmax threads (t = 0..127);
// returns the exclusive prefix, *total the sum.
__device__ __forceinline__ uint32_t group_exclusive_scan(uint32_t v, int t, uint32_t* buf,
                                                         GroupSync& gs, bool& ok,
                                                         uint32_t* total) {
  const int lane = t & 31, w = t >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) buf[w] = x;
  ok = ok && gs(40);
  uint32_t before = 0, sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t tw = buf[i];
    if (i < w) before += tw;
    sum += tw;
  }
  ok = ok && gs(41);  // buf may be reused after this
  *total = sum;
  return before + x - v;
}

}  // namespace dec

using namespace dec;

template <int REP, bool HIER>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + kNumBars) + 1;
  int32_t* sel_s = reinterpret_cast<int32_t*>(smem + OFF_SEL);
  int32_t* sel2_s = reinterpret_cast<int32_t*>(smem + OFF_SEL2);
  uint8_t* hmask_s = smem + OFF_HMASK;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % P.Hkv, seq = blockIdx.x / P.Hkv;
  const int nb = P.nG + P.nW + (HIER ? P.nB1 : 0) + P.nC;
  DeviceStatus* st = P.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bar[B_KF + s], 1);
      mbar_init(&bar[B_KE + s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bar[B_VF + s], 1);
      mbar_init(&bar[B_VE + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_SF + s], 1);
      mbar_init(&bar[B_SE + s], 128);
      mbar_init(&bar[B_PF + s], 128);
    }
    mbar_init(&bar[B_PD], 1);
    mbar_init(&bar[B_MX], 128);
    mbar_init(&bar[B_GS], 128);
    mbar_init(&bar[B_QR], 128);
    mbar_init(&bar[B_SELD], 128);
    mbar_init(&bar[B_SEL2], 128);
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
      prefetch_tmap(&P.gk);
      prefetch_tmap(&P.gv);
      prefetch_tmap(&P.ck);
      prefetch_tmap(&P.cv);
      prefetch_tmap(&P.ckc);
      prefetch_tmap(&P.cvc);
      if (HIER) {
        prefetch_tmap(&P.g1k);
        prefetch_tmap(&P.g1v);
      }
      const int ws = P.cache_len - P.window;
      const int cpb = kBlk / P.chunk;  // chunks per block
      int last_k = -1, last_v = -1;
      // block b of K (is_k) or V into its ring slot; false on timeout
      auto load = [&](bool is_k, int b) -> bool {
        const int ns = is_k ? kKStages : kVStages, s = b % ns;
        if (!mbar_wait(&bar[(is_k ? B_KE : B_VE) + s], ((b / ns) & 1) ^ 1, abort, st, 1))
          return false;
        uint8_t* dst = smem + (is_k ? OFF_K : OFF_V) + s * kTileBytes;
        uint64_t* full = &bar[(is_k ? B_KF : B_VF) + s];
        mbar_arrive_expect_tx(full, kTileBytes);
        int kind, idx;  // block kind and its index within the kind
        if constexpr (HIER) {
          const BlockOf bo(P, b);
          kind = bo.kind;
          idx = bo.idx;
        } else {
          kind = b < P.nG ? BK_GIST : (b < P.nG + P.nW ? BK_WIN : BK_CHUNK);
          idx = b < P.nG ? b : (b < P.nG + P.nW ? b - P.nG : b - P.nG - P.nW);
        }
        if (kind == BK_GIST || kind == BK_WIN) {  // a gist block or a window block
          const bool gist = kind == BK_GIST;
          const int row0 = gist ? idx * kBlk : ws + idx * kBlk;
          const CUtensorMap* map = gist ? (is_k ? &P.gk : &P.gv) : (is_k ? &P.ck : &P.cv);
          for (int at = 0; at < 2; ++at) tma_load_4d(dst + at * kAtom, map, full, at * 64, g, row0, seq);
        } else if (HIER && kind == BK_L1) {
          // the level-1 gists of 128 / fanout kept groups, one box per group
          const int gpb = kBlk / P.fanout;
          const CUtensorMap* map = is_k ? &P.g1k : &P.g1v;
          for (int i = 0; i < gpb; ++i) {
            const int slot = idx * gpb + i;
            // an empty slot loads group 0 (finite values; its keys are masked)
            const int c = (slot < P.top_k2 && sel2_s[slot] >= 0) ? sel2_s[slot] : 0;
            const uint32_t roff = (uint32_t)(i * P.fanout) * 128u;
            for (int at = 0; at < 2; ++at)
              tma_load_4d(dst + at * kAtom + roff, map, full, at * 64, g, c * P.fanout, seq);
          }
        } else {
          const int cb = idx;
          const CUtensorMap* map = is_k ? &P.ckc : &P.cvc;
          for (int i = 0; i < cpb; ++i) {
            const int slot = cb * cpb + i;
            // an empty slot loads chunk 0 (finite values; its keys are masked)
            const int c = (slot < P.n_slots && sel_s[slot] >= 0) ? sel_s[slot] : 0;
            const uint32_t roff = (uint32_t)(i * P.chunk) * 128u;
            for (int at = 0; at < 2; ++at)
              tma_load_4d(dst + at * kAtom + roff, map, full, at * 64, g, c * P.chunk, seq);
          }
        }
        if (is_k) last_k = b; else last_v = b;
        return true;
      };
      // K runs up to kKAhead blocks ahead of V. A chunk block's K needs the
      // selection: it is prefetched only once the selection is known, and
      // waited for only when it is the K of the current block (by then every
      // earlier V has been requested, so the softmax can reach the selection).
      bool ok = true, seld = P.nC == 0, sel2d = !HIER || P.nB1 == 0;
      int nk = 0;
      const int chunk0 = P.nG + P.nW + (HIER ? P.nB1 : 0);  // first chunk block
      for (int b = 0; ok && b < nb; ++b) {
        while (ok && nk < nb && nk <= b + kKAhead) {
          if (HIER && !sel2d && BlockOf(P, nk).kind == BK_L1) {  // needs the kept groups
            if (nk > b) break;
            if (!mbar_wait(&bar[B_SEL2], 0, abort, st, 5)) {
              ok = false;
              break;
            }
            sel2d = true;
          }
          if (nk >= chunk0 && !seld) {
            if (nk > b) break;
            if (!mbar_wait(&bar[B_SELD], 0, abort, st, 2)) {
              ok = false;
              break;
            }
            seld = true;
          }
          ok = load(true, nk++);
        }
        if (ok) ok = load(false, b);
      }
      // every copy this CTA started must land before the CTA may exit
      volatile int no_abort = 0;
      for (int s = 0; s < kKStages; ++s)
        if (last_k >= s) {
          const int bs = last_k - ((last_k - s) % kKStages);
          mbar_wait(&bar[B_KF + s], (bs / kKStages) & 1, &no_abort, nullptr, 3);
        }
      for (int s = 0; s < kVStages; ++s)
        if (last_v >= s) {
          const int bs = last_v - ((last_v - s) % kVStages);
          mbar_wait(&bar[B_VF + s], (bs / kVStages) & 1, &no_abort, nullptr, 4);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdQK = idesc_bf16_f32(kBlk, kN, false, false);
      constexpr uint32_t kIdPV = idesc_bf16_f32(kD, kN, true, false);
      bool ok = mbar_wait(&bar[B_QR], 0, abort, st, 10);
      for (int b = 0; ok && b <= nb; ++b) {
        if (b < nb) {
          const int s = b & 1, sk = b % kKStages;
          if (!mbar_wait(&bar[B_KF + sk], (b / kKStages) & 1, abort, st, 11) ||
              !mbar_wait(&bar[B_SE + s], ((b >> 1) & 1) ^ 1, abort, st, 12))
            break;
          tc_fence_after();
          const uint32_t kb = sb + OFF_K + sk * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(kb + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024);
            const uint64_t bd =
                smem_desc_sw128(sb + OFF_QT + (kk >> 2) * kQtAtom + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem + s * kN, ad, bd, kIdQK, kk > 0);
          }
          mma_commit(&bar[B_SF + s]);
          mma_commit(&bar[B_KE + sk]);
        }
        if (b >= 1) {
          const int bp = b - 1, s = bp & 1, sv = bp % kVStages;
          if (!mbar_wait(&bar[B_VF + sv], (bp / kVStages) & 1, abort, st, 15) ||
              !mbar_wait(&bar[B_PF + s], (bp >> 1) & 1, abort, st, 13))
            break;
          tc_fence_after();
          const uint32_t vb = sb + OFF_V + sv * kTileBytes;
          const uint32_t pb = sb + OFF_PT + s * 2 * kQtAtom;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk) {
            // A = V^T (dims x keys, dims contiguous), B = P^T (heads x keys, keys contiguous)
            const uint64_t ad = smem_desc_sw128(vb + kk * 2048, kAtom, 1024);
            const uint64_t bd = smem_desc_sw128(pb + (kk >> 2) * kQtAtom + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem + kTmemO, ad, bd, kIdPV, (bp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_PD]);
          mma_commit(&bar[B_VE + sv]);
        }
      }
      mma_commit(&bar[B_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[B_DRAIN], 0, &no_abort, nullptr, 14);
    }
  } else {
    // ------------------------------------------- softmax, selection, epilogue
    const int sw = warp - 2;                // softmax warp 0..3
    const int quarter = warp & 3;           // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;      // key row of a block / output dimension
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    GroupSync gs{&bar[B_GS], 0u, abort, st};
    float* scores = reinterpret_cast<float*>(smem + OFF_SCORE);
    float* red = reinterpret_cast<float*>(smem + OFF_RED);  // [2][4][kN]
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + OFF_HIST);
    uint32_t* scan = reinterpret_cast<uint32_t*>(smem + OFF_SCAN);

    // Q^T of the group (rows >= REP zero) and zeroed P^T buffers
    for (int x = r; x < kN * (kD / 8); x += 128) {
      const int h = x >> 4, c0 = (x & 15) * 8;
      uint32_t w4[4] = {0u, 0u, 0u, 0u};
      if (h < REP) {
        const __nv_bfloat16* qp = P.q + seq * P.qs[0] + (int64_t)(g * REP + h) * P.qs[1] + c0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w4[i] = pack_bf16(__bfloat162float(qp[2 * i]), __bfloat162float(qp[2 * i + 1]));
      }
      st_shared_v4(sb + OFF_QT + (c0 >> 6) * kQtAtom + sw128_offset(h, c0 & 63), w4[0], w4[1],
                   w4[2], w4[3]);
    }
    for (int x = r; x < (int)(2 * 2 * kQtAtom / 16); x += 128)
      st_shared_v4(sb + OFF_PT + x * 16, 0u, 0u, 0u, 0u);
    fence_async_shared();
    mbar_arrive(&bar[B_QR]);

    const float sl2 = P.scale * 1.4426950408889634f;
    float m_run[REP], l_part[REP];
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    const int wstart = P.cache_len - P.window, cpb = kBlk / P.chunk;
    bool ok = true;
    for (int b = 0; b < nb; ++b) {
      const int s = b & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_SF + s], (b >> 1) & 1, abort, st, 20))) {
        ok = false;
        break;
      }
      tc_fence_after();
      __syncwarp();
      float sv[kN];
      tmem_ld16(lane_addr + s * kN, sv);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar[B_SE + s]);
      bool valid;
      uint32_t hv = 0xFFFFFFFFu;  // heads that see this key (unfolded chunks of one head)
      int kind, idx;  // block kind and its index within the kind
      if constexpr (HIER) {
        const BlockOf bo(P, b);
        kind = bo.kind;
        idx = bo.idx;
      } else {
        kind = b < P.nG ? BK_GIST : (b < P.nG + P.nW ? BK_WIN : BK_CHUNK);
        idx = b < P.nG ? b : (b < P.nG + P.nW ? b - P.nG : b - P.nG - P.nW);
      }
      if (kind == BK_GIST) {
        const int key = idx * kBlk + r;
        valid = key < P.G;
        if (valid && (P.rule == SA_SELECT_SUM_PROBS_PER_GROUP || P.rule == SA_SELECT_TOP_K_PER_HEAD)) {
          float* lg = P.logits + (int64_t)(seq * P.Hkv + g) * REP * P.G + key;
#pragma unroll
          for (int h = 0; h < REP; ++h) lg[(int64_t)h * P.G] = sv[h];
        } else if (valid) {  // selection score: sum over the group's heads of q_h . k * scale
          float sum = 0.f;
#pragma unroll
          for (int h = 0; h < REP; ++h) sum += sv[h];
          scores[key] = sum * P.scale;
        }
      } else if (kind == BK_WIN) {
        valid = wstart + idx * kBlk + r < P.cache_len;
      } else if (HIER && kind == BK_L1) {
        // candidate c = 128 idx + r: level-1 gist c % fanout of kept group slot c / fanout
        const int slot = (idx * kBlk + r) / P.fanout;
        valid = slot < P.top_k2 && sel2_s[slot] >= 0;
        if (valid) {
          float sum = 0.f;
#pragma unroll
          for (int h = 0; h < REP; ++h) sum += sv[h];
          scores[idx * kBlk + r] = sum * P.scale;
        }
      } else {
        const int slot = idx * cpb + r / P.chunk;
        valid = slot < P.n_slots && sel_s[slot] >= 0;
        if (valid && P.rule == SA_SELECT_TOP_K_PER_HEAD) hv = hmask_s[slot];
      }
      // block maximum per head over the four softmax warps
      float* rb = red + s * 4 * kN;
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        float v = (valid && ((hv >> h) & 1u)) ? sv[h] : -INFINITY;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        if (lane == 0) rb[sw * kN + h] = v;
      }
      mbar_arrive(&bar[B_MX]);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_MX], b & 1, abort, st, 21))) {
        ok = false;
        break;
      }
      float alpha[REP], pv[REP];
      bool any_resc = false;
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        const float M = fmaxf(fmaxf(rb[h], rb[kN + h]), fmaxf(rb[2 * kN + h], rb[3 * kN + h]));
        const float m_new = fmaxf(m_run[h], M * sl2);  // scale > 0 keeps the order
        const bool resc = m_new > m_run[h] + 8.f;       // the same in every thread
        const float m_use = resc ? m_new : m_run[h];
        alpha[h] = !resc ? 1.f : (m_run[h] == -INFINITY ? 0.f : ex2(m_run[h] - m_use));
        pv[h] = (valid && ((hv >> h) & 1u) && m_use != -INFINITY) ? ex2(fmaf(sv[h], sl2, -m_use))
                                                                  : 0.f;
        l_part[h] = l_part[h] * alpha[h] + pv[h];
        m_run[h] = m_use;
        any_resc = any_resc || resc;
      }
      // P V(b - 1) is done: P^T buffer s (read by P V(b - 2)) is free, O^T is quiet
      if (b >= 1 &&
          !__all_sync(0xffffffffu, mbar_wait(&bar[B_PD], (b - 1) & 1, abort, st, 22))) {
        ok = false;
        break;
      }
      if (any_resc && b >= 1) {
        tc_fence_after();
        __syncwarp();
        float o[kN];
        tmem_ld16(lane_addr + kTmemO, o);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < REP; ++h) o[h] *= alpha[h];
        tmem_st16(lane_addr + kTmemO, o);
        tmem_wait_st();
      }
      uint8_t* pt = smem + OFF_PT + s * 2 * kQtAtom + (r >> 6) * kQtAtom;
#pragma unroll
      for (int h = 0; h < REP; ++h)
        *reinterpret_cast<__nv_bfloat16*>(pt + sw128_offset(h, r & 63)) = __float2bfloat16_rn(pv[h]);
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(&bar[B_PF + s]);

      // selection points: flat decode, the chunks after the gist blocks; gist of
      // gists, the groups after the level-2 blocks and the chunks after the
      // kept groups' level-1 blocks
      const bool sel_groups = HIER && b == P.nG - 1 && P.top_k2 > 0;
      const bool sel_chunks = P.top_k > 0 && b == (HIER ? P.nG + P.nW1 + P.nB1 - 1 : P.nG - 1);
      if (sel_groups || sel_chunks) {
        // ---------------------------------------------------- top-k select
        // mode 0: chunks by their gists (flat); 1: groups by their level-2
        // gists; 2: chunks among the kept groups' level-1 gists (candidate c is
        // level-1 gist c % fanout of kept group slot c / fanout)
        const int mode = !HIER ? 0 : (sel_groups ? 1 : 2);
        const int sel_n = mode == 2 ? P.nB1 * kBlk : P.G;
        const int sel_k = mode == 1 ? P.top_k2 : P.top_k;
        int32_t* sel_dst = mode == 1 ? sel2_s : sel_s;
        // thread r owns candidates [r * per, r * per + per): ascending index
        // order across threads, so an exclusive scan keeps the output ascending
        __threadfence_block();
        ok = ok && gs(30);  // every score (or logit) is written
        const int per = (sel_n + 127) / 128, j0 = r * per, j1 = min(sel_n, j0 + per);
        // Thread r visits its candidates starting at offset lane % per, so that
        // at per = 32 the lanes of a warp read 32 different banks of scores[]
        // (in index order every lane would read the same bank).
        const int o_first = per > 0 ? lane % per : 0;
        auto o_next = [&](int o) -> int { return o + 1 == per ? 0 : o + 1; };
        // sum or max over the 128 softmax threads (hist serves as scratch)
        auto group_reduce = [&](float v, bool is_max) -> float {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float y = __shfl_xor_sync(0xffffffffu, v, off);
            v = is_max ? fmaxf(v, y) : v + y;
          }
          float* buf = reinterpret_cast<float*>(hist);
          if (lane == 0) buf[sw] = v;
          ok = ok && gs(42);
          const float t = is_max ? fmaxf(fmaxf(buf[0], buf[1]), fmaxf(buf[2], buf[3]))
                                 : (buf[0] + buf[1]) + (buf[2] + buf[3]);
          ok = ok && gs(43);  // buf may be reused after this
          return t;
        };
        if (P.rule == SA_SELECT_SUM_PROBS_PER_GROUP) {
          // each head's softmax over all gists: the state after the gist blocks
          float inv_l[REP];
#pragma unroll
          for (int h = 0; h < REP; ++h) {
            const float l = group_reduce(l_part[h], false);
            inv_l[h] = l > 0.f ? 1.f / l : 0.f;
          }
          const float* lg = P.logits + (int64_t)(seq * P.Hkv + g) * REP * P.G;
          for (int t = 0, o = o_first; t < per; ++t, o = o_next(o)) {
            const int j = j0 + o;
            if (j >= j1) continue;
            float sum = 0.f;
#pragma unroll
            for (int h = 0; h < REP; ++h)
              sum += ex2(fmaf(lg[(int64_t)h * P.G + j], sl2, -m_run[h])) * inv_l[h];
            scores[j] = sum;
          }
        }
        const int64_t last_ok = (int64_t)P.cache_len - P.window;
        // a chunk (group) is eligible iff all its raw tokens lie before the
        // window; a candidate iff its group slot holds a kept group
        auto key_of = [&](int j) -> uint32_t {
          bool e;
          if (mode == 0) {
            e = (int64_t)(j + 1) * P.chunk <= last_ok;
          } else if (mode == 1) {
            e = (int64_t)(j + 1) * P.fanout * P.chunk <= last_ok;
          } else {
            const int sl = j / P.fanout;
            e = sl < P.top_k2 && sel2_s[sl] >= 0;
          }
          return e ? float_key(scores[j]) : 0u;
        };
        auto value_of = [&](int j) -> int32_t {
          return mode == 2 ? sel2_s[j / P.fanout] * P.fanout + j % P.fanout : j;
        };
        // top_k through a short list (per <= 32, sel_k <= 128): the thread's
        // keys are read once into registers, and the threshold comes from
        // ranking at most 128 listed candidates instead of radix passes, whose
        // shared-memory histogram serializes on the few bins that similar
        // scores share. Same result as the radix path; returns false (having
        // written nothing) when the list would exceed 128 entries, and the
        // radix path runs instead.
        auto list_select = [&](uint32_t& total) __attribute__((always_inline)) -> bool {
          uint32_t kr[32];  // slot t: candidate j0 + o_t, o_t = (o_first + t) mod per
          uint32_t n_elig = 0u, mx = 0u;
          {
            int o = o_first;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const uint32_t k = (t < per && j0 + o < j1) ? key_of(j0 + o) : 0u;
              kr[t] = k;
              n_elig += k != 0u ? 1u : 0u;
              mx = max(mx, k);
              o = o_next(o);
            }
          }
          // T0 <= the sel_k-th largest key: the sel_k-th largest thread
          // maximum (sel_k threads hold a key >= it). Each warp sorts its 32
          // maxima (bitonic, descending, in registers) into hist; a maximum's
          // rank among all 128 is its lane plus a binary search in each other
          // warp's list (ties: the lower warp first).
          uint32_t v = mx;
#pragma unroll
          for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
              const uint32_t y = __shfl_xor_sync(0xffffffffu, v, stride);
              const bool lower = (lane & stride) == 0;
              const bool desc = (lane & size) == 0 || size == 32;
              v = (lower == desc) ? max(v, y) : min(v, y);
            }
          }
          hist[sw * 32 + lane] = v;
          // the eligible total in the same exchange
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) n_elig += __shfl_xor_sync(0xffffffffu, n_elig, off);
          if (lane == 0) scan[8 + sw] = n_elig;
          ok = ok && gs(48);
          const uint32_t E = scan[8] + scan[9] + scan[10] + scan[11];
          uint32_t T = 0u, want = 0u;
          if (E > (uint32_t)sel_k) {
            // with at most 128 eligible keys every one is on the list
            uint32_t T0 = 1u;
            if (E > 128u) {
              uint32_t rank = (uint32_t)lane;
#pragma unroll
              for (int w2 = 0; w2 < 4; ++w2) {
                if (w2 == sw) continue;
                const uint32_t* L = hist + w2 * 32;
                // entries ranked above v (e > v, or e == v in a lower warp): a
                // prefix of the descending list, found a bit at a time
                int pos = 0;
#pragma unroll
                for (int step = 16; step >= 1; step >>= 1) {
                  const uint32_t e = L[pos + step - 1];
                  if (e > v || (e == v && w2 < sw)) pos += step;
                }
                if (pos == 31 && (L[31] > v || (L[31] == v && w2 < sw))) pos = 32;
                rank += (uint32_t)pos;
              }
              if (rank == (uint32_t)sel_k - 1u) scan[6] = v;
              ok = ok && gs(49);
              T0 = max(scan[6], 1u);
            }
            uint32_t nc = 0u;
#pragma unroll
            for (int t = 0; t < 32; ++t) nc += kr[t] >= T0 ? 1u : 0u;
            uint32_t C = 0u;
            // (its barriers also order the reads of hist above before the writes below)
            uint32_t pos = group_exclusive_scan(nc, r, scan, gs, ok, &C);
            if (C > 128u) return false;
            uint32_t* ckey = hist;        // the list, padded with zero keys to a
            uint32_t* cidx = hist + 128;  // multiple of 4 entries
            {
              int o = o_first;
#pragma unroll
              for (int t = 0; t < 32; ++t) {
                if (kr[t] >= T0) {
                  ckey[pos] = kr[t];
                  cidx[pos] = (uint32_t)(j0 + o);
                  ++pos;
                }
                o = o_next(o);
              }
            }
            const int C4 = ((int)C + 3) >> 2;
            if (r >= (int)C && r < 4 * C4) ckey[r] = 0u;
            ok = ok && gs(50);
            // rank by (key descending, index ascending): the entry of rank
            // sel_k - 1 is the threshold T; want = how many keys equal to T to take
            if (r < (int)C) {
              const uint32_t key = ckey[r], idx = cidx[r];
              const uint4* k4 = reinterpret_cast<const uint4*>(ckey);
              const uint4* i4 = reinterpret_cast<const uint4*>(cidx);
              uint32_t rank = 0u, gt = 0u;
#pragma unroll 4
              for (int c = 0; c < C4; ++c) {
                const uint4 kk = k4[c], ii = i4[c];
                gt += (kk.x > key ? 1u : 0u) + (kk.y > key ? 1u : 0u) + (kk.z > key ? 1u : 0u) +
                      (kk.w > key ? 1u : 0u);
                rank += (kk.x == key && ii.x < idx ? 1u : 0u) + (kk.y == key && ii.y < idx ? 1u : 0u) +
                        (kk.z == key && ii.z < idx ? 1u : 0u) + (kk.w == key && ii.w < idx ? 1u : 0u);
              }
              rank += gt;
              if (rank == (uint32_t)sel_k - 1u) {
                scan[4] = key;
                scan[5] = (uint32_t)sel_k - gt;
              }
            }
            ok = ok && gs(51);
            T = scan[4];
            want = scan[5];
          }
          // take key > T, and the first `want` keys equal to T in index order;
          // bit o of the masks is candidate j0 + o. One scan of the packed
          // counts (equal << 16 | greater) gives both prefixes: the threads
          // before r take min(want, equal keys before r) of the equal keys.
          uint32_t gtm = 0u, eqm = 0u;
          {
            int o = o_first;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const uint32_t bit = t < per ? 1u << o : 0u;
              gtm |= kr[t] > T ? bit : 0u;
              eqm |= (kr[t] == T && kr[t] != 0u) ? bit : 0u;
              o = o_next(o);
            }
          }
          const uint32_t n_eq = (uint32_t)__popc(eqm);
          uint32_t tot = 0u;
          const uint32_t pre = group_exclusive_scan((n_eq << 16) | (uint32_t)__popc(gtm), r, scan, gs,
                                                    ok, &tot);
          const uint32_t eq_before = pre >> 16;
          const uint32_t take_eq = want > eq_before ? min(n_eq, want - eq_before) : 0u;
          for (uint32_t u = 0; u < take_eq; ++u) {
            const uint32_t low = eqm & (0u - eqm);
            gtm |= low;
            eqm ^= low;
          }
          uint32_t off = (pre & 0xFFFFu) + min(want, eq_before);
          const uint32_t sel_total = (tot & 0xFFFFu) + min(want, tot >> 16);
          while (gtm != 0u) {
            const int o = __ffs(gtm) - 1;
            gtm &= gtm - 1u;
            if (off < (uint32_t)sel_k) sel_dst[off++] = value_of(j0 + o);
          }
          for (int x = r; x < sel_k; x += 128)
            if (x >= (int)sel_total) sel_dst[x] = -1;
          ok = ok && gs(35);
          total = sel_total;
          return true;
        };
        // top_k of scores[] into sel_s (ascending, -1 padded); returns the
        // number of eligible chunks taken
        // top_k of at most 256 candidates (one or two per thread: the
        // gist-of-gists selections, small flat decodes). Each warp sorts its
        // 64 candidates in registers (bitonic, descending by key, ties to the
        // lower index) into shared memory; a candidate's rank is its position
        // in its warp's list plus a binary search in each other warp's list.
        // Five group barriers, where the radix passes take about twenty; same
        // result.
        auto small_select = [&]() __attribute__((always_inline)) -> uint32_t {
          uint8_t* sidx = smem + OFF_SIDX;
          uint32_t* flags = scan + 8;  // 256 bits: the taken candidates
          // (key, 255 - index) packed: descending order is key descending,
          // then index ascending; absent or ineligible candidates are 0
          uint64_t x[2];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int j = j0 + t;
            const uint32_t key = (t < per && j < j1) ? key_of(j) : 0u;
            x[t] = key ? ((uint64_t)key << 32) | (uint32_t)(255 - j) : 0ull;
          }
#pragma unroll
          for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
              if (stride == 1) {  // both elements of the pair are this lane's
                const bool desc = ((2 * lane) & size) == 0;
                const uint64_t hi = x[0] > x[1] ? x[0] : x[1], lo = x[0] > x[1] ? x[1] : x[0];
                x[0] = desc ? hi : lo;
                x[1] = desc ? lo : hi;
              } else {
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                  const int e = 2 * lane + t;
                  const uint32_t yl = __shfl_xor_sync(0xffffffffu, (uint32_t)x[t], stride >> 1);
                  const uint32_t yh = __shfl_xor_sync(0xffffffffu, (uint32_t)(x[t] >> 32), stride >> 1);
                  const uint64_t y = ((uint64_t)yh << 32) | yl;
                  const bool keep_max = ((e & stride) == 0) == ((e & size) == 0);
                  x[t] = keep_max ? (x[t] > y ? x[t] : y) : (x[t] > y ? y : x[t]);
                }
              }
            }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            hist[sw * 64 + 2 * lane + t] = (uint32_t)(x[t] >> 32);
            sidx[sw * 64 + 2 * lane + t] = (uint8_t)(uint32_t)x[t];
          }
          if (r < 8) flags[r] = 0u;
          ok = ok && gs(53);
          // entries of list w2 ranked above x[t]: a prefix of the descending
          // list, found a bit at a time; the six searches (two elements, three
          // other lists) advance together so that their loads overlap
          auto above = [&](int w2, int i, uint64_t v) -> bool {
            const uint32_t k2 = hist[w2 * 64 + i];
            return k2 != 0u && (((uint64_t)k2 << 32) | sidx[w2 * 64 + i]) > v;
          };
          int pos[2][3] = {{0, 0, 0}, {0, 0, 0}};
#pragma unroll
          for (int step = 32; step >= 1; step >>= 1) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
              for (int u = 0; u < 3; ++u) {
                const int w2 = u + (u >= sw ? 1 : 0);
                if (above(w2, pos[t][u] + step - 1, x[t])) pos[t][u] += step;
              }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (x[t] == 0ull) continue;
            uint32_t rank = (uint32_t)(2 * lane + t);
#pragma unroll
            for (int u = 0; u < 3; ++u) {
              const int w2 = u + (u >= sw ? 1 : 0);
              rank += (uint32_t)(pos[t][u] == 63 && above(w2, 63, x[t]) ? 64 : pos[t][u]);
            }
            if (rank < (uint32_t)sel_k) {
              const int j = 255 - (int)(uint32_t)(x[t] & 0xffu);
              atomicOr(&flags[j >> 5], 1u << (j & 31));
            }
          }
          ok = ok && gs(54);
          uint32_t take = 0u, cnt = 0u;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int j = j0 + t;
            if (t < per && j < j1 && ((flags[j >> 5] >> (j & 31)) & 1u)) {
              take |= 1u << t;
              ++cnt;
            }
          }
          uint32_t sel_total = 0u;
          uint32_t off = group_exclusive_scan(cnt, r, scan, gs, ok, &sel_total);
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if ((take >> t) & 1u) sel_dst[off++] = value_of(j0 + t);
          for (int x2 = r; x2 < sel_k; x2 += 128)
            if (x2 >= (int)sel_total) sel_dst[x2] = -1;
          ok = ok && gs(35);  // (also orders hist's and the flags' reads before their next writes)
          return sel_total;
        };
        auto radix_select = [&]() __attribute__((always_inline)) -> uint32_t {
        if (per <= 2) return small_select();
        if constexpr (!HIER) {
          if (per >= 8 && per <= 32 && sel_k <= 128) {
            uint32_t total = 0u;
            if (list_select(total)) return total;
          }
        }
        uint32_t n_elig = 0;
        for (int j = j0; j < j1; ++j) n_elig += key_of(j) != 0u;
        uint32_t E = 0;
        group_exclusive_scan(n_elig, r, scan, gs, ok, &E);
        // threshold T and the number of keys equal to T to take (lowest indices)
        uint32_t T = 0u, want = 0u;
        if (E > (uint32_t)sel_k) {
          uint32_t prefix = 0u, pmask = 0u;
          want = (uint32_t)sel_k;
          for (int pass = 0; pass < 4 && ok; ++pass) {
            const int shift = 24 - 8 * pass;
            hist[r] = 0u;
            hist[r + 128] = 0u;
            ok = ok && gs(31);
            for (int j = j0; j < j1; ++j) {
              const uint32_t k = key_of(j);
              if (k != 0u && (k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
            }
            ok = ok && gs(32);
            if (sw == 0) {
              // lane l sums bins [8l, 8l + 8); suffix over lanes from the top
              uint32_t c8 = 0u;
#pragma unroll
              for (int i = 0; i < 8; ++i) c8 += hist[8 * lane + i];
              uint32_t suf = c8;
#pragma unroll
              for (int off = 1; off < 32; off <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32) suf += y;
              }
              const uint32_t mask = __ballot_sync(0xffffffffu, suf >= want);
              const int L = 31 - __clz(mask);  // highest lane whose suffix reaches want
              if (lane == L) {
                uint32_t above = suf - c8;  // keys in bins above this lane's
                int B = 8 * lane;
                for (int bb = 8 * lane + 7; bb >= 8 * lane; --bb) {
                  if (above + hist[bb] >= want) {
                    B = bb;
                    break;
                  }
                  above += hist[bb];
                }
                scan[4] = (uint32_t)B;
                scan[5] = want - above;
              }
            }
            ok = ok && gs(33);
            prefix |= scan[4] << shift;
            pmask |= 0xFFu << shift;
            want = scan[5];
            ok = ok && gs(34);  // scan[4..5] and hist are rewritten by the next pass
          }
          T = prefix;
        }
        // take key > T, and the first `want` keys equal to T in index order
        uint32_t n_gt = 0u, n_eq = 0u;
        for (int j = j0; j < j1; ++j) {
          const uint32_t k = key_of(j);
          n_gt += k > T;
          n_eq += (k == T && k != 0u);
        }
        uint32_t eq_total = 0u, sel_total = 0u;
        const uint32_t eq_before = group_exclusive_scan(n_eq, r, scan, gs, ok, &eq_total);
        const uint32_t take_eq = want > eq_before ? min(n_eq, want - eq_before) : 0u;
        uint32_t off = group_exclusive_scan(n_gt + take_eq, r, scan, gs, ok, &sel_total);
        uint32_t eq_seen = 0u;
        for (int j = j0; j < j1; ++j) {
          const uint32_t k = key_of(j);
          const bool take = k > T || (k == T && k != 0u && eq_seen++ < take_eq);
          if (take && off < (uint32_t)sel_k) sel_dst[off++] = value_of(j);
        }
        for (int x = r; x < sel_k; x += 128)
          if (x >= (int)sel_total) sel_dst[x] = -1;
        ok = ok && gs(35);
        return sel_total;
        };
        if (P.rule == SA_SELECT_TOP_K_PER_HEAD) {
          // each query head's own top_k from its logits, written to its row of
          // sel; then the union of the group's chunks (ascending) into sel_s
          // with, per slot, the heads that chose it
          const float* lg = P.logits + (int64_t)(seq * P.Hkv + g) * REP * P.G;
          int32_t* hsel = P.sel + (int64_t)(seq * P.Hkv + g) * REP * P.top_k;
          for (int h = 0; h < REP; ++h) {
            for (int t = 0, o = o_first; t < per; ++t, o = o_next(o))
              if (j0 + o < j1) scores[j0 + o] = lg[(int64_t)h * P.G + j0 + o] * P.scale;
            radix_select();
            for (int x = r; x < P.top_k; x += 128) hsel[h * P.top_k + x] = sel_s[x];
            __threadfence_block();
            ok = ok && gs(44);  // scores and sel_s are rewritten by the next head
          }
          uint32_t* bm = reinterpret_cast<uint32_t*>(scores);  // [REP][W] chunk bitmaps
          const int W = (P.G + 31) / 32;
          for (int x = r; x < REP * W; x += 128) bm[x] = 0u;
          ok = ok && gs(45);
          for (int x = r; x < REP * P.top_k; x += 128) {
            const int c = hsel[x];
            if (c >= 0) atomicOr(&bm[(x / P.top_k) * W + (c >> 5)], 1u << (c & 31));
          }
          ok = ok && gs(46);
          const int wper = (W + 127) / 128, w0 = r * wper, w1 = min(W, w0 + wper);
          uint32_t cnt = 0u;
          for (int w = w0; w < w1; ++w) {
            uint32_t u = 0u;
#pragma unroll
            for (int h = 0; h < REP; ++h) u |= bm[h * W + w];
            cnt += __popc(u);
          }
          uint32_t n_union = 0u;
          uint32_t pos = group_exclusive_scan(cnt, r, scan, gs, ok, &n_union);
          for (int w = w0; w < w1; ++w) {
            uint32_t u = 0u;
#pragma unroll
            for (int h = 0; h < REP; ++h) u |= bm[h * W + w];
            while (u != 0u && pos < (uint32_t)P.n_slots) {
              const int bit = __ffs(u) - 1;
              u &= u - 1u;
              uint32_t hm = 0u;
#pragma unroll
              for (int h = 0; h < REP; ++h) hm |= ((bm[h * W + w] >> bit) & 1u) << h;
              sel_s[pos] = w * 32 + bit;
              hmask_s[pos] = (uint8_t)hm;
              ++pos;
            }
          }
          for (int x = r; x < P.n_slots; x += 128)
            if (x >= (int)n_union) sel_s[x] = -1;
          ok = ok && gs(47);
        } else {
        const uint32_t sel_total = radix_select();
        const int nsel = min((int)sel_total, sel_k);
        if (P.rule == SA_SELECT_TOP_P_PER_GROUP && nsel > 0) {
          // softmax over the eligible chunks (the best score is among the
          // selected); selected entry x is kept iff the probability of the
          // entries ranked above it (score descending, lower index first) is
          // below p: the shortest prefix reaching p. Thread r decides for
          // entries 2r and 2r + 1, so a scan keeps the ascending order.
          float smax = -INFINITY;
          for (int x = r; x < nsel; x += 128) smax = fmaxf(smax, scores[sel_s[x]]);
          smax = group_reduce(smax, true);
          float z = 0.f;
          for (int t = 0, o = o_first; t < per; ++t, o = o_next(o))
            if (j0 + o < j1 && key_of(j0 + o) != 0u) z += __expf(scores[j0 + o] - smax);
          const float thr = P.top_p * group_reduce(z, false);
          int val[2];
          uint32_t nk = 0u;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int x = 2 * r + u;
            val[u] = -1;
            if (x < nsel) {
              const float sx = scores[sel_s[x]];
              float above = 0.f;
              for (int y = 0; y < nsel; ++y) {
                const float sy = scores[sel_s[y]];
                if (sy > sx || (sy == sx && y < x)) above += __expf(sy - smax);
              }
              if (above < thr) val[nk++] = sel_s[x];
            }
          }
          uint32_t kept = 0u;
          const uint32_t base = group_exclusive_scan(nk, r, scan, gs, ok, &kept);
          for (uint32_t u = 0; u < nk; ++u) sel_s[base + u] = val[u];
          for (int x = r; x < P.top_k; x += 128)
            if (x >= (int)kept) sel_s[x] = -1;
          ok = ok && gs(39);
        }
        int32_t* sel_out = mode == 1 ? P.sel2 + ((int64_t)seq * P.Hkv + g) * P.top_k2
                                     : P.sel + ((int64_t)seq * P.Hkv + g) * P.top_k;
        for (int x = r; x < sel_k; x += 128) sel_out[x] = sel_dst[x];
        }
        mbar_arrive(&bar[mode == 1 ? B_SEL2 : B_SELD]);  // release: the selection is complete
        if (!__all_sync(0xffffffffu, ok)) break;
      }
    }
    // -------------------------------------------------------------- epilogue
    if (ok && nb > 0 &&
        __all_sync(0xffffffffu, mbar_wait(&bar[B_PD], (nb - 1) & 1, abort, st, 23))) {
      float* lr = red + (nb & 1) * 4 * kN;  // the slot no thread reads any more
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        float v = l_part[h];
#pragma unroll
        for (int off2 = 16; off2 > 0; off2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off2);
        if (lane == 0) lr[sw * kN + h] = v;
      }
      if (gs(36)) {
        tc_fence_after();
        __syncwarp();
        float o[kN];
        tmem_ld16(lane_addr + kTmemO, o);  // lane = output dimension r
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          const float l = (lr[h] + lr[kN + h]) + (lr[2 * kN + h] + lr[3 * kN + h]);
          const int hq = g * REP + h;
          P.o[seq * P.os[0] + (int64_t)hq * P.os[1] + r] =
              __float2bfloat16_rn(l > 0.f ? o[h] / l : 0.f);
          if (r == 0)
            P.lse[(int64_t)seq * P.Hkv * REP + hq] =
                l > 0.f ? (m_run[h] + __log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// --------------------------------------------------------------- host side
// Shapes this kernel takes: 8 <= chunk <= 128 dividing 128 (a chunk is whole
// 8-row swizzle groups of a block), at least one full block of gists and of
// cache positions (TMA boxes of 128 rows), and whatever check_decode admits.
bool decode_tc_supported(const sa_decode_desc& d) {
  return d.head_dim == kD && d.chunk >= 8 && d.chunk <= kBlk && kBlk % d.chunk == 0 &&
         d.n_gists >= kBlk && d.n_gists <= kMaxG && d.cache_len >= kBlk &&
         d.top_k <= kMaxTopK && d.num_q_heads / d.num_kv_heads <= 8 &&
         (d.select_rule != SA_SELECT_TOP_K_PER_HEAD ||
          d.num_q_heads / d.num_kv_heads * d.top_k <= kMaxTopK);
}

template <int REP, bool HIER>
static cudaError_t decode_tc_launch(const Params& P, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<REP, HIER>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  decode_tc_kernel<REP, HIER><<<dim3(P.n_seq * P.Hkv), kThreads, kSmemBytes, s>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_decode_tc(const sa_decode_desc& d, const void* q, const void* gk,
                             const void* gv, const void* kc, const void* vc, int32_t* sel, void* o,
                             float* lse, void* ws, float* logits, cudaStream_t s) {
  Params P;
  memset(&P, 0, sizeof(P));
  const int64_t gstr[3] = {d.gist_strides[0], d.gist_strides[2], d.gist_strides[1]};
  const int64_t cstr[3] = {d.cache_strides[0], d.cache_strides[2], d.cache_strides[1]};
  if (!make_tile_map_box(&P.gk, gk, kD, d.num_kv_heads, d.n_gists, d.n_seq, gstr, kBlk) ||
      !make_tile_map_box(&P.gv, gv, kD, d.num_kv_heads, d.n_gists, d.n_seq, gstr, kBlk) ||
      !make_tile_map_box(&P.ck, kc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, kBlk) ||
      !make_tile_map_box(&P.cv, vc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, kBlk) ||
      !make_tile_map_box(&P.ckc, kc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, d.chunk) ||
      !make_tile_map_box(&P.cvc, vc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, d.chunk))
    return cudaErrorInvalidValue;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.o = static_cast<__nv_bfloat16*>(o);
  P.lse = lse;
  P.sel = sel;
  P.logits = logits;
  P.rule = d.select_rule;
  P.top_p = d.top_p;
  P.status = static_cast<DeviceStatus*>(ws);
  P.n_seq = d.n_seq;
  P.Hkv = d.num_kv_heads;
  P.rep = d.num_q_heads / d.num_kv_heads;
  P.G = d.n_gists;
  P.cache_len = d.cache_len;
  P.chunk = d.chunk;
  P.top_k = d.top_k;
  P.window = d.window;
  P.nG = (d.n_gists + kBlk - 1) / kBlk;
  P.nW = (d.window + kBlk - 1) / kBlk;
  const int cpb = kBlk / d.chunk;
  P.n_slots = d.select_rule == SA_SELECT_TOP_K_PER_HEAD ? P.rep * d.top_k : d.top_k;
  P.nC = (P.n_slots + cpb - 1) / cpb;
  P.scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.f / sqrtf((float)d.head_dim);
  for (int i = 0; i < 2; ++i) {
    P.qs[i] = d.q_strides[i];
    P.os[i] = d.o_strides[i];
  }
  switch (P.rep) {
    case 1: return decode_tc_launch<1, false>(P, s);
    case 2: return decode_tc_launch<2, false>(P, s);
    case 4: return decode_tc_launch<4, false>(P, s);
    case 8: return decode_tc_launch<8, false>(P, s);
    default: return cudaErrorInvalidValue;
  }
}

// ------------------------------------------------- gist of gists, host side
// Shapes the tensor-core kernel takes for the two-level decode: whole 8-row
// swizzle groups per chunk and per group of level-1 gists, a full 128-row box
// of level-2 gists and of cache positions, and the selection buffers' bounds.
bool hier_tc_supported(const sa_hier_decode_desc& d) {
  const int rep = d.num_q_heads / d.num_kv_heads;
  const int n2 = d.fanout > 0 ? d.n_gists / d.fanout : 0;
  return d.head_dim == kD && d.chunk >= 8 && d.chunk <= kBlk && kBlk % d.chunk == 0 &&
         d.fanout >= 8 && d.fanout <= kBlk && kBlk % d.fanout == 0 && n2 >= kBlk && n2 <= kMaxG &&
         d.cache_len >= kBlk && d.top_k <= kMaxTopK && d.top_k2 <= kMaxTopK &&
         d.top_k2 * d.fanout <= kMaxG && (rep == 1 || rep == 2 || rep == 4 || rep == 8);
}

cudaError_t launch_hier_decode_tc(const sa_hier_decode_desc& d, const void* q, const void* g2k,
                                  const void* g2v, const void* gk, const void* gv, const void* kc,
                                  const void* vc, int32_t* sel2, int32_t* sel1, void* o, float* lse,
                                  void* ws, cudaStream_t s) {
  Params P;
  memset(&P, 0, sizeof(P));
  const int n2 = d.n_gists / d.fanout;
  const int64_t g2str[3] = {d.gist2_strides[0], d.gist2_strides[2], d.gist2_strides[1]};
  const int64_t gstr[3] = {d.gist_strides[0], d.gist_strides[2], d.gist_strides[1]};
  const int64_t cstr[3] = {d.cache_strides[0], d.cache_strides[2], d.cache_strides[1]};
  if (!make_tile_map_box(&P.gk, g2k, kD, d.num_kv_heads, n2, d.n_seq, g2str, kBlk) ||
      !make_tile_map_box(&P.gv, g2v, kD, d.num_kv_heads, n2, d.n_seq, g2str, kBlk) ||
      !make_tile_map_box(&P.g1k, gk, kD, d.num_kv_heads, d.n_gists, d.n_seq, gstr, d.fanout) ||
      !make_tile_map_box(&P.g1v, gv, kD, d.num_kv_heads, d.n_gists, d.n_seq, gstr, d.fanout) ||
      !make_tile_map_box(&P.ck, kc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, kBlk) ||
      !make_tile_map_box(&P.cv, vc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, kBlk) ||
      !make_tile_map_box(&P.ckc, kc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, d.chunk) ||
      !make_tile_map_box(&P.cvc, vc, kD, d.num_kv_heads, d.cache_len, d.n_seq, cstr, d.chunk))
    return cudaErrorInvalidValue;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.o = static_cast<__nv_bfloat16*>(o);
  P.lse = lse;
  P.sel = sel1;
  P.sel2 = sel2;
  P.rule = SA_SELECT_SUM_LOGITS_PER_GROUP;
  P.top_p = 1.f;
  P.status = static_cast<DeviceStatus*>(ws);
  P.n_seq = d.n_seq;
  P.Hkv = d.num_kv_heads;
  P.rep = d.num_q_heads / d.num_kv_heads;
  P.G = n2;
  P.cache_len = d.cache_len;
  P.chunk = d.chunk;
  P.top_k = d.top_k;
  P.window = d.window;
  P.fanout = d.fanout;
  P.top_k2 = d.top_k2;
  P.nG = (n2 + kBlk - 1) / kBlk;
  P.nW = (d.window + kBlk - 1) / kBlk;
  P.nW1 = (P.nW + 1) / 2;  // half the window loads while the groups are selected
  P.nB1 = (d.top_k2 * d.fanout + kBlk - 1) / kBlk;
  P.n_slots = d.top_k;
  P.nC = (d.top_k + kBlk / d.chunk - 1) / (kBlk / d.chunk);
  P.scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.f / sqrtf((float)d.head_dim);
  for (int i = 0; i < 2; ++i) {
    P.qs[i] = d.q_strides[i];
    P.os[i] = d.o_strides[i];
  }
  switch (P.rep) {
    case 1: return decode_tc_launch<1, true>(P, s);
    case 2: return decode_tc_launch<2, true>(P, s);
    case 4: return decode_tc_launch<4, true>(P, s);
    case 8: return decode_tc_launch<8, true>(P, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
