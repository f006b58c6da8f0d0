// Block-sparse attention forward on the 5th-generation tensor cores (sm_100a).
//
// For one (128-query tile, head, sequence) per CTA, the listed 128-key tiles
// are visited in order; everything else is skipped ("UniGist ...", Approach:
// skipping non-visible blocks is what makes the sparse layout fast; "Gzip-
// guided sparse attention ...", Scope: dense-then-mask gives no speed-up).
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then K_j / V_j into a 2-stage ring
//               (128-byte swizzled, 64-column atoms), and TMEM allocation.
//   warp 1      one thread issues tcgen05.mma: S_j = Q K_j^T into one of two
//               TMEM S buffers, then O += P_j V_j into the TMEM O accumulator.
//               Completion is signalled with tcgen05.commit on mbarriers.
//   warps 2-5   softmax: thread t owns query row t (TMEM lane t). It reads its
//               S row, applies the element mask on MASKED/TAIL tiles, keeps a
//               running max in the log2 domain and rescales its O row only
//               when the max grew by more than 2^8 (the reference max is kept
//               otherwise, so P <= 256), writes P (bf16) into a swizzled
//               shared tile and hands it to the MMA thread. The epilogue
//               divides O by the row sum and writes O (bf16) and LSE (fp32).
// S is double-buffered so that S_{j+1} = Q K_{j+1}^T runs on the tensor core
// while the softmax of tile j runs. Every wait is bounded; on timeout the
// device status word is set and all roles leave after draining their copies
// and MMAs, freeing TMEM.
#include <cuda.h>

#include "attn_mask.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

struct FwdTcParams {
  CUtensorMap tmq, tmk, tmv;
  CUtensorMap tmkc, tmvc;  // gist mode: sinks + gists compacted in logical order
  AttnArgs a;
  MaskArgs m;
};

// Internal tile kind: only the first `cnt` columns hold keys (the last tile of
// the compacted sink/gist keys).
constexpr int kTileCount = 3;

// The CTA's visit list, the same in every role. Gzip mode: the tile list of
// (sequence, head class, query tile). Gist mode: the dense prefix of the
// compacted sink/gist keys that lie below the near tiles, then the near tiles
// Jlo..I of the physical sequence, which take the element rule.
struct WorkList {
  int gist, e0, n, nft, nf, jlo;
  __device__ void init(const MaskArgs& m, int list, int I) {
    gist = m.kind == SA_MASK_GIST;
    if (gist) {
      jlo = max(0, I - (m.window - 1 + kTile - 1) / kTile);
      nf = m.far_ptr[jlo];
      nft = (nf + kTile - 1) / kTile;
      n = nft + (I - jlo + 1);
      e0 = 0;
    } else {
      e0 = m.trp[list * (m.T + 1) + I];
      n = m.trp[list * (m.T + 1) + I + 1] - e0;
      nft = nf = jlo = 0;
    }
  }
  // source (0 = sequence, 1 = compacted keys), first key row, kind, valid columns
  __device__ void entry(const MaskArgs& m, int it, int& src, int& k0, int& kind, int& cnt) const {
    if (gist) {
      if (it < nft) {
        src = 1;
        k0 = it * kTile;
        cnt = min(kTile, nf - k0);
        kind = cnt == kTile ? SA_TILE_FULL : kTileCount;
      } else {
        src = 0;
        k0 = (jlo + it - nft) * kTile;
        kind = SA_TILE_MASKED;
        cnt = kTile;
      }
    } else {
      src = 0;
      k0 = m.tcol[e0 + it] * kTile;
      kind = m.tkind[e0 + it] == SA_TILE_FULL ? SA_TILE_FULL : SA_TILE_MASKED;
      cnt = kTile;
    }
  }
};

template <int D>
struct FwdLayout {
  static constexpr uint32_t kQ = 128 * D * 2;       // Q tile
  static constexpr uint32_t kKV = 128 * D * 2;      // one K or V tile
  static constexpr uint32_t kP = 128 * 128 * 2;     // one P tile
  static constexpr uint32_t kAtom = 128 * 128;      // [128 rows][64 bf16] swizzle atom
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k0 = kQ;
  static constexpr uint32_t v0 = kQ + 2 * kKV;
  static constexpr uint32_t p0 = kQ + 4 * kKV;
  static constexpr uint32_t bars = p0 + 2 * kP;    // 16 mbarriers + TMEM slot + flags
  static constexpr uint32_t bytes = bars + 256 + 1024;  // + alignment slack
};

enum { B_Q = 0, B_KVF = 1, B_KVE = 3, B_SF = 5, B_SE = 7, B_PF = 9, B_OD = 11, B_DRAIN = 13 };

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

template <int D>
__global__ void __launch_bounds__(192, 1) fwd_tc_kernel(const __grid_constant__ FwdTcParams P) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 16);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + 16) + 1;

  const AttnArgs& a = P.a;
  const MaskArgs& m = P.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = m.T;
  // late query tiles (long lists) of every head and sequence first
  const int hb = a.Hq * a.Bt;
  const int I = T - 1 - (int)(blockIdx.x / hb);
  const int h = (int)(blockIdx.x % hb) % a.Hq, bt = (int)(blockIdx.x % hb) / a.Hq;
  const int hk = h / (a.Hq / a.Hkv);
  const int list = list_of(m, bt, h);
  WorkList wl;
  wl.init(m, list, I);
  const int n = wl.n;
  const int q0 = I * kTile;
  DeviceStatus* st = a.status;

  if (threadIdx.x == 0) {
    mbar_init(&bar[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_KVF + s], 1);
      mbar_init(&bar[B_KVE + s], 1);
      mbar_init(&bar[B_SF + s], 1);
      mbar_init(&bar[B_SE + s], 128);
      mbar_init(&bar[B_PF + s], 128);
      mbar_init(&bar[B_OD + s], 1);
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
      if (wl.gist) {
        prefetch_tmap(&P.tmkc);
        prefetch_tmap(&P.tmvc);
      }
      mbar_arrive_expect_tx(&bar[B_Q], L::kQ);
      for (int at = 0; at < D / 64; ++at)
        tma_load_4d(smem + L::q + at * L::kAtom, &P.tmq, &bar[B_Q], at * 64, h, q0, bt);
      int last[2] = {-1, -1};
      for (int it = 0; it < n; ++it) {
        const int s = it & 1;
        if (!mbar_wait(&bar[B_KVE + s], ((it >> 1) & 1) ^ 1, abort, st, 1)) break;
        int src, k0, kind, cnt;
        wl.entry(m, it, src, k0, kind, cnt);
        const CUtensorMap* mk = src ? &P.tmkc : &P.tmk;
        const CUtensorMap* mv = src ? &P.tmvc : &P.tmv;
        mbar_arrive_expect_tx(&bar[B_KVF + s], 2 * L::kKV);
        for (int at = 0; at < D / 64; ++at) {
          tma_load_4d(smem + L::k0 + s * L::kKV + at * L::kAtom, mk, &bar[B_KVF + s], at * 64, hk,
                      k0, bt);
          tma_load_4d(smem + L::v0 + s * L::kKV + at * L::kAtom, mv, &bar[B_KVF + s], at * 64, hk,
                      k0, bt);
        }
        last[s] = it;
      }
      // every copy this CTA started must land before the CTA may exit
      volatile int no_abort = 0;
      mbar_wait(&bar[B_Q], 0, &no_abort, nullptr, 2);
      for (int s = 0; s < 2; ++s)
        if (last[s] >= 0) mbar_wait(&bar[B_KVF + s], (last[s] >> 1) & 1, &no_abort, nullptr, 3);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(&bar[B_Q], 0, abort, st, 10);
      for (int it = 0; ok && it <= n; ++it) {
        if (it < n) {
          const int s = it & 1;
          if (!mbar_wait(&bar[B_KVF + s], (it >> 1) & 1, abort, st, 11)) break;
          if (!mbar_wait(&bar[B_SE + s], ((it >> 1) & 1) ^ 1, abort, st, 12)) break;
          tc_fence_after();
          const uint32_t kbase = sb + L::k0 + s * L::kKV;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
            mma_bf16(tmem + s * 128, smem_desc_sw128(sb + L::q + off, 16, 1024),
                     smem_desc_sw128(kbase + off, 16, 1024), kIdQK, kk > 0);
          }
          mma_commit(&bar[B_SF + s]);
        }
        if (it >= 1) {
          const int j = it - 1, s = j & 1;
          if (!mbar_wait(&bar[B_PF + s], (j >> 1) & 1, abort, st, 13)) break;
          tc_fence_after();
          const uint32_t pbase = sb + L::p0 + s * L::kP;
          const uint32_t vbase = sb + L::v0 + s * L::kKV;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = smem_desc_sw128(pbase + (kk >> 2) * L::kAtom + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(vbase + kk * 2048, L::kAtom, 1024);
            mma_bf16(tmem + kTmemO, ad, bd, kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_OD + s]);
          mma_commit(&bar[B_KVE + s]);
        }
      }
      // drain: every MMA issued above has completed
      mma_commit(&bar[B_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[B_DRAIN], 0, &no_abort, nullptr, 14);
    }
  } else {
    // --------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int p = q0 + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    const int gzip = m.kind == SA_MASK_GZIP;
    const uint32_t* rowbits = nullptr;
    int li = 0;
    if (gzip && p < a.N) rowbits = m.bits + ((int64_t)list * m.B + p / m.b) * m.words;
    if (!gzip && p < a.N) li = m.perm[p];
    const int lb = (gzip && m.b < kTile) ? __ffs(m.b) - 1 : 0;  // b < 128 is a power of two
    // Every tcgen05.ld/st below is warp-collective: the branches around them
    // are made warp-uniform with __all_sync / __any_sync.
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int s = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_SF + s], (it >> 1) & 1, abort, st, 20))) {
        ok = false;
        break;
      }
      tc_fence_after();
      __syncwarp();  // tcgen05.ld is warp-collective (.sync.aligned)
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + s * 128 + c * 32, x + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar[B_SE + s]);

      int src, kbase, kind, cnt;
      wl.entry(m, it, src, kbase, kind, cnt);
      // The branch taken depends only on CTA-uniform values (kind, src,
      // kbase); rows past the end of the sequence are handled inside each.
      const bool row_ok = p < a.N;
      // scores stay unscaled here; the scale is folded into the exponent
      if (kind == SA_TILE_FULL && (src || kbase + kTile <= a.N)) {
        if (!row_ok) {
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = -INFINITY;
        }
      } else if (kind == kTileCount) {
        // compacted sink/gist keys, all visible: only the first cnt columns exist
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c < cnt && row_ok) ? x[c] : -INFINITY;
      } else if (gzip) {
        // this row's block bits over the key tile, then the causal cut
        if (m.b >= kTile) {
          const int jb = kbase / m.b;  // the whole key tile lies in one block
          const bool blk = row_ok && ((rowbits[jb >> 5] >> (jb & 31)) & 1u);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            x[c] = (blk && kbase + c <= p && kbase + c < a.N) ? x[c] : -INFINITY;
        } else if (lb >= 2) {
          const int kb0 = kbase >> lb;  // 128 / b <= 32 blocks, inside one word
          const uint32_t bb = row_ok ? (rowbits[kb0 >> 5] >> (kb0 & 31)) : 0u;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            x[c] = (((bb >> (c >> lb)) & 1u) && kbase + c <= p && kbase + c < a.N) ? x[c]
                                                                                   : -INFINITY;
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const int kq = kbase + c, jb = kq >> lb;
            const bool v = row_ok && kq <= p && kq < a.N && ((rowbits[jb >> 5] >> (jb & 31)) & 1u);
            x[c] = v ? x[c] : -INFINITY;
          }
        }
      } else {
        // gist near tile: each lane fetches 4 column codes (logical position |
        // always-visible bit), shared across the warp with shuffles
        int32_t cw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kq = kbase + 32 * j + lane;
          int32_t code = 0x3FFFFFFF;  // no key: never visible
          if (kq < a.N) {
            const int lj = m.perm[kq];
            const bool always = lj < m.sinks || ((m.gist_bits[lj >> 5] >> (lj & 31)) & 1u);
            code = lj | (always ? 0x40000000 : 0);
          }
          cw[j] = code;
        }
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int code = __shfl_sync(0xffffffffu, cw[c >> 5], c & 31);
          const int lj = code & 0x3FFFFFFF;
          const bool v = row_ok && lj <= li && ((code & 0x40000000) || li - lj < m.window);
          x[c] = v ? x[c] : -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, x[c]);
      const float m_new = fmaxf(m_run, mx * sl2);  // scale > 0 keeps the order
      const bool resc = m_new > m_run + 8.f;  // true on the first finite max
      const float m_use = resc ? m_new : m_run;
      float rowsum = 0.f;
      uint32_t pk[64];
      if (m_use == -INFINITY) {
#pragma unroll
        for (int c = 0; c < 64; ++c) pk[c] = 0u;
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ex2(fmaf(x[2 * c], sl2, -m_use));
          const float p1 = ex2(fmaf(x[2 * c + 1], sl2, -m_use));
          rowsum += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
      }
      const float alpha = !resc ? 1.f : (m_run == -INFINITY ? 0.f : ex2(m_run - m_use));
      // P tile s was last read by PV(it - 2)
      if (it >= 2 &&
          !__all_sync(0xffffffffu, mbar_wait(&bar[B_OD + s], ((it - 2) >> 1) & 1, abort, st, 21))) {
        ok = false;
        break;
      }
      if (it >= 1 && __any_sync(0xffffffffu, resc)) {
        // O must not be accumulated while it is rescaled: wait for PV(it-1).
        // The whole warp takes part; rows that keep their max use alpha = 1.
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_OD + ((it - 1) & 1)], ((it - 1) >> 1) & 1,
                                                abort, st, 22))) {
          ok = false;
          break;
        }
        tc_fence_after();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(lane_addr + kTmemO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(lane_addr + kTmemO + c * 32, o);
        }
        tmem_wait_st();
      }
      l_run = l_run * alpha + rowsum;
      m_run = m_use;
      const uint32_t prow = sb + L::p0 + s * L::kP;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {  // 16 chunks of 8 columns
        const int col = ch * 8;
        const uint32_t addr = prow + (col >> 6) * L::kAtom + sw128_offset(r, col & 63);
        st_shared_v4(addr, pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(&bar[B_PF + s]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && n > 0 &&
        __all_sync(0xffffffffu,
                   mbar_wait(&bar[B_OD + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort, st, 23))) {
      tc_fence_after();
      __syncwarp();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + bt * a.os[0] +
                            (int64_t)p * a.os[1] + (int64_t)h * a.os[2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(lane_addr + kTmemO + c * 32, o);  // all lanes: collective
        tmem_wait_ld();
        if (p < a.N) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16(o[v * 8 + 0] * inv, o[v * 8 + 1] * inv);
            w.y = pack_bf16(o[v * 8 + 2] * inv, o[v * 8 + 3] * inv);
            w.z = pack_bf16(o[v * 8 + 4] * inv, o[v * 8 + 5] * inv);
            w.w = pack_bf16(o[v * 8 + 6] * inv, o[v * 8 + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = w;
          }
        }
      }
      if (p < a.N)
        a.lse[((int64_t)bt * a.Hq + h) * a.N + p] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
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

// [Bt, N, H, d] bf16 with element strides {batch, seq, head}; box 64 x 1 x 128 x 1.
bool make_tile_map(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                     const int64_t* s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t sh = s[2] > 0 ? s[2] : d, sn = s[1];
  const int64_t sbat = (Bt > 1) ? s[0] : sn * N;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)Bt};
  cuuint64_t strides[3] = {(cuuint64_t)(sh * 2), (cuuint64_t)(sn * 2), (cuuint64_t)(sbat * 2)};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

template <int D>
static cudaError_t fwd_tc_launch(const AttnArgs& a, const MaskArgs& m, void* compact,
                                 cudaStream_t s) {
  FwdTcParams P;
  memset(&P, 0, sizeof(P));
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
    gist_gather_kernel<D><<<dim3((a.N + 7) / 8, a.Bt), 256, 0, s>>>(a, m, kc, vc);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  P.a = a;
  P.m = m;
  const int bytes = (int)FwdLayout<D>::bytes;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes);
  if (e != cudaSuccess) return e;
  fwd_tc_kernel<D><<<dim3(m.T * a.Hq * a.Bt), 192, bytes, s>>>(P);
  return cudaGetLastError();
}

// `compact`: gist mode only, 2 * Bt * N * Hkv * d bf16 of workspace.
cudaError_t launch_fwd_tc(int d, const AttnArgs& a, const MaskArgs& m, void* compact,
                          cudaStream_t s) {
  if (d == 64) return fwd_tc_launch<64>(a, m, compact, s);
  if (d == 128) return fwd_tc_launch<128>(a, m, compact, s);
  return cudaErrorInvalidValue;
}

}  // namespace sa
