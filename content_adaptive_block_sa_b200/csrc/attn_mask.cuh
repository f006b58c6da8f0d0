// Element mask and list addressing shared by the attention kernels.
// Internal header.
#pragma once

#include "sa_common.cuh"

namespace sa {

constexpr int kMaxHeads = 256;

// Everything an attention kernel needs to know about the mask.
struct MaskArgs {
  int kind;                 // SA_MASK_GZIP / SA_MASK_GIST
  int T;                    // query/key tiles
  const int32_t* trp;       // tile CSR row pointers  [lists*(T+1)]
  const int32_t* tcol;      // key tiles
  const int8_t* tkind;      // kinds
  const int32_t* tcp;       // tile CSC pointers      [lists*(T+1)]
  const int32_t* trow;      // query tiles
  const int8_t* tkind_t;
  // gzip
  const uint32_t* bits;     // [batch*3*B*words]
  int B, b, words;
  int wb;                   // window w in blocks
  // gzip, b = 64, tensor-core forward ("pair mode"): a 128-row query tile
  // holds two 64-row query blocks and a 128-key tile two 64-key blocks.
  // Per list l: P pairs of query blocks pair_q[l * P + k] = qa | qb << 16
  // (qb = 0xffff: none); the visits of pair k are visits[pair_ptr[l * (P + 1)
  // + k] .. pair_ptr[l * (P + 1) + k + 1]) (absolute), each j1 | j2 << 12 |
  // vis << 24 with j2 = 0xfff for none and vis bits (qa sees j1, qb sees j1,
  // qa sees j2, qb sees j2).
  int pair, P;
  const int32_t* pair_q;
  const int32_t* pair_ptr;
  const int32_t* visits;
  // gist
  const int32_t* perm;      // physical -> logical
  const uint32_t* gist_bits;
  const int32_t* far_idx;   // sinks + gists in logical order (physical indices)
  const int32_t* far_ptr;   // [T+1] far keys below each key tile
  int sinks, window;
  int period;               // coarse layout: positions per segment (raw + gists); 0: fine
  uint8_t head_class[kMaxHeads];  // gzip: class of each query head
};

// Pointers, shapes and strides (elements) of one attention call.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const void* dout;
  float* dq;
  float* dk;
  float* dv;
  float* delta;  // [Bt, Hq, N] rowsum(dO * O)
  int Bt, N, Hq, Hkv;
  float scale;
  int64_t qs[3], ks[3], vs[3], os[3];
  DeviceStatus* status;
};

// ---- gist visibility ("UniGist ...", Approach; "A Silver Bullet or a
// Compromise ...", sections 2 and 6). A sink or gist key j is seen by every
// query i >= j; a raw key by the queries of its window (fine layout: i - j <
// window) or of its own segment (coarse layout: segments of `period`
// positions after the sinks). Both are "(unsigned)(i - j) < reach(j)".
__host__ __device__ inline uint32_t gist_reach(bool always, int lj, int sinks, int window,
                                               int period) {
  if (always) return 0x80000000u;
  if (period > 0) return (uint32_t)(sinks + ((lj - sinks) / period + 1) * period - lj);
  return (uint32_t)window;
}

// First key tile that query tile I visits with the element rule: every key
// below it is seen by the whole tile if it is a sink or a gist, else by none
// of it. Fine layout: I - ceil((window - 1) / 128). Coarse layout: the tile
// holding the start of the segment of the tile's first row (I while that row
// is a sink).
__host__ __device__ inline int gist_near_lo(int I, int sinks, int window, int period) {
  if (period > 0) {
    const int p = I * kTile;
    return p < sinks ? I : (sinks + (p - sinks) / period * period) / kTile;
  }
  return max(0, I - (window - 1 + kTile - 1) / kTile);
}

// Bound on the near tiles of one query tile (I - gist_near_lo(I) + 1).
__host__ __device__ inline int gist_near_tiles(int window, int period) {
  if (period > 0) return (period + kTile - 2) / kTile + 1;
  return (window - 1 + kTile - 1) / kTile + 1;
}

// Index of the list used by (batch row, query head).
__device__ __forceinline__ int list_of(const MaskArgs& m, int bt, int h) {
  return m.kind == SA_MASK_GZIP ? bt * 3 + m.head_class[h] : 0;
}

// Is physical key q visible from physical query p (both < N)?
__device__ __forceinline__ bool element_visible(const MaskArgs& m, int list, int p, int q) {
  if (m.kind == SA_MASK_GZIP) {
    if (q > p) return false;
    const uint32_t* row = m.bits + ((int64_t)list * m.B + p / m.b) * m.words;
    const int j = q / m.b;
    return (row[j >> 5] >> (j & 31)) & 1u;
  }
  const int i = m.perm[p], j = m.perm[q];
  const bool g = (m.gist_bits[j >> 5] >> (j & 31)) & 1u;
  return (uint32_t)(i - j) < gist_reach(j < m.sinks || g, j, m.sinks, m.window, m.period);
}

// ---- visibility words of gzip tiles (forward and query-major backward)
// Bits [0, n) set, n clamped to [0, 32] (no branch).
__device__ __forceinline__ uint32_t prefix_bits(int n) {
  const int c = min(max(n, 0), 32);
  return (uint32_t)((1ull << c) - 1ull);
}

// Each set bit of e (nb bits) widened to a run of 2^lb bits (lb <= 4).
__device__ __forceinline__ uint32_t widen_bits(uint32_t e, int lb, int nb) {
  if (lb == 0) return e;
  uint32_t w = 0u;
  const uint32_t run = (1u << (1 << lb)) - 1u;
  for (int i = 0; i < nb; ++i)
    if ((e >> i) & 1u) w |= run << (i << lb);
  return w;
}

// One query row as the mask warp sees it: position, logical position (gist
// layout), in range, and its packed block bits (gzip).
struct RowCtx {
  int p, li;
  bool ok;
  const uint32_t* bits;
};

// Gzip tiles: words w = 0..3 of rows i = 0..3 of one lane (rows lane + 32 i),
// out[w * 128 + lane + 32 i]. Same rule as tile_word, arranged so that every
// bit-word load is issued before any of them is used: rc[i].bits always
// points at valid words (rows past N read some row and are cleared by lim).
__device__ __forceinline__ void gzip_tile_words(const MaskArgs& m, int lb, int N, const RowCtx* rc,
                                                int kbase, int kind, int lane, uint32_t* out) {
  if (kind == SA_TILE_FULL && kbase + kTile <= N) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int w = 0; w < 4; ++w) out[w * 128 + lane + 32 * i] = rc[i].ok ? 0xffffffffu : 0u;
    return;
  }
  int lim[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) lim[i] = rc[i].ok ? min(rc[i].p, N - 1) : -1;
  if (m.b >= kTile || lb >= 5) {
    // one block bit per (row, word): the whole tile (b >= 128) or 32 columns
    uint32_t u[4][4];
    int jb[4];
#pragma unroll
    for (int w = 0; w < 4; ++w)  // clamped: columns past N are cleared by lim anyway
      jb[w] = min(m.B - 1, m.b >= kTile ? kbase / m.b : (kbase + 32 * w) >> lb);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int w = 0; w < 4; ++w) u[i][w] = rc[i].bits[jb[w] >> 5];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t causal = prefix_bits(lim[i] - (kbase + 32 * w) + 1);
        out[w * 128 + lane + 32 * i] = ((u[i][w] >> (jb[w] & 31)) & 1u) ? causal : 0u;
      }
    return;
  }
  // b < 32: 32 >> lb blocks per word, inside one bit word
  const int nb = 32 >> lb;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int cw0 = kbase + 32 * w, kb = min(cw0 >> lb, m.B - 1);  // clamped as above
      const uint32_t e = (rc[i].bits[kb >> 5] >> (kb & 31)) & prefix_bits(nb);
      out[w * 128 + lane + 32 * i] = widen_bits(e, lb, nb) & prefix_bits(lim[i] - cw0 + 1);
    }
}

// ---- visit lists of a query tile (forward and query-major backward)
// Internal tile kind: only the first `cnt` columns hold keys (the last tile of
// the compacted sink/gist keys).
constexpr int kTileCount = 3;

// The visit list of one item, the same in every role. Gzip mode: the tile list
// of (sequence, head class, query tile). Gist mode: the dense prefix of the
// compacted sink/gist keys that lie below the near tiles, then the near tiles
// Jlo..I of the physical sequence, which take the element rule.
struct WorkList {
  int gist, e0, n, nft, nf, jlo;
  __device__ void init(const MaskArgs& m, int list, int I) {
    gist = m.kind == SA_MASK_GIST;
    if (m.pair) {  // I is the pair index
      e0 = m.pair_ptr[list * (m.P + 1) + I];
      n = m.pair_ptr[list * (m.P + 1) + I + 1] - e0;
      nft = nf = jlo = 0;
    } else if (gist) {
      jlo = gist_near_lo(I, m.sinks, m.window, m.period);
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
  // pair mode: first rows of the two 64-key blocks of visit it (the second
  // repeats the first when the visit has one block; its columns are masked)
  __device__ void pair_entry(const MaskArgs& m, int it, int& k0a, int& k0b) const {
    const uint32_t v = (uint32_t)m.visits[e0 + it];
    const int j1 = v & 0xfff, j2 = (v >> 12) & 0xfff;
    k0a = j1 * 64;
    k0b = (j2 == 0xfff ? j1 : j2) * 64;
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

// Visibility of key columns [32w, 32w + 32) of a tile from one row, for gzip
// tiles and compacted sink/gist tiles (gist near tiles take the element rule,
// evaluated with the whole warp in the mask role). Gzip: the row's block bits
// over the tile, then the causal cut ("Gzip-guided sparse attention ...", Core
// equations: M restricted to j <= i). Compacted tiles: the first cnt columns.
__device__ __forceinline__ uint32_t tile_word(const MaskArgs& m, int gzip, int lb, int N,
                                              const RowCtx& rc, int kbase, int kind, int cnt,
                                              int w) {
  if (!rc.ok) return 0u;
  if (!gzip) return kind == SA_TILE_FULL ? 0xffffffffu : prefix_bits(cnt - 32 * w);
  if (kind == SA_TILE_FULL && kbase + kTile <= N) return 0xffffffffu;
  const int cw0 = kbase + 32 * w;
  const uint32_t causal = prefix_bits(min(rc.p, N - 1) - cw0 + 1);
  if (causal == 0u) return 0u;
  if (m.b >= kTile) {
    const int jb = kbase / m.b;  // the whole key tile lies in one block
    return ((rc.bits[jb >> 5] >> (jb & 31)) & 1u) ? causal : 0u;
  }
  if (lb >= 5) {
    const int jb = cw0 >> lb;  // 32 columns lie in one block
    return ((rc.bits[jb >> 5] >> (jb & 31)) & 1u) ? causal : 0u;
  }
  const int kb = cw0 >> lb, nb = 32 >> lb;  // nb blocks inside one bit word
  const uint32_t e = (rc.bits[kb >> 5] >> (kb & 31)) & prefix_bits(nb);
  return widen_bits(e, lb, nb) & causal;
}

}  // namespace sa
