// Block-mask and gist-layout builders (integer work, bit-exact).
//
// Gzip mode ("Gzip-guided sparse attention: Selecting long-range content by
// compressibility", Core equations, mask equation): for every sequence and
// head class, the causal block mask
//   local   = M^local            (i - j <= w, which holds i == j)
//   literal = M^lit U I          (l_i = l_j = 1, or i == j)
//   hybrid  = M^lit U M^local U I
// emitted as CSR (query block -> key blocks), CSC (key block -> query
// blocks), packed bit rows, and 128x128 tile lists with a FULL/MASKED kind.
//
// Gist mode ("UniGist: Towards General and Hardware-aligned Sequence-level
// Long Context Compression", Approach): per logical position a gist bit, the
// per-tile shift permutation (raw tokens first, gists last, both stable) and
// the tile lists of the visibility rule
//   vis(i, j) = j <= i and (j < sinks or gist(j) or i - j < window)
// with FULL / MASKED / TAIL kinds. The segment-wise coarse layout ("A Silver
// Bullet or a Compromise for Full Attention? ...", sections 2 and 6: each
// segment's gists follow all of its raw tokens; full attention inside a
// segment) puts `seg` raw tokens and seg / ratio gists in every period after
// the sinks and replaces the window by the segment:
//   vis(i, j) = j <= i and (j < sinks or gist(j) or segment(i) == segment(j)).
// Both rules read "raw key j is seen by query i iff lo(i) <= j <= i".
//
// Gzip: five CTAs per (sequence, class) pair, one per output (block CSR, block
// CSC, bit rows, tile lists, transposed tile lists); counts become absolute
// offsets with a block-wide scan into fixed per-pair regions, and every list
// is filled by one warp per row (column) with its lanes over the entries.
// Gist: four launches, one warp per 128-position tile in each (bits and
// permutation; row and column counts; one-CTA scans; list fills), so no
// global scratch beyond the output lists is needed.
#include "sa_common.cuh"

namespace sa {

struct GzipBuild {
  const uint8_t* flags;  // [batch, B]
  int B, b, w, N, T, words;
  int64_t region, tregion;  // B(B+1)/2, T(T+1)/2
  int32_t *row_ptr, *col_idx, *col_ptr, *row_idx;
  uint32_t* bits;
  int32_t *trp, *tcol, *tcp, *trow;
  int8_t *tkind, *tkind_t;
};

// M_class[i][j] for j <= i (block units); f is this sequence's flag array.
__device__ __forceinline__ bool block_visible(int cls, const uint8_t* f, int w, int i, int j) {
  const bool loc = (i - j) <= w;
  const bool lit = (i == j) || (f[i] && f[j]);
  return cls == SA_CLASS_LOCAL ? loc : cls == SA_CLASS_LITERAL ? lit : (loc || lit);
}

// Kind of tile pair (I, J), or -1 when it holds no visible token pair
// (b < 128, a power of two: lb = log2 b).
__device__ int gzip_tile_kind(const GzipBuild& p, int lb, int cls, const uint8_t* f, int I, int J) {
  if (J > I) return -1;
  const int q_end = min(p.N, (I + 1) * kTile);
  if (J == I) return (q_end - I * kTile == 1) ? SA_TILE_FULL : SA_TILE_MASKED;
  const int qb0 = (I * kTile) >> lb, qb1 = (q_end - 1) >> lb;
  const int kb0 = (J * kTile) >> lb, kb1 = (min(p.N, (J + 1) * kTile) - 1) >> lb;
  bool any = false, all = true;
  for (int i = qb0; i <= qb1; ++i)
    for (int j = kb0; j <= kb1; ++j) {
      const bool v = block_visible(cls, f, p.w, i, j);
      any |= v;
      all &= v;
    }
  return any ? (all ? SA_TILE_FULL : SA_TILE_MASKED) : -1;
}

// Five roles per (sequence, class) pair, one CTA each (blockIdx.y): 0 the
// CSR block lists, 1 their transpose (CSC), 2 the packed bit rows, 3 the tile
// lists, 4 their transpose. Every role first derives the literal prefix counts
// and the ascending literal blocks from the flags; the block-list entries have
// closed forms in those, so no role reads another role's output.
__global__ void __launch_bounds__(1024) gzip_build_kernel(GzipBuild p) {
  extern __shared__ int32_t smem[];
  const int bc = blockIdx.x, bt = bc / 3, cls = bc % 3, role = blockIdx.y;
  const int B = p.B;
  int32_t* lp = smem;                 // [B+1]: literals in [0, i)
  int32_t* lit_idx = lp + B + 1;      // [B]: ascending literal blocks
  int32_t* rp = lit_idx + B;          // [B+1]: CSR row pointers (absolute)
  int32_t* cp = rp + B + 1;           // [B+1]: CSC column pointers (absolute)
  uint8_t* f = reinterpret_cast<uint8_t*>(cp + B + 1);  // [B]
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    f[i] = p.flags[(int64_t)bt * B + i] ? 1 : 0;
    lp[i + 1] = f[i];
  }
  if (threadIdx.x == 0) lp[0] = 0;
  __syncthreads();
  block_inclusive_scan(lp + 1, B, 0);
  for (int i = threadIdx.x; i < B; i += blockDim.x)
    if (f[i]) lit_idx[lp[i]] = i;
  __syncthreads();
  const int L = lp[B], w = p.w;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int32_t base = (int32_t)(bc * p.region);

  // Entry t of CSR row i (query block i -> ascending key blocks: literal blocks
  // below the window first, then the window lo..i; the literal class: literal
  // blocks up to i, or i alone).
  auto csr_entry = [&](int i, int t) -> int {
    const int lo = max(0, i - w);
    const int nlit = cls == SA_CLASS_LITERAL ? (f[i] ? lp[i + 1] : 0)
                     : (cls == SA_CLASS_HYBRID && f[i] ? lp[lo] : 0);
    return t < nlit ? lit_idx[t] : (cls == SA_CLASS_LITERAL ? i : lo + (t - nlit));
  };
  // Entry t of CSC column j (key block j -> ascending query blocks: the window
  // j..hi, then literal blocks above it; the literal class: literal blocks from
  // j, or j).
  auto csc_entry = [&](int j, int t) -> int {
    const int hi = min(B - 1, j + w);
    if (cls == SA_CLASS_LITERAL) return f[j] ? lit_idx[lp[j] + t] : j;
    return t <= hi - j ? j + t : lit_idx[lp[hi + 1] + (t - (hi - j + 1))];
  };
  // CSR row pointers (roles 0 and 3) and CSC column pointers (roles 1 and 4)
  if (role == 0 || role == 3) {
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
      const int lo = max(0, i - w);
      int cnt;
      if (cls == SA_CLASS_LOCAL) cnt = i - lo + 1;
      else if (cls == SA_CLASS_LITERAL) cnt = f[i] ? lp[i + 1] : 1;
      else cnt = (i - lo + 1) + (f[i] ? lp[lo] : 0);
      rp[i + 1] = cnt;
    }
    if (threadIdx.x == 0) rp[0] = base;
    __syncthreads();
    block_inclusive_scan(rp + 1, B, base);
  }
  if (role == 1 || role == 4) {
    for (int j = threadIdx.x; j < B; j += blockDim.x) {
      const int hi = min(B - 1, j + w);
      int cnt;
      if (cls == SA_CLASS_LOCAL) cnt = hi - j + 1;
      else if (cls == SA_CLASS_LITERAL) cnt = f[j] ? (L - lp[j]) : 1;
      else cnt = (hi - j + 1) + (f[j] ? (L - lp[hi + 1]) : 0);
      cp[j + 1] = cnt;
    }
    if (threadIdx.x == 0) cp[0] = base;
    __syncthreads();
    block_inclusive_scan(cp + 1, B, base);
  }

  if (role == 0) {  // ---- CSR
    int32_t* rpg = p.row_ptr + (int64_t)bc * (B + 1);
    for (int i = threadIdx.x; i <= B; i += blockDim.x) rpg[i] = rp[i];
    for (int i = warp; i < B; i += nwarps) {  // one warp per row, lanes over entries
      int32_t* out = p.col_idx + rp[i];
      const int n = rp[i + 1] - rp[i];
      for (int t = lane; t < n; t += 32) out[t] = csr_entry(i, t);
    }
    return;
  }
  if (role == 1) {  // ---- CSC
    int32_t* cpg = p.col_ptr + (int64_t)bc * (B + 1);
    for (int j = threadIdx.x; j <= B; j += blockDim.x) cpg[j] = cp[j];
    for (int j = warp; j < B; j += nwarps) {
      int32_t* out = p.row_idx + cp[j];
      const int n = cp[j + 1] - cp[j];
      for (int t = lane; t < n; t += 32) out[t] = csc_entry(j, t);
    }
    return;
  }
  if (role == 2) {  // ---- packed bit rows
    uint32_t* bits = p.bits + (int64_t)bc * B * p.words;
    for (int e = threadIdx.x; e < B * p.words; e += blockDim.x) {
      const int i = e / p.words, k = e % p.words;
      uint32_t word = 0;
      for (int t = 0; t < 32; ++t) {
        const int j = k * 32 + t;
        if (j <= i && j < B && block_visible(cls, f, w, i, j)) word |= 1u << t;
      }
      bits[e] = word;
    }
    return;
  }

  // ---- tile lists (role 3: CSR) and their transpose (role 4: CSC); the row
  // pointers are scanned in shared memory, after the block pointers
  const int T = p.T;
  const int32_t tbase = (int32_t)(bc * p.tregion);
  int32_t* tp = cp + B + 1 + (B + 3) / 4;  // [T+1] (after f)
  if (p.b >= kTile) {
    // r whole tiles per block: key tile J of a visited block kb is FULL,
    // except the diagonal tile; tiles of the diagonal block past I are skipped
    const int r = p.b / kTile;
    if (role == 3) {
      for (int I = threadIdx.x; I < T; I += blockDim.x) {
        const int i = I / r;
        tp[I + 1] = (rp[i + 1] - rp[i] - 1) * r + (I - i * r + 1);
      }
      if (threadIdx.x == 0) tp[0] = tbase;
      __syncthreads();
      block_inclusive_scan(tp + 1, T, tbase);
      int32_t* trp = p.trp + (int64_t)bc * (T + 1);
      for (int I = threadIdx.x; I <= T; I += blockDim.x) trp[I] = tp[I];
      for (int I = warp; I < T; I += nwarps) {
        // entry x of the row: block entry x / r (the diagonal block, last in
        // the list, contributes the tiles i r .. I)
        const int i = I / r, ne = rp[i + 1] - rp[i], n = tp[I + 1] - tp[I];
        for (int x = lane; x < n; x += 32) {
          const int k = min(x / r, ne - 1);
          const int J = k < ne - 1 ? csr_entry(i, k) * r + (x % r) : i * r + (x - (ne - 1) * r);
          p.tcol[tp[I] + x] = J;
          p.tkind[tp[I] + x] = (int8_t)(J == I ? SA_TILE_MASKED : SA_TILE_FULL);
        }
      }
    } else {
      for (int J = threadIdx.x; J < T; J += blockDim.x) {
        const int j = J / r;
        tp[J + 1] = (cp[j + 1] - cp[j] - 1) * r + (j * r + r - J);
      }
      if (threadIdx.x == 0) tp[0] = tbase;
      __syncthreads();
      block_inclusive_scan(tp + 1, T, tbase);
      int32_t* tcp = p.tcp + (int64_t)bc * (T + 1);
      for (int J = threadIdx.x; J <= T; J += blockDim.x) tcp[J] = tp[J];
      for (int J = warp; J < T; J += nwarps) {
        // the diagonal block, first in the column list, contributes J .. j r + r - 1
        const int j = J / r, n = tp[J + 1] - tp[J], nd = j * r + r - J;
        for (int x = lane; x < n; x += 32) {
          const int I = x < nd ? J + x : csc_entry(j, 1 + (x - nd) / r) * r + (x - nd) % r;
          p.trow[tp[J] + x] = I;
          p.tkind_t[tp[J] + x] = (int8_t)(I == J ? SA_TILE_MASKED : SA_TILE_FULL);
        }
      }
    }
    return;
  }
  // b < 128 (a power of two): the kind of every tile pair from the flags; one
  // warp per row (column), lanes over 32 candidate tiles at a time, compacted
  // with ballots
  const int lb = __ffs(p.b) - 1;
  const uint32_t below = (1u << lane) - 1u;
  if (role == 3) {
    for (int I = warp; I < T; I += nwarps) {
      int cnt = 0;
      for (int J0 = 0; J0 <= I; J0 += 32) {
        const int J = J0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, J <= I && gzip_tile_kind(p, lb, cls, f, I, J) >= 0));
      }
      if (lane == 0) tp[I + 1] = cnt;
    }
    if (threadIdx.x == 0) tp[0] = tbase;
    __syncthreads();
    block_inclusive_scan(tp + 1, T, tbase);
    int32_t* trp = p.trp + (int64_t)bc * (T + 1);
    for (int I = threadIdx.x; I <= T; I += blockDim.x) trp[I] = tp[I];
    for (int I = warp; I < T; I += nwarps) {
      int n = tp[I];
      for (int J0 = 0; J0 <= I; J0 += 32) {
        const int J = J0 + lane;
        const int k = J <= I ? gzip_tile_kind(p, lb, cls, f, I, J) : -1;
        const uint32_t m = __ballot_sync(0xffffffffu, k >= 0);
        if (k >= 0) {
          p.tcol[n + __popc(m & below)] = J;
          p.tkind[n + __popc(m & below)] = (int8_t)k;
        }
        n += __popc(m);
      }
    }
  } else {
    for (int J = warp; J < T; J += nwarps) {
      int cnt = 0;
      for (int I0 = J; I0 < T; I0 += 32) {
        const int I = I0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, I < T && gzip_tile_kind(p, lb, cls, f, I, J) >= 0));
      }
      if (lane == 0) tp[J + 1] = cnt;
    }
    if (threadIdx.x == 0) tp[0] = tbase;
    __syncthreads();
    block_inclusive_scan(tp + 1, T, tbase);
    int32_t* tcp = p.tcp + (int64_t)bc * (T + 1);
    for (int J = threadIdx.x; J <= T; J += blockDim.x) tcp[J] = tp[J];
    for (int J = warp; J < T; J += nwarps) {
      int n = tp[J];
      for (int I0 = J; I0 < T; I0 += 32) {
        const int I = I0 + lane;
        const int k = I < T ? gzip_tile_kind(p, lb, cls, f, I, J) : -1;
        const uint32_t m = __ballot_sync(0xffffffffu, k >= 0);
        if (k >= 0) {
          p.trow[n + __popc(m & below)] = I;
          p.tkind_t[n + __popc(m & below)] = (int8_t)k;
        }
        n += __popc(m);
      }
    }
  }
}

// ------------------------------------------------------------------ gist
struct GistBuild {
  const uint8_t* flags;  // [N] or null
  int N, T, sinks, ratio, window, tail;
  int seg, period;  // coarse layout: raw tokens and positions per segment; 0: fine
  int64_t tregion;
  uint32_t* gist_bits;
  int32_t* perm;
  int32_t *far_idx, *far_ptr;
  int32_t *trp, *tcol, *tcp, *trow;
  int8_t *tkind, *tkind_t;
};

__device__ __forceinline__ bool is_gist(const uint32_t* gb, int p) {
  return (gb[p >> 5] >> (p & 31)) & 1u;
}

// gists among positions [a, b)
__device__ int count_gists(const uint32_t* gb, int a, int b) {
  int n = 0;
  for (int p = a; p < b;) {
    const int w = p >> 5, lo = p & 31;
    const int hi = min(32, lo + (b - p));
    uint32_t m = gb[w] >> lo;
    if (hi - lo < 32) m &= (1u << (hi - lo)) - 1u;
    n += __popc(m);
    p += hi - lo;
  }
  return n;
}

// first raw (non-gist) position in [a, b), or -1 (one 32-bit word at a time)
__device__ int first_raw(const uint32_t* gb, int a, int b) {
  for (int p = a; p < b;) {
    const int lo = p & 31;
    const int span = min(32 - lo, b - p);
    uint32_t m = ~gb[p >> 5] >> lo;
    if (span < 32) m &= (1u << span) - 1u;
    if (m) return p + __ffs(m) - 1;
    p += span;
  }
  return -1;
}

// Smallest raw key position query i sees (any j <= i at or above it): the
// window's start, or the start of i's segment (0 for sink rows, whose keys
// are all sinks).
__device__ __forceinline__ int raw_lo(const GistBuild& p, int i) {
  if (p.period > 0) return i < p.sinks ? 0 : p.sinks + (i - p.sinks) / p.period * p.period;
  return i - p.window + 1;
}

// Kind of tile pair (I, J) under the gist visibility rule, or -1.
__device__ int gist_tile_kind(const GistBuild& p, int I, int J) {
  if (J > I) return -1;
  const int i_min = I * kTile, i_max = min(p.N, (I + 1) * kTile) - 1;
  const int j0 = J * kTile, j1 = min(p.N, (J + 1) * kTile);  // [j0, j1)
  if (J == I) return (i_max == i_min) ? SA_TILE_FULL : SA_TILE_MASKED;
  const uint32_t* gb = p.gist_bits;
  const int ng = count_gists(gb, j0, j1);
  const bool has_sink = j0 < p.sinks;
  const bool any = has_sink || ng > 0 || j1 - 1 >= raw_lo(p, i_min);
  if (!any) return -1;
  // all pairs visible iff every non-gist, non-sink key is seen by every query
  // (lo is non-decreasing in i: the last row binds)
  const int jr = first_raw(gb, max(j0, p.sinks), j1);
  if (jr < 0 || jr >= raw_lo(p, i_max)) return SA_TILE_FULL;
  // smallest physical column visible to some query of tile I
  const int n_raw = (j1 - j0) - ng;
  int min_col = kTile;
  if (ng > 0) min_col = n_raw;  // gists sit after the raw tokens
  int r = first_raw(gb, j0, min(j1, p.sinks));  // raw sink tokens
  if (r < 0) r = first_raw(gb, max(j0, raw_lo(p, i_min)), j1);  // raw window / segment tokens
  if (r >= 0) min_col = min(min_col, (r - j0) - count_gists(gb, j0, r));
  return (min_col >= kTile - p.tail) ? SA_TILE_TAIL : SA_TILE_MASKED;
}

// Gist bit of logical position pos (< N).
__device__ __forceinline__ bool gist_at(const GistBuild& p, int pos) {
  if (p.flags) return p.flags[pos] != 0;
  if (p.period > 0) return pos >= p.sinks && (pos - p.sinks) % p.period >= p.seg;
  return pos >= p.sinks && ((pos - p.sinks) % (p.ratio + 1)) == p.ratio;
}

// 1. One warp per 128-position tile J: its 4 gist-bit words, its part of the
// shift permutation (raw tokens first, then gists, both in order), and its
// count of keys visible to every later query (sinks and gists) in far_ptr[J + 1].
__global__ void __launch_bounds__(256) gist_tile_kernel(GistBuild p) {
  const int lane = threadIdx.x & 31, J = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (J >= p.T) return;
  const int N = p.N, j0 = J * kTile, n = min(kTile, N - j0);
  uint32_t gw[4];
  int ng = 0, nf = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int pos = j0 + c * 32 + lane;
    const bool ok = pos < N;
    const bool g = ok && gist_at(p, pos);
    gw[c] = __ballot_sync(0xffffffffu, g);
    nf += __popc(__ballot_sync(0xffffffffu, ok && (pos < p.sinks || g)));
    ng += __popc(gw[c]);
    if (lane == 0 && j0 + c * 32 < N) p.gist_bits[(j0 >> 5) + c] = gw[c];
  }
  int before = 0;  // gists of this tile before the current 32-chunk
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int off = c * 32 + lane;
    if (off < n) {
      const int gb = before + __popc(gw[c] & ((1u << lane) - 1u));
      const bool g = (gw[c] >> lane) & 1u;
      p.perm[j0 + (g ? (n - ng) + gb : off - gb)] = j0 + off;
    }
    before += __popc(gw[c]);
  }
  if (lane == 0) p.far_ptr[J + 1] = nf;
}

// 2. One warp per query tile I (row counts) and per key tile J = I (column
// counts) of the tile lists.
__global__ void __launch_bounds__(256) gist_count_kernel(GistBuild p) {
  const int lane = threadIdx.x & 31, X = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (X >= p.T) return;
  int rows = 0, cols = 0;
  for (int J0 = 0; J0 <= X; J0 += 32) {
    const int J = J0 + lane;
    rows += __popc(__ballot_sync(0xffffffffu, J <= X && gist_tile_kind(p, X, J) >= 0));
  }
  for (int I0 = X; I0 < p.T; I0 += 32) {
    const int I = I0 + lane;
    cols += __popc(__ballot_sync(0xffffffffu, I < p.T && gist_tile_kind(p, I, X) >= 0));
  }
  if (lane == 0) {
    p.trp[X + 1] = rows;
    p.tcp[X + 1] = cols;
  }
}

// 3. Counts -> offsets (one CTA: T is at most 2^17).
__global__ void __launch_bounds__(1024) gist_scan_kernel(GistBuild p) {
  if (threadIdx.x == 0) {
    p.trp[0] = 0;
    p.tcp[0] = 0;
    p.far_ptr[0] = 0;
  }
  block_inclusive_scan(p.trp + 1, p.T, 0);
  block_inclusive_scan(p.tcp + 1, p.T, 0);
  block_inclusive_scan(p.far_ptr + 1, p.T, 0);
}

// 4. One warp per tile: the row list of query tile X, the column list of key
// tile X, and the physical index of every sink / gist of tile X at its
// logical-order slot of far_idx.
__global__ void __launch_bounds__(256) gist_fill_kernel(GistBuild p) {
  const int lane = threadIdx.x & 31, X = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (X >= p.T) return;
  const uint32_t below = (1u << lane) - 1u;
  int n = p.trp[X];
  for (int J0 = 0; J0 <= X; J0 += 32) {
    const int J = J0 + lane;
    const int k = J <= X ? gist_tile_kind(p, X, J) : -1;
    const uint32_t m = __ballot_sync(0xffffffffu, k >= 0);
    if (k >= 0) {
      p.tcol[n + __popc(m & below)] = J;
      p.tkind[n + __popc(m & below)] = (int8_t)k;
    }
    n += __popc(m);
  }
  n = p.tcp[X];
  for (int I0 = X; I0 < p.T; I0 += 32) {
    const int I = I0 + lane;
    const int k = I < p.T ? gist_tile_kind(p, I, X) : -1;
    const uint32_t m = __ballot_sync(0xffffffffu, k >= 0);
    if (k >= 0) {
      p.trow[n + __popc(m & below)] = I;
      p.tkind_t[n + __popc(m & below)] = (int8_t)k;
    }
    n += __popc(m);
  }
  const int j0 = X * kTile, nt = min(kTile, p.N - j0);
  const int ng = count_gists(p.gist_bits, j0, j0 + nt);
  int f = p.far_ptr[X], gbefore = 0;
  for (int c = 0; c < kTile / 32; ++c) {
    const int off = c * 32 + lane, pos = j0 + off;
    const bool ok = pos < p.N;
    const bool g = ok && is_gist(p.gist_bits, pos);
    const bool far = ok && (pos < p.sinks || g);
    const uint32_t gmask = __ballot_sync(0xffffffffu, g);
    const uint32_t fmask = __ballot_sync(0xffffffffu, far);
    if (far) {
      const int gb = gbefore + __popc(gmask & below);
      p.far_idx[f + __popc(fmask & below)] = j0 + (g ? (nt - ng) + gb : off - gb);
    }
    f += __popc(fmask);
    gbefore += __popc(gmask);
  }
}

// ------------------------------------------------------------ host launch
cudaError_t launch_gzip_build(const sa_mask_desc& d, const uint8_t* flags,
                              const sa_block_lists& L, cudaStream_t s) {
  GzipBuild p{};
  p.flags = flags;
  p.B = (int)(d.seq_len / d.block_size);
  p.b = d.block_size;
  p.w = d.window;
  p.N = (int)d.seq_len;
  p.T = (p.N + kTile - 1) / kTile;
  p.words = (p.B + 31) / 32;
  p.region = (int64_t)p.B * (p.B + 1) / 2;
  p.tregion = (int64_t)p.T * (p.T + 1) / 2;
  p.row_ptr = L.row_ptr; p.col_idx = L.col_idx; p.col_ptr = L.col_ptr; p.row_idx = L.row_idx;
  p.bits = L.bits;
  p.trp = L.tile_row_ptr; p.tcol = L.tile_col; p.tkind = L.tile_kind;
  p.tcp = L.tile_col_ptr; p.trow = L.tile_row; p.tkind_t = L.tile_kind_t;
  // lp, lit_idx, rp, cp (ints), the flags (bytes, rounded to ints), tile pointers
  const size_t smem = ((size_t)4 * p.B + 3 + (p.B + 3) / 4 + p.T + 1) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gzip_build_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  gzip_build_kernel<<<dim3(d.batch * 3, 5), 1024, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gist_build(const sa_mask_desc& d, const uint8_t* flags,
                              const sa_block_lists& L, cudaStream_t s) {
  GistBuild p{};
  p.flags = flags;
  p.N = (int)d.seq_len;
  p.T = (p.N + kTile - 1) / kTile;
  p.sinks = d.sinks;
  p.ratio = d.gist_ratio;
  p.window = d.window;
  p.seg = d.block_size;
  p.period = d.block_size > 0 ? d.block_size + d.block_size / d.gist_ratio : 0;
  p.tail = d.gist_tail > 0 ? d.gist_tail : 32;
  p.tregion = (int64_t)p.T * (p.T + 1) / 2;
  p.gist_bits = L.gist_bits;
  p.perm = L.perm;
  p.far_idx = L.far_idx;
  p.far_ptr = L.far_ptr;
  p.trp = L.tile_row_ptr; p.tcol = L.tile_col; p.tkind = L.tile_kind;
  p.tcp = L.tile_col_ptr; p.trow = L.tile_row; p.tkind_t = L.tile_kind_t;
  const unsigned grid = (unsigned)((p.T + 7) / 8);
  gist_tile_kernel<<<grid, 256, 0, s>>>(p);
  gist_count_kernel<<<grid, 256, 0, s>>>(p);
  gist_scan_kernel<<<1, 1024, 0, s>>>(p);
  gist_fill_kernel<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
