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
// with FULL / MASKED / TAIL kinds.
//
// One CTA builds one (sequence, class) pair (gzip) or the whole layout
// (gist); counts are turned into absolute offsets with a block-wide scan into
// fixed per-pair regions, so no global scratch and no second launch is
// needed.
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

__global__ void __launch_bounds__(1024) gzip_build_kernel(GzipBuild p) {
  extern __shared__ int32_t smem[];
  const int bc = blockIdx.x, bt = bc / 3, cls = bc % 3;
  const int B = p.B;
  int32_t* lp = smem;            // [B+1]: literals in [0, i)
  int32_t* lit_idx = lp + B + 1;  // [B]: ascending literal blocks
  uint8_t* f = reinterpret_cast<uint8_t*>(lit_idx + B);  // [B]
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

  // ---- CSR: query block i -> ascending key blocks
  int32_t* rp = p.row_ptr + (int64_t)bc * (B + 1);
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const int lo = max(0, i - w);
    int cnt;
    if (cls == SA_CLASS_LOCAL) cnt = i - lo + 1;
    else if (cls == SA_CLASS_LITERAL) cnt = f[i] ? lp[i + 1] : 1;
    else cnt = (i - lo + 1) + (f[i] ? lp[lo] : 0);
    rp[i + 1] = cnt;
  }
  if (threadIdx.x == 0) rp[0] = (int32_t)(bc * p.region);
  __syncthreads();
  block_inclusive_scan(rp + 1, B, (int32_t)(bc * p.region));
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    int32_t* out = p.col_idx + rp[i];
    const int lo = max(0, i - w);
    int n = 0;
    if (cls == SA_CLASS_LITERAL) {
      if (f[i]) for (int t = 0; t < lp[i + 1]; ++t) out[n++] = lit_idx[t];
      else out[n++] = i;
    } else {
      if (cls == SA_CLASS_HYBRID && f[i])
        for (int t = 0; t < lp[lo]; ++t) out[n++] = lit_idx[t];
      for (int j = lo; j <= i; ++j) out[n++] = j;
    }
  }

  // ---- CSC: key block j -> ascending query blocks
  int32_t* cp = p.col_ptr + (int64_t)bc * (B + 1);
  for (int j = threadIdx.x; j < B; j += blockDim.x) {
    const int hi = min(B - 1, j + w);
    int cnt;
    if (cls == SA_CLASS_LOCAL) cnt = hi - j + 1;
    else if (cls == SA_CLASS_LITERAL) cnt = f[j] ? (L - lp[j]) : 1;
    else cnt = (hi - j + 1) + (f[j] ? (L - lp[hi + 1]) : 0);
    cp[j + 1] = cnt;
  }
  if (threadIdx.x == 0) cp[0] = (int32_t)(bc * p.region);
  __syncthreads();
  block_inclusive_scan(cp + 1, B, (int32_t)(bc * p.region));
  for (int j = threadIdx.x; j < B; j += blockDim.x) {
    int32_t* out = p.row_idx + cp[j];
    const int hi = min(B - 1, j + w);
    int n = 0;
    if (cls == SA_CLASS_LITERAL) {
      if (f[j]) for (int t = lp[j]; t < L; ++t) out[n++] = lit_idx[t];
      else out[n++] = j;
    } else {
      for (int i = j; i <= hi; ++i) out[n++] = i;
      if (cls == SA_CLASS_HYBRID && f[j])
        for (int t = lp[hi + 1]; t < L; ++t) out[n++] = lit_idx[t];
    }
  }

  // ---- packed bit rows
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

  // ---- tile lists (CSR) and their transpose (CSC)
  __syncthreads();  // the block lists above are read below
  const int T = p.T;
  int32_t* trp = p.trp + (int64_t)bc * (T + 1);
  int32_t* tcp = p.tcp + (int64_t)bc * (T + 1);
  if (p.b >= kTile) {
    // r whole tiles per block: key tile J of a visited block kb is FULL,
    // except the diagonal tile; tiles of the diagonal block past I are skipped
    const int r = p.b / kTile;
    for (int I = threadIdx.x; I < T; I += blockDim.x) {
      const int i = I / r;
      trp[I + 1] = (rp[i + 1] - rp[i] - 1) * r + (I - i * r + 1);
    }
    if (threadIdx.x == 0) trp[0] = (int32_t)(bc * p.tregion);
    __syncthreads();
    block_inclusive_scan(trp + 1, T, (int32_t)(bc * p.tregion));
    for (int I = threadIdx.x; I < T; I += blockDim.x) {
      const int i = I / r;
      int n = trp[I];
      for (int e = rp[i]; e < rp[i + 1]; ++e) {
        const int kb = p.col_idx[e];
        const int last = kb < i ? kb * r + r - 1 : I;
        for (int J = kb * r; J <= last; ++J) {
          p.tcol[n] = J;
          p.tkind[n] = (int8_t)(J == I ? SA_TILE_MASKED : SA_TILE_FULL);
          ++n;
        }
      }
    }
    for (int J = threadIdx.x; J < T; J += blockDim.x) {
      const int j = J / r;
      tcp[J + 1] = (cp[j + 1] - cp[j] - 1) * r + (j * r + r - J);
    }
    if (threadIdx.x == 0) tcp[0] = (int32_t)(bc * p.tregion);
    __syncthreads();
    block_inclusive_scan(tcp + 1, T, (int32_t)(bc * p.tregion));
    for (int J = threadIdx.x; J < T; J += blockDim.x) {
      const int j = J / r;
      int n = tcp[J];
      for (int e = cp[j]; e < cp[j + 1]; ++e) {
        const int qb = p.row_idx[e];
        for (int I = qb == j ? J : qb * r; I < qb * r + r; ++I) {
          p.trow[n] = I;
          p.tkind_t[n] = (int8_t)(I == J ? SA_TILE_MASKED : SA_TILE_FULL);
          ++n;
        }
      }
    }
    return;
  }
  const int lb = __ffs(p.b) - 1;  // b divides 128: a power of two
  for (int I = threadIdx.x; I < T; I += blockDim.x) {
    int cnt = 0;
    for (int J = 0; J <= I; ++J) cnt += gzip_tile_kind(p, lb, cls, f, I, J) >= 0;
    trp[I + 1] = cnt;
  }
  if (threadIdx.x == 0) trp[0] = (int32_t)(bc * p.tregion);
  __syncthreads();
  block_inclusive_scan(trp + 1, T, (int32_t)(bc * p.tregion));
  for (int I = threadIdx.x; I < T; I += blockDim.x) {
    int n = trp[I];
    for (int J = 0; J <= I; ++J) {
      const int k = gzip_tile_kind(p, lb, cls, f, I, J);
      if (k >= 0) { p.tcol[n] = J; p.tkind[n] = (int8_t)k; ++n; }
    }
  }
  for (int J = threadIdx.x; J < T; J += blockDim.x) {
    int cnt = 0;
    for (int I = J; I < T; ++I) cnt += gzip_tile_kind(p, lb, cls, f, I, J) >= 0;
    tcp[J + 1] = cnt;
  }
  if (threadIdx.x == 0) tcp[0] = (int32_t)(bc * p.tregion);
  __syncthreads();
  block_inclusive_scan(tcp + 1, T, (int32_t)(bc * p.tregion));
  for (int J = threadIdx.x; J < T; J += blockDim.x) {
    int n = tcp[J];
    for (int I = J; I < T; ++I) {
      const int k = gzip_tile_kind(p, lb, cls, f, I, J);
      if (k >= 0) { p.trow[n] = I; p.tkind_t[n] = (int8_t)k; ++n; }
    }
  }
}

// ------------------------------------------------------------------ gist
struct GistBuild {
  const uint8_t* flags;  // [N] or null
  int N, T, sinks, ratio, window, tail;
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

// Kind of tile pair (I, J) under the gist visibility rule, or -1.
__device__ int gist_tile_kind(const GistBuild& p, int I, int J) {
  if (J > I) return -1;
  const int i_min = I * kTile, i_max = min(p.N, (I + 1) * kTile) - 1;
  const int j0 = J * kTile, j1 = min(p.N, (J + 1) * kTile);  // [j0, j1)
  if (J == I) return (i_max == i_min) ? SA_TILE_FULL : SA_TILE_MASKED;
  const uint32_t* gb = p.gist_bits;
  const int ng = count_gists(gb, j0, j1);
  const bool has_sink = j0 < p.sinks;
  const bool any = has_sink || ng > 0 || (i_min - (j1 - 1) < p.window);
  if (!any) return -1;
  // all pairs visible iff every non-gist, non-sink key is in every query's window
  const int jr = first_raw(gb, max(j0, p.sinks), j1);
  if (jr < 0 || i_max - jr < p.window) return SA_TILE_FULL;
  // smallest physical column visible to some query of tile I
  const int n_raw = (j1 - j0) - ng;
  int min_col = kTile;
  if (ng > 0) min_col = n_raw;  // gists sit after the raw tokens
  int r = first_raw(gb, j0, min(j1, p.sinks));  // raw sink tokens
  if (r < 0) r = first_raw(gb, max(j0, i_min - p.window + 1), j1);  // raw window tokens
  if (r >= 0) min_col = min(min_col, (r - j0) - count_gists(gb, j0, r));
  return (min_col >= kTile - p.tail) ? SA_TILE_TAIL : SA_TILE_MASKED;
}

__global__ void __launch_bounds__(1024) gist_build_kernel(GistBuild p) {
  const int N = p.N, T = p.T;
  const int nwords = (N + 31) / 32;
  for (int k = threadIdx.x; k < nwords; k += blockDim.x) {
    uint32_t word = 0;
    for (int t = 0; t < 32; ++t) {
      const int pos = k * 32 + t;
      if (pos >= N) break;
      bool g;
      if (p.flags) g = p.flags[pos] != 0;
      else g = pos >= p.sinks && ((pos - p.sinks) % (p.ratio + 1)) == p.ratio;
      if (g) word |= 1u << t;
    }
    p.gist_bits[k] = word;
  }
  __syncthreads();
  // shift permutation: one warp per tile
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int J = warp; J < T; J += nwarps) {
    const int j0 = J * kTile, n = min(kTile, N - j0);
    const int ng = count_gists(p.gist_bits, j0, j0 + n);
    int before = 0;  // gists of this tile before the current 32-chunk
    for (int c = 0; c < kTile / 32; ++c) {
      const int off = c * 32 + lane, pos = j0 + off;
      const uint32_t word = (j0 + c * 32 < N) ? p.gist_bits[(j0 >> 5) + c] : 0u;
      const uint32_t valid = (n - c * 32 >= 32) ? 0xffffffffu
                             : (n - c * 32 <= 0) ? 0u : ((1u << (n - c * 32)) - 1u);
      const uint32_t gw = word & valid;
      if (off < n) {
        const int gb = before + __popc(gw & ((1u << lane) - 1u));
        const bool g = (gw >> lane) & 1u;
        const int phys = j0 + (g ? (n - ng) + gb : off - gb);
        p.perm[phys] = pos;
      }
      before += __popc(gw);
    }
    // keys visible to every later query: sinks and gists of this tile
    int nf = 0;
    for (int c = 0; c < kTile / 32; ++c) {
      const int pos = j0 + c * 32 + lane;
      nf += __popc(__ballot_sync(0xffffffffu, pos < N && (pos < p.sinks || is_gist(p.gist_bits, pos))));
    }
    if (lane == 0) p.far_ptr[J + 1] = nf;
  }
  if (threadIdx.x == 0) p.far_ptr[0] = 0;
  __syncthreads();
  block_inclusive_scan(p.far_ptr + 1, T, 0);
  // far_idx: the physical index of every sink / gist, in logical order
  for (int J = warp; J < T; J += nwarps) {
    const int j0 = J * kTile, n = min(kTile, N - j0);
    const int ng = count_gists(p.gist_bits, j0, j0 + n);
    int f = p.far_ptr[J], gbefore = 0;
    for (int c = 0; c < kTile / 32; ++c) {
      const int off = c * 32 + lane, pos = j0 + off;
      const bool ok = pos < N;
      const bool g = ok && is_gist(p.gist_bits, pos);
      const bool far = ok && (pos < p.sinks || g);
      const uint32_t gmask = __ballot_sync(0xffffffffu, g);
      const uint32_t fmask = __ballot_sync(0xffffffffu, far);
      const uint32_t below = (1u << lane) - 1u;
      if (far) {
        const int gb = gbefore + __popc(gmask & below);
        p.far_idx[f + __popc(fmask & below)] = j0 + (g ? (n - ng) + gb : off - gb);
      }
      f += __popc(fmask);
      gbefore += __popc(gmask);
    }
  }
  __syncthreads();
  for (int I = threadIdx.x; I < T; I += blockDim.x) {
    int cnt = 0;
    for (int J = 0; J <= I; ++J) cnt += gist_tile_kind(p, I, J) >= 0;
    p.trp[I + 1] = cnt;
  }
  if (threadIdx.x == 0) p.trp[0] = 0;
  __syncthreads();
  block_inclusive_scan(p.trp + 1, T, 0);
  for (int I = threadIdx.x; I < T; I += blockDim.x) {
    int n = p.trp[I];
    for (int J = 0; J <= I; ++J) {
      const int k = gist_tile_kind(p, I, J);
      if (k >= 0) { p.tcol[n] = J; p.tkind[n] = (int8_t)k; ++n; }
    }
  }
  for (int J = threadIdx.x; J < T; J += blockDim.x) {
    int cnt = 0;
    for (int I = J; I < T; ++I) cnt += gist_tile_kind(p, I, J) >= 0;
    p.tcp[J + 1] = cnt;
  }
  if (threadIdx.x == 0) p.tcp[0] = 0;
  __syncthreads();
  block_inclusive_scan(p.tcp + 1, T, 0);
  for (int J = threadIdx.x; J < T; J += blockDim.x) {
    int n = p.tcp[J];
    for (int I = J; I < T; ++I) {
      const int k = gist_tile_kind(p, I, J);
      if (k >= 0) { p.trow[n] = I; p.tkind_t[n] = (int8_t)k; ++n; }
    }
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
  const size_t smem = (size_t)(2 * p.B + 1) * 4 + p.B;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gzip_build_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  gzip_build_kernel<<<d.batch * 3, 1024, smem, s>>>(p);
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
  p.tail = d.gist_tail > 0 ? d.gist_tail : 32;
  p.tregion = (int64_t)p.T * (p.T + 1) / 2;
  p.gist_bits = L.gist_bits;
  p.perm = L.perm;
  p.far_idx = L.far_idx;
  p.far_ptr = L.far_ptr;
  p.trp = L.tile_row_ptr; p.tcol = L.tile_col; p.tkind = L.tile_kind;
  p.tcp = L.tile_col_ptr; p.trow = L.tile_row; p.tkind_t = L.tile_kind_t;
  gist_build_kernel<<<1, 1024, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
