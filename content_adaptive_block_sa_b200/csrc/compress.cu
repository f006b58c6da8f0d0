// On-device literal flags from raw bytes.
//
// "Gzip-guided sparse attention: Selecting long-range content by
// compressibility" (Core equations) flags block i as literal when its
// compression ratio r_i = c_i / b exceeds the mean, c_i being the block's
// gzip level-1 size. Here c_i is computed on the GPU by a plain DEFLATE
// encoder defined from "RFC 1951: DEFLATE Compressed Data Format
// Specification version 1.3", so the sizes are an ESTIMATE of gzip's:
//   * greedy LZ77 parse with the candidate table of the specification's
//     section 4 in its fast form: at position p the candidate is the most
//     recent ENTERED earlier position with the same three bytes; the match is
//     their common prefix, at most 258 bytes and within the block; 3 or more
//     bytes are emitted as a match and skipped, otherwise the byte is a
//     literal. Positions the parse stops at are entered, and so are the
//     positions inside a match of at most 4 bytes; the inside of a longer
//     match is not;
//   * each block is one final block of the smallest of the three types:
//     fixed Huffman codes (section 3.2.6), dynamic Huffman codes (section
//     3.2.7: Huffman's construction, two queues, leaves before merged nodes
//     of equal weight; code lengths run-length coded under a code of at most
//     7 bits, made by package-merge when Huffman's exceeds 7), or stored
//     (section 3.2.4);
//   * c_i = ceil(bits / 8).
// Two launches: one warp per block, then one CTA per sequence for
// l_i = 1[c_i * B > sum_j c_j] in 64-bit integers.
//
// The warp's steps: a bitonic sort of (three-byte key, position) pairs gives
// every position its nearest earlier position with the same key and their
// common prefix; lane 0 walks the parse, a run of positions without such a
// position in one step (the table rule only matters where the nearest
// position lies inside a long match, and then the walk follows the same-key
// chain further back); the symbol counts are gathered in parallel; lane 0
// runs the two-queue merges; the run-length coding of the code lengths is
// counted in closed form per run.
#include "sa_common.cuh"

namespace sa {

constexpr int kMaxBlockBytes = 1024;
constexpr int kBlocksPerCta = 4;  // one warp per block
constexpr int kCompThreads = 32 * kBlocksPerCta;
constexpr int kNumLitLen = 286, kNumDist = 30, kNumCl = 19;
constexpr int kNumSyms = kNumLitLen + kNumDist + kNumCl;  // symbol counts and code lengths
constexpr int kMaxNodes = 2 * kNumLitLen - 1;
constexpr int kMaxInsert = 4;  // longest match whose inside positions are entered

// RFC 1951 section 3.2.7: order of the code-length code lengths in the header
__constant__ uint8_t kClOrder[kNumCl] = {16, 17, 18, 0, 8, 7, 9, 6, 10, 5,
                                         11, 4, 12, 3, 13, 2, 14, 1, 15};

// Length symbol (257..285) of a match length 3..258 and its extra bits
// (RFC 1951 section 3.2.5): lengths 3..10 have one symbol each; above, each
// power-of-two range [2^k, 2^(k+1)) of n - 3 (k = 3..7) holds four symbols of
// k - 2 extra bits; 258 is symbol 285.
__device__ __forceinline__ int length_symbol(int n, int& extra) {
  if (n == 258) {
    extra = 0;
    return 285;
  }
  const int l = n - 3;
  if (l < 8) {
    extra = 0;
    return 257 + l;
  }
  const int k = 31 - __clz(l);
  extra = k - 2;
  return 257 + 4 * (k - 1) + ((l >> (k - 2)) & 3);
}
// Distance code (0..29) and its extra bits: distances 1..4 have codes 0..3;
// above, each range (2^k, 2^(k+1)] (k >= 2) holds two codes of k - 1 extra bits.
__device__ __forceinline__ int distance_code(int d, int& extra) {
  const int e = d - 1;
  if (e < 4) {
    extra = 0;
    return e;
  }
  const int k = 31 - __clz(e);
  extra = k - 1;
  return 2 * k + ((e >> (k - 1)) & 1);
}
// Fixed code length of a literal/length symbol (section 3.2.6)
__device__ __forceinline__ int fixed_bits(int sym) {
  return sym <= 143 ? 8 : sym <= 255 ? 9 : sym <= 279 ? 7 : 8;
}

__host__ __device__ constexpr int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}
__host__ __device__ constexpr size_t align16(size_t n) { return (n + 15) / 16 * 16; }

// Per-warp shared memory, each part 16-byte aligned
struct DeflateSmem {
  uint64_t* srt;   // [pow2 >= b] (key, position) pairs
  uint16_t* mlen;  // [b + 1] common prefix with the nearest same-key position (0: none)
  uint16_t* mdist; // [b + 1] distance to it
  uint8_t* xs;     // [b + 1] the block's bytes
  uint32_t* skip;  // [32] bit p: p lies inside a match longer than kMaxInsert
  uint32_t* vis;   // [32] bit p: the parse stops at p
  uint32_t* mat;   // [32] bit p: ... with a match
  uint32_t* cand;  // [32] bit p: p has an earlier position with its key
  uint32_t* runs;  // [16] run starts of the code-length sequence
  uint32_t* freq;  // [kNumSyms] literal/length, distance, code-length symbol counts
  uint8_t* len;    // [kNumSyms] their code lengths
  uint32_t* hkey;  // [kNumLitLen] used symbols as (count << 9 | symbol), ascending
  uint32_t* hw;    // [kMaxNodes] node weights
  uint16_t* hpar;  // [kMaxNodes] node parents
};

__host__ __device__ constexpr size_t deflate_warp_smem(int b) {
  return align16(8 * (size_t)pow2_at_least(b)) + 2 * align16(2 * ((size_t)b + 1)) +
         align16((size_t)b + 1) + 4 * 32 * 4 + 4 * 16 + align16(4 * kNumSyms) +
         align16(kNumSyms) + align16(4 * kNumLitLen) + align16(4 * kMaxNodes) +
         align16(2 * kMaxNodes);
}

static_assert(kBlocksPerCta * deflate_warp_smem(kMaxBlockBytes) <= 227 * 1024,
              "the warps' shared memory exceeds a CTA's");

__device__ DeflateSmem deflate_carve(uint8_t* base, int b) {
  DeflateSmem m;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    uint8_t* ptr = base + o;
    o += align16(bytes);
    return ptr;
  };
  m.srt = reinterpret_cast<uint64_t*>(take(8 * (size_t)pow2_at_least(b)));
  m.mlen = reinterpret_cast<uint16_t*>(take(2 * ((size_t)b + 1)));
  m.mdist = reinterpret_cast<uint16_t*>(take(2 * ((size_t)b + 1)));
  m.xs = take((size_t)b + 1);
  m.skip = reinterpret_cast<uint32_t*>(take(4 * 32 * 4));
  m.vis = m.skip + 32;
  m.mat = m.skip + 64;
  m.cand = m.skip + 96;
  m.runs = reinterpret_cast<uint32_t*>(take(4 * 16));
  m.freq = reinterpret_cast<uint32_t*>(take(4 * kNumSyms));
  m.len = take(kNumSyms);
  m.hkey = reinterpret_cast<uint32_t*>(take(4 * kNumLitLen));
  m.hw = reinterpret_cast<uint32_t*>(take(4 * kMaxNodes));
  m.hpar = reinterpret_cast<uint16_t*>(take(2 * kMaxNodes));
  return m;
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Package-merge (Larmore and Hirschberg, 1990) for the code-length code:
// m <= 19 leaves (their (count << 9 | symbol) keys ascending in hkey), code
// lengths at most `limit`. Level 0 lists the leaves; level k merges the leaves
// with the pairs (2j, 2j + 1) of level k - 1, ordered by weight with a leaf
// before a package of equal weight; the first 2m - 2 entries of the last
// level are expanded, each leaf occurrence adding one to its symbol's length.
// Lane 0 only.
__device__ void package_merge(const DeflateSmem& S, int m, int limit, uint8_t* len) {
  constexpr int kStride = 2 * kNumCl - 1;
  uint32_t* pw = S.hw;                                     // [limit][kStride] weights
  int16_t* ptag = reinterpret_cast<int16_t*>(S.hpar);      // leaf index, or -(pair + 1)
  uint16_t* pcnt = S.hpar + 7 * kStride;                   // selections of each entry
  int size[8];
  for (int i = 0; i < m; ++i) {
    pw[i] = S.hkey[i] >> 9;
    ptag[i] = (int16_t)i;
  }
  size[0] = m;
  for (int k = 1; k < limit; ++k) {
    const uint32_t* lw = pw + (k - 1) * kStride;
    uint32_t* w = pw + k * kStride;
    int16_t* tg = ptag + k * kStride;
    const int npk = size[k - 1] / 2;
    int li = 0, pi = 0, o = 0;
    while (li < m || pi < npk) {
      const uint32_t pkw = pi < npk ? lw[2 * pi] + lw[2 * pi + 1] : 0u;
      if (li < m && (pi >= npk || (S.hkey[li] >> 9) <= pkw)) {
        w[o] = S.hkey[li] >> 9;
        tg[o++] = (int16_t)li++;
      } else {
        w[o] = pkw;
        tg[o++] = (int16_t)(-(pi++) - 1);
      }
    }
    size[k] = o;
  }
  for (int i = 0; i < limit * kStride; ++i) pcnt[i] = 0;
  for (int i = 0; i < 2 * m - 2; ++i) pcnt[(limit - 1) * kStride + i] = 1;
  for (int i = 0; i < m; ++i) len[S.hkey[i] & 511u] = 0;
  for (int k = limit - 1; k >= 0; --k) {
    for (int i = 0; i < size[k]; ++i) {
      const uint16_t c = pcnt[k * kStride + i];
      if (c == 0) continue;
      const int t = ptag[k * kStride + i];
      if (t >= 0) {
        len[S.hkey[t] & 511u] += (uint8_t)c;
      } else {
        const int j = -t - 1;
        pcnt[(k - 1) * kStride + 2 * j] += c;
        pcnt[(k - 1) * kStride + 2 * j + 1] += c;
      }
    }
  }
}

// Code lengths of the symbols with freq > 0 among n (the others get 0), by
// Huffman's construction: leaves in ascending (count, symbol) order, merged
// nodes in creation order, each step joining the two lightest fronts with a
// leaf taken before a merged node of equal weight; a length is the leaf's
// depth; one used symbol gets length 1. Longer than `limit`: package-merge.
// A literal/length or distance code never exceeds 15 here: a Huffman code of
// depth 15 needs a total count of at least F(17) = 1597 (Fibonacci), and a
// block of at most 1024 bytes has at most 1025 symbols; so only the
// code-length code (19 symbols, limit 7) reaches package-merge.
// Whole warp; ends with __syncwarp.
__device__ void huffman_lengths(const DeflateSmem& S, const uint32_t* freq, int n, int limit,
                                uint8_t* len, int lane) {
  int m = 0;
  for (int base = 0; base < n; base += 32) {
    const int s = base + lane;
    const bool used = s < n && freq[s] > 0u;
    const uint32_t bal = __ballot_sync(0xffffffffu, used);
    if (used) S.hw[m + __popc(bal & ((1u << lane) - 1u))] = (freq[s] << 9) | (uint32_t)s;
    if (s < n) len[s] = 0;
    m += __popc(bal);
  }
  __syncwarp();
  if (m == 0) return;
  if (m == 1) {
    if (lane == 0) len[S.hw[0] & 511u] = 1;
    __syncwarp();
    return;
  }
  for (int i = lane; i < m; i += 32) {  // rank sort of the distinct keys
    const uint32_t k = S.hw[i];
    int rank = 0;
    for (int j = 0; j < m; ++j) rank += S.hw[j] < k ? 1 : 0;
    S.hkey[rank] = k;
  }
  __syncwarp();
  if (lane == 0) {
    // the fronts of both queues stay in registers; each take loads the next
    uint32_t* w = S.hw;
    for (int i = 0; i < m; ++i) w[i] = S.hkey[i] >> 9;
    int li = 0, ii = m, nn = m;  // next leaf, next merged node to take, next node id
    uint32_t wl = w[0], wi = 0u;  // their weights (wi valid while ii < nn)
    for (int step = 0; step < m - 1; ++step) {
      int who[2];
      uint32_t sum = 0u;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (li < m && (ii >= nn || wl <= wi)) {
          who[u] = li++;
          sum += wl;
          wl = w[li];  // (w[m] is the first merged node: read, never used as a leaf)
        } else {
          who[u] = ii++;
          sum += wi;
          wi = w[ii];
        }
      }
      w[nn] = sum;
      if (ii == nn) wi = sum;  // the merged queue was empty: the new node is its front
      S.hpar[who[0]] = (uint16_t)nn;
      S.hpar[who[1]] = (uint16_t)nn;
      ++nn;
    }
  }
  __syncwarp();
  // a leaf's length is its depth: the steps up to the root (node 2m - 2)
  int maxd = 0;
  for (int k = lane; k < m; k += 32) {
    int node = k, d = 0;
    while (node != 2 * m - 2) {
      node = S.hpar[node];
      ++d;
    }
    len[S.hkey[k] & 511u] = (uint8_t)d;
    maxd = max(maxd, d);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) maxd = max(maxd, __shfl_xor_sync(0xffffffffu, maxd, off));
  __syncwarp();
  if (maxd > limit && m <= kNumCl) {
    if (lane == 0) package_merge(S, m, limit, len);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kCompThreads) deflate_size_kernel(const uint8_t* x, int64_t n_bytes,
                                                                    int b, int B, uint32_t* sizes) {
  extern __shared__ __align__(16) uint8_t dyn_s[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x * kBlocksPerCta + warp, bt = blockIdx.y;
  if (blk >= B) return;  // warp-uniform; no CTA-wide barrier below
  const int np2 = pow2_at_least(b);
  const DeflateSmem S = deflate_carve(dyn_s + (size_t)warp * deflate_warp_smem(b), b);
  const uint8_t* src = x + (int64_t)bt * n_bytes + (int64_t)blk * b;
  for (int i = lane; i < b; i += 32) S.xs[i] = src[i];
  for (int i = lane; i < kNumSyms; i += 32) S.freq[i] = 0u;
  for (int i = lane; i < 128; i += 32) S.skip[i] = 0u;  // skip, vis, mat, cand
  __syncwarp();
  // (three-byte key, position) of every position with three bytes left,
  // padded with the largest value; sorted ascending, an entry whose
  // predecessor has the same key finds there its nearest earlier position
  // with that key
  for (int i = lane; i < np2; i += 32) {
    uint64_t v = ~0ull;
    if (i + 3 <= b)
      v = ((uint64_t)((uint32_t)S.xs[i] | ((uint32_t)S.xs[i + 1] << 8) |
                      ((uint32_t)S.xs[i + 2] << 16)) << 32) | (uint32_t)i;
    S.srt[i] = v;
    if (i <= b) S.mlen[i] = 0;
  }
  __syncwarp();
  for (int size = 2; size <= np2; size <<= 1) {  // bitonic sort, ascending
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < np2 / 2; i += 32) {
        const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t a = S.srt[lo], c = S.srt[hi];
        if ((a > c) == up) {
          S.srt[lo] = c;
          S.srt[hi] = a;
        }
      }
      __syncwarp();
    }
  }
  // common prefix with the nearest same-key position (at least its 3 bytes)
  for (int t = 1 + lane; t < np2; t += 32) {
    const uint64_t cur = S.srt[t], prev = S.srt[t - 1];
    if (cur != ~0ull && (cur >> 32) == (prev >> 32)) {
      const int p = (int)(uint32_t)cur, q = (int)(uint32_t)prev;
      int m = 3;
      while (p + m < b && m < 258 && S.xs[q + m] == S.xs[p + m]) ++m;
      S.mlen[p] = (uint16_t)m;
      S.mdist[p] = (uint16_t)(p - q);
    }
  }
  __syncwarp();
  for (int base = 0; base < b; base += 32) {
    const uint32_t cb = __ballot_sync(0xffffffffu, base + lane < b && S.mlen[base + lane] >= 3);
    if (lane == 0) S.cand[base >> 5] = cb;
  }
  __syncwarp();
  // the parse (lane 0): a run of positions without a same-key position is a
  // run of literals; elsewhere the nearest same-key position q is the
  // candidate unless it lies inside a long match, and then the chain of
  // same-key positions (each one's own nearest) is followed back to an
  // entered one
  if (lane == 0) {
    auto set_bits = [&](uint32_t* bm, int lo, int hi) {  // bits [lo, hi)
      for (int i = lo; i < hi;) {
        const int sh = i & 31, nbit = min(32 - sh, hi - i);
        bm[i >> 5] |= (nbit == 32 ? 0xffffffffu : ((1u << nbit) - 1u)) << sh;
        i += nbit;
      }
    };
    const int nwords = (b + 31) >> 5;
    int p = 0;
    while (p < b) {
      int w = p >> 5;
      uint32_t c = S.cand[w] & (0xffffffffu << (p & 31));
      while (c == 0u && ++w < nwords) c = S.cand[w];
      const int nx = c ? (w << 5) + __ffs(c) - 1 : b;
      if (nx > p) {  // literals p .. nx - 1
        set_bits(S.vis, p, nx);
        p = nx;
        continue;
      }
      int m = S.mlen[p];
      int q = p - S.mdist[p];
      if ((S.skip[q >> 5] >> (q & 31)) & 1u) {
        do {
          q = S.mlen[q] >= 3 ? q - S.mdist[q] : -1;
        } while (q >= 0 && ((S.skip[q >> 5] >> (q & 31)) & 1u));
        if (q < 0) {
          m = 0;
        } else {
          m = 3;
          while (p + m < b && m < 258 && S.xs[q + m] == S.xs[p + m]) ++m;
          S.mlen[p] = (uint16_t)m;
          S.mdist[p] = (uint16_t)(p - q);
        }
      }
      S.vis[p >> 5] |= 1u << (p & 31);
      if (m >= 3) {
        S.mat[p >> 5] |= 1u << (p & 31);
        if (m > kMaxInsert) set_bits(S.skip, p + 1, p + m);  // not entered
        p += m;
      } else {
        p += 1;
      }
    }
  }
  __syncwarp();
  // symbol counts; the fixed code's bits and the extra bits (same in both codes)
  uint32_t* ll = S.freq;
  uint32_t* dd = S.freq + kNumLitLen;
  uint32_t* cf = S.freq + kNumLitLen + kNumDist;
  uint32_t fixed = 0u, extra = 0u;
  for (int p = lane; p < b; p += 32) {
    const uint32_t bit = 1u << (p & 31);
    if (!(S.vis[p >> 5] & bit)) continue;
    if (S.mat[p >> 5] & bit) {
      int el, ed;
      const int sym = length_symbol(S.mlen[p], el);
      const int code = distance_code(S.mdist[p], ed);
      atomicAdd(&ll[sym], 1u);
      atomicAdd(&dd[code], 1u);
      fixed += (uint32_t)(fixed_bits(sym) + 5);
      extra += (uint32_t)(el + ed);
    } else {
      const int c = S.xs[p];
      atomicAdd(&ll[c], 1u);
      fixed += (uint32_t)fixed_bits(c);
    }
  }
  if (lane == 0) ll[256] = 1u;  // end of block
  fixed = warp_sum(fixed);
  extra = warp_sum(extra);
  __syncwarp();
  // dynamic code: literal/length and distance code lengths
  uint8_t* Lll = S.len;
  uint8_t* Ldd = S.len + kNumLitLen;
  uint8_t* Lcl = S.len + kNumLitLen + kNumDist;
  huffman_lengths(S, ll, kNumLitLen, 15, Lll, lane);
  huffman_lengths(S, dd, kNumDist, 15, Ldd, lane);
  int last_ll = 0, last_dd = -1;
  for (int base = 0; base < kNumLitLen; base += 32) {
    const uint32_t bal = __ballot_sync(0xffffffffu, base + lane < kNumLitLen && Lll[base + lane] > 0);
    if (bal) last_ll = base + 31 - __clz(bal);
  }
  {
    const uint32_t bal = __ballot_sync(0xffffffffu, lane < kNumDist && Ldd[lane] > 0);
    if (bal) last_dd = 31 - __clz(bal);
  }
  const int hlit = max(257, last_ll + 1), hdist = max(1, last_dd + 1);
  const int ncl = hlit + hdist;
  auto cl_value = [&](int i) -> int { return i < hlit ? Lll[i] : Ldd[i - hlit]; };
  // run-length coding of the code lengths (section 3.2.7), counted per run:
  // a run of R zeros sends 18 (11..138 zeros) while 11 or more remain, then
  // 17 (3..10) if 3 or more remain, then single zeros; a run of R copies of a
  // length v sends v, then 16 (3..6 repeats) while 3 or more remain, then v
  for (int base = 0; base < ncl; base += 32) {
    const int i = base + lane;
    const bool st = i < ncl && (i == 0 || cl_value(i) != cl_value(i - 1));
    const uint32_t bal = __ballot_sync(0xffffffffu, st);
    if (lane == 0) S.runs[base >> 5] = bal;
  }
  __syncwarp();
  const int nwords = (ncl + 31) >> 5;
  uint32_t rle_extra = 0u;
  for (int i = lane; i < ncl; i += 32) {
    if (!((S.runs[i >> 5] >> (i & 31)) & 1u)) continue;
    int w = i >> 5;
    uint32_t rest = (i & 31) == 31 ? 0u : S.runs[w] & ~((2u << (i & 31)) - 1u);
    while (rest == 0u && ++w < nwords) rest = S.runs[w];
    const int next = rest ? (w << 5) + __ffs(rest) - 1 : ncl;
    const int R = next - i, v = cl_value(i);
    if (v == 0) {
      int n18 = R / 138, rem = R % 138;
      if (rem >= 11) {
        ++n18;
        rem = 0;
      }
      const int n17 = rem >= 3 ? 1 : 0;
      if (n17) rem = 0;
      if (n18) atomicAdd(&cf[18], (uint32_t)n18);
      if (n17) atomicAdd(&cf[17], 1u);
      if (rem) atomicAdd(&cf[0], (uint32_t)rem);
      rle_extra += (uint32_t)(7 * n18 + 3 * n17);
    } else {
      int n16 = (R - 1) / 6, rem = (R - 1) % 6;
      if (rem >= 3) {
        ++n16;
        rem = 0;
      }
      atomicAdd(&cf[v], (uint32_t)(1 + rem));
      if (n16) atomicAdd(&cf[16], (uint32_t)n16);
      rle_extra += (uint32_t)(2 * n16);
    }
  }
  rle_extra = warp_sum(rle_extra);
  __syncwarp();
  huffman_lengths(S, cf, kNumCl, 7, Lcl, lane);
  const uint32_t clbal = __ballot_sync(0xffffffffu, lane < kNumCl && Lcl[kClOrder[lane < kNumCl ? lane : 0]] > 0);
  const int hclen = max(4, clbal ? 32 - __clz(clbal) : 0);
  uint32_t dyn = 0u;
  for (int s = lane; s < kNumSyms; s += 32) dyn += S.freq[s] * S.len[s];
  dyn = warp_sum(dyn);
  if (lane == 0) {
    const uint32_t dyn_bits = 3 + 5 + 5 + 4 + 3 * (uint32_t)hclen + rle_extra + dyn + extra;
    const uint32_t fixed_bits_total = 3 + fixed + 7 + extra;  // + end of block (symbol 256)
    const uint32_t stored_bits = 3 + 5 + 32 + 8 * (uint32_t)b;
    const uint32_t bits = min(min(dyn_bits, fixed_bits_total), stored_bits);
    sizes[(int64_t)bt * B + blk] = (bits + 7) / 8;
  }
}

__global__ void __launch_bounds__(256) literal_flags_kernel(const uint32_t* sizes, int B,
                                                            uint8_t* flags) {
  __shared__ unsigned long long part[8];
  const int bt = blockIdx.x;
  const uint32_t* c = sizes + (int64_t)bt * B;
  unsigned long long sum = 0ull;
  for (int i = threadIdx.x; i < B; i += blockDim.x) sum += c[i];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sum;
  __syncthreads();
  unsigned long long total = 0ull;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += part[w];
  for (int i = threadIdx.x; i < B; i += blockDim.x)
    flags[(int64_t)bt * B + i] = (unsigned long long)c[i] * (unsigned long long)B > total ? 1 : 0;
}

cudaError_t launch_literal_flags_device(const uint8_t* bytes, int batch, int64_t n_bytes, int b,
                                        uint32_t* sizes, uint8_t* flags, cudaStream_t s) {
  const int B = (int)(n_bytes / b);
  const size_t smem = kBlocksPerCta * deflate_warp_smem(b);  // <= 79 KB (b <= 1024)
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(deflate_size_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  deflate_size_kernel<<<dim3((B + kBlocksPerCta - 1) / kBlocksPerCta, batch), kCompThreads, smem, s>>>(
      bytes, n_bytes, b, B, sizes);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  literal_flags_kernel<<<batch, 256, 0, s>>>(sizes, B, flags);
  return cudaGetLastError();
}

}  // namespace sa
