// On-device literal flags from raw bytes.
//
// "Gzip-guided sparse attention: Selecting long-range content by
// compressibility" (Core equations) flags block i as literal when its
// compression ratio r_i = c_i / b exceeds the mean, c_i being the block's
// gzip level-1 size. Here c_i is computed on the GPU by a plain DEFLATE
// encoder defined from "RFC 1951: DEFLATE Compressed Data Format
// Specification version 1.3", so the sizes (and the flags) are an ESTIMATE of
// gzip's, not equal to them:
//   * each block is one final block with the fixed Huffman codes (section
//     3.2.6): 3 header bits, the symbols, the end-of-block symbol 256;
//   * greedy LZ77 parse: at position p the candidate is the nearest earlier q
//     with the same three bytes (p - q <= 32768); the match is their common
//     prefix, at most 258 bytes and within the block; 3 or more bytes are
//     emitted as a match and skipped, otherwise the byte is a literal;
//   * literals 0..143 cost 8 bits and 144..255 9; length symbols 256..279 7
//     bits and 280..287 8; distance codes 5 bits; plus the extra bits of
//     section 3.2.5's length and distance tables;
//   * c_i = ceil(bits / 8).
// Two launches: one warp per block (a bitonic sort of (three-byte key,
// position) pairs in shared memory gives every position its nearest earlier
// match; binary lifting over the next-position pointers marks the positions
// the greedy parse visits; the code lengths are in closed form), then one CTA
// per sequence for l_i = 1[c_i * B > sum_j c_j] in 64-bit integers.
#include "sa_common.cuh"

namespace sa {

constexpr int kMaxBlockBytes = 1024;
constexpr int kBlocksPerCta = 4;  // one warp per block
constexpr int kCompThreads = 32 * kBlocksPerCta;

// Code lengths in closed form (RFC 1951 section 3.2.5 and 3.2.6).
// Length n: symbols 257..279 take 7 bits, 280..287 8; with the symbol's
// extra bits a match length costs 7 (3..10), 8 (11..18), 9 (19..34),
// 10 (35..66), 11 (67..114, symbols 277..279), 12 (115..130, symbol 280),
// 13 (131..257) or 8 (258, symbol 285) bits.
__device__ __forceinline__ int length_bits(int n) {
  return n <= 10 ? 7 : n <= 18 ? 8 : n <= 34 ? 9 : n <= 66 ? 10 : n <= 114 ? 11
       : n <= 130 ? 12 : n <= 257 ? 13 : 8;
}
// Distance d: a 5-bit code; distances 1..4 have no extra bits, and the two
// codes covering (2^k, 2^(k+1)] carry k - 1 extra bits.
__device__ __forceinline__ int distance_bits(int d) {
  return 5 + (d <= 4 ? 0 : (31 - __clz(d - 1)) - 1);
}

__host__ __device__ constexpr int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Per warp: the sort buffer (uint64 [pow2 >= b]), match lengths and
// distances, next-position pointers (uint16 [b + 1] each), parse marks and
// the block's bytes (uint8 [b + 1] each), 16-byte aligned.
__host__ __device__ constexpr size_t deflate_warp_smem(int b) {
  return ((size_t)8 * pow2_at_least(b) + 6 * ((size_t)b + 1) + 2 * ((size_t)b + 1) + 15) / 16 * 16;
}

__device__ __forceinline__ int position_bits(const uint16_t* mlen, const uint16_t* mdist,
                                             const uint8_t* xs, int p) {
  const int m = mlen[p];
  return m >= 3 ? length_bits(m) + distance_bits(mdist[p]) : (xs[p] <= 143 ? 8 : 9);
}

__global__ void __launch_bounds__(kCompThreads) deflate_size_kernel(const uint8_t* x, int64_t n_bytes,
                                                                    int b, int B, uint32_t* sizes) {
  extern __shared__ __align__(16) uint8_t dyn_s[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x * kBlocksPerCta + warp, bt = blockIdx.y;
  if (blk >= B) return;  // warp-uniform; no CTA-wide barrier below
  const int np2 = pow2_at_least(b);
  uint8_t* base = dyn_s + (size_t)warp * deflate_warp_smem(b);
  uint64_t* srt = reinterpret_cast<uint64_t*>(base);
  uint16_t* mlen = reinterpret_cast<uint16_t*>(base + 8 * (size_t)np2);
  uint16_t* mdist = mlen + (b + 1);
  uint16_t* nxt = mdist + (b + 1);
  uint8_t* mark = reinterpret_cast<uint8_t*>(nxt + (b + 1));
  uint8_t* xs = mark + (b + 1);
  const uint8_t* src = x + (int64_t)bt * n_bytes + (int64_t)blk * b;
  for (int i = lane; i < b; i += 32) xs[i] = src[i];
  __syncwarp();
  // (three-byte key, position) of every position with three bytes left,
  // padded with the largest value; sorted ascending, an entry whose
  // predecessor has the same key finds there its nearest earlier match
  for (int i = lane; i < np2; i += 32) {
    uint64_t v = ~0ull;
    if (i + 3 <= b)
      v = ((uint64_t)((uint32_t)xs[i] | ((uint32_t)xs[i + 1] << 8) | ((uint32_t)xs[i + 2] << 16)) << 32) |
          (uint32_t)i;
    srt[i] = v;
    if (i <= b) mlen[i] = 0;
  }
  __syncwarp();
  for (int size = 2; size <= np2; size <<= 1) {  // bitonic sort, ascending
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < np2 / 2; i += 32) {
        const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t a = srt[lo], c = srt[hi];
        if ((a > c) == up) {
          srt[lo] = c;
          srt[hi] = a;
        }
      }
      __syncwarp();
    }
  }
  for (int t = 1 + lane; t < np2; t += 32) {
    const uint64_t cur = srt[t], prev = srt[t - 1];
    if (cur != ~0ull && (cur >> 32) == (prev >> 32)) {
      const int p = (int)(uint32_t)cur, q = (int)(uint32_t)prev;
      int m = 3;
      while (p + m < b && m < 258 && xs[q + m] == xs[p + m]) ++m;
      mlen[p] = (uint16_t)m;
      mdist[p] = (uint16_t)(p - q);
    }
  }
  __syncwarp();
  // the greedy parse visits 0, next(0), next(next(0)), ... with next(p) =
  // p + (match length or 1): mark that orbit by binary lifting (round k
  // follows next^(2^k) from every marked position), then sum the costs
  for (int p = lane; p <= b; p += 32) {
    nxt[p] = (uint16_t)(p == b ? b : p + (mlen[p] >= 3 ? mlen[p] : 1));
    mark[p] = p == 0 ? 1 : 0;
  }
  __syncwarp();
  for (int span = 1; span < 2 * b; span <<= 1) {
    for (int p = lane; p < b; p += 32)
      if (mark[p]) mark[nxt[p]] = 1;
    __syncwarp();
    uint16_t j2[kMaxBlockBytes / 32 + 1];
    int c = 0;
    for (int p = lane; p <= b; p += 32) j2[c++] = nxt[nxt[p]];
    __syncwarp();
    c = 0;
    for (int p = lane; p <= b; p += 32) nxt[p] = j2[c++];
    __syncwarp();
  }
  int bits = 0;
  for (int p = lane; p < b; p += 32)
    if (mark[p]) bits += position_bits(mlen, mdist, xs, p);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) bits += __shfl_xor_sync(0xffffffffu, bits, off);
  if (lane == 0)  // + block header (3) + end of block (symbol 256: 7 bits)
    sizes[(int64_t)bt * B + blk] = (uint32_t)((bits + 10 + 7) / 8);
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
  const size_t smem = kBlocksPerCta * deflate_warp_smem(b);  // <= 73 KB (b <= 1024)
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
