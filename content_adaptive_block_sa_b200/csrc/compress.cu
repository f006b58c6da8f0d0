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
// Two launches: one warp per block (lanes find every position's nearest
// match over 32-bit three-byte keys in shared memory, then one lane walks the
// greedy parse with the code lengths in closed form), then one CTA per
// sequence for l_i = 1[c_i * B > sum_j c_j] in 64-bit integers.
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

__host__ __device__ constexpr size_t deflate_warp_smem(int b) {
  return ((size_t)9 * b + 15) / 16 * 16;
}

__global__ void __launch_bounds__(kCompThreads) deflate_size_kernel(const uint8_t* x, int64_t n_bytes,
                                                                    int b, int B, uint32_t* sizes) {
  // per warp, deflate_warp_smem(b) bytes: keys (x[p] | x[p+1] << 8 | x[p+2] << 16),
  // match lengths, match distances, the block's bytes
  extern __shared__ __align__(16) uint8_t dyn_s[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x * kBlocksPerCta + warp, bt = blockIdx.y;
  if (blk >= B) return;  // warp-uniform; no CTA-wide barrier below
  uint8_t* base = dyn_s + (size_t)warp * deflate_warp_smem(b);
  uint32_t* key = reinterpret_cast<uint32_t*>(base);
  uint16_t* mlen = reinterpret_cast<uint16_t*>(base + 4 * b);
  uint16_t* mdist = mlen + b;
  uint8_t* xs = base + 8 * b;
  const uint8_t* src = x + (int64_t)bt * n_bytes + (int64_t)blk * b;
  for (int i = lane; i < b; i += 32) xs[i] = src[i];
  __syncwarp();
  for (int p = lane; p + 3 <= b; p += 32)
    key[p] = (uint32_t)xs[p] | ((uint32_t)xs[p + 1] << 8) | ((uint32_t)xs[p + 2] << 16);
  __syncwarp();
  for (int p = lane; p < b; p += 32) {
    int m = 0, dist = 0;
    if (p + 3 <= b) {
      const uint32_t k = key[p];
      for (int q = p - 1; q >= 0 && p - q <= 32768; --q) {
        if (key[q] == k) {  // the nearest earlier position with the same three bytes
          m = 3;
          while (p + m < b && m < 258 && xs[q + m] == xs[p + m]) ++m;
          dist = p - q;
          break;
        }
      }
    }
    mlen[p] = (uint16_t)m;
    mdist[p] = (uint16_t)dist;
  }
  __syncwarp();
  if (lane == 0) {
    int bits = 3 + 7;  // block header, end of block (symbol 256: 7 bits)
    for (int p = 0; p < b;) {
      const int m = mlen[p];
      if (m >= 3) {
        bits += length_bits(m) + distance_bits(mdist[p]);
        p += m;
      } else {
        bits += xs[p] <= 143 ? 8 : 9;
        ++p;
      }
    }
    sizes[(int64_t)bt * B + blk] = (uint32_t)((bits + 7) / 8);
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
  const size_t smem = kBlocksPerCta * deflate_warp_smem(b);  // <= 36 KB (b <= 1024)
  deflate_size_kernel<<<dim3((B + kBlocksPerCta - 1) / kBlocksPerCta, batch), kCompThreads, smem, s>>>(
      bytes, n_bytes, b, B, sizes);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  literal_flags_kernel<<<batch, 256, 0, s>>>(sizes, B, flags);
  return cudaGetLastError();
}

}  // namespace sa
