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
// Two launches: one CTA per block (threads find every position's match in
// shared memory, then one thread walks the greedy parse), then one CTA per
// sequence for l_i = 1[c_i * B > sum_j c_j] in 64-bit integers.
#include "sa_common.cuh"

namespace sa {

constexpr int kMaxBlockBytes = 1024;
constexpr int kCompThreads = 128;

// RFC 1951 section 3.2.5: first length of symbols 257..285 with their extra
// bits, and first distance of codes 0..29 with theirs.
__constant__ int16_t c_len_base[29] = {3,  4,  5,  6,  7,  8,  9,  10, 11,  13,  15,  17,  19,  23, 27,
                                       31, 35, 43, 51, 59, 67, 83, 99, 115, 131, 163, 195, 227, 258};
__constant__ int8_t c_len_extra[29] = {0, 0, 0, 0, 0, 0, 0, 0, 1, 1, 1, 1, 2, 2, 2,
                                       2, 3, 3, 3, 3, 4, 4, 4, 4, 5, 5, 5, 5, 0};
__constant__ int32_t c_dist_base[30] = {1,    2,    3,    4,    5,    7,     9,     13,    17,  25,
                                        33,   49,   65,   97,   129,  193,   257,   385,   513, 769,
                                        1025, 1537, 2049, 3073, 4097, 6145, 8193, 12289, 16385, 24577};
__constant__ int8_t c_dist_extra[30] = {0, 0, 0, 0, 1, 1, 2, 2,  3,  3,  4,  4,  5,  5,  6,
                                        6, 7, 7, 8, 8, 9, 9, 10, 10, 11, 11, 12, 12, 13, 13};

// Bits of a match: length symbol (7 or 8 bits) + its extra bits + distance
// code (5 bits) + its extra bits.
__device__ int match_bits(int len, int dist) {
  int s = 28;
  while (c_len_base[s] > len) --s;
  int d = 29;
  while (c_dist_base[d] > dist) --d;
  return (257 + s <= 279 ? 7 : 8) + c_len_extra[s] + 5 + c_dist_extra[d];
}

__global__ void __launch_bounds__(kCompThreads) deflate_size_kernel(const uint8_t* x, int64_t n_bytes,
                                                                    int b, int B, uint32_t* sizes) {
  __shared__ uint8_t xs[kMaxBlockBytes];
  __shared__ uint16_t mlen[kMaxBlockBytes];
  __shared__ uint16_t mdist[kMaxBlockBytes];
  const int blk = blockIdx.x, bt = blockIdx.y;
  const uint8_t* src = x + (int64_t)bt * n_bytes + (int64_t)blk * b;
  for (int i = threadIdx.x; i < b; i += blockDim.x) xs[i] = src[i];
  __syncthreads();
  for (int p = threadIdx.x; p < b; p += blockDim.x) {
    int m = 0, dist = 0;
    if (p + 3 <= b) {
      const uint8_t a0 = xs[p], a1 = xs[p + 1], a2 = xs[p + 2];
      for (int q = p - 1; q >= 0 && p - q <= 32768; --q) {
        if (xs[q] == a0 && xs[q + 1] == a1 && xs[q + 2] == a2) {  // nearest earlier match
          while (p + m < b && m < 258 && xs[q + m] == xs[p + m]) ++m;
          dist = p - q;
          break;
        }
      }
    }
    mlen[p] = (uint16_t)m;
    mdist[p] = (uint16_t)dist;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t bits = 3 + 7;  // block header, end of block (symbol 256: 7 bits)
    for (int p = 0; p < b;) {
      const int m = mlen[p];
      if (m >= 3) {
        bits += match_bits(m, mdist[p]);
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
  deflate_size_kernel<<<dim3(B, batch), kCompThreads, 0, s>>>(bytes, n_bytes, b, B, sizes);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  literal_flags_kernel<<<batch, 256, 0, s>>>(sizes, B, flags);
  return cudaGetLastError();
}

}  // namespace sa
